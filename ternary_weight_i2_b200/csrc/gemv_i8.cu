// gemv_i8.cu -- the I8_S linear layer: int8 weights x per-token int8
// activations, exact int32 sums, fp32 epilogue.
//
// "VibeVoice-ASR-BitNet Technical Report", §2.2.1 (I8_S: weights, activations
// and operator boundaries all INT8) and §2.4.2 (the I8_S kernel works on
// blocks of Q_K = 32 elements through the same multiply-add pipeline as
// I2_S; on the CPU a sign trick makes the unsigned x signed instruction do a
// signed product).  The reading taken: plain int8 weights [N, K] with one
// fp32 scale per tensor, each row stored as whole Q_K blocks (32*ceil(K/32)
// bytes); activations quantised per token as for I2_S.  On sm_100a the
// signed x signed product is native (dp4a.s32.s32), so no sign trick is
// needed.
//
// Decode shape: a weight row is 1 byte per element, so the kernel streams
// rows with 16-byte loads, one warp per row, the rows of a grid-stride loop
// dealt to the warps; activations (at most 8 tokens, already quantised into
// a [m, kpad] int8 buffer) are read through L1.  No shared-memory pipeline
// and no waits.
#include "common.cuh"
#include "gemv_i8.cuh"

namespace bitnet {

constexpr int kI8Warps = 8;          // warps (rows in flight) per CTA
constexpr int kI8CtasPerSm = 8;

constexpr int kI8MaxGroup = 64;     // linears per grouped launch

// One linear of a launch: its weights, this token slice's activations and
// outputs, and its epilogue operands.
struct I8Linear {
    const int8_t *w;
    const int8_t *q;          // int8 activations [MT, kpad] of this slice
    const float *s_act;       // [MT]
    float *y;                 // [MT, n] of this slice
    int32_t *acc;             // [MT, n] or null
    const float *bias, *gamma, *res;
    int64_t n, rowb, kpad;
    int64_t row0;             // first row of this linear in the launch's row numbering
    float s_w;
    int32_t relu;
};

struct I8Params {
    int32_t count;
    int64_t total_rows;
    I8Linear lin[kI8MaxGroup];
};
static_assert(sizeof(I8Params) <= 32760, "I8_S parameter block too large");

// The rows of all the launch's linears form one numbering; warps take rows
// of it round-robin.
template <int MT>
__global__ void __launch_bounds__(kI8Warps * 32) i8_gemv_kernel(const __grid_constant__ I8Params p)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int64_t grow = int64_t(blockIdx.x) * kI8Warps + warp; grow < p.total_rows;
         grow += int64_t(gridDim.x) * kI8Warps) {
        int li = 0;
        while (li + 1 < p.count && p.lin[li + 1].row0 <= grow) ++li;
        const I8Linear &L = p.lin[li];
        const int64_t row = grow - L.row0, n = L.n, rowb = L.rowb, kpad = L.kpad;
        const int8_t *__restrict__ q = L.q;
        const int64_t chunks = rowb / 16;        // 16-byte chunks per row
        const int4 *wr = reinterpret_cast<const int4 *>(L.w + row * rowb);
        int32_t acc[MT];
#pragma unroll
        for (int t = 0; t < MT; ++t) acc[t] = 0;
        // two chunks per lane per step: 1 KB of the row in flight per warp
        int64_t c = lane;
        for (; c + 32 < chunks; c += 64) {
            const int4 w0 = __ldcs(wr + c), w1 = __ldcs(wr + c + 32);
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                const int4 *qr = reinterpret_cast<const int4 *>(q + t * kpad);
                const int4 a0 = __ldg(qr + c), a1 = __ldg(qr + c + 32);
                acc[t] = __dp4a(w0.x, a0.x, acc[t]);
                acc[t] = __dp4a(w0.y, a0.y, acc[t]);
                acc[t] = __dp4a(w0.z, a0.z, acc[t]);
                acc[t] = __dp4a(w0.w, a0.w, acc[t]);
                acc[t] = __dp4a(w1.x, a1.x, acc[t]);
                acc[t] = __dp4a(w1.y, a1.y, acc[t]);
                acc[t] = __dp4a(w1.z, a1.z, acc[t]);
                acc[t] = __dp4a(w1.w, a1.w, acc[t]);
            }
        }
        if (c < chunks) {
            const int4 w0 = __ldcs(wr + c);
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                const int4 a0 = __ldg(reinterpret_cast<const int4 *>(q + t * kpad) + c);
                acc[t] = __dp4a(w0.x, a0.x, acc[t]);
                acc[t] = __dp4a(w0.y, a0.y, acc[t]);
                acc[t] = __dp4a(w0.z, a0.z, acc[t]);
                acc[t] = __dp4a(w0.w, a0.w, acc[t]);
            }
        }
        // integer sums: any reduction order gives the same result
#pragma unroll
        for (int t = 0; t < MT; ++t)
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
        // lane t writes token t: y = ((float)acc * s_act) * s_w, then the
        // optional fused epilogue (one rounding per step)
#pragma unroll
        for (int t = 0; t < MT; ++t) {
            if (lane == t) {
                const size_t o = size_t(t) * size_t(n) + size_t(row);
                float v = __fmul_rn(__fmul_rn(float(acc[t]), L.s_act[t]), L.s_w);
                if (L.bias) v = __fadd_rn(v, L.bias[row]);
                if (L.relu) v = v > 0.f ? v : 0.f;
                if (L.gamma) v = __fmul_rn(L.gamma[row], v);
                if (L.res) v = __fadd_rn(L.res[o], v);
                L.y[o] = v;
                if (L.acc) L.acc[o] = acc[t];
            }
        }
    }
}

static_assert(kI8MaxGroup == BITNET_I8_GROUP_MAX, "group limit");

cudaError_t launch_gemv_i8_group(const I8Job *jobs, int count, int64_t m, int sm_count, cudaStream_t st)
{
    if (count < 1 || count > kI8MaxGroup) return cudaErrorInvalidValue;
    static thread_local I8Params p;
    int64_t total = 0;
    for (int i = 0; i < count; ++i) total += jobs[i].n;
    const int64_t want = (total + kI8Warps - 1) / kI8Warps;
    const int64_t cap = int64_t(sm_count) * kI8CtasPerSm;
    const int grid = int(want < cap ? want : cap);
    for (int64_t m0 = 0; m0 < m; m0 += 8) {
        const int mt = int(m - m0 < 8 ? m - m0 : 8);
        p.count = count;
        p.total_rows = total;
        int64_t row0 = 0;
        for (int i = 0; i < count; ++i) {
            const I8Job &J = jobs[i];
            I8Linear &L = p.lin[i];
            L.w = J.w;
            L.n = J.n;
            L.rowb = 32 * ((J.k + 31) / 32);
            L.kpad = 128 * ((J.k + 127) / 128);
            L.q = J.q + m0 * L.kpad;
            L.s_act = J.s_act + m0;
            L.y = J.y + m0 * J.n;
            L.acc = J.acc ? J.acc + m0 * J.n : nullptr;
            L.bias = J.epi ? J.epi->bias : nullptr;
            L.gamma = J.epi ? J.epi->gamma : nullptr;
            L.res = (J.epi && J.epi->residual) ? J.epi->residual + m0 * J.n : nullptr;
            L.relu = (J.epi && J.epi->relu) ? 1 : 0;
            L.s_w = J.s_w;
            L.row0 = row0;
            row0 += J.n;
        }
        const dim3 blk(kI8Warps * 32);
        switch (mt) {
        case 1: i8_gemv_kernel<1><<<grid, blk, 0, st>>>(p); break;
        case 2: i8_gemv_kernel<2><<<grid, blk, 0, st>>>(p); break;
        case 3: i8_gemv_kernel<3><<<grid, blk, 0, st>>>(p); break;
        case 4: i8_gemv_kernel<4><<<grid, blk, 0, st>>>(p); break;
        case 5: i8_gemv_kernel<5><<<grid, blk, 0, st>>>(p); break;
        case 6: i8_gemv_kernel<6><<<grid, blk, 0, st>>>(p); break;
        case 7: i8_gemv_kernel<7><<<grid, blk, 0, st>>>(p); break;
        default: i8_gemv_kernel<8><<<grid, blk, 0, st>>>(p); break;
        }
        cudaError_t r = cudaGetLastError();
        if (r != cudaSuccess) return r;
    }
    return cudaSuccess;
}

cudaError_t launch_gemv_i8(const int8_t *w, int64_t n, int64_t k, float s_w, const int8_t *q, const float *s_act,
                           int64_t m, const bitnet_epilogue *e, float *y, int32_t *acc, int sm_count,
                           cudaStream_t st)
{
    const I8Job j{w, n, k, s_w, q, s_act, y, acc, e};
    return launch_gemv_i8_group(&j, 1, m, sm_count, st);
}

}  // namespace bitnet
