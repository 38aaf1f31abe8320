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

namespace bitnet {

constexpr int kI8Warps = 8;          // warps (rows in flight) per CTA
constexpr int kI8CtasPerSm = 8;

struct I8Epilogue {
    const float *bias, *gamma, *res;
    int relu;
};

template <int MT>
__global__ void __launch_bounds__(kI8Warps * 32) i8_gemv_kernel(const int8_t *__restrict__ w, int64_t n,
                                                             int64_t rowb, const int8_t *__restrict__ q,
                                                             int64_t kpad, const float *__restrict__ s_act,
                                                             float s_w, I8Epilogue epi, float *y, int32_t *acc_out)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t chunks = rowb / 16;            // 16-byte chunks per row
    for (int64_t row = int64_t(blockIdx.x) * kI8Warps + warp; row < n; row += int64_t(gridDim.x) * kI8Warps) {
        const int4 *wr = reinterpret_cast<const int4 *>(w + row * rowb);
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
                float v = __fmul_rn(__fmul_rn(float(acc[t]), s_act[t]), s_w);
                if (epi.bias) v = __fadd_rn(v, epi.bias[row]);
                if (epi.relu) v = v > 0.f ? v : 0.f;
                if (epi.gamma) v = __fmul_rn(epi.gamma[row], v);
                if (epi.res) v = __fadd_rn(epi.res[o], v);
                y[o] = v;
                if (acc_out) acc_out[o] = acc[t];
            }
        }
    }
}

template <int MT>
static cudaError_t launch_mt(const int8_t *w, int64_t n, int64_t rowb, const int8_t *q, int64_t kpad,
                             const float *s_act, float s_w, I8Epilogue epi, float *y, int32_t *acc, int grid,
                             cudaStream_t st)
{
    i8_gemv_kernel<MT><<<grid, kI8Warps * 32, 0, st>>>(w, n, rowb, q, kpad, s_act, s_w, epi, y, acc);
    return cudaGetLastError();
}

// Quantised activations q [m, kpad] and scales [m] are already in device
// memory; runs the tokens in slices of at most 8.
cudaError_t launch_gemv_i8(const int8_t *w, int64_t n, int64_t k, float s_w, const int8_t *q, const float *s_act,
                           int64_t m, const bitnet_epilogue *e, float *y, int32_t *acc, int sm_count,
                           cudaStream_t st)
{
    const int64_t rowb = 32 * ((k + 31) / 32), kpad = 128 * ((k + 127) / 128);
    const int64_t want = (n + kI8Warps - 1) / kI8Warps;
    const int64_t cap = int64_t(sm_count) * kI8CtasPerSm;
    const int grid = int(want < cap ? want : cap);
    for (int64_t m0 = 0; m0 < m; m0 += 8) {
        const int mt = int(m - m0 < 8 ? m - m0 : 8);
        I8Epilogue epi{nullptr, nullptr, nullptr, 0};
        if (e) epi = I8Epilogue{e->bias, e->gamma, e->residual ? e->residual + m0 * n : nullptr, e->relu ? 1 : 0};
        const int8_t *qs = q + m0 * kpad;
        const float *ss = s_act + m0;
        float *ys = y + m0 * n;
        int32_t *as = acc ? acc + m0 * n : nullptr;
        cudaError_t r;
        switch (mt) {
        case 1: r = launch_mt<1>(w, n, rowb, qs, kpad, ss, s_w, epi, ys, as, grid, st); break;
        case 2: r = launch_mt<2>(w, n, rowb, qs, kpad, ss, s_w, epi, ys, as, grid, st); break;
        case 3: r = launch_mt<3>(w, n, rowb, qs, kpad, ss, s_w, epi, ys, as, grid, st); break;
        case 4: r = launch_mt<4>(w, n, rowb, qs, kpad, ss, s_w, epi, ys, as, grid, st); break;
        case 5: r = launch_mt<5>(w, n, rowb, qs, kpad, ss, s_w, epi, ys, as, grid, st); break;
        case 6: r = launch_mt<6>(w, n, rowb, qs, kpad, ss, s_w, epi, ys, as, grid, st); break;
        case 7: r = launch_mt<7>(w, n, rowb, qs, kpad, ss, s_w, epi, ys, as, grid, st); break;
        default: r = launch_mt<8>(w, n, rowb, qs, kpad, ss, s_w, epi, ys, as, grid, st); break;
        }
        if (r != cudaSuccess) return r;
    }
    return cudaSuccess;
}

}  // namespace bitnet
