// gemv.cu -- streaming ternary GEMV for the decode path (M <= 8 tokens).
//
// What it computes ("VibeVoice-ASR-BitNet Technical Report", §2.2.2, §2.4.2,
// Figure 4): for every layer i of the launch and token m,
//   q      = per-token int8 quantisation of x_i[m, :]           (fused here)
//   acc[n] = sum_k q[k] * w_i[n, k]                              (exact int32)
//   y[m,n] = ((float)acc[n] * s_act[m]) * s_w,i
// Decode is bound by reading the 2-bit weights once per token (technical
// report §3.2, Figure 6b), so the kernel is built as a weight stream:
//
// * One CTA per SM works through a contiguous byte range of the launch's
//   weights (host-balanced).  Each warp is an independent pipeline over the
//   32-row tiles dealt to it: its lanes issue 1-D bulk (TMA) copies of their
//   own row chunk into a padded shared-memory slot, two slots deep, and wait
//   on an mbarrier; no register staging of weights.
// * Lane r owns weight row r of the tile, so there is no cross-lane reduction;
//   the int8 activations are broadcast from shared memory (all lanes read the
//   same address).
// * Decode in registers: a 32-bit word of codes holds 16 weights, four 2-bit
//   fields per byte; masking field g (one LOP3) leaves 4^g * code in each byte,
//   and dp4a multiplies those unsigned bytes by the signed activations.  With
//   code = w + 1 the exact sum is  sum(code*x) - sum(x); the four fields keep
//   separate accumulators and are recombined as (64*a0+16*a1+4*a2+a3) >> 6.
//   This is the unpack-then-multiply-add formulation of the technical report
//   (codes as unsigned bytes times signed int8, like maddubs) on the dp4a unit.
// * Every CTA quantises the activation rows its range needs straight into
//   shared memory, laid out so one 16-byte read gives the four activation
//   words a code word needs.
#include <cstdio>

#include "common.cuh"
#include "gemv.cuh"

namespace bitnet {

template <int M>
struct GemvMeta {
    uint64_t bar[8 * kSlotsPerWarp];
    uint64_t stall_bar;
    int32_t tcum[kMaxRangeSegs + 1];
    int32_t seg_lin[kMaxRangeSegs];
    int32_t seg_slot[kMaxRangeSegs];
    int32_t seg_tile0[kMaxRangeSegs];
    int32_t xoff[kMaxRangeInputs];
    int32_t kpad[kMaxRangeInputs];
    int32_t wstart[kMaxRangeInputs * M + 1];   // job word starts (job = slot*M + m)
    uint32_t amax[kMaxRangeInputs * M];
    int32_t nonfin[kMaxRangeInputs * M];
    float inv[kMaxRangeInputs * M];
    float s_act[kMaxRangeInputs * M];
    int32_t sumx[kMaxRangeInputs * M];
};
static_assert(sizeof(GemvMeta<8>) <= kMetaBytes, "meta area too small");

__device__ __forceinline__ uint32_t perm_offset(int p)
{
    // word p (elements 4p..4p+3) of a row -> byte offset in the broadcast
    // layout: block j = p/32, field g = (p/8)%4, word-in-field t = p%8
    return uint32_t((p >> 5) * 128 + (p & 7) * 16 + ((p >> 3) & 3) * 4);
}

template <int M, int NW>
__global__ void __launch_bounds__(NW * 32, 1) gemv_stack_kernel(const __grid_constant__ GemvParams p)
{
    constexpr int T = NW * 32;
    constexpr int QB = 16;   // float4 words a thread holds per quantiser batch
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *xarea = smem + gemv_ring_bytes(NW);
    GemvMeta<M> *meta = reinterpret_cast<GemvMeta<M> *>(xarea + p.x_bytes);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const GemvRange &R = p.rng[blockIdx.x];
    const int nin = R.nin, nseg = R.nseg;
    const uint64_t limit = p.wait_limit;

    // ---------------------------------------------------------- set-up
    if (tid == 0) {
        meta->tcum[0] = 0;
        for (int s = 0; s < nseg; ++s) {
            const GemvSeg &sg = p.seg[R.seg0 + s];
            meta->tcum[s + 1] = meta->tcum[s] + (sg.tile1 - sg.tile0);
            meta->seg_lin[s] = sg.lin;
            meta->seg_slot[s] = sg.slot;
            meta->seg_tile0[s] = sg.tile0;
        }
        int off = 0, w = 0;
        for (int u = 0; u < nin; ++u) {
            const int kp = 128 * p.inp[R.in[u]].kb;
            meta->xoff[u] = off;
            meta->kpad[u] = kp;
            off += M * kp;
            for (int m = 0; m < M; ++m) {
                meta->wstart[u * M + m] = w;
                w += kp / 4;
            }
        }
        meta->wstart[nin * M] = w;
        mbar_init(smem_u32(&meta->stall_bar), 1);
    }
    if (lane == 0)
        for (int s = 0; s < kSlotsPerWarp; ++s) mbar_init(smem_u32(&meta->bar[warp * kSlotsPerWarp + s]), 1);
    for (int j = tid; j < nin * M; j += T) {
        meta->amax[j] = 0u;
        meta->nonfin[j] = 0;
        meta->sumx[j] = 0;
    }
    fence_mbar_init();
    __syncthreads();

    if (p.force_stall) {
        // Test aid: wait on a barrier nobody arrives at; the bounded wait
        // must expire, raise the timeout flag and return cleanly.
        if (!mbar_wait(smem_u32(&meta->stall_bar), 0, limit)) raise_flag(p.flags, BITNET_FLAG_TIMEOUT);
        return;
    }

    const int ttot = meta->tcum[nseg];
    const uint32_t ring = smem_u32(smem) + warp * kSlotsPerWarp * kSlotBytes;
    const uint32_t bar0 = smem_u32(&meta->bar[warp * kSlotsPerWarp]);

    auto nchunks = [&](int s) { return (p.lin[meta->seg_lin[s]].kb + kChunkBlocks - 1) / kChunkBlocks; };
    auto advance = [&](int &i, int &s, int &c) {
        if (++c == nchunks(s)) {
            c = 0;
            i += NW;
            while (s < nseg && i >= meta->tcum[s + 1]) ++s;
        }
    };
    auto issue = [&](int i, int s, int c, int slot) {
        const GemvLinear &L = p.lin[meta->seg_lin[s]];
        const int row0 = (meta->seg_tile0[s] + (i - meta->tcum[s])) * kTileRows;
        const int rows = min(kTileRows, L.n - row0);
        const int cb0 = c * kChunkBlocks;
        const int bytes = 32 * min(kChunkBlocks, L.kb - cb0);
        const uint32_t bar = bar0 + 8 * slot;
        if (lane == 0) mbar_arrive_expect_tx(bar, uint32_t(rows * bytes));
        __syncwarp();
        if (lane < rows)
            bulk_g2s(ring + slot * kSlotBytes + lane * kSlotPitch,
                     L.packed + size_t(row0 + lane) * size_t(32 * L.kb) + 32 * cb0, uint32_t(bytes), bar);
    };

    // producer iterator: start streaming weights before quantising
    int pi = warp, ps = 0, pc = 0;
    while (ps < nseg && pi >= meta->tcum[ps + 1]) ++ps;
    int issued = 0;
    for (int sl = 0; sl < kSlotsPerWarp && pi < ttot; ++sl) {
        issue(pi, ps, pc, sl);
        advance(pi, ps, pc);
        ++issued;
    }

    // ------------------------------------------- activation quantiser
    {
        const int W = meta->wstart[nin * M];
        const int nbatch = (W + QB * T - 1) / (QB * T);
        float4 xr[QB];
        auto load_word = [&](int J, int word) -> float4 {
            const int u = J / M, m = J - u * M;
            const GemvInput &in = p.inp[R.in[u]];
            const int pw = word - meta->wstart[J];
            const int k0 = 4 * pw;
            const float *row = static_cast<const float *>(in.x) + size_t(m) * size_t(in.k);
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (k0 + 3 < in.k && (reinterpret_cast<uintptr_t>(row) & 15) == 0) {
                v = __ldg(reinterpret_cast<const float4 *>(row + k0));
            } else {
                if (k0 + 0 < in.k) v.x = __ldg(row + k0 + 0);
                if (k0 + 1 < in.k) v.y = __ldg(row + k0 + 1);
                if (k0 + 2 < in.k) v.z = __ldg(row + k0 + 2);
                if (k0 + 3 < in.k) v.w = __ldg(row + k0 + 3);
            }
            return v;
        };
        if (!p.prequant) {
            // pass 1: absmax and finiteness per job (token row of an input)
            for (int b = 0; b < nbatch; ++b) {
                int J = 0;
#pragma unroll
                for (int q = 0; q < QB; ++q) {
                    const int word = (b * QB + q) * T + tid;   // warp-uniform job
                    if (word - lane >= W) break;
                    while (word - lane >= meta->wstart[J + 1]) ++J;
                    xr[q] = word < W ? load_word(J, word) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
                J = 0;
#pragma unroll
                for (int q = 0; q < QB; ++q) {
                    const int word = (b * QB + q) * T + tid;
                    if (word - lane >= W) break;
                    while (word - lane >= meta->wstart[J + 1]) ++J;
                    const float4 v = xr[q];
                    const bool fin = isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w);
                    float a = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
                    if (!fin) a = 0.f;
                    a = warp_max(a);
                    const bool anynf = __any_sync(0xffffffffu, !fin);
                    if (lane == 0) {
                        atomicMax(&meta->amax[J], __float_as_uint(a));
                        if (anynf) meta->nonfin[J] = 1;
                    }
                }
            }
            __syncthreads();
            for (int J = tid; J < nin * M; J += T) {
                const float amax = __uint_as_float(meta->amax[J]);
                const bool bad = meta->nonfin[J] != 0;
                if (bad) raise_flag(p.flags, BITNET_FLAG_NONFINITE);
                meta->inv[J] = (bad || amax == 0.f) ? 0.f : __fdiv_rn(127.0f, amax);
                meta->s_act[J] = (bad || amax == 0.f) ? 0.f : __fdiv_rn(amax, 127.0f);
            }
            __syncthreads();
            // pass 2: codes into the broadcast layout, and sum(q) per job
            for (int b = 0; b < nbatch; ++b) {
                int J = 0;
#pragma unroll
                for (int q = 0; q < QB; ++q) {
                    const int word = (b * QB + q) * T + tid;
                    if (word - lane >= W) break;
                    while (word - lane >= meta->wstart[J + 1]) ++J;
                    const float4 v = (nbatch == 1) ? xr[q]
                                                   : (word < W ? load_word(J, word) : make_float4(0.f, 0.f, 0.f, 0.f));
                    const float inv = meta->inv[J];
                    int32_t q0 = 0, q1 = 0, q2 = 0, q3 = 0;
                    if (word < W && inv != 0.f) {
                        q0 = quant_one(v.x, inv);
                        q1 = quant_one(v.y, inv);
                        q2 = quant_one(v.z, inv);
                        q3 = quant_one(v.w, inv);
                    }
                    const int32_t s = warp_sum(q0 + q1 + q2 + q3);
                    if (word < W) {
                        const int u = J / M, m = J - u * M;
                        const int pw = word - meta->wstart[J];
                        *reinterpret_cast<uint32_t *>(xarea + meta->xoff[u] + m * meta->kpad[u] + perm_offset(pw)) =
                            pack4(q0, q1, q2, q3);
                    }
                    if (lane == 0) atomicAdd(&meta->sumx[J], s);
                }
            }
        } else {
            // pre-quantised int8 rows [m, kpad] with given scales
            for (int word = tid; word - lane < W; word += T) {
                int J = 0;
                while (word - lane >= meta->wstart[J + 1]) ++J;
                const int u = J / M, m = J - u * M;
                const GemvInput &in = p.inp[R.in[u]];
                const int pw = word - meta->wstart[J];
                uint32_t v = 0;
                int32_t s = 0;
                if (word < W) {
                    v = __ldg(reinterpret_cast<const uint32_t *>(static_cast<const int8_t *>(in.x) +
                                                                 size_t(m) * size_t(meta->kpad[u])) +
                              pw);
                    s = int32_t(int8_t(v)) + int32_t(int8_t(v >> 8)) + int32_t(int8_t(v >> 16)) +
                        int32_t(int8_t(v >> 24));
                    *reinterpret_cast<uint32_t *>(xarea + meta->xoff[u] + m * meta->kpad[u] + perm_offset(pw)) = v;
                }
                s = warp_sum(s);
                if (lane == 0) atomicAdd(&meta->sumx[J], s);
            }
            for (int J = tid; J < nin * M; J += T) {
                const int u = J / M, m = J - u * M;
                meta->s_act[J] = p.inp[R.in[u]].scale[m];
            }
        }
    }
    __syncthreads();

    // ------------------------------------------------- stream and multiply
    int ci = warp, cs = 0, cc = 0;
    while (cs < nseg && ci >= meta->tcum[cs + 1]) ++cs;
    int slot = 0, consumed = 0;
    uint32_t phase = 0;
    int32_t acc[M][4];
#pragma unroll
    for (int m = 0; m < M; ++m) acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0;
    bool timed_out = false;

    while (ci < ttot) {
        const bool landed = mbar_wait(bar0 + 8 * slot, (phase >> slot) & 1u, limit);
        if (!__all_sync(0xffffffffu, landed)) {   // warp-uniform decision
            timed_out = true;
            break;
        }
        phase ^= 1u << slot;
        const int lin = meta->seg_lin[cs];
        const GemvLinear &L = p.lin[lin];
        const int u = meta->seg_slot[cs];
        const int kp = meta->kpad[u];
        const int cb0 = cc * kChunkBlocks;
        const int nblk = min(kChunkBlocks, L.kb - cb0);
        const uint32_t wrow = ring + slot * kSlotBytes + lane * kSlotPitch;
        const uint32_t xb = smem_u32(xarea) + meta->xoff[u] + cb0 * 128;
#pragma unroll 2
        for (int jj = 0; jj < nblk; ++jj) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint4 wv = lds128(wrow + jj * 32 + h * 16);
                const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t c0 = wd[i] & 0x03030303u, c1 = wd[i] & 0x0C0C0C0Cu;
                    const uint32_t c2 = wd[i] & 0x30303030u, c3 = wd[i] & 0xC0C0C0C0u;
#pragma unroll
                    for (int m = 0; m < M; ++m) {
                        const uint4 xv = lds128(xb + m * kp + jj * 128 + (4 * h + i) * 16);
                        acc[m][0] = dp4a_us(c0, xv.x, acc[m][0]);
                        acc[m][1] = dp4a_us(c1, xv.y, acc[m][1]);
                        acc[m][2] = dp4a_us(c2, xv.z, acc[m][2]);
                        acc[m][3] = dp4a_us(c3, xv.w, acc[m][3]);
                    }
                }
            }
        }
        if (cc == nchunks(cs) - 1) {
            const int row0 = (meta->seg_tile0[cs] + (ci - meta->tcum[cs])) * kTileRows;
            const int row = row0 + lane;
            if (row < L.n) {
#pragma unroll
                for (int m = 0; m < M; ++m) {
                    const int32_t s64 = acc[m][0] * 64 + acc[m][1] * 16 + acc[m][2] * 4 + acc[m][3];
                    const int32_t a = (s64 >> 6) - meta->sumx[u * M + m];
                    const float yv = __fmul_rn(__fmul_rn(float(a), meta->s_act[u * M + m]), L.scale);
                    L.y[size_t(m) * size_t(L.n) + row] = yv;
                    if (L.acc) L.acc[size_t(m) * size_t(L.n) + row] = a;
                }
            }
#pragma unroll
            for (int m = 0; m < M; ++m) acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0;
        }
        __syncwarp();
        ++consumed;
        if (pi < ttot) {
            issue(pi, ps, pc, slot);
            advance(pi, ps, pc);
            ++issued;
        }
        advance(ci, cs, cc);
        slot = (slot + 1 == kSlotsPerWarp) ? 0 : slot + 1;
    }

    if (timed_out) {
        raise_flag(p.flags, BITNET_FLAG_TIMEOUT);
        // let this warp's copies in flight land before the CTA exits
        for (int k = consumed; k < issued; ++k) {
            mbar_wait(bar0 + 8 * slot, (phase >> slot) & 1u, kDrainWaitLimit);
            phase ^= 1u << slot;
            slot = (slot + 1 == kSlotsPerWarp) ? 0 : slot + 1;
        }
    }
}

// ------------------------------------------------------------- launcher

template <int M, int NW>
static cudaError_t launch_one(const GemvParams &p, size_t smem, cudaStream_t st)
{
    static bool configured = false;   // per instantiation, set once
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(gemv_stack_kernel<M, NW>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    gemv_stack_kernel<M, NW><<<p.num_ranges, NW * 32, smem, st>>>(p);
    return cudaGetLastError();
}

template <int NW>
static cudaError_t launch_nw(const GemvParams &p, size_t smem, cudaStream_t st)
{
    switch (p.m) {
    case 1: return launch_one<1, NW>(p, smem, st);
    case 2: return launch_one<2, NW>(p, smem, st);
    case 3: return launch_one<3, NW>(p, smem, st);
    case 4: return launch_one<4, NW>(p, smem, st);
    case 5: return launch_one<5, NW>(p, smem, st);
    case 6: return launch_one<6, NW>(p, smem, st);
    case 7: return launch_one<7, NW>(p, smem, st);
    case 8: return launch_one<8, NW>(p, smem, st);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_gemv(const GemvParams &p, int nw, cudaStream_t st)
{
    const size_t smem = size_t(gemv_ring_bytes(nw)) + size_t(p.x_bytes) + size_t(kMetaBytes);
    if (smem > size_t(kSmemLimit)) return cudaErrorInvalidValue;
    switch (nw) {
    case 8: return launch_nw<8>(p, smem, st);
    case 6: return launch_nw<6>(p, smem, st);
    case 4: return launch_nw<4>(p, smem, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace bitnet
