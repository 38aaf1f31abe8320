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
// * One CTA per SM works through a contiguous, byte-balanced range of the
//   launch's weight tiles.  Each warp is an independent pipeline over the
//   32-row tiles dealt to it: per unit it issues BOX 2-D tiled TMA loads
//   (128 bytes x 32 rows each, 128-byte swizzle) from the layer's tensor map
//   into a shared-memory slot, kSlotsPerWarp deep, and waits on an mbarrier;
//   no register staging of weights.  Ragged tails (rows past N, bytes past
//   the row end) are zero-filled by the tensor map and never used.
// * Lane r owns weight row r of the tile, so there is no cross-lane reduction;
//   the swizzle puts the 32 lanes' 16-byte reads of one column in distinct
//   bank groups, and the int8 activations are broadcast from shared memory
//   (all lanes read the same address).
// * Decode in registers: a 32-bit word of codes holds 16 weights, four 2-bit
//   fields per byte; masking field g (one LOP3) leaves 4^g * code in each byte,
//   and dp4a multiplies those unsigned bytes by the signed activations.  With
//   code = w + 1 the exact sum is  sum(code*x) - sum(x); the four fields keep
//   separate accumulators and are recombined as (64*a0+16*a1+4*a2+a3) >> 6.
//   This is the unpack-then-multiply-add formulation of the technical report
//   (codes as unsigned bytes times signed int8, like maddubs) on the dp4a unit.
//   Even and odd blocks use separate accumulator sets for instruction-level
//   parallelism.
// * Every CTA quantises the activation rows its range needs straight into
//   shared memory, laid out so one 16-byte read gives the four activation
//   words a code word needs.  The activation loads are issued before the
//   weight prefetch so that they are not queued behind it.
#include <cstdio>

#include "common.cuh"
#include "gemv.cuh"

namespace bitnet {

struct SegInfo {
    const void *tmap;
    float *y;
    int32_t *acc;
    int32_t n;
    int32_t rowb;    // packed bytes per row
    int32_t kb;      // blocks per row
    int32_t nch;     // chunks per tile
    int32_t slot;    // range-local input slot
    int32_t tile0;   // first tile of the layer in this range
    int32_t tcum;    // range-local index of the segment's first tile
    int32_t lin;     // index of the layer in the launch (its epilogue operands)
    float scale;
};

template <int M>
struct GemvMeta {
    uint64_t bar[kMaxWarps * kSlotsPerWarp];
    uint64_t stall_bar;
    SegInfo seg[kMaxRangeSegs];
    int32_t ttot;
    int32_t xoff[kMaxRangeInputs];
    int32_t kpad[kMaxRangeInputs];
    int32_t wstart[kMaxRangeInputs * M + 1];   // job word starts (job = slot*M + m)
    const void *xptr[kMaxRangeInputs];
    const float *xscale[kMaxRangeInputs];
    int32_t xk[kMaxRangeInputs];
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

// Block jj of a unit for lane r: box jj/4, 128-byte line r of that box, 16-byte
// chunks 2*(jj%4)+h placed by the 128-byte swizzle (chunk ^ (r & 7)).
template <int M>
__device__ __forceinline__ void block_dot(uint32_t wrow, uint32_t rx, uint32_t xb, int kp, int jj,
                                          int32_t (&acc)[M][4])
{
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t ch = uint32_t((jj & 3) * 2 + h) ^ rx;
        const uint4 wv = lds128(wrow + (jj >> 2) * kBoxBytes + ch * 16);
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

template <int M, int NW, int BOX>
__global__ void __launch_bounds__(NW * 32, 1) gemv_stack_kernel(const __grid_constant__ GemvParams p)
{
    constexpr int T = NW * 32;
    constexpr int QB = (NW >= 16) ? 8 : 16;   // float4 words a thread holds per quantiser batch
    constexpr int SLOT = slot_bytes(BOX);
    constexpr int UNIT_BYTES = BOX * 128;     // bytes of each row per unit
    constexpr int UNIT_BLOCKS = BOX * kBoxBlocks;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // swizzled boxes need 1024-byte aligned destinations
    uint8_t *smem = smem_raw + ((kAlignPad - (smem_u32(smem_raw) & (kAlignPad - 1))) & (kAlignPad - 1));
    uint8_t *xarea = smem + ring_bytes(NW, BOX);
    GemvMeta<M> *meta = reinterpret_cast<GemvMeta<M> *>(xarea + p.x_bytes);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const GemvRange &R = p.rng[blockIdx.x];
    const int nin = R.nin, nseg = R.nseg;
    const uint64_t limit = p.wait_limit;

    // ---------------------------------------------------------- set-up
    // warp 0: one lane per segment; warp 1: one lane per input slot
    if (warp == 0) {
        int cnt = 0;
        if (lane < nseg) {
            const GemvSeg sg = p.seg[R.seg0 + lane];
            const GemvLinear &L = p.lin[sg.lin];
            SegInfo &si = meta->seg[lane];
            si.tmap = L.tmap;
            si.y = L.y;
            si.acc = L.acc;
            si.n = L.n;
            si.kb = L.kb;
            si.rowb = 32 * L.kb;
            si.nch = (32 * L.kb + UNIT_BYTES - 1) / UNIT_BYTES;
            si.slot = sg.slot;
            si.tile0 = sg.tile0;
            si.scale = L.scale;
            si.lin = sg.lin;
            cnt = sg.tile1 - sg.tile0;
        }
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane < nseg) meta->seg[lane].tcum = incl - cnt;
        if (lane == 31) meta->ttot = incl;
        if (lane == 0) mbar_init(smem_u32(&meta->stall_bar), 1);
    } else if (warp == 1) {
        int bytes = 0, kp = 0;
        if (lane < nin) {
            const GemvInput &in = p.inp[R.in[lane]];
            kp = 128 * in.kb;
            bytes = M * kp;
            meta->xptr[lane] = in.x;
            meta->xscale[lane] = in.scale;
            meta->xk[lane] = in.k;
            meta->kpad[lane] = kp;
        }
        int incl = bytes;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane < nin) {
            const int off = incl - bytes;
            meta->xoff[lane] = off;
            for (int m = 0; m < M; ++m) meta->wstart[lane * M + m] = (off + m * kp) / 4;
        }
        if (lane == 31) meta->wstart[nin * M] = incl / 4;
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
    uint64_t *trace = p.trace ? p.trace + (size_t(blockIdx.x) * NW + warp) * kTraceEvents : nullptr;
    auto stamp = [&](int ev) {
        if (trace && lane == 0) trace[ev] = globaltimer();
    };
    stamp(0);

    if (p.force_stall) {
        // Test aid: wait on a barrier nobody arrives at; the bounded wait
        // must expire, raise the timeout flag and return cleanly.
        if (!mbar_wait(smem_u32(&meta->stall_bar), 0, limit)) raise_flag(p.flags, BITNET_FLAG_TIMEOUT);
        return;
    }

    // ------------------------------- activation loads (pass-1 registers)
    const int W = meta->wstart[nin * M];
    const int nbatch = (W + QB * T - 1) / (QB * T);
    float4 xr[QB];
    auto load_word = [&](int J, int word) -> float4 {
        const int u = J / M, m = J - u * M;
        const int k = meta->xk[u];
        const int pw = word - meta->wstart[J];
        const int k0 = 4 * pw;
        const float *row = static_cast<const float *>(meta->xptr[u]) + size_t(m) * size_t(k);
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (k0 + 3 < k && (reinterpret_cast<uintptr_t>(row) & 15) == 0) {
            v = __ldg(reinterpret_cast<const float4 *>(row + k0));
        } else {
            if (k0 + 0 < k) v.x = __ldg(row + k0 + 0);
            if (k0 + 1 < k) v.y = __ldg(row + k0 + 1);
            if (k0 + 2 < k) v.z = __ldg(row + k0 + 2);
            if (k0 + 3 < k) v.w = __ldg(row + k0 + 3);
        }
        return v;
    };
    auto load_batch = [&](int b) {
        int J = 0;
#pragma unroll
        for (int q = 0; q < QB; ++q) {
            const int word = (b * QB + q) * T + tid;   // warp-uniform job
            if (word - lane >= W) break;
            while (word - lane >= meta->wstart[J + 1]) ++J;
            xr[q] = load_word(J, word);
        }
    };
    if (!p.prequant) load_batch(0);

    // ------------------------------------------------ weight prefetch
    const int ttot = meta->ttot;
    const uint64_t policy = l2_evict_first_policy();
    const uint32_t ring = smem_u32(smem) + warp * kSlotsPerWarp * SLOT;
    const uint32_t bar0 = smem_u32(&meta->bar[warp * kSlotsPerWarp]);
    auto seg_end = [&](int s) { return s + 1 < nseg ? meta->seg[s + 1].tcum : ttot; };
    auto advance = [&](int &i, int &s, int &c) {
        if (++c == meta->seg[s].nch) {
            c = 0;
            i += NW;
            while (s < nseg && i >= seg_end(s)) ++s;
        }
    };
    auto issue = [&](int i, int s, int c, int slot) {
        const SegInfo &si = meta->seg[s];
        const int row0 = (si.tile0 + (i - si.tcum)) * kTileRows;
        const int x0 = c * UNIT_BYTES;
        const int nbox = min(BOX, (si.rowb - x0 + 127) / 128);   // boxes that start inside the row
        const uint32_t bar = bar0 + 8 * slot;
        if (lane == 0) mbar_arrive_expect_tx(bar, uint32_t(nbox * kBoxBytes));
        __syncwarp();
        if (lane < nbox)
            tma_load_2d(ring + slot * SLOT + lane * kBoxBytes, si.tmap, x0 + lane * 128, row0, bar, policy);
    };
    // lanes that issue TMA loads acquire every map of the range once when the
    // maps' bytes may have changed at an address the TMA unit has cached
    if (p.fence_maps && lane < BOX)
        for (int s = 0; s < nseg; ++s) tensormap_acquire(meta->seg[s].tmap);
    int pi = warp, ps = 0, pc = 0;
    while (ps < nseg && pi >= seg_end(ps)) ++ps;
    int issued = 0;
    for (int sl = 0; sl < kSlotsPerWarp && pi < ttot; ++sl) {
        issue(pi, ps, pc, sl);
        advance(pi, ps, pc);
        ++issued;
    }
    stamp(1);

    // ------------------------------------------- activation quantiser
    if (!p.prequant) {
        // pass 1: absmax and finiteness per job (token row of an input)
        for (int b = 0; b < nbatch; ++b) {
            if (b > 0) load_batch(b);
            int J = 0;
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
            if (nbatch > 1) load_batch(b);
            int J = 0;
#pragma unroll
            for (int q = 0; q < QB; ++q) {
                const int word = (b * QB + q) * T + tid;
                if (word - lane >= W) break;
                while (word - lane >= meta->wstart[J + 1]) ++J;
                const float4 v = xr[q];
                const float inv = meta->inv[J];
                int32_t q0 = 0, q1 = 0, q2 = 0, q3 = 0;
                if (inv != 0.f) {
                    q0 = quant_one(v.x, inv);
                    q1 = quant_one(v.y, inv);
                    q2 = quant_one(v.z, inv);
                    q3 = quant_one(v.w, inv);
                }
                const int32_t s = warp_sum(q0 + q1 + q2 + q3);
                const int u = J / M, m = J - u * M;
                const int pw = word - meta->wstart[J];
                *reinterpret_cast<uint32_t *>(xarea + meta->xoff[u] + m * meta->kpad[u] + perm_offset(pw)) =
                    pack4(q0, q1, q2, q3);
                if (lane == 0) atomicAdd(&meta->sumx[J], s);
            }
        }
    } else {
        // pre-quantised int8 rows [m, kpad] with given scales
        for (int word = tid; word - lane < W; word += T) {
            int J = 0;
            while (word - lane >= meta->wstart[J + 1]) ++J;
            const int u = J / M, m = J - u * M;
            const int pw = word - meta->wstart[J];
            const uint32_t v = __ldg(reinterpret_cast<const uint32_t *>(static_cast<const int8_t *>(meta->xptr[u]) +
                                                                       size_t(m) * size_t(meta->kpad[u])) +
                                     pw);
            int32_t s = int32_t(int8_t(v)) + int32_t(int8_t(v >> 8)) + int32_t(int8_t(v >> 16)) +
                        int32_t(int8_t(v >> 24));
            *reinterpret_cast<uint32_t *>(xarea + meta->xoff[u] + m * meta->kpad[u] + perm_offset(pw)) = v;
            s = warp_sum(s);
            if (lane == 0) atomicAdd(&meta->sumx[J], s);
        }
        for (int J = tid; J < nin * M; J += T) {
            const int u = J / M, m = J - u * M;
            meta->s_act[J] = meta->xscale[u][m];
        }
    }
    __syncthreads();
    stamp(2);

    // ------------------------------------------------- stream and multiply
    int ci = warp, cs = 0, cc = 0;
    while (cs < nseg && ci >= seg_end(cs)) ++cs;
    int slot = 0, consumed = 0;
    uint32_t phase = 0;
    int32_t acc0[M][4], acc1[M][4];
#pragma unroll
    for (int m = 0; m < M; ++m)
#pragma unroll
        for (int g = 0; g < 4; ++g) acc0[m][g] = acc1[m][g] = 0;
    bool timed_out = false;

    while (ci < ttot) {
        const bool landed = mbar_wait(bar0 + 8 * slot, (phase >> slot) & 1u, limit);
        if (!__all_sync(0xffffffffu, landed)) {   // warp-uniform decision
            timed_out = true;
            break;
        }
        phase ^= 1u << slot;
        if (consumed == 0) stamp(3);
        const SegInfo &si = meta->seg[cs];
        const int u = si.slot;
        const int kp = meta->kpad[u];
        const int cb0 = cc * UNIT_BLOCKS;
        const int nblk = min(UNIT_BLOCKS, si.kb - cb0);
        const uint32_t wrow = ring + slot * SLOT + lane * 128;
        const uint32_t rx = uint32_t(lane & 7);
        const uint32_t xb = smem_u32(xarea) + meta->xoff[u] + cb0 * 128;
        int jj = 0;
#pragma unroll 1
        for (; jj + 1 < nblk; jj += 2) {
            block_dot<M>(wrow, rx, xb, kp, jj, acc0);
            block_dot<M>(wrow, rx, xb, kp, jj + 1, acc1);
        }
        if (jj < nblk) block_dot<M>(wrow, rx, xb, kp, jj, acc0);
        if (cc == si.nch - 1) {
            const int row = (si.tile0 + (ci - si.tcum)) * kTileRows + lane;
            if (row < si.n && !p.has_epi) {
#pragma unroll
                for (int m = 0; m < M; ++m) {
                    const int32_t s64 = (acc0[m][0] + acc1[m][0]) * 64 + (acc0[m][1] + acc1[m][1]) * 16 +
                                        (acc0[m][2] + acc1[m][2]) * 4 + (acc0[m][3] + acc1[m][3]);
                    const int32_t a = (s64 >> 6) - meta->sumx[u * M + m];
                    const float yv = __fmul_rn(__fmul_rn(float(a), meta->s_act[u * M + m]), si.scale);
                    si.y[size_t(m) * size_t(si.n) + row] = yv;
                    if (si.acc) si.acc[size_t(m) * size_t(si.n) + row] = a;
                }
            } else if (row < si.n) {
                // fused epilogue operands (technical report §2.4.1): bias and
                // ReLU, then the layer-scaled residual add; one rounding per step
                const GemvLinear &L = p.lin[si.lin];
                const float *res = L.res;
                const bool relu = L.relu != 0;
                const float bias = L.bias ? __ldg(L.bias + row) : 0.f;
                const float gamma = L.gamma ? __ldg(L.gamma + row) : 1.f;
                const bool has_bias = L.bias != nullptr, has_gamma = L.gamma != nullptr;
#pragma unroll
                for (int m = 0; m < M; ++m) {
                    const int32_t s64 = (acc0[m][0] + acc1[m][0]) * 64 + (acc0[m][1] + acc1[m][1]) * 16 +
                                        (acc0[m][2] + acc1[m][2]) * 4 + (acc0[m][3] + acc1[m][3]);
                    const int32_t a = (s64 >> 6) - meta->sumx[u * M + m];
                    float yv = __fmul_rn(__fmul_rn(float(a), meta->s_act[u * M + m]), si.scale);
                    if (has_bias) yv = __fadd_rn(yv, bias);
                    if (relu) yv = yv > 0.f ? yv : 0.f;
                    if (has_gamma) yv = __fmul_rn(gamma, yv);
                    const size_t o = size_t(m) * size_t(si.n) + row;
                    if (res) yv = __fadd_rn(res[o], yv);
                    si.y[o] = yv;
                    if (si.acc) si.acc[o] = a;
                }
            }
#pragma unroll
            for (int m = 0; m < M; ++m)
#pragma unroll
                for (int g = 0; g < 4; ++g) acc0[m][g] = acc1[m][g] = 0;
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
    stamp(4);

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

template <int M, int NW, int BOX>
static cudaError_t launch_one(const GemvParams &p, size_t smem, cudaStream_t st)
{
    static bool configured = false;   // per instantiation, set once
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(gemv_stack_kernel<M, NW, BOX>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    gemv_stack_kernel<M, NW, BOX><<<p.num_ranges, NW * 32, smem, st>>>(p);
    return cudaGetLastError();
}

template <int NW, int BOX, int MAXM>
static cudaError_t launch_variant(const GemvParams &p, size_t smem, cudaStream_t st)
{
    switch (p.m) {
    case 1: return launch_one<1, NW, BOX>(p, smem, st);
    case 2: if constexpr (MAXM >= 2) return launch_one<2, NW, BOX>(p, smem, st); break;
    case 3: if constexpr (MAXM >= 3) return launch_one<3, NW, BOX>(p, smem, st); break;
    case 4: if constexpr (MAXM >= 4) return launch_one<4, NW, BOX>(p, smem, st); break;
    case 5: if constexpr (MAXM >= 5) return launch_one<5, NW, BOX>(p, smem, st); break;
    case 6: if constexpr (MAXM >= 6) return launch_one<6, NW, BOX>(p, smem, st); break;
    case 7: if constexpr (MAXM >= 7) return launch_one<7, NW, BOX>(p, smem, st); break;
    case 8: if constexpr (MAXM >= 8) return launch_one<8, NW, BOX>(p, smem, st); break;
    default: break;
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_gemv(const GemvParams &p, int variant, cudaStream_t st)
{
    if (variant < 0 || variant >= kNumVariants || p.m > kVariantMaxM[variant]) return cudaErrorInvalidValue;
    const GemvVariant v = kVariants[variant];
    const size_t smem =
        size_t(kAlignPad) + size_t(ring_bytes(v.nw, v.boxes)) + size_t(p.x_bytes) + size_t(kMetaBytes);
    if (smem > size_t(kSmemLimit)) return cudaErrorInvalidValue;
    switch (variant) {
    case 0: return launch_variant<kVariants[0].nw, kVariants[0].boxes, kVariantMaxM[0]>(p, smem, st);
    case 1: return launch_variant<kVariants[1].nw, kVariants[1].boxes, kVariantMaxM[1]>(p, smem, st);
    case 2: return launch_variant<kVariants[2].nw, kVariants[2].boxes, kVariantMaxM[2]>(p, smem, st);
    case 3: return launch_variant<kVariants[3].nw, kVariants[3].boxes, kVariantMaxM[3]>(p, smem, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace bitnet
