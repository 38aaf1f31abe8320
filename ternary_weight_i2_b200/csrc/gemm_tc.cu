// gemm_tc.cu -- prefill path (M > 8 tokens): ternary x int8 GEMM on the
// 5th-generation tensor cores (tcgen05, kind::i8).
//
// What it computes ("VibeVoice-ASR-BitNet Technical Report", §2.2.2, §2.4.2,
// Figure 4; prefill in §3.2, Figure 6a): for int8 activations q [M, Kpad]
// (per-token quantised, scales s_act[M]) and packed ternary weights
// W [N, 32*KB],
//   acc[m,n] = sum_k q[m,k] * w[n,k]       (exact int32)
//   y[m,n]   = ((float)acc[m,n] * s_act[m]) * s_w
// The report's kernel unpacks the 2-bit weights to INT8 and feeds them to the
// same multiply-add as its INT8 path; here the unpacked INT8 tile feeds the
// tensor cores.
//
// One CTA per SM, persistent over 128 x 256 output tiles; per 128-element
// K block (one packed block per weight row):
//   warp 0      TMA: the activation tile (128 rows x 128 B, 128-byte swizzle,
//               the canonical K-major layout of the MMA) and the packed weight
//               tile (256 rows x 32 B) into a 6-stage shared-memory ring;
//   warps 3-6   expand the packed tile into the canonical K-major
//               128-byte-swizzled layout of operand B (two buffers), as the
//               unsigned codes w + 1 in {0, 1, 2}: one mask per 2-bit field;
//   warp 2      sums each activation row of the tile (sum_k q), so that the
//               epilogue can remove the +1 of the codes: acc = D - sum_k q;
//   warp 1      one thread issues 4 tcgen05.mma (M=128, N=256, K=32, signed A
//               x unsigned B) per block into a TMEM accumulator (two 256-column
//               accumulators, so the epilogue of one tile overlaps the next
//               tile's K loop) and commits to mbarriers;
//   warps 7-10  epilogue: tcgen05.ld the accumulator (one TMEM lane = one
//               output row per thread), subtract the row sum, dequantise in
//               fp32, store.
// Every wait is bounded; on expiry the CTA raises BITNET_FLAG_TIMEOUT, the
// other roles stop, in-flight copies and MMAs are drained (bounded) and TMEM
// is freed before exit.  No TMA multicast.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <vector>

#include "common.cuh"

namespace bitnet {

constexpr int kBM = 128, kBN = 256, kBK = 128;
constexpr int kStages = 5;                         // TMA ring (activations + packed weights)
constexpr int kBBufs = 2;                          // expanded weight tiles
constexpr int kAStage = kBM * kBK;                 // 16 KB int8 activations
constexpr int kBStage = kBN * kBK;                 // 32 KB expanded weight codes
constexpr int kPStage = kBN * 32;                  // 8 KB packed weights
constexpr int kStageOut = 32 * 128;                // one 32 x 32 fp32 output chunk (128-byte rows)
constexpr int kAOff = 0, kPOff = kStages * kAStage, kBOff = kPOff + kStages * kPStage;
constexpr int kOOff = kBOff + 2 * kBStage;         // 4 epilogue warps x 2 output staging buffers
constexpr int kGemmThreads = 352;                  // 11 warps
constexpr int kExpandWarp0 = 3, kExpandWarps = 4, kExpandThreads = 32 * kExpandWarps;
constexpr int kEpiWarp0 = 7, kEpiThreads = 128;
constexpr int kTmemCols = 2 * kBN;                 // two int32 accumulators
constexpr int kGemmSmem = 1024 + kOOff + 4 * 2 * kStageOut;

struct GemmProblem {
    CUtensorMap tmap_a;       // int8 q [M, Kpad]: dims {Kpad, M}, box {128, 128}, 128-byte swizzle
    CUtensorMap tmap_b;       // packed [N, 32*KB]: dims {32*KB, N}, box {32, 256}, no swizzle
    CUtensorMap tmap_y;       // fp32 y [M, N]: dims {N, M}, box {32, 32}, 128-byte swizzle (when tma_out)
    CUtensorMap tmap_acc;     // int32 acc [M, N], same shape (when tma_out and acc)
    const float *act_scale;   // [M]
    float *y;                 // [M, N]
    int32_t *acc;             // [M, N] or null
    float w_scale;
    int32_t m, n, kb;
    int32_t tiles_m, tiles_n;
    int32_t tma_out;          // outputs through TMA stores (N % 4 == 0), else direct stores
    int32_t tile0;            // first id of this problem's tiles in the launch's tile numbering
};

constexpr int kMaxGroup = 8;         // problems (layers) per launch
constexpr int kMaxGemmCtas = 160;
constexpr int kMaxGemmTiles = 3072;  // tiles per launch

struct GemmParams {
    GemmProblem prob[kMaxGroup];
    int32_t nprob;
    int32_t ntiles_total;
    int32_t *flags;
    uint64_t wait_limit;
    uint64_t *trace;          // optional: CTA 0 per-K-block globaltimer stamps (kGemmTraceBlocks x 8)
    int32_t cta_off[kMaxGemmCtas + 1];   // CTA c runs tiles[cta_off[c] .. cta_off[c+1])
    int32_t tiles[kMaxGemmTiles];        // tile ids, heaviest first within each CTA
};
static_assert(sizeof(GemmParams) <= 32760, "GEMM parameter block too large");

struct TileRef {
    int g, m_tile, n_tile;
};

__device__ __forceinline__ TileRef decode_tile(const GemmParams &p, int id)
{
    int g = 0;
    while (g + 1 < p.nprob && id >= p.prob[g + 1].tile0) ++g;
    const int local = id - p.prob[g].tile0;
    return TileRef{g, local % p.prob[g].tiles_m, local / p.prob[g].tiles_m};
}

// Trace of CTA 0 (profiling aid), per K block it < kGemmTraceBlocks:
// [it*8 + 0] producer issued, 1 MMA saw full, 2 MMA saw B ready, 3 MMA issued,
// 4 expander saw full, 5 expander saw B free, 6 expander done, 7 row sums done;
// then [kGemmTraceBlocks*8 + 0] kernel entry, +1 set-up done, +2 all roles
// done, +8+t epilogue of the CTA's tile t (t < 8) done.
constexpr int kGemmTraceBlocks = 64;

// ------------------------------------------------------------ tcgen05 PTX

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes, 8-row groups 1024 bytes apart (SBO); LBO unused for this layout.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr)
{
    uint64_t d = uint64_t((saddr >> 4) & 0x3FFFu);
    d |= uint64_t(1) << 16;              // leading byte offset (16-byte units)
    d |= uint64_t(1024 >> 4) << 32;      // stride byte offset (16-byte units)
    d |= uint64_t(1) << 46;              // descriptor version for sm_100
    d |= uint64_t(2) << 61;              // layout: 128-byte swizzle
    return d;
}

// Instruction descriptor: kind::i8, D int32, A signed int8, B unsigned int8,
// both K-major, M = 128, N = 256, dense.
constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (0u << 10) | (uint32_t(kBN >> 3) << 17) | (uint32_t(kBM >> 4) << 24);

__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// 2-D TMA store of a shared-memory box to global memory (bulk-group completion).
__device__ __forceinline__ void tma_store_2d(const void *tmap, uint32_t src, int32_t x, int32_t y)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(tmap), "r"(x),
                 "r"(y), "r"(src)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Codes w + 1 of field g of a packed word as unsigned bytes: elements
// 32g + b .. 32g + b + 3 of the block.
__device__ __forceinline__ uint32_t expand_field(uint32_t v, int g)
{
    return (v >> (2 * g)) & 0x03030303u;
}

// Wait on an mbarrier phase; false on timeout or when another role aborted.
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, uint64_t limit, volatile int *abort_flag)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = clock64();
    for (int spin = 0;; ++spin) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((spin & 63) == 0 && *abort_flag) return false;
        if (clock64() - t0 > limit) return false;
    }
}

__global__ void __launch_bounds__(kGemmThreads, 1) gemm_i2_kernel(const __grid_constant__ GemmParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
    __shared__ __align__(8) uint64_t bready_bar[kBBufs], bfree_bar[kBBufs];
    __shared__ __align__(8) uint64_t accf_bar[2], acce_bar[2], drain_bar;
    __shared__ int32_t rowsum[2][kBM];
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;
    volatile int *abort_flag = &abort_s;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint64_t limit = p.wait_limit;
    const int tbeg = p.cta_off[blockIdx.x], tend = p.cta_off[blockIdx.x + 1];
    const uint32_t sbase = smem_u32(smem);
    uint64_t *ctrace = (p.trace && blockIdx.x == 0) ? p.trace + kGemmTraceBlocks * 8 : nullptr;
    if (ctrace && tid == 0) ctrace[0] = globaltimer();

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&empty_bar[s]), 1 + kExpandWarps + 1);   // MMA, expanders, row sums
        }
        for (int b = 0; b < kBBufs; ++b) {
            mbar_init(smem_u32(&bready_bar[b]), kExpandThreads);
            mbar_init(smem_u32(&bfree_bar[b]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&accf_bar[b]), 2);                       // MMA, row sums
            mbar_init(smem_u32(&acce_bar[b]), kEpiThreads);
        }
        mbar_init(smem_u32(&drain_bar), 1);
        abort_s = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_s)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_s;
    if (ctrace && tid == 0) ctrace[1] = globaltimer();

    auto fail = [&]() {
        abort_s = 1;
        raise_flag(p.flags, BITNET_FLAG_TIMEOUT);
    };
    uint64_t *trace = (p.trace && blockIdx.x == 0) ? p.trace : nullptr;
    auto stamp = [&](int it, int ev) {
        if (trace && it < kGemmTraceBlocks) trace[it * 8 + ev] = globaltimer();
    };

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol_w = l2_evict_first_policy();
            int it = 0, last = -1;
            bool ok = true;
            for (int ti = tbeg; ti < tend && ok; ++ti) {
                const TileRef tr = decode_tile(p, p.tiles[ti]);
                const GemmProblem &P = p.prob[tr.g];
                const int m_tile = tr.m_tile, n_tile = tr.n_tile, kblocks = P.kb;
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const int s = it % kStages, r = it / kStages;
                    if (r > 0 && !wait_or_abort(smem_u32(&empty_bar[s]), (r - 1) & 1, limit, abort_flag)) {
                        fail();
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&full_bar[s]);
                    mbar_arrive_expect_tx(fb, kAStage + kPStage);
                    asm volatile(
                        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                        " [%0], [%1, {%2, %3}], [%4];" ::"r"(sbase + kAOff + s * kAStage),
                        "l"(&P.tmap_a), "r"(kb * kBK), "r"(m_tile * kBM), "r"(fb)
                        : "memory");
                    tma_load_2d(sbase + kPOff + s * kPStage, &P.tmap_b, kb * 32, n_tile * kBN, fb, pol_w);
                    stamp(it, 0);
                    last = it;
                }
            }
            if (!ok)   // let copies already issued land before the CTA can exit
                for (int j = (last >= kStages ? last - kStages + 1 : 0); j <= last; ++j)
                    mbar_wait(smem_u32(&full_bar[j % kStages]), (j / kStages) & 1, kDrainWaitLimit);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int it = 0, tcount = 0;
            bool ok = true, any = false;
            for (int ti = tbeg; ti < tend && ok; ++ti, ++tcount) {
                const int kblocks = p.prob[decode_tile(p, p.tiles[ti]).g].kb;
                const int b = tcount & 1, ur = tcount >> 1;
                if (ur > 0 && !wait_or_abort(smem_u32(&acce_bar[b]), (ur - 1) & 1, limit, abort_flag)) {
                    fail();
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + uint32_t(b * kBN);
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const int s = it % kStages, r = it / kStages;
                    const int bb = it % kBBufs, rb = it / kBBufs;
                    const bool f1 = wait_or_abort(smem_u32(&full_bar[s]), r & 1, limit, abort_flag);
                    stamp(it, 1);
                    if (!f1 || !wait_or_abort(smem_u32(&bready_bar[bb]), rb & 1, limit, abort_flag)) {
                        fail();
                        ok = false;
                        break;
                    }
                    stamp(it, 2);
                    tc_fence_after();
                    const uint32_t a0 = sbase + kAOff + s * kAStage;
                    const uint32_t b0 = sbase + kBOff + bb * kBStage;
#pragma unroll
                    for (int ks = 0; ks < kBK / 32; ++ks)
                        mma_i8(d_tmem, sw128_desc(a0 + ks * 32), sw128_desc(b0 + ks * 32),
                               (kb > 0 || ks > 0) ? 1u : 0u);
                    mma_commit(smem_u32(&empty_bar[s]));
                    mma_commit(smem_u32(&bfree_bar[bb]));
                    stamp(it, 3);
                    any = true;
                }
                if (ok) mma_commit(smem_u32(&accf_bar[b]));
            }
            if (any) {
                // all MMAs this thread issued are complete before TMEM is freed
                mma_commit(smem_u32(&drain_bar));
                mbar_wait(smem_u32(&drain_bar), 0, kDrainWaitLimit);
            }
        }
    } else if (warp == 2) {
        // -------------------------------------------- activation row sums
        // lane = (row group rg = lane/8, 16-byte chunk c = lane%8); rows 4i+rg
        const int c = lane & 7, rg = lane >> 3;
        int it = 0, tcount = 0;
        bool ok = true;
        for (int ti = tbeg; ti < tend && ok; ++ti, ++tcount) {
            const int kblocks = p.prob[decode_tile(p, p.tiles[ti]).g].kb;
            const int b = tcount & 1, ur = tcount >> 1;
            int32_t ps[kBM / 4];
#pragma unroll
            for (int i = 0; i < kBM / 4; ++i) ps[i] = 0;
            for (int kb = 0; kb < kblocks; ++kb, ++it) {
                const int s = it % kStages, r = it / kStages;
                const bool landed = wait_or_abort(smem_u32(&full_bar[s]), r & 1, limit, abort_flag);
                if (!__all_sync(0xffffffffu, landed)) {
                    if (lane == 0) fail();
                    ok = false;
                    break;
                }
                const uint32_t a0 = sbase + kAOff + s * kAStage;
#pragma unroll
                for (int i = 0; i < kBM / 4; ++i) {
                    const uint4 v = lds128(a0 + (4 * i + rg) * 128 + c * 16);
                    int32_t acc = ps[i];
                    asm("dp4a.s32.s32 %0, %1, %2, %0;" : "+r"(acc) : "r"(v.x), "r"(0x01010101));
                    asm("dp4a.s32.s32 %0, %1, %2, %0;" : "+r"(acc) : "r"(v.y), "r"(0x01010101));
                    asm("dp4a.s32.s32 %0, %1, %2, %0;" : "+r"(acc) : "r"(v.z), "r"(0x01010101));
                    asm("dp4a.s32.s32 %0, %1, %2, %0;" : "+r"(acc) : "r"(v.w), "r"(0x01010101));
                    ps[i] = acc;
                }
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(smem_u32(&empty_bar[s]));
                    stamp(it, 7);
                }
            }
            if (!ok) break;
            if (ur > 0) {
                const bool freed = wait_or_abort(smem_u32(&acce_bar[b]), (ur - 1) & 1, limit, abort_flag);
                if (!__all_sync(0xffffffffu, freed)) {
                    if (lane == 0) fail();
                    break;
                }
            }
#pragma unroll
            for (int i = 0; i < kBM / 4; ++i) {
                int32_t v = ps[i];
                v += __shfl_xor_sync(0xffffffffu, v, 1);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                v += __shfl_xor_sync(0xffffffffu, v, 4);
                if (c == 0) rowsum[b][4 * i + rg] = v;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&accf_bar[b]));
        }
    } else if (warp < kEpiWarp0) {
        // ------------------------------------------------------- expanders
        const int et = tid - 32 * kExpandWarp0;
        int it = 0;
        bool ok = true;
        for (int ti = tbeg; ti < tend && ok; ++ti) {
            const int kblocks = p.prob[decode_tile(p, p.tiles[ti]).g].kb;
            for (int kb = 0; kb < kblocks; ++kb, ++it) {
                const int s = it % kStages, r = it / kStages;
                const int bb = it % kBBufs, rb = it / kBBufs;
                bool go = wait_or_abort(smem_u32(&full_bar[s]), r & 1, limit, abort_flag);
                if (et == 0) stamp(it, 4);
                if (go && rb > 0) go = wait_or_abort(smem_u32(&bfree_bar[bb]), (rb - 1) & 1, limit, abort_flag);
                if (et == 0) stamp(it, 5);
                if (!__all_sync(0xffffffffu, go)) {
                    if (lane == 0) fail();
                    ok = false;
                    break;
                }
                const uint32_t bsm = sbase + kBOff + bb * kBStage;
                const uint32_t psm = sbase + kPOff + s * kPStage;
#pragma unroll
                for (int i = 0; i < (kBN * 2) / kExpandThreads; ++i) {
                    // task q: 8 consecutive rows with the same quad per quarter-warp
                    const int q = et + kExpandThreads * i;
                    const int quad = (q >> 3) & 1, row = (q & 7) + 8 * (q >> 4);
                    const uint4 v = lds128(psm + row * 32 + quad * 16);
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const uint32_t chunk = uint32_t(2 * g + quad) ^ uint32_t(row & 7);
                        const uint32_t dst = bsm + row * 128 + chunk * 16;
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst),
                                     "r"(expand_field(v.x, g)), "r"(expand_field(v.y, g)), "r"(expand_field(v.z, g)),
                                     "r"(expand_field(v.w, g))
                                     : "memory");
                    }
                }
                // generic-proxy writes -> visible to the tensor core (async proxy)
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_arrive(smem_u32(&bready_bar[bb]));
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&empty_bar[s]));   // packed tile consumed
                if (et == 0) stamp(it, 6);
            }
        }
    } else {
        // -------------------------------------------------------- epilogue
        const int sub = warp & 3;            // TMEM lanes 32*sub .. 32*sub+31
        const uint32_t stage0 = sbase + kOOff + uint32_t(sub) * 2 * kStageOut;
        int tcount = 0, chunk_no = 0;
        for (int ti = tbeg; ti < tend; ++ti, ++tcount) {
            const TileRef tr = decode_tile(p, p.tiles[ti]);
            const GemmProblem &P = p.prob[tr.g];
            const int m_tile = tr.m_tile, n_tile = tr.n_tile;
            const int b = tcount & 1, ur = tcount >> 1;
            const bool ready = wait_or_abort(smem_u32(&accf_bar[b]), ur & 1, limit, abort_flag);
            if (!__all_sync(0xffffffffu, ready)) {
                if (lane == 0) fail();
                break;
            }
            tc_fence_after();
            const int rloc = 32 * sub + lane;
            const int row = m_tile * kBM + rloc;
            const bool row_ok = row < P.m;
            const float sa = row_ok ? P.act_scale[row] : 0.f;
            const int32_t rs = rowsum[b][rloc];
            const uint32_t taddr = tmem_base + (uint32_t(32 * sub) << 16) + uint32_t(b * kBN);
#pragma unroll 1
            for (int c0 = 0; c0 < kBN; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(taddr + uint32_t(c0), v);
                const int col0 = n_tile * kBN + c0;
                if (col0 >= P.n) continue;
                if (P.tma_out) {
                    // stage the 32 x 32 chunk (row = lane) in the 128-byte swizzled
                    // layout and store it with one TMA store; tails are clipped by
                    // the tensor map
                    const uint32_t stg = stage0 + uint32_t(chunk_no & 1) * kStageOut;
                    if (lane == 0) bulk_wait_read<1>();   // the store that used this buffer has read it
                    __syncwarp();
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int32_t a0 = int32_t(v[4 * j + 0]) - rs, a1 = int32_t(v[4 * j + 1]) - rs;
                        const int32_t a2 = int32_t(v[4 * j + 2]) - rs, a3 = int32_t(v[4 * j + 3]) - rs;
                        const uint32_t dst = stg + uint32_t(lane) * 128 + (uint32_t(j ^ (lane & 7)) << 4);
                        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(dst),
                                     "f"(__fmul_rn(__fmul_rn(float(a0), sa), P.w_scale)),
                                     "f"(__fmul_rn(__fmul_rn(float(a1), sa), P.w_scale)),
                                     "f"(__fmul_rn(__fmul_rn(float(a2), sa), P.w_scale)),
                                     "f"(__fmul_rn(__fmul_rn(float(a3), sa), P.w_scale))
                                     : "memory");
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&P.tmap_y, stg, col0, m_tile * kBM + 32 * sub);
                        bulk_commit();
                    }
                    ++chunk_no;
                    if (P.acc) {
                        const uint32_t stg2 = stage0 + uint32_t(chunk_no & 1) * kStageOut;
                        if (lane == 0) bulk_wait_read<1>();
                        __syncwarp();
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const uint32_t dst = stg2 + uint32_t(lane) * 128 + (uint32_t(j ^ (lane & 7)) << 4);
                            asm volatile("st.shared.v4.s32 [%0], {%1, %2, %3, %4};" ::"r"(dst),
                                         "r"(int32_t(v[4 * j + 0]) - rs), "r"(int32_t(v[4 * j + 1]) - rs),
                                         "r"(int32_t(v[4 * j + 2]) - rs), "r"(int32_t(v[4 * j + 3]) - rs)
                                         : "memory");
                        }
                        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&P.tmap_acc, stg2, col0, m_tile * kBM + 32 * sub);
                            bulk_commit();
                        }
                        ++chunk_no;
                    }
                } else {
                    if (!row_ok) continue;
                    float *yr = P.y + size_t(row) * size_t(P.n) + col0;
                    int32_t *ar = P.acc ? P.acc + size_t(row) * size_t(P.n) + col0 : nullptr;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (col0 + j < P.n) {
                            const int32_t a = int32_t(v[j]) - rs;
                            yr[j] = __fmul_rn(__fmul_rn(float(a), sa), P.w_scale);
                            if (ar) ar[j] = a;
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&acce_bar[b]));
            if (ctrace && tid == 32 * kEpiWarp0 && tcount < 8) ctrace[8 + tcount] = globaltimer();
        }
        if (lane == 0) bulk_wait_all();   // every output store has completed
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (ctrace && tid == 0) ctrace[2] = globaltimer();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                     : "memory");
}

// ------------------------------------------------------------------ host

static PFN_cuTensorMapEncodeTiled_v12000 gemm_encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    return fn;
}

bool gemm_available() { return true; }

// One or more grouped launches over `count` (<= kMaxGroup) problems sharing
// the token count m.  Tiles are dealt heaviest-first to the least-loaded CTA
// (cost = K blocks + a fixed epilogue share), so layers of different K
// balance inside one persistent launch.
cudaError_t launch_gemm_grouped(const int8_t *const *xq, const float *const *act_scale, int64_t m,
                                const bitnet_tw *w, int count, float *const *y, int32_t *const *acc,
                                int32_t *flags, uint64_t wait_limit, int sm_count, uint64_t *trace, cudaStream_t st)
{
    if (count < 1 || count > kMaxGroup) return cudaErrorInvalidValue;
    auto enc = gemm_encode_fn();
    if (!enc) return cudaErrorNotSupported;
    static thread_local GemmParams p;   // staging; copied into each launch
    struct Tile {
        int id, cost;
    };
    static thread_local std::vector<Tile> all;
    all.clear();
    int tile0 = 0;
    for (int g = 0; g < count; ++g) {
        GemmProblem &P = p.prob[g];
        const int64_t kb = (w[g].k + 127) / 128;
        const cuuint32_t es[2] = {1u, 1u};
        {
            const cuuint64_t dims[2] = {cuuint64_t(128 * kb), cuuint64_t(m)};
            const cuuint64_t strides[1] = {cuuint64_t(128 * kb)};
            const cuuint32_t box[2] = {uint32_t(kBK), uint32_t(kBM)};
            if (enc(&P.tmap_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(xq[g]), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
        }
        {
            const cuuint64_t dims[2] = {cuuint64_t(32 * kb), cuuint64_t(w[g].n)};
            const cuuint64_t strides[1] = {cuuint64_t(32 * kb)};
            const cuuint32_t box[2] = {32u, uint32_t(kBN)};
            if (enc(&P.tmap_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(w[g].packed), dims, strides, box,
                    es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
        }
        P.tma_out = (w[g].n % 4 == 0) ? 1 : 0;
        int32_t *accg = acc ? acc[g] : nullptr;
        if (P.tma_out) {
            const cuuint64_t dims[2] = {cuuint64_t(w[g].n), cuuint64_t(m)};
            const cuuint64_t strides[1] = {cuuint64_t(w[g].n) * 4};
            const cuuint32_t box[2] = {32u, 32u};
            if (enc(&P.tmap_y, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, y[g], dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
            if (accg && enc(&P.tmap_acc, CU_TENSOR_MAP_DATA_TYPE_INT32, 2, accg, dims, strides, box, es,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
        }
        P.act_scale = act_scale[g];
        P.y = y[g];
        P.acc = accg;
        P.w_scale = w[g].scale;
        P.m = int32_t(m);
        P.n = int32_t(w[g].n);
        P.kb = int32_t(kb);
        P.tiles_m = int32_t((m + kBM - 1) / kBM);
        P.tiles_n = int32_t((w[g].n + kBN - 1) / kBN);
        P.tile0 = tile0;
        const int nt = P.tiles_m * P.tiles_n;
        for (int i = 0; i < nt; ++i) all.push_back(Tile{tile0 + i, int(kb) + 3});
        tile0 += nt;
    }
    p.nprob = count;
    p.ntiles_total = tile0;
    p.flags = flags;
    p.wait_limit = wait_limit;
    p.trace = trace;
    std::stable_sort(all.begin(), all.end(), [](const Tile &a, const Tile &b) { return a.cost > b.cost; });
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(gemm_i2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    static thread_local std::vector<int> owner, fill;
    for (size_t c0 = 0; c0 < all.size(); c0 += kMaxGemmTiles) {
        const int n = int(std::min<size_t>(kMaxGemmTiles, all.size() - c0));
        const int G = std::min(std::min(sm_count, kMaxGemmCtas), n);
        // least-loaded CTA first (loads are small integers: linear scan)
        static thread_local std::vector<long long> load;
        load.assign(G, 0);
        owner.assign(n, 0);
        std::vector<int> count_of(G, 0);
        for (int i = 0; i < n; ++i) {
            int best = 0;
            for (int c = 1; c < G; ++c)
                if (load[c] < load[best]) best = c;
            load[best] += all[c0 + i].cost;
            owner[i] = best;
            ++count_of[best];
        }
        p.cta_off[0] = 0;
        for (int c = 0; c < G; ++c) p.cta_off[c + 1] = p.cta_off[c] + count_of[c];
        fill.assign(G, 0);
        for (int i = 0; i < n; ++i) {
            const int c = owner[i];
            p.tiles[p.cta_off[c] + fill[c]++] = all[c0 + i].id;
        }
        gemm_i2_kernel<<<G, kGemmThreads, kGemmSmem, st>>>(p);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_gemm(const int8_t *xq, const float *act_scale, int64_t m, const bitnet_tw *w, float *y,
                        int32_t *acc, int32_t *flags, uint64_t wait_limit, int sm_count, uint64_t *trace,
                        cudaStream_t st)
{
    const int8_t *xqa[1] = {xq};
    const float *sa[1] = {act_scale};
    float *ya[1] = {y};
    int32_t *aa[1] = {acc};
    return launch_gemm_grouped(xqa, sa, m, w, 1, ya, acc ? aa : nullptr, flags, wait_limit, sm_count, trace, st);
}

}  // namespace bitnet
