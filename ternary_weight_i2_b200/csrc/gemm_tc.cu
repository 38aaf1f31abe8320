// gemm_tc.cu -- prefill path (M > 8 tokens): ternary x int8 GEMM on the
// 5th-generation tensor cores (tcgen05, kind::i8), two SMs per MMA.
//
// What it computes ("VibeVoice-ASR-BitNet Technical Report", §2.2.2, §2.4.2,
// Figure 4; prefill in §3.2, Figure 6a): for int8 activations q [M, Kpad]
// (per-token quantised, scales s_act[M]) and packed ternary weights
// W [N, 32*KB],
//   acc[m,n] = sum_k q[m,k] * w[n,k]       (exact int32)
//   y[m,n]   = ((float)acc[m,n] * s_act[m]) * s_w
// The report's kernel unpacks the 2-bit weights to INT8 and feeds them to the
// same multiply-add as its INT8 path; here the unpacked INT8 weights feed the
// tensor cores.
//
// Operand roles.  The weights are the MMA's A operand and live in tensor
// memory (TMEM); the activations are B and come from shared memory, so the
// accumulator is D[n, m] = sum_k w[n,k] q[m,k]: one TMEM lane per output
// feature, one column per token.  Expanded weights never touch shared memory.
//
// Two SMs per MMA.  A cluster of two CTAs computes tiles of 256 features x up
// to 192 tokens with tcgen05.mma.cta_group::2 (M = 256): each CTA holds 128
// weight rows in its own TMEM and half of the tile's tokens in its own
// shared memory, and its TMEM receives its 128 rows of D.  Per K block an SM
// thus loads 96 activation rows + 128 packed weight rows (16 KB) for the
// work of 128 x 192 x 128 MACs: half the activation traffic of one SM doing
// the same tile alone, and room for a 12-stage copy ring.
//
// Roles per CTA (16 warps), per 128-element K block:
//   warps 0, 3     TMA producers: this CTA's 96 x 128 B activation half
//                  (128-byte swizzle, the canonical K-major layout of B) and
//                  its 128 x 32 B packed weight rows, into a 12-stage ring;
//   warps 4-11     expanders, one thread per weight row: the row's 32 packed
//                  bytes become 128 signed int8 weights (logic ops and one
//                  add per 4 weights) written to one of 4 TMEM A buffers with
//                  one tcgen05.st; two groups of four warps take alternate K
//                  blocks;
//   warps 12-15    epilogue: tcgen05.ld 32 tokens of a feature per thread,
//                  dequantise in fp32, store (a warp writes 32 consecutive
//                  features of one token per store);
//   warp 1         (first CTA of the pair) issues the four tcgen05.mma of each
//                  K block for both SMs and commits to the barriers of both
//                  CTAs at once (multicast commit);
//   warp 2         (first CTA) relay: turns the second CTA's remote mbarrier
//                  signals into named-barrier arrivals for the MMA warp.
// The MMA warp waits only on hardware named barriers (an mbarrier poll in
// the issuing warp idles the tensor core for over a hundred cycles per K
// block); every other wait is bounded, and every role arrives exactly once
// per barrier phase, also after a timeout, so the MMA warp always completes.
// No TMA multicast: each CTA loads only into its own shared memory.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <vector>

#include "common.cuh"

namespace bitnet {

constexpr int kBF = 128;                           // weight rows per CTA (TMEM lanes); 256 per pair
constexpr int kPairF = 2 * kBF;                    // features per tile: MMA M
constexpr int kBT = 192;                           // tokens per tile: MMA N (at most)
constexpr int kHalfT = kBT / 2;                    // activation rows per CTA
constexpr int kBK = 128;                           // K per block: one packed block per row
constexpr int kStages = 12;                        // TMA ring (activation half + packed weights)
constexpr int kABufs = 4;                          // expanded weight tiles in TMEM
constexpr int kActStage = kHalfT * kBK;            // 12 KB int8 activations
constexpr int kPStage = kBF * 32;                  // 4 KB packed weights
constexpr int kActOff = 0, kPOff = kStages * kActStage;
constexpr int kGemmSmem = 1024 + kPOff + kStages * kPStage;
constexpr int kGemmThreads = 512;                  // 16 warps
constexpr int kProducers = 2;                      // TMA-issuing warps: 0, 3
constexpr int kExpandWarp0 = 4, kExpandGroupWarps = 4, kExpandGroups = 2;
constexpr int kEpiWarp0 = 12, kEpiWarps = 4;
constexpr int kACol0 = 2 * kBT;                    // TMEM columns of the A buffers
constexpr int kTmemCols = 512;
static_assert(kACol0 + 32 * kABufs <= kTmemCols, "TMEM budget");
static_assert(kGemmSmem <= 232448, "shared-memory budget");
static_assert(kActStage % 1024 == 0, "128-byte-swizzled stages need 1024-byte alignment");
static_assert(kEpiWarp0 % 4 == 0 && kExpandWarp0 % 4 == 0, "TMEM lane quadrant = warp % 4");

struct GemmProblem {
    CUtensorMap tmap_q;       // int8 q [M, Kpad]: dims {Kpad, M}, box {128, 96}, 128-byte swizzle
    CUtensorMap tmap_w;       // packed [N, 32*KB]: dims {32*KB, N}, box {32, 128}, no swizzle
    const float *act_scale;   // [M]
    float *y;                 // [M, N]
    int32_t *acc;             // [M, N] or null
    float w_scale;
    int32_t m, n, kb;
    int32_t tiles_t, tiles_f;
    int32_t tile0;            // first id of this problem's tiles in the launch's tile numbering
};

constexpr int kMaxGroup = 8;         // problems (layers) per launch
constexpr int kMaxGemmPairs = 80;
constexpr int kMaxGemmTiles = 7168;  // tiles per launch

struct GemmParams {
    GemmProblem prob[kMaxGroup];
    int32_t nprob;
    int32_t ntiles_total;
    int32_t *flags;
    uint64_t wait_limit;
    int32_t force_stall;      // test aid: K block kStallBlock's copies are never issued
    uint64_t *trace;          // optional: the first pair's stamps (2 * kGemmTraceStride entries)
    int32_t pair_off[kMaxGemmPairs + 1];   // pair c runs tiles[pair_off[c] .. pair_off[c+1])
    int32_t tiles[kMaxGemmTiles];          // tile ids, heaviest first within each pair
};
static_assert(sizeof(GemmParams) <= 32760, "GEMM parameter block too large");

struct TileRef {
    int g, f_tile, t_tile;
};

__device__ __forceinline__ TileRef decode_tile(const GemmParams &p, int id)
{
    int g = 0;
    while (g + 1 < p.nprob && id >= p.prob[g + 1].tile0) ++g;
    const int local = id - p.prob[g].tile0;
    return TileRef{g, local / p.prob[g].tiles_t, local % p.prob[g].tiles_t};
}

// Trace of the first pair's two CTAs, CTA r at [r * kGemmTraceStride + ...]
// (profiling aid; a stamp right after a named barrier may be taken before the
// barrier has completed): SM clock stamps per K block it <
// kGemmTraceBlocks at [it*16 + e]: 0 producer issued, 1 relay saw the second
// CTA's A half written, 2 MMA warp passed the A barrier, 3 MMAs issued, 4+q / 8+q / 12+q expander warp of lane quadrant q
// saw full / saw its A buffer free / wrote it; then at kGemmTraceMisc + 0
// kernel entry, +1 set-up done, +2 all roles done, +3 / +4 globaltimer at
// entry / end, +8+t epilogue of tile t done, +24+t MMA warp passed tile t's
// accumulator barrier (t < 16), +40+16t+2c (+1) epilogue warp 0 loaded
// (stored) chunk c of tile t (t < 2).
constexpr int kGemmTraceBlocks = 48, kGemmTraceEv = 16;
constexpr int kGemmTraceMisc = kGemmTraceBlocks * kGemmTraceEv;
constexpr int kGemmTraceStride = 1024;             // entries per traced CTA (CTAs 0 and 1)

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

// Instruction descriptor: kind::i8, D int32, A and B signed int8, both
// K-major, M = 256 (two SMs), N = n (a multiple of 16, at most 256), dense.
__device__ __forceinline__ uint32_t idesc_i8(int n)
{
    return (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(kPairF >> 4) << 24);
}

// One K block for both SMs of the pair, issued by one thread of the first
// CTA: four MMAs (K = 32 each) into d_tmem -- the activation descriptor of K
// step ks is qdesc + 2*ks (32 bytes further, in 16-byte units; the
// start-address field cannot carry out for shared-memory addresses) -- then
// commits, to the barriers at the same offsets in both CTAs, that free the
// activation stage and the A buffer.
__device__ __forceinline__ void mma_kblock(uint32_t d_tmem, uint32_t a_tmem, uint64_t qdesc, uint32_t idesc,
                                           uint32_t accumulate, uint32_t bar_stage, uint32_t bar_abuf)
{
    asm volatile(
        "{\n\t.reg .pred p0, p1;\n\t"
        "setp.ne.b32 p0, %4, 0;\n\t"
        "setp.eq.u32 p1, %4, %4;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], [%1], %2, %3, p0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], [%6], %7, %3, p1;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], [%8], %9, %3, p1;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], [%10], %11, %3, p1;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%5], %13;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%12], %13;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(qdesc), "r"(idesc), "r"(accumulate), "r"(bar_stage), "r"(a_tmem + 8u),
          "l"(qdesc + 2u), "r"(a_tmem + 16u), "l"(qdesc + 4u), "r"(a_tmem + 24u), "l"(qdesc + 6u), "r"(bar_abuf),
          "h"(uint16_t(3))
        : "memory");
}

// Commit to the barrier at this offset in both CTAs of the pair.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
        "h"(uint16_t(3))
        : "memory");
}

// Commit to this CTA's barrier only.
__device__ __forceinline__ void mma_commit_local(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// Named (hardware) barriers of the first CTA between the MMA warp and the
// warps that feed or drain TMEM: ids 1..4 "A buffer a written in both CTAs"
// (the CTA's expander group of four warps + the relay warp + the MMA warp),
// ids 5..6 "accumulator b drained in both CTAs" (four epilogue warps + relay
// + MMA warp).  The MMA warp waits (bar.sync); the others arrive
// (bar.arrive, release), exactly once per phase.
constexpr uint32_t kNbAbuf0 = 1, kNbAcc0 = 5, kNbThreads = 192;
static_assert(kNbThreads == 32 * (kExpandGroupWarps + 2) && kNbThreads == 32 * (kEpiWarps + 2), "barrier sizes");
__device__ __forceinline__ void nb_arrive(uint32_t id)
{
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(kNbThreads) : "memory");
}
__device__ __forceinline__ void nb_sync(uint32_t id)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(kNbThreads) : "memory");
}

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// All threads of both CTAs (release / acquire at cluster scope).
__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on the barrier at this offset in CTA `rank`.  Relaxed: what it
// signals is the completion of this thread's TMEM accesses (tcgen05.wait::st
// / wait::ld, then tcgen05.fence::before_thread_sync, precede it); a release
// would also wait for every earlier global store of the thread (the
// epilogue's outputs), which the MMA warp does not need.
__device__ __forceinline__ void remote_arrive(uint32_t bar, uint32_t rank)
{
    asm volatile(
        "{\n\t.reg .b32 ra;\n\t"
        "mapa.shared::cluster.u32 ra, %0, %1;\n\t"
        "mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [ra];\n\t}" ::"r"(bar),
        "r"(rank)
        : "memory");
}

// SM clock read ordered with the surrounding volatile asm (barriers, MMAs),
// for the trace.
__device__ __forceinline__ uint64_t clock_ordered()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%clock64;" : "=l"(t)::"memory");
    return t;
}

// K block whose copies a test stalls (force_stall)
constexpr int kStallBlock = 2;

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

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
        ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
          "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
          "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]),
          "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Signed int8 weights w = code - 1 of field g of a packed word: elements
// 32g + b .. 32g + b + 3 of the block.  Bit 7 is set in every byte before
// the subtraction so that no byte borrows from its neighbour; the xor then
// clears it again: codes 0, 1, 2 -> 0xFF, 0x00, 0x01.
__device__ __forceinline__ uint32_t expand_signed(uint32_t v, int g)
{
    const uint32_t c = ((v >> (2 * g)) & 0x03030303u) | 0x80808080u;
    return (c - 0x01010101u) ^ 0x80808080u;
}

// Suspend-time hint of every wait: a waiting thread that polls without one
// takes issue slots from the warps that work (the expanders above all), and
// one suspended for long is not reliably woken at once by arrivals from the
// other SM or from the asynchronous units -- a short hint bounds both.
constexpr uint32_t kSleepNs = 100;

// Wait on an mbarrier phase; false on timeout or when another role aborted.
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, uint64_t limit, volatile int *abort_flag)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = clock64();
    for (int spin = 0;; ++spin) {
        if (mbar_try_wait_sleep(bar, parity, kSleepNs)) return true;
        if ((spin & 15) == 0 && *abort_flag) return false;
        if (clock64() - t0 > limit) return false;
    }
}

// Cluster-scope acquire poll with the short suspend-time hint (the phases
// it waits for may be completed by the other CTA's remote arrivals).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kSleepNs)
        : "memory");
    return ok != 0;
}

// Warp-wide wait: lane 0 polls, the others take its result (and, through
// __syncwarp, the ordering its successful wait established).
__device__ __forceinline__ bool warp_wait_or_abort(uint32_t bar, uint32_t parity, uint64_t limit,
                                                   volatile int *abort_flag)
{
    bool ok = false;
    if ((threadIdx.x & 31) == 0) ok = wait_or_abort(bar, parity, limit, abort_flag);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    return ok;
}

// Warp-wide wait for a phase that is bound to complete: one the MMA warp's
// commits complete (it never stops) -- `cluster` false -- or one the other
// CTA's roles complete with remote arrivals (they arrive once per phase
// whatever happens) -- `cluster` true, cluster-scope acquire.  No abort
// check, only the long limit.
__device__ __forceinline__ bool warp_wait_progress(uint32_t bar, uint32_t parity, uint64_t long_limit,
                                                   bool cluster = false)
{
    bool ok = false;
    if ((threadIdx.x & 31) == 0) {
        const uint64_t t0 = clock64();
        while (!(ok = cluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait_sleep(bar, parity, kSleepNs)) &&
               clock64() - t0 <= long_limit) {
        }
    }
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    return ok;
}

// Tokens of tile t_tile.
__device__ __forceinline__ int tile_tokens(const GemmProblem &P, int t_tile)
{
    return min(kBT, P.m - t_tile * kBT);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_i2_kernel(const __grid_constant__ GemmParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
    __shared__ __align__(8) uint64_t aempty_bar[kABufs], accf_bar[2], drain_bar;
    __shared__ __align__(8) uint64_t peer_ready_bar[kABufs], peer_drained_bar[2];   // first CTA only
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;
    volatile int *abort_flag = &abort_s;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_rank();              // 0: issues the MMAs; 1: its peer
    const bool leader = rank == 0;
    const uint64_t limit = p.wait_limit;
    // limit of the waits that are bound to end (see warp_wait_progress): far
    // above the time one failed copy wait can hold the pipeline up
    const uint64_t long_limit = (limit > (kDrainWaitLimit >> 2)) ? (limit << 2) : kDrainWaitLimit;
    const int pair = blockIdx.x >> 1;
    const int tbeg = p.pair_off[pair], tend = p.pair_off[pair + 1];
    const uint32_t sbase = smem_u32(smem);
    // trace: the first pair, each CTA in its own kGemmTraceStride block
    uint64_t *const tbase = (p.trace && blockIdx.x < 2) ? p.trace + blockIdx.x * kGemmTraceStride : nullptr;
    uint64_t *ctrace = tbase ? tbase + kGemmTraceMisc : nullptr;
    if (ctrace && tid == 0) {
        ctrace[0] = clock_ordered();
        ctrace[3] = globaltimer();
    }

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&empty_bar[s]), 1 + kExpandGroupWarps);   // MMA commit, expander warps
        }
        for (int a = 0; a < kABufs; ++a) {
            mbar_init(smem_u32(&aempty_bar[a]), 1);
            mbar_init(smem_u32(&peer_ready_bar[a]), kExpandGroupWarps);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&accf_bar[b]), 1);
            mbar_init(smem_u32(&peer_drained_bar[b]), kEpiWarps);
        }
        mbar_init(smem_u32(&drain_bar), 1);
        abort_s = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_s)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    // both CTAs' barriers are initialised (and TMEM allocated) before either
    // CTA touches the other's
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_s;
    if (ctrace && tid == 0) ctrace[1] = clock_ordered();

    auto fail = [&]() {
        abort_s = 1;
        raise_flag(p.flags, BITNET_FLAG_TIMEOUT);
    };
    uint64_t *trace = tbase;
    auto stamp = [&](int it, int ev) {
        if (trace && it < kGemmTraceBlocks) trace[it * kGemmTraceEv + ev] = clock_ordered();
    };

    if (warp == 0 || warp == 3) {
        // ----------------------------------------------------- TMA producers
        // The whole warp runs the loop and lane 0 issues the copies (a lone
        // diverged lane is starved by busy warps of its sub-partition).
        const int pidx = (warp == 0) ? 0 : 1;
        int it = 0, last = -1;
        bool ok = true;
        for (int ti = tbeg; ti < tend && ok; ++ti) {
            const TileRef tr = decode_tile(p, p.tiles[ti]);
            const GemmProblem &P = p.prob[tr.g];
            const int kblocks = P.kb;
            // this CTA's token half of the tile: the MMA's B rows [0, n/2) come
            // from the first CTA, [n/2, n) from the second.  Box origins stay
            // inside the tensors (a short last tile or a ragged feature count
            // would otherwise start a box past the end); rows read in place of
            // the missing ones only reach outputs that are never stored.
            const int half = ((tile_tokens(P, tr.t_tile) + 15) & ~15) >> 1;
            const int t_row = min(tr.t_tile * kBT + int(rank) * half, P.m - 1);
            const int f_row = min(tr.f_tile * kPairF + int(rank) * kBF, P.n - 1);
            for (int kb = 0; kb < kblocks; ++kb, ++it) {
                if (it % kProducers != pidx) continue;
                const int s = it % kStages, r = it / kStages;
                if (r > 0 && !warp_wait_or_abort(smem_u32(&empty_bar[s]), (r - 1) & 1, limit, abort_flag)) {
                    if (lane == 0) fail();
                    ok = false;
                    break;
                }
                if (p.force_stall && it == kStallBlock) continue;   // test aid: this block's copies never come
                if (lane == 0) {
                    const uint32_t fb = smem_u32(&full_bar[s]);
                    mbar_arrive_expect_tx(fb, kActStage + kPStage);
                    asm volatile(
                        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                        " [%0], [%1, {%2, %3}], [%4];" ::"r"(sbase + kActOff + s * kActStage),
                        "l"(&P.tmap_q), "r"(kb * kBK), "r"(t_row), "r"(fb)
                        : "memory");
                    asm volatile(
                        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                        " [%0], [%1, {%2, %3}], [%4];" ::"r"(sbase + kPOff + s * kPStage),
                        "l"(&P.tmap_w), "r"(kb * 32), "r"(f_row), "r"(fb)
                        : "memory");
                    stamp(it, 0);
                }
                __syncwarp();
                last = it;
            }
        }
        if (!ok && lane == 0)   // let copies already issued land before the CTA can exit
            for (int j = (last >= kStages ? last - kStages + 1 : 0); j <= last; ++j)
                if (j % kProducers == pidx && !(p.force_stall && j == kStallBlock))
                    mbar_wait(smem_u32(&full_bar[j % kStages]), (j / kStages) & 1, kDrainWaitLimit);
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        // First CTA only.  Waits only on named barriers, never gives up,
        // always commits: every other role's waits on its commits therefore
        // end.  The expanders (and, through the relay, the second CTA's)
        // arrive for a K block only after they saw its stage's TMA
        // transaction complete, so the barrier covers both operands.
        if (leader) {
            const uint64_t qdesc0 = sw128_desc(sbase + kActOff);          // stage 0; + s * (kActStage >> 4)
            const uint32_t a_tm0 = tmem_base + uint32_t(kACol0);          // A buffer 0; + 32 * a
            const uint32_t empty0 = smem_u32(&empty_bar[0]), aempty0 = smem_u32(&aempty_bar[0]);
            int it = 0, tcount = 0, s = 0, a = 0;
            for (int ti = tbeg; ti < tend; ++ti, ++tcount) {
                const TileRef tr = decode_tile(p, p.tiles[ti]);
                const GemmProblem &P = p.prob[tr.g];
                const int kblocks = P.kb;
                const uint32_t idesc = idesc_i8((tile_tokens(P, tr.t_tile) + 15) & ~15);
                const int b = tcount & 1;
                if (tcount >= 2) nb_sync(kNbAcc0 + uint32_t(b));   // both epilogues drained tile tcount-2
                if (ctrace && lane == 0 && tcount < 16) ctrace[24 + tcount] = clock_ordered();
                const uint32_t d_tmem = tmem_base + uint32_t(b * kBT);
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    nb_sync(kNbAbuf0 + uint32_t(a));                   // both CTAs' A buffer a hold K block it
                    if (lane == 0) stamp(it, 2);
                    tc_fence_after();
                    if (lane == 0)
                        mma_kblock(d_tmem, a_tm0 + 32u * uint32_t(a), qdesc0 + uint64_t(s) * (kActStage >> 4),
                                   idesc, kb > 0 ? 1u : 0u, empty0 + 8u * uint32_t(s), aempty0 + 8u * uint32_t(a));
                    __syncwarp();
                    if (lane == 0) stamp(it, 3);
                    s = (s + 1 == kStages) ? 0 : s + 1;
                    a = (a + 1) & (kABufs - 1);
                }
                if (lane == 0) mma_commit_pair(smem_u32(&accf_bar[b]));
                __syncwarp();
            }
            // the epilogues' arrivals for the last two tiles
            for (int t = (tcount > 2 ? tcount - 2 : 0); t < tcount; ++t) nb_sync(kNbAcc0 + uint32_t(t & 1));
            if (tcount > 0 && lane == 0) {
                // all MMAs are complete (and their commits delivered) before
                // either CTA frees TMEM or exits
                mma_commit_local(smem_u32(&drain_bar));
                mbar_wait(smem_u32(&drain_bar), 0, kDrainWaitLimit);
            }
            __syncwarp();
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ relay
        // First CTA only: walks the MMA warp's sequence of named-barrier
        // phases and, for each, waits for the second CTA's matching remote
        // arrivals (its expanders for an A buffer, its epilogue for an
        // accumulator), then arrives.  Those arrivals come once per phase
        // whatever happens, so these waits end; after the long limit (a bug)
        // it raises the flag and arrives anyway.
        if (leader) {
            int it = 0, tcount = 0;
            for (int ti = tbeg; ti < tend; ++ti, ++tcount) {
                const int kblocks = p.prob[decode_tile(p, p.tiles[ti]).g].kb;
                const int b = tcount & 1;
                if (tcount >= 2) {
                    if (!warp_wait_progress(smem_u32(&peer_drained_bar[b]), ((tcount - 2) >> 1) & 1, long_limit,
                                            true) &&
                        lane == 0)
                        fail();
                    nb_arrive(kNbAcc0 + uint32_t(b));
                }
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const int a = it % kABufs;
                    if (!warp_wait_progress(smem_u32(&peer_ready_bar[a]), (it / kABufs) & 1, long_limit, true) &&
                        lane == 0)
                        fail();
                    if (lane == 0) stamp(it, 1);
                    nb_arrive(kNbAbuf0 + uint32_t(a));
                }
            }
            for (int t = (tcount > 2 ? tcount - 2 : 0); t < tcount; ++t) {
                if (!warp_wait_progress(smem_u32(&peer_drained_bar[t & 1]), (t >> 1) & 1, long_limit, true) &&
                    lane == 0)
                    fail();
                nb_arrive(kNbAcc0 + uint32_t(t & 1));
            }
        }
    } else if (warp < kEpiWarp0) {
        // ------------------------------------------------------- expanders
        // Every K block of the group ends with one arrival for its A buffer,
        // in order, also after a failed wait (the work is then skipped): in
        // the first CTA at the named barrier, in the second on the first
        // CTA's peer_ready barrier (relayed).  Before writing a buffer again
        // the group waits for the MMA warp's commit of its previous use, so
        // it never arrives twice in one phase.
        const int grp = (warp - kExpandWarp0) / kExpandGroupWarps;
        const int quad = warp & 3;                       // TMEM lanes 32*quad .. 32*quad+31
        const int row = 32 * quad + lane;                // weight row of this CTA's half
        const uint32_t lane_addr = uint32_t(32 * quad) << 16;
        int it = 0;
        bool aborted = false;
        for (int ti = tbeg; ti < tend; ++ti) {
            const int kblocks = p.prob[decode_tile(p, p.tiles[ti]).g].kb;
            for (int kb = 0; kb < kblocks; ++kb, ++it) {
                if ((it % kExpandGroups) != grp) continue;
                const int s = it % kStages, a = it % kABufs, ra = it / kABufs;
                if (!aborted) {
                    const bool landed =
                        warp_wait_or_abort(smem_u32(&full_bar[s]), (it / kStages) & 1, limit, abort_flag);
                    if (lane == 0) stamp(it, 4 + quad);
                    if (!landed) {
                        if (lane == 0) fail();
                        aborted = true;
                    }
                }
                uint32_t wv[32];
                if (!aborted) {
                    const uint32_t psm = sbase + kPOff + s * kPStage + uint32_t(row) * 32;
                    const uint4 lo = lds128(psm), hi = lds128(psm + 16);
                    const uint32_t pw[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
                    for (int g = 0; g < 4; ++g)
#pragma unroll
                        for (int j = 0; j < 8; ++j) wv[8 * g + j] = expand_signed(pw[j], g);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&empty_bar[s]));   // packed tile read (or given up)
                if (ra > 0 && !warp_wait_progress(smem_u32(&aempty_bar[a]), (ra - 1) & 1, long_limit)) {
                    if (lane == 0) fail();
                    aborted = true;
                }
                if (lane == 0) stamp(it, 8 + quad);
                if (!aborted) {
                    tc_fence_after();
                    tmem_st32(tmem_base + lane_addr + uint32_t(kACol0 + 32 * a), wv);
                }
                tc_fence_before();
                __syncwarp();
                if (leader) {
                    nb_arrive(kNbAbuf0 + uint32_t(a));
                } else if (lane == 0) {
                    remote_arrive(smem_u32(&peer_ready_bar[a]), 0);
                }
                if (lane == 0) stamp(it, 12 + quad);
            }
        }
    } else {
        // -------------------------------------------------------- epilogue
        // One arrival per tile (first CTA: named barrier; second CTA: the
        // first CTA's peer_drained barrier, relayed), in order, after the MMA
        // warp's commit of that tile, so never twice in one phase; outputs
        // are skipped once the launch has failed.
        const int quad = warp & 3;                       // TMEM lanes 32*quad .. 32*quad+31
        const uint32_t lane_addr = uint32_t(32 * quad) << 16;
        int tcount = 0;
        for (int ti = tbeg; ti < tend; ++ti, ++tcount) {
            const TileRef tr = decode_tile(p, p.tiles[ti]);
            // the tile's fields in registers: the stores below go through
            // generic pointers, which the compiler cannot prove do not alias
            // the parameter block, so reading these from it inside the store
            // loop would reload them after every store
            const GemmProblem &P = p.prob[tr.g];
            const int n = P.n, t0 = tr.t_tile * kBT, nt = tile_tokens(P, tr.t_tile);
            float *const y = P.y;
            int32_t *const acc = P.acc;
            const float *const act_scale = P.act_scale;
            const float sw = P.w_scale;
            const int b = tcount & 1, ur = tcount >> 1;
            // the tile's activation scales, token 32c + lane in sa_t[c], fetched
            // while the accumulator is still being computed
            float sa_t[kBT / 32];
#pragma unroll
            for (int c = 0; c < kBT / 32; ++c) sa_t[c] = (32 * c + lane < nt) ? act_scale[t0 + 32 * c + lane] : 0.f;
            bool live = warp_wait_progress(smem_u32(&accf_bar[b]), ur & 1, long_limit);
            if (!live && lane == 0) fail();
            live = __shfl_sync(0xffffffffu, (live && *abort_flag == 0) ? 1 : 0, 0) != 0;
            tc_fence_after();
            const int f = tr.f_tile * kPairF + int(rank) * kBF + 32 * quad + lane;
            const bool f_ok = f < n;
            const uint32_t taddr = tmem_base + lane_addr + uint32_t(b * kBT);
            if (live) {
#pragma unroll
                for (int c = 0; c < kBT / 32; ++c) {
                    const int c0 = 32 * c;
                    if (c0 >= nt) break;
                    uint32_t v[32];
                    tmem_ld32(taddr + uint32_t(c0), v);
                    if (ctrace && quad == 0 && lane == 0 && tcount < 2) ctrace[40 + 16 * tcount + 2 * c] = clock_ordered();
                    // dequantise all 32 in place first (straight-line code, so the
                    // shuffle -> convert -> multiply chains overlap), then store;
                    // a per-element branch here would serialise those chains
                    const float sa_l = sa_t[c];
                    const bool full = c0 + 32 <= nt;
                    if (acc && f_ok) {
                        int32_t *ac = acc + size_t(t0 + c0) * size_t(n) + f;
                        if (full) {
#pragma unroll
                            for (int j = 0; j < 32; ++j) ac[size_t(j) * size_t(n)] = int32_t(v[j]);
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                if (c0 + j < nt) ac[size_t(j) * size_t(n)] = int32_t(v[j]);
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        v[j] = __float_as_uint(
                            __fmul_rn(__fmul_rn(float(int32_t(v[j])), __shfl_sync(0xffffffffu, sa_l, j)), sw));
                    if (f_ok) {
                        float *yc = y + size_t(t0 + c0) * size_t(n) + f;
                        if (full) {
#pragma unroll
                            for (int j = 0; j < 32; ++j) yc[size_t(j) * size_t(n)] = __uint_as_float(v[j]);
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                if (c0 + j < nt) yc[size_t(j) * size_t(n)] = __uint_as_float(v[j]);
                        }
                    }
                    if (ctrace && quad == 0 && lane == 0 && tcount < 2) ctrace[41 + 16 * tcount + 2 * c] = clock_ordered();
                }
            }
            tc_fence_before();
            __syncwarp();
            if (leader) {
                nb_arrive(kNbAcc0 + uint32_t(b));
            } else if (lane == 0) {
                remote_arrive(smem_u32(&peer_drained_bar[b]), 0);
            }
            if (ctrace && tid == 32 * kEpiWarp0 && tcount < 16) ctrace[8 + tcount] = clock_ordered();
        }
    }

    // neither CTA frees TMEM or exits while the other may still use its
    // barriers, shared memory or TMEM
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (ctrace && tid == 0) {
        ctrace[2] = clock_ordered();
        ctrace[4] = globaltimer();
    }
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
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
// the token count m.  Tiles are dealt heaviest-first to the least-loaded SM
// pair (cost = MMA work of the tile's K loop plus a fixed epilogue share), so
// layers of different K balance inside one persistent launch.
cudaError_t launch_gemm_grouped(const int8_t *const *xq, const float *const *act_scale, int64_t m,
                                const bitnet_tw *w, int count, float *const *y, int32_t *const *acc,
                                int32_t *flags, uint64_t wait_limit, int force_stall, int sm_count, uint64_t *trace,
                                cudaStream_t st)
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
    const int tiles_t = int((m + kBT - 1) / kBT);
    for (int g = 0; g < count; ++g) {
        GemmProblem &P = p.prob[g];
        const int64_t kb = (w[g].k + 127) / 128;
        const cuuint32_t es[2] = {1u, 1u};
        {
            const cuuint64_t dims[2] = {cuuint64_t(128 * kb), cuuint64_t(m)};
            const cuuint64_t strides[1] = {cuuint64_t(128 * kb)};
            const cuuint32_t box[2] = {uint32_t(kBK), uint32_t(kHalfT)};
            if (enc(&P.tmap_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(xq[g]), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
        }
        {
            const cuuint64_t dims[2] = {cuuint64_t(32 * kb), cuuint64_t(w[g].n)};
            const cuuint64_t strides[1] = {cuuint64_t(32 * kb)};
            const cuuint32_t box[2] = {32u, uint32_t(kBF)};
            if (enc(&P.tmap_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(w[g].packed), dims, strides, box,
                    es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
        }
        P.act_scale = act_scale[g];
        P.y = y[g];
        P.acc = acc ? acc[g] : nullptr;
        P.w_scale = w[g].scale;
        P.m = int32_t(m);
        P.n = int32_t(w[g].n);
        P.kb = int32_t(kb);
        P.tiles_t = tiles_t;
        P.tiles_f = int32_t((w[g].n + kPairF - 1) / kPairF);
        P.tile0 = tile0;
        for (int ft = 0; ft < P.tiles_f; ++ft)
            for (int tt = 0; tt < tiles_t; ++tt) {
                const int64_t nt = std::min<int64_t>(kBT, m - int64_t(tt) * kBT);
                const int n16 = int((nt + 15) / 16);
                all.push_back(Tile{tile0 + ft * tiles_t + tt, int(kb + 2) * n16});
            }
        tile0 += P.tiles_f * tiles_t;
    }
    p.nprob = count;
    p.ntiles_total = tile0;
    p.flags = flags;
    p.wait_limit = wait_limit;
    p.force_stall = force_stall;
    p.trace = trace;
    std::stable_sort(all.begin(), all.end(), [](const Tile &a, const Tile &b) { return a.cost > b.cost; });
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    static bool configured[64] = {};
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        cudaError_t e = cudaFuncSetAttribute(gemm_i2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    static thread_local std::vector<int> owner, fill, count_of;
    static thread_local std::vector<long long> load;
    for (size_t c0 = 0; c0 < all.size(); c0 += kMaxGemmTiles) {
        const int n = int(std::min<size_t>(kMaxGemmTiles, all.size() - c0));
        const int G = std::min(std::min(sm_count / 2, kMaxGemmPairs), n);   // SM pairs
        if (G < 1) return cudaErrorInvalidConfiguration;
        // least-loaded pair first (loads are small integers: linear scan)
        load.assign(G, 0);
        owner.assign(n, 0);
        count_of.assign(G, 0);
        for (int i = 0; i < n; ++i) {
            int best = 0;
            for (int c = 1; c < G; ++c)
                if (load[c] < load[best]) best = c;
            load[best] += all[c0 + i].cost;
            owner[i] = best;
            ++count_of[best];
        }
        p.pair_off[0] = 0;
        for (int c = 0; c < G; ++c) p.pair_off[c + 1] = p.pair_off[c] + count_of[c];
        fill.assign(G, 0);
        for (int i = 0; i < n; ++i) {
            const int c = owner[i];
            p.tiles[p.pair_off[c] + fill[c]++] = all[c0 + i].id;
        }
        // grid = 2 CTAs per pair; the cluster shape (2, 1, 1) is compiled in
        gemm_i2_kernel<<<2 * G, kGemmThreads, kGemmSmem, st>>>(p);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_gemm(const int8_t *xq, const float *act_scale, int64_t m, const bitnet_tw *w, float *y,
                        int32_t *acc, int32_t *flags, uint64_t wait_limit, int force_stall, int sm_count,
                        uint64_t *trace, cudaStream_t st)
{
    const int8_t *xqa[1] = {xq};
    const float *sa[1] = {act_scale};
    float *ya[1] = {y};
    int32_t *aa[1] = {acc};
    return launch_gemm_grouped(xqa, sa, m, w, 1, ya, acc ? aa : nullptr, flags, wait_limit, force_stall, sm_count,
                               trace, st);
}

}  // namespace bitnet
