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
// same multiply-add as its INT8 path; here the unpacked INT8 weights feed the
// tensor cores.
//
// Operand roles.  The weights are the MMA's A operand and live in tensor
// memory (TMEM); the activations are B and come from shared memory, so the
// accumulator is D[n, m] = sum_k w[n,k] q[m,k]: one TMEM lane per output
// feature, one column per token.  The expanded weights never touch shared
// memory: per K block shared memory carries only the TMA-landed activation
// and packed-weight tiles and the tensor core's read of the activations
// (shared-memory bandwidth, not the tensor pipe, bounds a design that stages
// expanded weights there).
//
// One CTA per SM, persistent over tiles of 128 features x up to 192 tokens;
// per 128-element K block (one packed block per weight row):
//   warps 0, 2, 3  TMA: the activation tile (192 tokens x 128 B, 128-byte
//                  swizzle: the canonical K-major layout of B) and the packed
//                  weight tile (128 rows x 32 B) into a 7-stage ring; K block
//                  `it` is issued by producer it % 3;
//   warps 4-11     expanders, one thread per weight row: read the row's 32
//                  packed bytes, turn the 2-bit codes into signed int8 w in
//                  registers (three logic ops and one add per 4 weights, no
//                  multiply) and write the row's 128 values, 32 TMEM columns,
//                  with one tcgen05.st into one of 4 A buffers; two groups of
//                  four warps take alternate K blocks;
//   warp 1         one thread issues 4 tcgen05.mma (M=128, N<=192, K=32, A
//                  from TMEM, B from shared memory, both signed) per K block
//                  into one of two TMEM accumulators, so the epilogue of one
//                  tile overlaps the next tile's K loop, and commits to
//                  mbarriers;
//   warps 12-15    epilogue: tcgen05.ld gives each thread 32 tokens of one
//                  feature; dequantise in fp32 and store, each warp writing 32
//                  consecutive features (128 bytes) of one token per store.
// Every wait is bounded; on expiry the CTA raises BITNET_FLAG_TIMEOUT, the
// other roles stop, in-flight copies and MMAs are drained (bounded) and TMEM
// is freed before exit.  No TMA multicast.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <vector>

#include "common.cuh"

namespace bitnet {

constexpr int kBF = 128;                           // features per tile: MMA M, TMEM lanes
constexpr int kBT = 192;                           // tokens per tile: MMA N (at most)
constexpr int kBK = 128;                           // K per block: one packed block per row
constexpr int kStages = 7;                         // TMA ring (activations + packed weights)
constexpr int kABufs = 4;                          // expanded weight tiles in TMEM
constexpr int kActStage = kBT * kBK;               // 24 KB int8 activations
constexpr int kPStage = kBF * 32;                  // 4 KB packed weights
constexpr int kActOff = 0, kPOff = kStages * kActStage;
constexpr int kGemmSmem = 1024 + kPOff + kStages * kPStage;
constexpr int kGemmThreads = 512;                  // 16 warps
constexpr int kProducers = 3;                      // TMA-issuing warps: 0, 2, 3
constexpr int kExpandWarp0 = 4, kExpandGroupWarps = 4, kExpandGroups = 2;
constexpr int kEpiWarp0 = 12, kEpiWarps = 4;
constexpr int kACol0 = 2 * kBT;                    // TMEM columns of the A buffers
constexpr int kTmemCols = 512;
static_assert(kACol0 + 32 * kABufs <= kTmemCols, "TMEM budget");
static_assert(kGemmSmem <= 232448, "shared-memory budget");
static_assert(kEpiWarp0 % 4 == 0 && kExpandWarp0 % 4 == 0, "TMEM lane quadrant = warp % 4");

struct GemmProblem {
    CUtensorMap tmap_q;       // int8 q [M, Kpad]: dims {Kpad, M}, box {128, 192}, 128-byte swizzle
    CUtensorMap tmap_w;       // packed [N, 32*KB]: dims {32*KB, N}, box {32, 128}, no swizzle
    const float *act_scale;   // [M]
    float *y;                 // [M, N]
    int32_t *acc;             // [M, N] or null
    const float *bias;        // fused epilogue: [N] or null
    const float *gamma;       // [N] or null (layer scale)
    const float *res;         // [M, N] or null (residual; may be y)
    int32_t relu;             // ReLU after the bias
    float w_scale;
    int32_t m, n, kb;
    int32_t tiles_t, tiles_f;
    int32_t tile0;            // first id of this problem's tiles in the launch's tile numbering
};

constexpr int kMaxGroup = 8;         // problems (layers) per launch
constexpr int kMaxGemmCtas = 160;
constexpr int kMaxGemmTiles = 7168;  // tiles per launch

struct GemmParams {
    GemmProblem prob[kMaxGroup];
    int32_t nprob;
    int32_t ntiles_total;
    int32_t *flags;
    uint64_t wait_limit;
    int32_t force_stall;      // test aid: K block kStallBlock's copies are never issued
    int32_t has_epi;          // some problem of the launch has a fused-epilogue operand
    uint64_t *trace;          // optional: CTA 0 stamps (kGemmTraceMisc + 72 entries)
    int32_t cta_off[kMaxGemmCtas + 1];   // CTA c runs tiles[cta_off[c] .. cta_off[c+1])
    int32_t tiles[kMaxGemmTiles];        // tile ids, heaviest first within each CTA
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

// Trace of CTA 0 (profiling aid): SM clock stamps per K block it <
// kGemmTraceBlocks at [it*16 + e]: 0 producer issued, 1 (a value, not a
// stamp) 1 if the MMA thread's look-ahead found the block ready, else 2, 2 MMA
// saw A ready, 3 MMA issued, 4+q / 8+q / 12+q expander warp of lane quadrant
// q saw full / saw its A buffer free / wrote it; then at kGemmTraceMisc + 0
// kernel entry, +1 set-up done, +2 all roles done, +3 / +4 globaltimer at
// entry / end, +8+t epilogue of tile t done, +24+t MMA found tile t's
// accumulator free (t < 16).
constexpr int kGemmTraceBlocks = 48, kGemmTraceEv = 16;
constexpr int kGemmTraceMisc = kGemmTraceBlocks * kGemmTraceEv;

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
// K-major, M = 128, N = n (a multiple of 16, at most 256), dense.
__device__ __forceinline__ uint32_t idesc_i8(int n)
{
    return (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(kBF >> 4) << 24);
}

// One K block, issued by one thread: four MMAs (K = 32 each) into d_tmem --
// the activation descriptor of K step ks is qdesc + 2*ks (32 bytes further,
// in 16-byte units; the start-address field cannot carry out for
// shared-memory addresses) -- then commits to the barriers that free the
// activation stage and the A buffer.
__device__ __forceinline__ void mma_kblock(uint32_t d_tmem, uint32_t a_tmem, uint64_t qdesc, uint32_t idesc,
                                           uint32_t accumulate, uint32_t bar_stage, uint32_t bar_abuf)
{
    asm volatile(
        "{\n\t.reg .pred p0, p1;\n\t"
        "setp.ne.b32 p0, %4, 0;\n\t"
        "setp.eq.u32 p1, %4, %4;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%6], %7, %3, p1;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%8], %9, %3, p1;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%10], %11, %3, p1;\n\t"
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%5];\n\t"
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%12];\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(qdesc), "r"(idesc), "r"(accumulate), "r"(bar_stage), "r"(a_tmem + 8u),
          "l"(qdesc + 2u), "r"(a_tmem + 16u), "l"(qdesc + 4u), "r"(a_tmem + 24u), "l"(qdesc + 6u), "r"(bar_abuf)
        : "memory");
}

// Named (hardware) barriers between the MMA warp and the warps that feed or
// drain the tensor memory: ids 1..4 "A buffer a written" (expander group of
// four warps + the MMA warp), ids 5..6 "accumulator b drained" (four epilogue
// warps + the MMA warp).  The MMA warp waits (bar.sync), the others arrive
// (bar.arrive, release); each phase has exactly one arrival per warp.
constexpr uint32_t kNbAbuf0 = 1, kNbAcc0 = 5, kNbThreads = 160;
static_assert(kNbThreads == 32 * (kExpandGroupWarps + 1) && kNbThreads == 32 * (kEpiWarps + 1), "barrier sizes");
__device__ __forceinline__ void nb_arrive(uint32_t id)
{
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(kNbThreads) : "memory");
}
__device__ __forceinline__ void nb_sync(uint32_t id)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(kNbThreads) : "memory");
}

// K block whose copies a test stalls (force_stall)
constexpr int kStallBlock = 2;

__device__ __forceinline__ void mma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

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

// Wait on an mbarrier phase; false on timeout or when another role aborted.
// Between polls the thread may sleep up to `sleep_ns` (it wakes as soon as
// the phase completes), so roles that wait do not take issue slots from the
// ones that work.
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, uint64_t limit, volatile int *abort_flag,
                                              uint32_t sleep_ns = 0)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = clock64();
    for (int spin = 0;; ++spin) {
        if (sleep_ns ? mbar_try_wait_sleep(bar, parity, sleep_ns) : mbar_try_wait(bar, parity)) return true;
        if ((spin & 15) == 0 && *abort_flag) return false;
        if (clock64() - t0 > limit) return false;
    }
}
// Suspend-time hint of the waiting roles: without one, a polling thread takes
// issue slots from the warps that work; with a long one, a thread is not
// reliably woken at once by arrivals of the asynchronous units (TMA, tensor
// core commits) and the pipeline stalls -- a short hint bounds both.
constexpr uint32_t kSleepNs = 100;

// Warp-wide wait: lane 0 polls, the others take its result (and, through
// __syncwarp, the ordering its successful wait established).  One poller per
// warp instead of 32 keeps the barrier traffic of the waiting roles low.
__device__ __forceinline__ bool warp_wait_or_abort(uint32_t bar, uint32_t parity, uint64_t limit,
                                                   volatile int *abort_flag, uint32_t sleep_ns = kSleepNs)
{
    bool ok = false;
    if ((threadIdx.x & 31) == 0) ok = wait_or_abort(bar, parity, limit, abort_flag, sleep_ns);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    return ok;
}

// Warp-wide wait for a phase the MMA warp's commits complete: no abort
// check (those commits always come), only the long limit.
__device__ __forceinline__ bool warp_wait_progress(uint32_t bar, uint32_t parity, uint64_t long_limit)
{
    bool ok = false;
    if ((threadIdx.x & 31) == 0) {
        ok = mbar_try_wait(bar, parity);
        if (!ok) {
            const uint64_t t0 = clock64();
            while (!(ok = mbar_try_wait_sleep(bar, parity, kSleepNs)) && clock64() - t0 <= long_limit) {
            }
        }
    }
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    return ok;
}

// Tokens of tile t_tile and the MMA's N for them (a multiple of 16).
__device__ __forceinline__ int tile_tokens(const GemmProblem &P, int t_tile)
{
    return min(kBT, P.m - t_tile * kBT);
}

// kEpi: the launch has a fused-epilogue operand on some problem.  The plain
// instantiation carries none of the epilogue code.
template <bool kEpi>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_i2_kernel(const __grid_constant__ GemmParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
    __shared__ __align__(8) uint64_t aempty_bar[kABufs], accf_bar[2], drain_bar;
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;
    volatile int *abort_flag = &abort_s;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint64_t limit = p.wait_limit;
    // limit of the waits on the MMA warp's commits, which always come (the MMA
    // warp never stops): far above the time one failed copy wait can hold
    // the pipeline up
    const uint64_t long_limit = (limit > (kDrainWaitLimit >> 2)) ? (limit << 2) : kDrainWaitLimit;
    const int tbeg = p.cta_off[blockIdx.x], tend = p.cta_off[blockIdx.x + 1];
    const uint32_t sbase = smem_u32(smem);
    uint64_t *ctrace = (p.trace && blockIdx.x == 0) ? p.trace + kGemmTraceMisc : nullptr;
    if (ctrace && tid == 0) {
        ctrace[0] = clock64();
        ctrace[3] = globaltimer();
    }

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&empty_bar[s]), 1 + kExpandGroupWarps);   // MMA commit, expander warps
        }
        for (int a = 0; a < kABufs; ++a) mbar_init(smem_u32(&aempty_bar[a]), 1);
        for (int b = 0; b < 2; ++b) mbar_init(smem_u32(&accf_bar[b]), 1);
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
    if (ctrace && tid == 0) ctrace[1] = clock64();

    auto fail = [&]() {
        abort_s = 1;
        raise_flag(p.flags, BITNET_FLAG_TIMEOUT);
    };
    uint64_t *trace = (p.trace && blockIdx.x == 0) ? p.trace : nullptr;
    auto stamp = [&](int it, int ev) {
        if (trace && it < kGemmTraceBlocks) trace[it * kGemmTraceEv + ev] = clock64();
    };

    if (warp == 0 || warp == 2 || warp == 3) {
        // ----------------------------------------------------- TMA producers
        // The whole warp runs the loop and lane 0 issues the copies (a lone
        // diverged lane is starved by busy warps of its sub-partition).
        const int pidx = (warp == 0) ? 0 : warp - 1;
        int it = 0, last = -1;
        bool ok = true;
        for (int ti = tbeg; ti < tend && ok; ++ti) {
            const TileRef tr = decode_tile(p, p.tiles[ti]);
            const GemmProblem &P = p.prob[tr.g];
            const int kblocks = P.kb;
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
                        "l"(&P.tmap_q), "r"(kb * kBK), "r"(tr.t_tile * kBT), "r"(fb)
                        : "memory");
                    asm volatile(
                        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                        " [%0], [%1, {%2, %3}], [%4];" ::"r"(sbase + kPOff + s * kPStage),
                        "l"(&P.tmap_w), "r"(kb * 32), "r"(tr.f_tile * kBF), "r"(fb)
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
        // Waits only on the named barriers the expanders and the epilogue
        // arrive at (an mbarrier poll here costs the tensor core more than a
        // hundred cycles per K block), never gives up, always commits: every
        // other role's waits on its commits therefore end.  The expanders
        // arrive for a K block only after they saw its stage's TMA
        // transaction complete, so the barrier covers both operands.
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
            if (tcount >= 2) nb_sync(kNbAcc0 + uint32_t(b));   // the epilogue drained tile tcount-2
            if (ctrace && lane == 0 && tcount < 16) ctrace[24 + tcount] = clock64();
            const uint32_t d_tmem = tmem_base + uint32_t(b * kBT);
            for (int kb = 0; kb < kblocks; ++kb, ++it) {
                nb_sync(kNbAbuf0 + uint32_t(a));                   // A buffer a holds K block it
                if (lane == 0) stamp(it, 2);
                tc_fence_after();
                if (lane == 0)
                    mma_kblock(d_tmem, a_tm0 + 32u * uint32_t(a), qdesc0 + uint64_t(s) * (kActStage >> 4), idesc,
                               kb > 0 ? 1u : 0u, empty0 + 8u * uint32_t(s), aempty0 + 8u * uint32_t(a));
                __syncwarp();
                if (lane == 0) stamp(it, 3);
                s = (s + 1 == kStages) ? 0 : s + 1;
                a = (a + 1) & (kABufs - 1);
            }
            if (lane == 0) mma_commit(smem_u32(&accf_bar[b]));
            __syncwarp();
        }
        // the epilogue's arrivals for the last two tiles
        for (int t = (tcount > 2 ? tcount - 2 : 0); t < tcount; ++t) nb_sync(kNbAcc0 + uint32_t(t & 1));
        if (tcount > 0 && lane == 0) {
            // all MMAs this warp issued are complete before TMEM is freed
            mma_commit(smem_u32(&drain_bar));
            mbar_wait(smem_u32(&drain_bar), 0, kDrainWaitLimit);
        }
        __syncwarp();
    } else if (warp < kEpiWarp0) {
        // ------------------------------------------------------- expanders
        // Every K block of the group ends with one arrival at its A buffer's
        // named barrier, in order, also after a failed wait (the work is then
        // skipped): the MMA warp waits there without a limit.  Before writing
        // a buffer again the group waits for the MMA warp's commit of its
        // previous use, so it can never arrive twice in one barrier phase.
        const int grp = (warp - kExpandWarp0) / kExpandGroupWarps;
        const int quad = warp & 3;                       // TMEM lanes 32*quad .. 32*quad+31
        const int row = 32 * quad + lane;                // weight row of the tile
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
                nb_arrive(kNbAbuf0 + uint32_t(a));
                if (lane == 0) stamp(it, 12 + quad);
            }
        }
    } else {
        // -------------------------------------------------------- epilogue
        // One arrival per tile at the accumulator's named barrier, in order,
        // after the MMA warp's commit of that tile (so never twice in one
        // phase); the outputs are skipped once the launch has failed.
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
            const float *const res = kEpi ? P.res : nullptr;
            const bool has_bias = kEpi && P.bias != nullptr, has_gamma = kEpi && P.gamma != nullptr;
            const bool relu = kEpi && P.relu != 0;
            const float *const bias_p = P.bias, *const gamma_p = P.gamma;
            const int b = tcount & 1, ur = tcount >> 1;
            // the tile's activation scales, token 32c + lane in sa_t[c], fetched
            // while the accumulator is still being computed
            float sa_t[kBT / 32];
#pragma unroll
            for (int c = 0; c < kBT / 32; ++c) sa_t[c] = (32 * c + lane < nt) ? act_scale[t0 + 32 * c + lane] : 0.f;
            const int f = tr.f_tile * kBF + 32 * quad + lane;
            const bool f_ok = f < n;
            // fused epilogue operands of this thread's feature (technical
            // report §2.4.1: bias + ReLU, then the layer-scaled residual add)
            const float bias_f = (has_bias && f_ok) ? bias_p[f] : 0.f;
            const float gamma_f = (has_gamma && f_ok) ? gamma_p[f] : 1.f;
            const bool has_res = res != nullptr && f_ok;
            bool live = warp_wait_progress(smem_u32(&accf_bar[b]), ur & 1, long_limit);
            if (!live && lane == 0) fail();
            live = __shfl_sync(0xffffffffu, (live && *abort_flag == 0) ? 1 : 0, 0) != 0;
            tc_fence_after();
            const uint32_t taddr = tmem_base + lane_addr + uint32_t(b * kBT);
            if (live) {
#pragma unroll
                for (int c = 0; c < kBT / 32; ++c) {
                    const int c0 = 32 * c;
                    if (c0 >= nt) break;
                    uint32_t v[32];
                    tmem_ld32(taddr + uint32_t(c0), v);
                    if (ctrace && quad == 0 && lane == 0 && tcount < 2) ctrace[40 + 16 * tcount + 2 * c] = clock64();
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
                    // each step one rounding, in straight-line loops (the
                    // branches are uniform over the tile)
                    if (has_bias) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__fadd_rn(__uint_as_float(v[j]), bias_f));
                    }
                    if (relu) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(v[j]) > 0.f ? v[j] : 0u;
                    }
                    if (has_gamma) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__fmul_rn(gamma_f, __uint_as_float(v[j])));
                    }
                    if (has_res) {
                        const float *rc = res + size_t(t0 + c0) * size_t(n) + f;
                        if (full) {
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                v[j] = __float_as_uint(__fadd_rn(rc[size_t(j) * size_t(n)], __uint_as_float(v[j])));
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                if (c0 + j < nt)
                                    v[j] = __float_as_uint(__fadd_rn(rc[size_t(j) * size_t(n)], __uint_as_float(v[j])));
                        }
                    }
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
                    if (ctrace && quad == 0 && lane == 0 && tcount < 2) ctrace[41 + 16 * tcount + 2 * c] = clock64();
                }
            }
            tc_fence_before();
            __syncwarp();
            nb_arrive(kNbAcc0 + uint32_t(b));
            if (ctrace && tid == 32 * kEpiWarp0 && tcount < 16) ctrace[8 + tcount] = clock64();
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (ctrace && tid == 0) {
        ctrace[2] = clock64();
        ctrace[4] = globaltimer();
    }
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
// (cost = MMA work of the tile's K loop plus a fixed epilogue share), so
// layers of different K balance inside one persistent launch.
cudaError_t launch_gemm_grouped(const int8_t *const *xq, const float *const *act_scale, int64_t m,
                                const bitnet_tw *w, const bitnet_epilogue *epi, int count, float *const *y,
                                int32_t *const *acc,
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
            const cuuint32_t box[2] = {uint32_t(kBK), uint32_t(kBT)};
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
        P.bias = epi ? epi[g].bias : nullptr;
        P.gamma = epi ? epi[g].gamma : nullptr;
        P.res = epi ? epi[g].residual : nullptr;
        P.relu = (epi && epi[g].relu) ? 1 : 0;
        P.w_scale = w[g].scale;
        P.m = int32_t(m);
        P.n = int32_t(w[g].n);
        P.kb = int32_t(kb);
        P.tiles_t = tiles_t;
        P.tiles_f = int32_t((w[g].n + kBF - 1) / kBF);
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
    p.has_epi = 0;
    for (int g = 0; g < count; ++g)
        if (p.prob[g].bias || p.prob[g].gamma || p.prob[g].res || p.prob[g].relu) p.has_epi = 1;
    std::stable_sort(all.begin(), all.end(), [](const Tile &a, const Tile &b) { return a.cost > b.cost; });
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    static bool configured[64] = {};
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        cudaError_t e = cudaFuncSetAttribute(gemm_i2_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kGemmSmem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(gemm_i2_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    static thread_local std::vector<int> owner, fill, count_of;
    static thread_local std::vector<long long> load;
    for (size_t c0 = 0; c0 < all.size(); c0 += kMaxGemmTiles) {
        const int n = int(std::min<size_t>(kMaxGemmTiles, all.size() - c0));
        const int G = std::min(std::min(sm_count, kMaxGemmCtas), n);
        // least-loaded CTA first (loads are small integers: linear scan)
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
        p.cta_off[0] = 0;
        for (int c = 0; c < G; ++c) p.cta_off[c + 1] = p.cta_off[c] + count_of[c];
        fill.assign(G, 0);
        for (int i = 0; i < n; ++i) {
            const int c = owner[i];
            p.tiles[p.cta_off[c] + fill[c]++] = all[c0 + i].id;
        }
        if (p.has_epi)
            gemm_i2_kernel<true><<<G, kGemmThreads, kGemmSmem, st>>>(p);
        else
            gemm_i2_kernel<false><<<G, kGemmThreads, kGemmSmem, st>>>(p);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_gemm(const int8_t *xq, const float *act_scale, int64_t m, const bitnet_tw *w,
                        const bitnet_epilogue *epi, float *y, int32_t *acc, int32_t *flags, uint64_t wait_limit,
                        int force_stall, int sm_count, uint64_t *trace, cudaStream_t st)
{
    const int8_t *xqa[1] = {xq};
    const float *sa[1] = {act_scale};
    float *ya[1] = {y};
    int32_t *aa[1] = {acc};
    return launch_gemm_grouped(xqa, sa, m, w, epi, 1, ya, acc ? aa : nullptr, flags, wait_limit, force_stall,
                               sm_count, trace, st);
}

}  // namespace bitnet
