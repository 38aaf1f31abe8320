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
//               tile (256 rows x 32 B) into a 3-stage shared-memory ring;
//   warps 2-3   expand the packed tile to signed int8 (code - 1) straight into
//               the canonical K-major 128-byte-swizzled layout of operand B;
//   warp 1      one thread issues 4 tcgen05.mma (M=128, N=256, K=32) per
//               block into a TMEM accumulator (two 256-column accumulators,
//               so the epilogue of one tile overlaps the next tile's K loop)
//               and commits to mbarriers;
//   warps 4-7   epilogue: tcgen05.ld the accumulator (one TMEM lane = one
//               output row per thread), dequantise in fp32, store.
// Every wait is bounded; on expiry the CTA raises BITNET_FLAG_TIMEOUT, the
// other roles stop, in-flight copies and MMAs are drained (bounded) and TMEM
// is freed before exit.  No TMA multicast.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace bitnet {

constexpr int kBM = 128, kBN = 256, kBK = 128;
constexpr int kStages = 3;
constexpr int kAStage = kBM * kBK;                 // 16 KB int8 activations
constexpr int kBStage = kBN * kBK;                 // 32 KB expanded int8 weights
constexpr int kPStage = kBN * 32;                  // 8 KB packed weights
constexpr int kStageBytes = kAStage + kBStage + kPStage;
constexpr int kGemmThreads = 256;
constexpr int kExpandThreads = 64;                 // warps 2-3
constexpr int kEpiThreads = 128;                   // warps 4-7
constexpr int kTmemCols = 2 * kBN;                 // two int32 accumulators
constexpr int kGemmSmem = 1024 + kStages * kStageBytes;

struct GemmParams {
    CUtensorMap tmap_a;       // int8 q [M, Kpad]: dims {Kpad, M}, box {128, 128}, 128-byte swizzle
    CUtensorMap tmap_b;       // packed [N, 32*KB]: dims {32*KB, N}, box {32, 256}, no swizzle
    const float *act_scale;   // [M]
    float *y;                 // [M, N]
    int32_t *acc;             // [M, N] or null
    float w_scale;
    int32_t m, n, kb;
    int32_t tiles_m, tiles_n;
    int32_t *flags;
    uint64_t wait_limit;
};

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
// K-major, M = 128, N = 256, dense.
constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(kBN >> 3) << 17) | (uint32_t(kBM >> 4) << 24);

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

// Signed int8 weights (code - 1) of field g of a packed word: one byte per
// element, elements 32g + b .. 32g + b + 3 of the block.
__device__ __forceinline__ uint32_t expand_field(uint32_t v, int g)
{
    const uint32_t c = (v >> (2 * g)) & 0x03030303u;   // codes 0, 1, 2 per byte
    return (c + 0x7F7F7F7Fu) ^ 0x80808080u;            // 0x7F+c has no carry; ^0x80 -> c - 1
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
    __shared__ __align__(8) uint64_t full_bar[kStages], expd_bar[kStages], empty_bar[kStages];
    __shared__ __align__(8) uint64_t accf_bar[2], acce_bar[2], drain_bar;
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;
    volatile int *abort_flag = &abort_s;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint64_t limit = p.wait_limit;
    const int ntiles = p.tiles_m * p.tiles_n;
    const int kblocks = p.kb;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&expd_bar[s]), kExpandThreads);
            mbar_init(smem_u32(&empty_bar[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&accf_bar[b]), 1);
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

    auto fail = [&]() {
        abort_s = 1;
        raise_flag(p.flags, BITNET_FLAG_TIMEOUT);
    };

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol_w = l2_evict_first_policy();
            int it = 0, issued_tail = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                const int m_tile = t % p.tiles_m, n_tile = t / p.tiles_m;
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const int s = it % kStages, r = it / kStages;
                    if (r > 0 && !wait_or_abort(smem_u32(&empty_bar[s]), (r - 1) & 1, limit, abort_flag)) {
                        fail();
                        ok = false;
                        break;
                    }
                    uint8_t *st = smem + s * kStageBytes;
                    const uint32_t fb = smem_u32(&full_bar[s]);
                    mbar_arrive_expect_tx(fb, kAStage + kPStage);
                    asm volatile(
                        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(st)),
                        "l"(&p.tmap_a), "r"(kb * kBK), "r"(m_tile * kBM), "r"(fb)
                        : "memory");
                    tma_load_2d(smem_u32(st + kAStage + kBStage), &p.tmap_b, kb * 32, n_tile * kBN, fb, pol_w);
                    issued_tail = it;
                }
            }
            if (!ok) {
                // let copies already issued land before the CTA can exit
                for (int j = (issued_tail >= kStages ? issued_tail - kStages + 1 : 0); j <= issued_tail; ++j)
                    mbar_wait(smem_u32(&full_bar[j % kStages]), (j / kStages) & 1, kDrainWaitLimit);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int it = 0, tcount = 0;
            bool ok = true, any = false;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++tcount) {
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
                    if (!wait_or_abort(smem_u32(&full_bar[s]), r & 1, limit, abort_flag) ||
                        !wait_or_abort(smem_u32(&expd_bar[s]), r & 1, limit, abort_flag)) {
                        fail();
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(smem + s * kStageBytes);
                    const uint32_t b0 = a0 + kAStage;
#pragma unroll
                    for (int ks = 0; ks < kBK / 32; ++ks)
                        mma_i8(d_tmem, sw128_desc(a0 + ks * 32), sw128_desc(b0 + ks * 32),
                               (kb > 0 || ks > 0) ? 1u : 0u);
                    mma_commit(smem_u32(&empty_bar[s]));
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
    } else if (warp < 4) {
        // ------------------------------------------------------- expanders
        const int et = tid - 64;
        int it = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            for (int kb = 0; kb < kblocks; ++kb, ++it) {
                const int s = it % kStages, r = it / kStages;
                const bool landed = wait_or_abort(smem_u32(&full_bar[s]), r & 1, limit, abort_flag);
                if (!landed) {
                    fail();
                    ok = false;
                    break;
                }
                uint8_t *st = smem + s * kStageBytes;
                const uint32_t bsm = smem_u32(st + kAStage);
                const uint32_t psm = smem_u32(st + kAStage + kBStage);
#pragma unroll 2
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
                mbar_arrive(smem_u32(&expd_bar[s]));
            }
        }
    } else {
        // -------------------------------------------------------- epilogue
        const int sub = warp & 3;            // TMEM lanes 32*sub .. 32*sub+31
        int tcount = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++tcount) {
            const int m_tile = t % p.tiles_m, n_tile = t / p.tiles_m;
            const int b = tcount & 1, ur = tcount >> 1;
            const bool ready = wait_or_abort(smem_u32(&accf_bar[b]), ur & 1, limit, abort_flag);
            if (!__all_sync(0xffffffffu, ready)) {
                if (lane == 0) fail();
                ok = false;
                break;
            }
            tc_fence_after();
            const int row = m_tile * kBM + 32 * sub + lane;
            const bool row_ok = row < p.m;
            const float sa = row_ok ? p.act_scale[row] : 0.f;
            const uint32_t taddr = tmem_base + (uint32_t(32 * sub) << 16) + uint32_t(b * kBN);
            const bool vec = (p.n % 4) == 0;
#pragma unroll 1
            for (int c0 = 0; c0 < kBN; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(taddr + uint32_t(c0), v);
                const int col0 = n_tile * kBN + c0;
                if (!row_ok || col0 >= p.n) continue;
                float *yr = p.y + size_t(row) * size_t(p.n) + col0;
                int32_t *ar = p.acc ? p.acc + size_t(row) * size_t(p.n) + col0 : nullptr;
                if (vec && col0 + 32 <= p.n) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        float4 o;
                        o.x = __fmul_rn(__fmul_rn(float(int32_t(v[j + 0])), sa), p.w_scale);
                        o.y = __fmul_rn(__fmul_rn(float(int32_t(v[j + 1])), sa), p.w_scale);
                        o.z = __fmul_rn(__fmul_rn(float(int32_t(v[j + 2])), sa), p.w_scale);
                        o.w = __fmul_rn(__fmul_rn(float(int32_t(v[j + 3])), sa), p.w_scale);
                        *reinterpret_cast<float4 *>(yr + j) = o;
                        if (ar)
                            *reinterpret_cast<int4 *>(ar + j) =
                                make_int4(int32_t(v[j]), int32_t(v[j + 1]), int32_t(v[j + 2]), int32_t(v[j + 3]));
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (col0 + j < p.n) {
                            yr[j] = __fmul_rn(__fmul_rn(float(int32_t(v[j])), sa), p.w_scale);
                            if (ar) ar[j] = int32_t(v[j]);
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&acce_bar[b]));
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
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

cudaError_t launch_gemm(const int8_t *xq, const float *act_scale, int64_t m, const bitnet_tw *w, float *y,
                        int32_t *acc, int32_t *flags, uint64_t wait_limit, int sm_count, cudaStream_t st)
{
    auto enc = gemm_encode_fn();
    if (!enc) return cudaErrorNotSupported;
    static thread_local GemmParams p;   // staging; copied into the launch
    const int64_t kb = (w->k + 127) / 128;
    {
        const cuuint64_t dims[2] = {cuuint64_t(128 * kb), cuuint64_t(m)};
        const cuuint64_t strides[1] = {cuuint64_t(128 * kb)};
        const cuuint32_t box[2] = {uint32_t(kBK), uint32_t(kBM)};
        const cuuint32_t es[2] = {1u, 1u};
        if (enc(&p.tmap_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(xq), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[2] = {cuuint64_t(32 * kb), cuuint64_t(w->n)};
        const cuuint64_t strides[1] = {cuuint64_t(32 * kb)};
        const cuuint32_t box[2] = {32u, uint32_t(kBN)};
        const cuuint32_t es[2] = {1u, 1u};
        if (enc(&p.tmap_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(w->packed), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    p.act_scale = act_scale;
    p.y = y;
    p.acc = acc;
    p.w_scale = w->scale;
    p.m = int32_t(m);
    p.n = int32_t(w->n);
    p.kb = int32_t(kb);
    p.tiles_m = int32_t((m + kBM - 1) / kBM);
    p.tiles_n = int32_t((w->n + kBN - 1) / kBN);
    p.flags = flags;
    p.wait_limit = wait_limit;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(gemm_i2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    const int64_t tiles = int64_t(p.tiles_m) * p.tiles_n;
    const int grid = int(tiles < sm_count ? tiles : sm_count);
    gemm_i2_kernel<<<grid, kGemmThreads, kGemmSmem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace bitnet
