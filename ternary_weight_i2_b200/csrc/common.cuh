// common.cuh -- device helpers shared by the sm_100a kernels of the library.
//
// Only inline PTX for the primitives the kernels use: mbarriers, 1-D bulk
// (TMA) copies global->shared, dp4a, bounded waits.  Every wait is bounded by
// a clock limit; on expiry the caller raises BITNET_FLAG_TIMEOUT and returns.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/bitnet.h"

// The library is written for B200 only.  Building the device code for any
// other architecture is an error, not a silent empty kernel.
#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ != 1000)
#error "bitnet kernels target sm_100a (B200) only: build with -gencode arch=compute_100a,code=sm_100a"
#endif

namespace bitnet {

constexpr uint64_t kDefaultWaitLimit = (1ull << 31);   // ~1 s at 2 GHz
constexpr uint64_t kDrainWaitLimit = (1ull << 31);

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void raise_flag(int32_t *flags, int32_t bit)
{
    if (flags) atomicOr(flags, bit);
}

// 4-byte asynchronous copy global -> shared (no registers held while in
// flight), committed as a group and waited for by the issuing thread.
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// ------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Make mbarrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// As mbar_try_wait, but a thread whose phase is not complete yet may be
// suspended for up to `ns` nanoseconds (it resumes early when the phase
// completes): waiting warps then stop competing for issue slots.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t ns)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

// Wait for the phase of parity `parity` to complete; false if `limit` SM
// cycles pass first.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t limit)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = clock64();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - t0 > limit) return false;
    }
}

// ------------------------------------------------------------ bulk copies

// 1-D bulk asynchronous copy global -> shared (TMA engine), completion
// counted in bytes on `bar`.  dst, src 16-byte aligned; bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Order this thread's later TMA uses of the tensor map at `tmap` (global
// memory) after writes to it made before the launch (host copies): a map's
// bytes may have been rewritten at an address the TMA unit has seen before.
__device__ __forceinline__ void tensormap_acquire(const void *tmap)
{
    asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(tmap) : "memory");
}

// L2 policy for data read exactly once per launch (the weight stream): evict
// first, so that it does not push activations and outputs out of L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// 2-D tiled TMA load of one box of a tensor map (global CUtensorMap) into
// shared memory with an L2 cache policy; coordinates in elements, x innermost
// (x * elemsize must be a multiple of 16 bytes).  No multicast.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void *tmap, int32_t x, int32_t y, uint32_t bar,
                                            uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(tmap), "r"(x), "r"(y), "r"(bar), "l"(policy)
        : "memory");
}

// ----------------------------------------------------------- arithmetic

// Four-way byte dot product: unsigned bytes of a times signed bytes of b,
// accumulated into c (the u8 x s8 multiply-add of the unpack-and-madd
// formulation).
__device__ __forceinline__ int32_t dp4a_us(uint32_t a, uint32_t b, int32_t c)
{
    int32_t d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ int32_t warp_sum(int32_t v)
{
    return __reduce_add_sync(0xffffffffu, v);
}

// Per-token activation quantiser of one element given inv = 127/amax
// (round half to even, clamp to +-127, zero stays zero).
__device__ __forceinline__ int32_t quant_one(float x, float inv)
{
    if (x == 0.0f) return 0;
    float v = __fmul_rn(x, inv);
    v = fminf(fmaxf(v, -127.0f), 127.0f);
    return __float2int_rn(v);
}

__device__ __forceinline__ uint32_t pack4(int32_t a, int32_t b, int32_t c, int32_t d)
{
    return (uint32_t(a) & 0xffu) | ((uint32_t(b) & 0xffu) << 8) | ((uint32_t(c) & 0xffu) << 16) |
           ((uint32_t(d) & 0xffu) << 24);
}

}  // namespace bitnet
