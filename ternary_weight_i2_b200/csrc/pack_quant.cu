// pack_quant.cu -- load-time pack/unpack of the 2-bit ternary format and the
// standalone per-token int8 activation quantiser (prefill input).
//
// Format ("VibeVoice-ASR-BitNet Technical Report", §2.2.2: ternary weights in
// 2 bits; 128-element groups per the ARM debugging blog post, second
// postscript): element k = 128j + 32g + b of a row sits in byte 32j + b, bits
// [2g, 2g+1], as code w + 1; tail positions hold code 1 (weight 0).
#include "common.cuh"

namespace bitnet {

// One thread per packed byte: gathers the four elements 128j + 32g + b.
__global__ void pack_kernel(const int8_t *__restrict__ w, int64_t n, int64_t k, int64_t kb,
                            uint8_t *__restrict__ packed, int32_t *flags)
{
    const int64_t rowb = 32 * kb;
    const int64_t total = n * rowb;
    bool bad = false;
    for (int64_t idx = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; idx < total;
         idx += int64_t(gridDim.x) * blockDim.x) {
        const int64_t r = idx / rowb, byte = idx - r * rowb;
        const int64_t j = byte >> 5, b = byte & 31;
        uint32_t out = 0;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const int64_t kk = 128 * j + 32 * g + b;
            uint32_t code = 1;
            if (kk < k) {
                const int v = w[r * k + kk];
                if (v >= -1 && v <= 1) code = uint32_t(v + 1);
                else bad = true;
            }
            out |= code << (2 * g);
        }
        packed[idx] = uint8_t(out);
    }
    const unsigned mask = __ballot_sync(0xffffffffu, bad);
    if (mask != 0u && (threadIdx.x & 31) == unsigned(__ffs(mask) - 1)) raise_flag(flags, BITNET_FLAG_NOT_TERNARY);
}

__global__ void unpack_kernel(const uint8_t *__restrict__ packed, int64_t n, int64_t k, int64_t kb,
                              int8_t *__restrict__ w)
{
    const int64_t rowb = 32 * kb;
    const int64_t total = n * rowb;
    for (int64_t idx = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; idx < total;
         idx += int64_t(gridDim.x) * blockDim.x) {
        const int64_t r = idx / rowb, byte = idx - r * rowb;
        const int64_t j = byte >> 5, b = byte & 31;
        const uint32_t v = packed[idx];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const int64_t kk = 128 * j + 32 * g + b;
            if (kk < k) w[r * k + kk] = int8_t(int((v >> (2 * g)) & 3u) - 1);
        }
    }
}

// Per-token quantiser: one CTA per row.  Pass 1 finds absmax (and whether the
// row is finite), pass 2 writes rint(x * 127/amax) as int8 in natural order,
// four codes per 32-bit store, pads zero.
template <int NT>
__global__ void __launch_bounds__(NT) quant_kernel(const float *__restrict__ x, int64_t m, int64_t k,
                                                   int64_t kpad, int8_t *__restrict__ xq,
                                                   float *__restrict__ scale, int32_t *flags)
{
    __shared__ float s_max[NT / 32];
    __shared__ int s_bad[NT / 32];
    const int64_t r = blockIdx.x;
    const float *row = x + r * k;
    const bool vec = ((reinterpret_cast<uintptr_t>(row) & 15) == 0);
    const int64_t nw = kpad / 4;
    float a = 0.f;
    bool bad = false;
    auto load = [&](int64_t wi) -> float4 {
        const int64_t k0 = 4 * wi;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (vec && k0 + 3 < k) {
            v = __ldg(reinterpret_cast<const float4 *>(row + k0));
        } else {
            if (k0 + 0 < k) v.x = __ldg(row + k0 + 0);
            if (k0 + 1 < k) v.y = __ldg(row + k0 + 1);
            if (k0 + 2 < k) v.z = __ldg(row + k0 + 2);
            if (k0 + 3 < k) v.w = __ldg(row + k0 + 3);
        }
        return v;
    };
    for (int64_t wi = threadIdx.x; wi < nw; wi += NT) {
        const float4 v = load(wi);
        const bool fin = isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w);
        if (!fin) bad = true;
        else a = fmaxf(a, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
    a = warp_max(a);
    const bool wbad = __any_sync(0xffffffffu, bad);
    if ((threadIdx.x & 31) == 0) {
        s_max[threadIdx.x >> 5] = a;
        s_bad[threadIdx.x >> 5] = wbad ? 1 : 0;
    }
    __syncthreads();
    float amax = 0.f;
    int anybad = 0;
#pragma unroll
    for (int i = 0; i < NT / 32; ++i) {
        amax = fmaxf(amax, s_max[i]);
        anybad |= s_bad[i];
    }
    const bool zero = anybad || amax == 0.f;
    const float inv = zero ? 0.f : __fdiv_rn(127.0f, amax);
    uint32_t *out = reinterpret_cast<uint32_t *>(xq + r * kpad);
    for (int64_t wi = threadIdx.x; wi < nw; wi += NT) {
        uint32_t word = 0;
        if (!zero) {
            const float4 v = load(wi);
            word = pack4(quant_one(v.x, inv), quant_one(v.y, inv), quant_one(v.z, inv), quant_one(v.w, inv));
        }
        out[wi] = word;
    }
    if (threadIdx.x == 0) {
        scale[r] = zero ? 0.f : __fdiv_rn(amax, 127.0f);
        if (anybad) raise_flag(flags, BITNET_FLAG_NONFINITE);
    }
}

// ------------------------------------------------------------- absmean
// Absmean ternary quantiser fused with the pack.  The ternary weights of the
// report's §2.2.2 come from a full-precision tensor by a recipe the report
// cites but does not print; the reading taken: scale = mean |W| over the
// tensor, summed in fp64 and rounded once to fp32; w = clamp(rint(W /
// scale), -1, 1) with the quotient and the rounding in fp32 (half to even);
// an all-zero tensor gives scale 0 and w = 0; a non-finite element gives
// scale 0, w = 0 and BITNET_FLAG_NONFINITE.
//
// Two launches, each deterministic.  The first writes per-CTA fp64 partial
// sums of |W| over a fixed grid, so the summation order, hence the scale, is
// the same on every call and every device.  The second has every CTA sum the
// partials by the same fixed tree (each CTA finds the same scale; CTA 0
// publishes it) and then quantises and packs.
//
// The rounding decision without a divide.  With s > 0 the code is 0 exactly
// when rint(fl(|W| / s)) == 0, i.e. when fl(|W| / s) <= 1/2 (1/2 is even).
// Rounding is monotone and the floats next to 1/2 are 1/2 - 2^-25 and
// 1/2 + 2^-24, so fl(q) <= 1/2 exactly when the real quotient q <= 1/2 +
// 2^-25 (the midpoint rounds to the even 1/2), i.e. |W| <= s * (1/2 + 2^-25).
// That product has at most 49 significant bits and is exact in fp64, as is
// |W|, so the fp64 comparison takes the same decision as the fp32 divide
// followed by rint.  Any other quotient rounds to a nonzero integer and
// clamps to sign(W).

constexpr int kAbsmeanCtas = 1024, kAbsmeanThreads = 256, kAbsmeanPackCtasPerSm = 4;
constexpr double kHalfPlusHalfUlp = 0.5 + 0x1p-25;

struct AbsmeanScratch {
    double partial[kAbsmeanCtas];
    int32_t bad[kAbsmeanCtas];
};
static_assert(sizeof(AbsmeanScratch) <= 16384, "absmean workspace");

// Four consecutive elements 4u .. 4u+3 of the flattened tensor; positions
// past the end read as 0 (adding +0.0 leaves a sum of magnitudes unchanged,
// so the vector and scalar forms give the same sums).
__device__ __forceinline__ void load_unit(const float *__restrict__ W, int64_t total, bool vec4, int64_t u,
                                          float v[4])
{
    const int64_t e = 4 * u;
    if (vec4 && e + 3 < total) {
        const float4 f = __ldg(reinterpret_cast<const float4 *>(W + e));
        v[0] = f.x, v[1] = f.y, v[2] = f.z, v[3] = f.w;
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = e + i < total ? W[e + i] : 0.f;
    }
}

// Block-wide fp64 sum and OR of `bad` by a fixed tree (xor shuffles within
// each warp, then the warps in order); the result is valid in thread 0.
__device__ __forceinline__ void block_sum_fixed(double &s, int &bad)
{
    __shared__ double wsum[kAbsmeanThreads / 32];
    __shared__ int wbad[kAbsmeanThreads / 32];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    bad = __any_sync(0xffffffffu, bad) ? 1 : 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        wsum[warp] = s;
        wbad[warp] = bad;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        s = 0.0;
        bad = 0;
        for (int w = 0; w < kAbsmeanThreads / 32; ++w) {
            s += wsum[w];
            bad |= wbad[w];
        }
    }
}

__global__ void __launch_bounds__(kAbsmeanThreads) absmean_partial_kernel(const float *__restrict__ W, int64_t total,
                                                                       bool vec4, AbsmeanScratch *scratch)
{
    const int64_t units = (total + 3) / 4, stride = int64_t(gridDim.x) * blockDim.x;
    int64_t u = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
    double s = 0.0;
    int bad = 0;
    // four units (64 bytes) in flight per thread; the adds keep unit order
    for (; u + 3 * stride < units; u += 4 * stride) {
        float v[4][4];
#pragma unroll
        for (int q = 0; q < 4; ++q) load_unit(W, total, vec4, u + q * stride, v[q]);
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                bad |= !isfinite(v[q][i]);
                s += fabs(double(v[q][i]));
            }
    }
    for (; u < units; u += stride) {
        float v[4];
        load_unit(W, total, vec4, u, v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            bad |= !isfinite(v[i]);
            s += fabs(double(v[i]));
        }
    }
    block_sum_fixed(s, bad);
    if (threadIdx.x == 0) {
        scratch->partial[blockIdx.x] = s;
        scratch->bad[blockIdx.x] = bad;
    }
}

// One thread per packed 32-bit word: bytes 4t .. 4t+3 of block j hold, in
// field g, elements 128j + 32g + 4t + i (i = 0..3) -- four consecutive
// weights per field, read by 8 consecutive threads as 128 contiguous bytes.
__global__ void __launch_bounds__(kAbsmeanThreads) absmean_pack_kernel(
    const float *__restrict__ W, int64_t n, int64_t k, int64_t kb, bool vec4, const AbsmeanScratch *scratch,
    float *scale_out, int32_t *flags, uint32_t *__restrict__ packed)
{
    __shared__ float s_shared;
    {
        double p = 0.0;
        int bad = 0;
        for (int i = threadIdx.x; i < kAbsmeanCtas; i += kAbsmeanThreads) {
            p += scratch->partial[i];
            bad |= scratch->bad[i];
        }
        block_sum_fixed(p, bad);
        if (threadIdx.x == 0) {
            const int64_t total = n * k;
            const float s = bad ? 0.f : float(p / double(total));
            s_shared = s;
            if (blockIdx.x == 0) {
                *scale_out = s;
                if (bad) raise_flag(flags, BITNET_FLAG_NONFINITE);
            }
        }
        __syncthreads();
    }
    const float s = s_shared;
    const double zero_below = double(s) * kHalfPlusHalfUlp;   // |W| <= this  <=>  code 0
    const int64_t row_words = 8 * kb, total_words = n * row_words;
    for (int64_t idx = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; idx < total_words;
         idx += int64_t(gridDim.x) * blockDim.x) {
        const int64_t r = idx / row_words, wi = idx - r * row_words;
        const int64_t j = wi >> 3, t = wi & 7;
        const float *wr = W + r * k;
        uint32_t out = 0;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const int64_t k0 = 128 * j + 32 * g + 4 * t;
            float v[4];
            if (vec4 && k0 + 3 < k) {
                const float4 f = __ldg(reinterpret_cast<const float4 *>(wr + k0));
                v[0] = f.x, v[1] = f.y, v[2] = f.z, v[3] = f.w;
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) v[i] = k0 + i < k ? wr[k0 + i] : 0.f;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                // weight 0 for tails, for every weight when s == 0, and for |W| <= s/2
                uint32_t code = 1;
                if (k0 + i < k && s != 0.f && fabs(double(v[i])) > zero_below) code = v[i] > 0.f ? 2u : 0u;
                out |= code << (8 * i + 2 * g);
            }
        }
        packed[idx] = out;
    }
}

static int grid_for(int64_t work, int threads)
{
    int64_t g = (work + threads - 1) / threads;
    if (g > 148 * 32) g = 148 * 32;
    return int(g < 1 ? 1 : g);
}

cudaError_t launch_pack(const int8_t *w, int64_t n, int64_t k, uint8_t *packed, int32_t *flags, cudaStream_t st)
{
    const int64_t kb = (k + 127) / 128;
    pack_kernel<<<grid_for(n * 32 * kb, 256), 256, 0, st>>>(w, n, k, kb, packed, flags);
    return cudaGetLastError();
}

cudaError_t launch_unpack(const uint8_t *packed, int64_t n, int64_t k, int8_t *w, cudaStream_t st)
{
    const int64_t kb = (k + 127) / 128;
    unpack_kernel<<<grid_for(n * 32 * kb, 256), 256, 0, st>>>(packed, n, k, kb, w);
    return cudaGetLastError();
}

cudaError_t launch_quant(const float *x, int64_t m, int64_t k, int8_t *xq, float *scale, int32_t *flags,
                         cudaStream_t st)
{
    const int64_t kpad = 128 * ((k + 127) / 128);
    quant_kernel<256><<<unsigned(m), 256, 0, st>>>(x, m, k, kpad, xq, scale, flags);
    return cudaGetLastError();
}

cudaError_t launch_quantize_pack(const float *w, int64_t n, int64_t k, uint8_t *packed, float *scale, void *workspace,
                                 int32_t *flags, int sm_count, cudaStream_t st)
{
    const int64_t kb = (k + 127) / 128, words = n * 8 * kb;
    auto *scratch = static_cast<AbsmeanScratch *>(workspace);
    const bool aligned16 = (reinterpret_cast<uintptr_t>(w) & 15) == 0;
    absmean_partial_kernel<<<kAbsmeanCtas, kAbsmeanThreads, 0, st>>>(w, n * k, aligned16, scratch);
    // the pack's float4 loads need every row start 16-byte aligned: W aligned and k % 4 == 0
    const int64_t want = (words + kAbsmeanThreads - 1) / kAbsmeanThreads;
    const int grid = int(want < int64_t(kAbsmeanPackCtasPerSm) * sm_count ? want : int64_t(kAbsmeanPackCtasPerSm) * sm_count);
    absmean_pack_kernel<<<grid, kAbsmeanThreads, 0, st>>>(w, n, k, kb, aligned16 && k % 4 == 0, scratch, scale,
                                                          flags, reinterpret_cast<uint32_t *>(packed));
    return cudaGetLastError();
}

}  // namespace bitnet
