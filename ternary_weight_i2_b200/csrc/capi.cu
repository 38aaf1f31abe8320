// capi.cu -- the C ABI declared in include/bitnet.h: argument checks, the
// device check, work partitioning for the streaming GEMV, and dispatch.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "common.cuh"
#include "gemv_i8.cuh"
#include "gemv.cuh"

namespace bitnet {
cudaError_t launch_gemv(const GemvParams &p, int variant, cudaStream_t st);
cudaError_t launch_pack(const int8_t *w, int64_t n, int64_t k, uint8_t *packed, int32_t *flags, cudaStream_t st);
cudaError_t launch_unpack(const uint8_t *packed, int64_t n, int64_t k, int8_t *w, cudaStream_t st);
cudaError_t launch_quant(const float *x, int64_t m, int64_t k, int8_t *xq, float *scale, int32_t *flags,
                         cudaStream_t st);
cudaError_t launch_quantize_pack(const float *w, int64_t n, int64_t k, uint8_t *packed, float *scale, void *workspace,
                                 int32_t *flags, int sm_count, cudaStream_t st);
bool gemm_available();
cudaError_t launch_gemv_i8(const int8_t *w, int64_t n, int64_t k, float s_w, const int8_t *q, const float *s_act,
                           int64_t m, const bitnet_epilogue *e, float *y, int32_t *acc, int sm_count,
                           cudaStream_t st);

cudaError_t launch_gemm(const int8_t *xq, const float *act_scale, int64_t m, const bitnet_tw *w,
                        const bitnet_epilogue *epi, float *y, int32_t *acc, int32_t *flags, uint64_t wait_limit,
                        int force_stall, int sm_count, uint64_t *trace, cudaStream_t st);
cudaError_t launch_gemm_grouped(const int8_t *const *xq, const float *const *act_scale, int64_t m,
                                const bitnet_tw *w, const bitnet_epilogue *epi, int count, float *const *y,
                                int32_t *const *acc, int32_t *flags, uint64_t wait_limit, int force_stall,
                                int sm_count, uint64_t *trace, cudaStream_t st);
}  // namespace bitnet

using namespace bitnet;

namespace {

thread_local char g_err[512] = "";
uint64_t g_wait_limit = 0;   // 0: built-in bound
int g_force_stall = 0;       // test aid: kernels wait on a barrier nobody arrives at
uint64_t *g_trace = nullptr; // optional device buffer for per-warp phase timestamps

bitnet_status fail(bitnet_status s, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

bitnet_status cuda_fail(cudaError_t e, const char *what)
{
    return fail(BITNET_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int64_t blocks_of(int64_t k) { return (k + 127) / 128; }

struct DevInfo {
    int sm_count = 0;
    int ordinal = 0;
    bool ok = false;
};

// Device check: the kernels are built for sm_100a only, so any other device
// is refused up front instead of running a kernel image that is not there.
// BITNET_TEST_FORCE_SM (test aid) overrides the detected "major*10+minor".
bitnet_status check_device(DevInfo *info)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    static DevInfo cache[64];
    static bool cached[64] = {false};
    if (dev < 0 || dev >= 64) return fail(BITNET_ERR_UNSUPPORTED_DEVICE, "device ordinal %d out of range", dev);
    int major = 0, minor = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    int sm = major * 10 + minor;
    if (const char *f = getenv("BITNET_TEST_FORCE_SM")) sm = atoi(f);
    if (sm != 100)
        return fail(BITNET_ERR_UNSUPPORTED_DEVICE, "device %d is sm_%d; this library runs on sm_100 (B200) only",
                    dev, sm);
    if (!cached[dev]) {
        int n = 0;
        e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
        cache[dev].sm_count = n;
        cache[dev].ordinal = dev;
        cache[dev].ok = true;
        cached[dev] = true;
    }
    *info = cache[dev];
    return BITNET_OK;
}

bitnet_status check_tw(const bitnet_tw &w, int64_t i)
{
    if (!w.packed) return fail(BITNET_ERR_INVALID_ARG, "layer %lld: packed is NULL", (long long)i);
    if (!aligned(w.packed, 16)) return fail(BITNET_ERR_INVALID_ARG, "layer %lld: packed not 16-byte aligned", (long long)i);
    if (w.n < 1 || w.n > (int64_t(1) << 30))
        return fail(BITNET_ERR_INVALID_ARG, "layer %lld: n=%lld out of range", (long long)i, (long long)w.n);
    if (w.k < 1 || w.k > BITNET_MAX_K)
        return fail(BITNET_ERR_INVALID_ARG, "layer %lld: k=%lld out of range [1, %d]", (long long)i, (long long)w.k,
                    BITNET_MAX_K);
    return BITNET_OK;
}

// A fused-epilogue descriptor (may be NULL: no epilogue).
bitnet_status check_epi(const bitnet_epilogue *e, int64_t i)
{
    if (!e) return BITNET_OK;
    if (e->reserved != 0) return fail(BITNET_ERR_INVALID_ARG, "layer %lld: epilogue reserved field not 0", (long long)i);
    if (!aligned(e->bias, 4) || !aligned(e->gamma, 4) || !aligned(e->residual, 4))
        return fail(BITNET_ERR_INVALID_ARG, "layer %lld: epilogue operand not 4-byte aligned", (long long)i);
    return BITNET_OK;
}

uint64_t wait_limit() { return g_wait_limit ? g_wait_limit : kDefaultWaitLimit; }

// ------------------------------------------------------- tensor-map cache
//
// The GEMV streams each packed weight matrix through a 2-D tiled TMA tensor
// map (uint8, dims {32*kb bytes, n rows}, box {128, 32}, 128-byte swizzle,
// zero fill out of bounds).  A map depends only on (address, n, kb), so maps
// are encoded once on the host and kept, per device, in device memory that
// lives until bitnet_release_device_cache() or process exit.  The first call
// that meets a new weight tensor allocates and copies (it must not run under
// stream capture); later calls only look the map up.

struct TmapKey {
    const void *p;
    int64_t n, kb;
    bool operator==(const TmapKey &o) const { return p == o.p && n == o.n && kb == o.kb; }
};
struct TmapKeyHash {
    size_t operator()(const TmapKey &k) const
    {
        return std::hash<const void *>()(k.p) ^ (std::hash<int64_t>()(k.n) * 31u) ^ (std::hash<int64_t>()(k.kb) * 131u);
    }
};
constexpr int kTmapChunk = 1024;
struct TmapChunk {
    CUtensorMap *dev = nullptr;
    CUtensorMap *host = nullptr;   // pinned mirror, each entry written once
    int used = 0;
};
struct DeviceTmaps {
    std::unordered_map<TmapKey, const CUtensorMap *, TmapKeyHash> index;
    std::vector<TmapChunk> chunks;
};
std::mutex g_tmap_mu;
DeviceTmaps g_tmaps[64];
uint64_t g_tmap_generation = 1;   // bumped when a cache is released

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
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

bitnet_status encode_weight_map(CUtensorMap *out, const void *packed, int64_t n, int64_t kb)
{
    auto fn = encode_fn();
    if (!fn) return fail(BITNET_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const cuuint64_t dims[2] = {cuuint64_t(32 * kb), cuuint64_t(n)};
    const cuuint64_t strides[1] = {cuuint64_t(32 * kb)};
    const cuuint32_t box[2] = {128u, cuuint32_t(kTileRows)};
    const cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(out, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(packed), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(BITNET_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
    return BITNET_OK;
}

// Device tensor maps of `count` weight tensors; new ones are encoded and
// copied in one batch per chunk.
bitnet_status weight_maps(int dev, const bitnet_tw *const *w, int count, const void **out)
{
    std::lock_guard<std::mutex> lock(g_tmap_mu);
    DeviceTmaps &D = g_tmaps[dev];
    std::vector<std::pair<int, int>> fresh;   // (chunk, first new entry)
    for (int i = 0; i < count; ++i) {
        const TmapKey key{w[i]->packed, w[i]->n, blocks_of(w[i]->k)};
        auto it = D.index.find(key);
        if (it != D.index.end()) {
            out[i] = it->second;
            continue;
        }
        if (D.chunks.empty() || D.chunks.back().used == kTmapChunk) {
            TmapChunk c;
            cudaError_t e = cudaMalloc(&c.dev, kTmapChunk * sizeof(CUtensorMap));
            if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(tensor-map cache)");
            e = cudaMallocHost(&c.host, kTmapChunk * sizeof(CUtensorMap));
            if (e != cudaSuccess) {
                cudaFree(c.dev);
                return cuda_fail(e, "cudaMallocHost(tensor-map cache)");
            }
            D.chunks.push_back(c);
        }
        TmapChunk &c = D.chunks.back();
        const int ci = int(D.chunks.size()) - 1;
        if (fresh.empty() || fresh.back().first != ci) fresh.emplace_back(ci, c.used);
        bitnet_status s = encode_weight_map(&c.host[c.used], key.p, key.n, key.kb);
        if (s != BITNET_OK) return s;
        const CUtensorMap *d = c.dev + c.used;
        ++c.used;
        D.index.emplace(key, d);
        out[i] = d;
    }
    for (auto &f : fresh) {
        TmapChunk &c = D.chunks[f.first];
        cudaError_t e = cudaMemcpy(c.dev + f.second, c.host + f.second, size_t(c.used - f.second) * sizeof(CUtensorMap),
                                   cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_fail(e, "tensor-map upload");
    }
    return BITNET_OK;
}

// ---------------------------------------------------------------- GEMV plan

struct LayerReq {
    const void *x;         // this slice's activation rows (fp32, or int8 when prequant)
    const float *xscale;   // prequant: per-token scales
    bitnet_tw w;
    float *y;
    int32_t *acc;
    const float *bias;     // fused epilogue operands (null when absent)
    const float *gamma;
    const float *res;      // this slice's residual rows
    int64_t relu;
};

// Kernel variant for m tokens whose activation area holds an input of
// max_kpad columns; BITNET_TEST_GEMV_VARIANT (tuning aid) forces one.
int pick_variant(int m, int64_t max_kpad)
{
    static const int pref[9][4] = {{-1}, {0, 1, 3, -1}, {0, 2, 3, -1}, {2, 3, -1}, {2, 3, -1}, {2, 3, -1},
                                   {3, -1}, {3, -1}, {3, -1}};
    if (const char *f = getenv("BITNET_TEST_GEMV_VARIANT")) {
        const int v = atoi(f);
        if (v >= 0 && v < kNumVariants && m <= kVariantMaxM[v] &&
            int64_t(m) * max_kpad <= x_cap(kVariants[v].nw, kVariants[v].boxes))
            return v;
    }
    for (int i = 0; i < 4 && pref[m][i] >= 0; ++i) {
        const int v = pref[m][i];
        if (int64_t(m) * max_kpad <= x_cap(kVariants[v].nw, kVariants[v].boxes)) return v;
    }
    return -1;
}

// Plans of recent launches, reused when a call repeats its arguments exactly
// (decode loops call the same stack with the same buffers every step).
struct PlanKey {
    std::vector<LayerReq> layers;
    int m = 0;
    bool prequant = false;
    int32_t *flags = nullptr;
    int ordinal = -1;
    uint64_t generation = 0, wait_limit = 0;
    int force_stall = 0;
    uint64_t *trace = nullptr;
    bool matches(const std::vector<LayerReq> &L, int m_, bool pq, int32_t *fl, int dev, uint64_t gen) const
    {
        if (m != m_ || prequant != pq || flags != fl || ordinal != dev || generation != gen ||
            wait_limit != g_wait_limit || force_stall != g_force_stall ||
            trace != g_trace || layers.size() != L.size())
            return false;
        return std::memcmp(layers.data(), L.data(), L.size() * sizeof(LayerReq)) == 0;
    }
};
struct CachedPlan {
    PlanKey key;
    GemvParams params;
    int variant = -1;
};
constexpr int kPlanCacheSize = 8;
thread_local std::vector<CachedPlan> g_plans;
thread_local int g_plan_next = 0;

// Split the layers' 32-row tiles into contiguous ranges, one CTA each: tile
// t goes to range floor((bytes before t + half of t) * G / total), so every
// range holds within half a tile of total/G bytes (G = SM count).  A range is
// split further when it would exceed a per-CTA limit (distinct inputs,
// segments, shared memory for the quantised activations).
bitnet_status plan_and_launch(const std::vector<LayerReq> &L, int m, bool prequant, int32_t *flags,
                              cudaStream_t st, const DevInfo &dev)
{
    uint64_t gen;
    {
        std::lock_guard<std::mutex> lock(g_tmap_mu);
        gen = g_tmap_generation;
    }
    for (const CachedPlan &c : g_plans)
        if (c.key.matches(L, m, prequant, flags, dev.ordinal, gen)) {
            cudaError_t e = launch_gemv(c.params, c.variant, st);
            return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "gemv launch");
        }
    if (int(g_plans.size()) < kPlanCacheSize) g_plans.emplace_back();
    CachedPlan &slot_plan = g_plans[g_plan_next];
    g_plan_next = (g_plan_next + 1) % kPlanCacheSize;
    slot_plan.variant = -1;   // invalid until the plan below succeeds
    GemvParams &p = slot_plan.params;
    static thread_local std::vector<int> input_of;
    const int count = int(L.size());
    {
        static thread_local std::vector<const bitnet_tw *> wp;
        static thread_local std::vector<const void *> maps;
        wp.resize(count);
        maps.resize(count);
        for (int i = 0; i < count; ++i) wp[i] = &L[i].w;
        bitnet_status s = weight_maps(dev.ordinal, wp.data(), count, maps.data());
        if (s != BITNET_OK) return s;
        for (int i = 0; i < count; ++i) p.lin[i].tmap = maps[i];
    }
    int ninp = 0;
    input_of.assign(count, -1);
    int64_t max_kpad = 0;
    for (int i = 0; i < count; ++i) {
        int found = -1;
        for (int j = 0; j < ninp; ++j)
            if (p.inp[j].x == L[i].x && p.inp[j].k == int32_t(L[i].w.k) && p.inp[j].scale == L[i].xscale) {
                found = j;
                break;
            }
        if (found < 0) {
            if (ninp == kMaxInputs) return fail(BITNET_ERR_INVALID_ARG, "more than %d distinct inputs", kMaxInputs);
            found = ninp++;
            p.inp[found].x = L[i].x;
            p.inp[found].scale = L[i].xscale;
            p.inp[found].k = int32_t(L[i].w.k);
            p.inp[found].kb = int32_t(blocks_of(L[i].w.k));
        }
        input_of[i] = found;
        const int64_t kp = 128 * blocks_of(L[i].w.k);
        if (kp > max_kpad) max_kpad = kp;
        p.lin[i].y = L[i].y;
        p.lin[i].acc = L[i].acc;
        p.lin[i].n = int32_t(L[i].w.n);
        p.lin[i].kb = int32_t(blocks_of(L[i].w.k));
        p.lin[i].scale = L[i].w.scale;
        p.lin[i].input = int16_t(found);
        p.lin[i].bias = L[i].bias;
        p.lin[i].gamma = L[i].gamma;
        p.lin[i].res = L[i].res;
        p.lin[i].relu = L[i].relu ? 1 : 0;
    }
    p.has_epi = 0;
    for (int i = 0; i < count; ++i)
        if (L[i].bias || L[i].gamma || L[i].res || L[i].relu) p.has_epi = 1;
    const int variant = pick_variant(m, max_kpad);
    if (variant < 0)
        return fail(BITNET_ERR_INVALID_ARG, "m=%d x kpad=%lld exceeds the GEMV activation area", m,
                    (long long)max_kpad);
    const int64_t xcap = x_cap(kVariants[variant].nw, kVariants[variant].boxes);

    int64_t total = 0;
    for (int i = 0; i < count; ++i) total += L[i].w.n * 32 * blocks_of(L[i].w.k);
    const int64_t G = dev.sm_count;

    int nr = 0, ns = 0;
    int64_t cur_x = 0, xmax = 0, cum = 0;
    int cur_target = -1;   // balanced-range index the open range belongs to
    bool open = false;
    auto close_range = [&]() {
        if (open && p.rng[nr].nseg > 0) {
            xmax = cur_x > xmax ? cur_x : xmax;
            ++nr;
        }
        open = false;
    };
    for (int i = 0; i < count; ++i) {
        const int64_t rowb = 32 * blocks_of(L[i].w.k);
        const int64_t tiles = (L[i].w.n + kTileRows - 1) / kTileRows;
        const int64_t xin = int64_t(m) * 128 * blocks_of(L[i].w.k);
        for (int64_t t = 0; t < tiles; ++t) {
            const int64_t rows = (t + 1 < tiles) ? kTileRows : L[i].w.n - t * kTileRows;
            const int64_t tb = rows * rowb;
            const int target = int((cum + tb / 2) * G / total);
            cum += tb;
            if (open && target != cur_target) close_range();
            for (;;) {
                if (!open) {
                    if (nr == kMaxRanges) return fail(BITNET_ERR_INVALID_ARG, "stack needs more than %d CTAs", kMaxRanges);
                    GemvRange &r = p.rng[nr];
                    r.seg0 = int16_t(ns);
                    r.nseg = 0;
                    r.nin = 0;
                    cur_x = 0;
                    cur_target = target;
                    open = true;
                }
                GemvRange &r = p.rng[nr];
                int slot = -1;
                for (int u = 0; u < r.nin; ++u)
                    if (r.in[u] == input_of[i]) slot = u;
                const bool same_seg = r.nseg > 0 && p.seg[ns - 1].lin == i && p.seg[ns - 1].tile1 == t;
                const bool need_in = slot < 0;
                const bool need_seg = !same_seg;
                if ((need_in && (r.nin == kMaxRangeInputs || cur_x + xin > xcap)) ||
                    (need_seg && (r.nseg == kMaxRangeSegs || ns == kMaxSegs))) {
                    if (r.nseg == 0 || ns == kMaxSegs)
                        return fail(BITNET_ERR_INVALID_ARG, "stack too large for one launch (%d segments)", ns);
                    close_range();
                    continue;
                }
                if (need_in) {
                    slot = r.nin;
                    r.in[r.nin++] = int16_t(input_of[i]);
                    cur_x += xin;
                }
                if (need_seg) {
                    GemvSeg &sg = p.seg[ns++];
                    sg.lin = int16_t(i);
                    sg.slot = int16_t(slot);
                    sg.tile0 = int32_t(t);
                    sg.tile1 = int32_t(t + 1);
                    r.nseg++;
                } else {
                    p.seg[ns - 1].tile1 = int32_t(t + 1);
                }
                break;
            }
        }
    }
    close_range();
    p.m = m;
    p.num_ranges = nr;
    p.prequant = prequant ? 1 : 0;
    p.force_stall = g_force_stall;
    p.flags = flags;
    p.wait_limit = wait_limit();
    p.trace = g_trace;
    p.x_bytes = int32_t((xmax + 127) / 128 * 128);
    // cache entries are never rewritten, but after a release a new chunk can
    // reuse the address of a freed one
    p.fence_maps = gen > 1 ? 1 : 0;
    cudaError_t e = launch_gemv(p, variant, st);
    if (e != cudaSuccess) return cuda_fail(e, "gemv launch");
    slot_plan.variant = variant;
    slot_plan.key.layers = L;
    slot_plan.key.m = m;
    slot_plan.key.prequant = prequant;
    slot_plan.key.flags = flags;
    slot_plan.key.ordinal = dev.ordinal;
    slot_plan.key.generation = gen;
    slot_plan.key.wait_limit = g_wait_limit;
    slot_plan.key.force_stall = g_force_stall;
    slot_plan.key.trace = g_trace;
    return BITNET_OK;
}

}  // namespace

extern "C" {

int bitnet_version(void) { return 100; }

const char *bitnet_status_str(bitnet_status s)
{
    switch (s) {
    case BITNET_OK: return "ok";
    case BITNET_ERR_INVALID_ARG: return "invalid argument";
    case BITNET_ERR_NOT_TERNARY: return "weight outside {-1,0,+1}";
    case BITNET_ERR_UNSUPPORTED_DEVICE: return "unsupported device (needs sm_100)";
    case BITNET_ERR_CUDA: return "CUDA error";
    case BITNET_ERR_NONFINITE: return "non-finite activation";
    case BITNET_ERR_TIMEOUT: return "device-side wait timed out";
    case BITNET_ERR_WORKSPACE: return "workspace too small";
    }
    return "unknown status";
}

const char *bitnet_last_error(void) { return g_err; }

bitnet_status bitnet_status_from_flags(int32_t flags)
{
    if (flags & BITNET_FLAG_TIMEOUT) return BITNET_ERR_TIMEOUT;
    if (flags & BITNET_FLAG_NONFINITE) return BITNET_ERR_NONFINITE;
    if (flags & BITNET_FLAG_NOT_TERNARY) return BITNET_ERR_NOT_TERNARY;
    return BITNET_OK;
}

size_t bitnet_packed_bytes(int64_t n, int64_t k)
{
    if (n < 1 || k < 1 || k > BITNET_MAX_K) return 0;
    return size_t(n) * size_t(32 * blocks_of(k));
}

int64_t bitnet_kpad(int64_t k)
{
    if (k < 1 || k > BITNET_MAX_K) return 0;
    return 128 * blocks_of(k);
}

bitnet_status bitnet_debug_set_wait_limit(uint64_t cycles)
{
    g_wait_limit = cycles;
    return BITNET_OK;
}

bitnet_status bitnet_release_device_cache(void)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) return fail(BITNET_ERR_UNSUPPORTED_DEVICE, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_tmap_mu);
    DeviceTmaps &D = g_tmaps[dev];
    e = cudaDeviceSynchronize();
    for (auto &c : D.chunks) {
        cudaFree(c.dev);
        cudaFreeHost(c.host);
    }
    D.chunks.clear();
    D.index.clear();
    ++g_tmap_generation;
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "cudaDeviceSynchronize");
}

bitnet_status bitnet_debug_set_trace(void *d_trace)
{
    g_trace = static_cast<uint64_t *>(d_trace);
    return BITNET_OK;
}

bitnet_status bitnet_debug_force_stall(int on)
{
    g_force_stall = on ? 1 : 0;
    return BITNET_OK;
}

bitnet_status bitnet_pack_ternary(const int8_t *w, int64_t n, int64_t k, uint8_t *packed, int32_t *d_flags,
                                  void *stream)
{
    if (!w || !packed) return fail(BITNET_ERR_INVALID_ARG, "pack: NULL pointer");
    if (n < 1 || k < 1 || k > BITNET_MAX_K) return fail(BITNET_ERR_INVALID_ARG, "pack: bad sizes n=%lld k=%lld",
                                                        (long long)n, (long long)k);
    if (!aligned(packed, 16)) return fail(BITNET_ERR_INVALID_ARG, "pack: packed not 16-byte aligned");
    DevInfo dev;
    bitnet_status s = check_device(&dev);
    if (s != BITNET_OK) return s;
    cudaError_t e = launch_pack(w, n, k, packed, d_flags, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "pack launch");
}

size_t bitnet_quantize_pack_workspace_bytes(void) { return 16384; }

bitnet_status bitnet_quantize_pack(const float *w, int64_t n, int64_t k, uint8_t *packed, float *d_scale,
                                   void *workspace, size_t workspace_bytes, int32_t *d_flags, void *stream)
{
    if (!w || !packed || !d_scale || !workspace) return fail(BITNET_ERR_INVALID_ARG, "quantize_pack: NULL pointer");
    if (n < 1 || k < 1 || k > BITNET_MAX_K)
        return fail(BITNET_ERR_INVALID_ARG, "quantize_pack: bad sizes n=%lld k=%lld", (long long)n, (long long)k);
    if (!aligned(w, 4) || !aligned(packed, 16) || !aligned(d_scale, 4) || !aligned(workspace, 8))
        return fail(BITNET_ERR_INVALID_ARG, "quantize_pack: misaligned pointer");
    if (workspace_bytes < bitnet_quantize_pack_workspace_bytes())
        return fail(BITNET_ERR_WORKSPACE, "quantize_pack: workspace %zu < %zu bytes", workspace_bytes,
                    bitnet_quantize_pack_workspace_bytes());
    DevInfo dev;
    bitnet_status s = check_device(&dev);
    if (s != BITNET_OK) return s;
    cudaError_t e = launch_quantize_pack(w, n, k, packed, d_scale, workspace, d_flags, dev.sm_count,
                                         static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "quantize_pack launch");
}

bitnet_status bitnet_unpack_ternary(const uint8_t *packed, int64_t n, int64_t k, int8_t *w, void *stream)
{
    if (!w || !packed) return fail(BITNET_ERR_INVALID_ARG, "unpack: NULL pointer");
    if (n < 1 || k < 1 || k > BITNET_MAX_K) return fail(BITNET_ERR_INVALID_ARG, "unpack: bad sizes");
    DevInfo dev;
    bitnet_status s = check_device(&dev);
    if (s != BITNET_OK) return s;
    cudaError_t e = launch_unpack(packed, n, k, w, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "unpack launch");
}

bitnet_status bitnet_quant_act(const float *x, int64_t m, int64_t k, int8_t *xq, float *act_scale,
                               int32_t *d_flags, void *stream)
{
    if (!x || !xq || !act_scale) return fail(BITNET_ERR_INVALID_ARG, "quant: NULL pointer");
    if (m < 1 || m > (int64_t(1) << 31) - 1 || k < 1 || k > BITNET_MAX_K)
        return fail(BITNET_ERR_INVALID_ARG, "quant: bad sizes m=%lld k=%lld", (long long)m, (long long)k);
    if (!aligned(x, 16) || !aligned(xq, 16)) return fail(BITNET_ERR_INVALID_ARG, "quant: x/xq not 16-byte aligned");
    DevInfo dev;
    bitnet_status s = check_device(&dev);
    if (s != BITNET_OK) return s;
    cudaError_t e = launch_quant(x, m, k, xq, act_scale, d_flags, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "quant launch");
}

size_t bitnet_linear_workspace_bytes(int64_t m, int64_t k)
{
    if (m < 1 || k < 1 || k > BITNET_MAX_K) return 0;
    if (m <= BITNET_GEMV_MAX_M) return 0;
    const size_t a = size_t(m) * size_t(128 * blocks_of(k));
    return (a + 255) / 256 * 256 + size_t(m) * sizeof(float);
}

static bitnet_status gemv_slices(const float *const *x, const int8_t *const *xq, const float *const *xs, int64_t m,
                                 const bitnet_tw *w, const bitnet_epilogue *epi, int64_t count, float *const *y,
                                 int32_t *const *acc, int32_t *d_flags, cudaStream_t st, const DevInfo &dev)
{
    std::vector<LayerReq> L;
    L.resize(static_cast<size_t>(count));
    std::memset(static_cast<void *>(L.data()), 0, L.size() * sizeof(LayerReq));   // plan keys compare bytes
    for (int64_t m0 = 0; m0 < m; m0 += BITNET_GEMV_MAX_M) {
        const int ms = int((m - m0) < BITNET_GEMV_MAX_M ? (m - m0) : BITNET_GEMV_MAX_M);
        for (int64_t i = 0; i < count; ++i) {
            const int64_t kpad = 128 * blocks_of(w[i].k);
            if (xq) {
                L[i].x = xq[i] + m0 * kpad;
                L[i].xscale = xs[i] + m0;
            } else {
                L[i].x = x[i] + m0 * w[i].k;
                L[i].xscale = nullptr;
            }
            L[i].w = w[i];
            L[i].y = y[i] + m0 * w[i].n;
            L[i].acc = (acc && acc[i]) ? acc[i] + m0 * w[i].n : nullptr;
            L[i].bias = epi ? epi[i].bias : nullptr;
            L[i].gamma = epi ? epi[i].gamma : nullptr;
            L[i].res = (epi && epi[i].residual) ? epi[i].residual + m0 * w[i].n : nullptr;
            L[i].relu = (epi && epi[i].relu) ? 1 : 0;
        }
        bitnet_status s = plan_and_launch(L, ms, xq != nullptr, d_flags, st, dev);
        if (s != BITNET_OK) return s;
    }
    return BITNET_OK;
}

bitnet_status bitnet_linear_ex(const float *x, int64_t m, const bitnet_tw *w, const bitnet_epilogue *epi, float *y,
                               int32_t *acc_out, void *workspace, size_t workspace_bytes, int32_t *d_flags,
                               void *stream)
{
    if (!x || !w || !y) return fail(BITNET_ERR_INVALID_ARG, "linear: NULL pointer");
    if (m < 1 || m > (int64_t(1) << 31) - 1) return fail(BITNET_ERR_INVALID_ARG, "linear: bad m=%lld", (long long)m);
    bitnet_status s = check_tw(*w, 0);
    if (s != BITNET_OK) return s;
    s = check_epi(epi, 0);
    if (s != BITNET_OK) return s;
    if (!aligned(x, 16)) return fail(BITNET_ERR_INVALID_ARG, "linear: x not 16-byte aligned");
    const size_t need = bitnet_linear_workspace_bytes(m, w->k);
    if (need > 0 && (!workspace || workspace_bytes < need))
        return fail(BITNET_ERR_WORKSPACE, "linear: workspace of %zu bytes needed, %zu given", need, workspace_bytes);
    if (need > 0 && !aligned(workspace, 256)) return fail(BITNET_ERR_INVALID_ARG, "linear: workspace not 256-byte aligned");
    DevInfo dev;
    s = check_device(&dev);
    if (s != BITNET_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (m <= BITNET_GEMV_MAX_M || !gemm_available()) {
        if (need > 0) {
            // quantise once into the workspace, then stream in token slices
            int8_t *xq = static_cast<int8_t *>(workspace);
            const size_t qa = (size_t(m) * size_t(128 * blocks_of(w->k)) + 255) / 256 * 256;
            float *xs = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + qa);
            cudaError_t e = launch_quant(x, m, w->k, xq, xs, d_flags, st);
            if (e != cudaSuccess) return cuda_fail(e, "quant launch");
            const int8_t *xqa[1] = {xq};
            const float *xsa[1] = {xs};
            float *ya[1] = {y};
            int32_t *aa[1] = {acc_out};
            return gemv_slices(nullptr, xqa, xsa, m, w, epi, 1, ya, aa, d_flags, st, dev);
        }
        const float *xa[1] = {x};
        float *ya[1] = {y};
        int32_t *aa[1] = {acc_out};
        return gemv_slices(xa, nullptr, nullptr, m, w, epi, 1, ya, aa, d_flags, st, dev);
    }
    int8_t *xq = static_cast<int8_t *>(workspace);
    const size_t qa = (size_t(m) * size_t(128 * blocks_of(w->k)) + 255) / 256 * 256;
    float *xs = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + qa);
    cudaError_t e = launch_quant(x, m, w->k, xq, xs, d_flags, st);
    if (e != cudaSuccess) return cuda_fail(e, "quant launch");
    e = launch_gemm(xq, xs, m, w, epi, y, acc_out, d_flags, wait_limit(), g_force_stall, dev.sm_count, g_trace, st);
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "gemm launch");
}

bitnet_status bitnet_linear(const float *x, int64_t m, const bitnet_tw *w, float *y, int32_t *acc_out,
                            void *workspace, size_t workspace_bytes, int32_t *d_flags, void *stream)
{
    return bitnet_linear_ex(x, m, w, nullptr, y, acc_out, workspace, workspace_bytes, d_flags, stream);
}

bitnet_status bitnet_linear_q_ex(const int8_t *xq, const float *act_scale, int64_t m, const bitnet_tw *w,
                                 const bitnet_epilogue *epi, float *y, int32_t *acc_out, int32_t *d_flags,
                                 void *stream)
{
    if (!xq || !act_scale || !w || !y) return fail(BITNET_ERR_INVALID_ARG, "linear_q: NULL pointer");
    if (m < 1 || m > (int64_t(1) << 31) - 1) return fail(BITNET_ERR_INVALID_ARG, "linear_q: bad m");
    bitnet_status s = check_tw(*w, 0);
    if (s != BITNET_OK) return s;
    s = check_epi(epi, 0);
    if (s != BITNET_OK) return s;
    if (!aligned(xq, 16)) return fail(BITNET_ERR_INVALID_ARG, "linear_q: xq not 16-byte aligned");
    DevInfo dev;
    s = check_device(&dev);
    if (s != BITNET_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (m <= BITNET_GEMV_MAX_M || !gemm_available()) {
        const int8_t *xqa[1] = {xq};
        const float *xsa[1] = {act_scale};
        float *ya[1] = {y};
        int32_t *aa[1] = {acc_out};
        return gemv_slices(nullptr, xqa, xsa, m, w, epi, 1, ya, aa, d_flags, st, dev);
    }
    cudaError_t e = launch_gemm(xq, act_scale, m, w, epi, y, acc_out, d_flags, wait_limit(), g_force_stall,
                                dev.sm_count, g_trace, st);
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "gemm launch");
}

bitnet_status bitnet_linear_q(const int8_t *xq, const float *act_scale, int64_t m, const bitnet_tw *w, float *y,
                              int32_t *acc_out, int32_t *d_flags, void *stream)
{
    return bitnet_linear_q_ex(xq, act_scale, m, w, nullptr, y, acc_out, d_flags, stream);
}

bitnet_status bitnet_linear_q_grouped_ex(const int8_t *const *xq, const float *const *act_scale, int64_t m,
                                         const bitnet_tw *w, const bitnet_epilogue *epi, int64_t count,
                                         float *const *y, int32_t *const *acc_out, int32_t *d_flags, void *stream)
{
    if (!xq || !act_scale || !w || !y) return fail(BITNET_ERR_INVALID_ARG, "linear_q_grouped: NULL array");
    if (count < 1 || count > BITNET_GROUP_MAX)
        return fail(BITNET_ERR_INVALID_ARG, "linear_q_grouped: count=%lld out of range [1, %d]", (long long)count,
                    BITNET_GROUP_MAX);
    if (m < 1 || m > (int64_t(1) << 31) - 1) return fail(BITNET_ERR_INVALID_ARG, "linear_q_grouped: bad m");
    for (int64_t i = 0; i < count; ++i) {
        bitnet_status s = check_tw(w[i], i);
        if (s != BITNET_OK) return s;
        if (!xq[i] || !act_scale[i] || !y[i])
            return fail(BITNET_ERR_INVALID_ARG, "linear_q_grouped: layer %lld has a NULL pointer", (long long)i);
        if (!aligned(xq[i], 16) || !aligned(y[i], 16))
            return fail(BITNET_ERR_INVALID_ARG, "linear_q_grouped: layer %lld xq or y not 16-byte aligned",
                        (long long)i);
        if (epi) {
            s = check_epi(epi + i, i);
            if (s != BITNET_OK) return s;
        }
    }
    DevInfo dev;
    bitnet_status s = check_device(&dev);
    if (s != BITNET_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (m <= BITNET_GEMV_MAX_M)
        return gemv_slices(nullptr, xq, act_scale, m, w, epi, count, y, acc_out, d_flags, st, dev);
    cudaError_t e = launch_gemm_grouped(xq, act_scale, m, w, epi, int(count), y, acc_out, d_flags, wait_limit(),
                                        g_force_stall, dev.sm_count, g_trace, st);
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "grouped gemm launch");
}

bitnet_status bitnet_linear_q_grouped(const int8_t *const *xq, const float *const *act_scale, int64_t m,
                                      const bitnet_tw *w, int64_t count, float *const *y, int32_t *const *acc_out,
                                      int32_t *d_flags, void *stream)
{
    return bitnet_linear_q_grouped_ex(xq, act_scale, m, w, nullptr, count, y, acc_out, d_flags, stream);
}

bitnet_status bitnet_linear_stack_ex(const float *const *x, int64_t m, const bitnet_tw *w, const bitnet_epilogue *epi,
                                     int64_t count, float *const *y, int32_t *const *acc_out, int32_t *d_flags,
                                     void *stream)
{
    if (!x || !w || !y) return fail(BITNET_ERR_INVALID_ARG, "stack: NULL array");
    if (count < 1 || count > BITNET_STACK_MAX)
        return fail(BITNET_ERR_INVALID_ARG, "stack: count=%lld out of range [1, %d]", (long long)count,
                    BITNET_STACK_MAX);
    if (m < 1 || m > (int64_t(1) << 31) - 1) return fail(BITNET_ERR_INVALID_ARG, "stack: bad m");
    for (int64_t i = 0; i < count; ++i) {
        bitnet_status s = check_tw(w[i], i);
        if (s != BITNET_OK) return s;
        if (!x[i] || !y[i]) return fail(BITNET_ERR_INVALID_ARG, "stack: layer %lld has a NULL x or y", (long long)i);
        if (!aligned(x[i], 16)) return fail(BITNET_ERR_INVALID_ARG, "stack: layer %lld x not 16-byte aligned", (long long)i);
        if (epi) {
            bitnet_status s = check_epi(epi + i, i);
            if (s != BITNET_OK) return s;
        }
    }
    DevInfo dev;
    bitnet_status s = check_device(&dev);
    if (s != BITNET_OK) return s;
    return gemv_slices(x, nullptr, nullptr, m, w, epi, count, y, acc_out, d_flags, static_cast<cudaStream_t>(stream),
                       dev);
}

bitnet_status bitnet_linear_stack(const float *const *x, int64_t m, const bitnet_tw *w, int64_t count,
                                  float *const *y, int32_t *const *acc_out, int32_t *d_flags, void *stream)
{
    return bitnet_linear_stack_ex(x, m, w, nullptr, count, y, acc_out, d_flags, stream);
}

size_t bitnet_i8_row_bytes(int64_t k)
{
    if (k < 1 || k > BITNET_MAX_K) return 0;
    return size_t(32 * ((k + 31) / 32));
}

size_t bitnet_linear_i8_workspace_bytes(int64_t m, int64_t k)
{
    if (m < 1 || m > (int64_t(1) << 31) - 1 || k < 1 || k > BITNET_MAX_K) return 0;
    const size_t a = size_t(m) * size_t(128 * blocks_of(k));
    return (a + 255) / 256 * 256 + size_t(m) * sizeof(float);
}

}  // extern "C"

namespace {

// Workspace layout of a grouped I8_S call: for each distinct input (same x
// pointer and k, in order of first use) its int8 rows [m, kpad] and then its
// scales [m], each area rounded up to 256 bytes.  input_of[i] = the distinct
// input of layer i; offsets of its two areas in q_off / s_off.
struct I8Plan {
    std::vector<int> input_of;
    std::vector<size_t> q_off, s_off;
    std::vector<int64_t> first;   // a layer that uses the input
    size_t bytes = 0;
};

void plan_i8(const float *const *x, int64_t m, const bitnet_i8w *w, int64_t count, I8Plan &P)
{
    P.input_of.assign(size_t(count), -1);
    P.q_off.clear();
    P.s_off.clear();
    P.first.clear();
    size_t off = 0;
    for (int64_t i = 0; i < count; ++i) {
        int found = -1;
        for (size_t j = 0; j < P.first.size(); ++j)
            if (x[P.first[j]] == x[i] && w[P.first[j]].k == w[i].k) found = int(j);
        if (found < 0) {
            found = int(P.first.size());
            P.first.push_back(i);
            const size_t qa = size_t(m) * size_t(128 * blocks_of(w[i].k));
            P.q_off.push_back(off);
            off += (qa + 255) / 256 * 256;
            P.s_off.push_back(off);
            off += (size_t(m) * sizeof(float) + 255) / 256 * 256;
        }
        P.input_of[size_t(i)] = found;
    }
    P.bytes = off;
}

}  // namespace

extern "C" {

size_t bitnet_linear_i8_grouped_workspace_bytes(const float *const *x, int64_t m, const bitnet_i8w *w, int64_t count)
{
    if (!x || !w || count < 1 || count > BITNET_I8_GROUP_MAX || m < 1 || m > (int64_t(1) << 31) - 1) return 0;
    for (int64_t i = 0; i < count; ++i)
        if (w[i].k < 1 || w[i].k > BITNET_MAX_K) return 0;
    I8Plan P;
    plan_i8(x, m, w, count, P);
    return P.bytes;
}

bitnet_status bitnet_linear_i8_grouped(const float *const *x, int64_t m, const bitnet_i8w *w,
                                       const bitnet_epilogue *epi, int64_t count, float *const *y,
                                       int32_t *const *acc_out, void *workspace, size_t workspace_bytes,
                                       int32_t *d_flags, void *stream)
{
    if (!x || !w || !y) return fail(BITNET_ERR_INVALID_ARG, "linear_i8_grouped: NULL array");
    if (count < 1 || count > BITNET_I8_GROUP_MAX)
        return fail(BITNET_ERR_INVALID_ARG, "linear_i8_grouped: count=%lld out of range [1, %d]", (long long)count,
                    BITNET_I8_GROUP_MAX);
    if (m < 1 || m > (int64_t(1) << 31) - 1) return fail(BITNET_ERR_INVALID_ARG, "linear_i8_grouped: bad m");
    for (int64_t i = 0; i < count; ++i) {
        if (!x[i] || !y[i] || !w[i].w)
            return fail(BITNET_ERR_INVALID_ARG, "linear_i8_grouped: layer %lld has a NULL pointer", (long long)i);
        if (w[i].n < 1 || w[i].n > (int64_t(1) << 30) || w[i].k < 1 || w[i].k > BITNET_MAX_K)
            return fail(BITNET_ERR_INVALID_ARG, "linear_i8_grouped: layer %lld bad sizes", (long long)i);
        if (!aligned(w[i].w, 16) || !aligned(x[i], 16))
            return fail(BITNET_ERR_INVALID_ARG, "linear_i8_grouped: layer %lld weights or x not 16-byte aligned",
                        (long long)i);
        if (epi) {
            bitnet_status s = check_epi(epi + i, i);
            if (s != BITNET_OK) return s;
        }
    }
    static thread_local I8Plan P;
    plan_i8(x, m, w, count, P);
    if (!workspace || workspace_bytes < P.bytes)
        return fail(BITNET_ERR_WORKSPACE, "linear_i8_grouped: workspace of %zu bytes needed, %zu given", P.bytes,
                    workspace_bytes);
    if (!aligned(workspace, 256))
        return fail(BITNET_ERR_INVALID_ARG, "linear_i8_grouped: workspace not 256-byte aligned");
    DevInfo dev;
    bitnet_status s = check_device(&dev);
    if (s != BITNET_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    for (size_t j = 0; j < P.first.size(); ++j) {
        const int64_t i = P.first[j];
        cudaError_t e = launch_quant(x[i], m, w[i].k, reinterpret_cast<int8_t *>(ws + P.q_off[j]),
                                     reinterpret_cast<float *>(ws + P.s_off[j]), d_flags, st);
        if (e != cudaSuccess) return cuda_fail(e, "quant launch");
    }
    static thread_local std::vector<I8Job> jobs;
    jobs.resize(size_t(count));
    for (int64_t i = 0; i < count; ++i) {
        const int j = P.input_of[size_t(i)];
        jobs[size_t(i)] = I8Job{w[i].w, w[i].n, w[i].k, w[i].scale, reinterpret_cast<const int8_t *>(ws + P.q_off[j]),
                                reinterpret_cast<const float *>(ws + P.s_off[j]), y[i],
                                acc_out ? acc_out[i] : nullptr, epi ? epi + i : nullptr};
    }
    cudaError_t e = launch_gemv_i8_group(jobs.data(), int(count), m, dev.sm_count, st);
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "i8 gemv launch");
}

bitnet_status bitnet_linear_i8(const float *x, int64_t m, const bitnet_i8w *w, const bitnet_epilogue *epi, float *y,
                               int32_t *acc_out, void *workspace, size_t workspace_bytes, int32_t *d_flags,
                               void *stream)
{
    if (!x || !w || !y || !w->w) return fail(BITNET_ERR_INVALID_ARG, "linear_i8: NULL pointer");
    if (m < 1 || m > (int64_t(1) << 31) - 1) return fail(BITNET_ERR_INVALID_ARG, "linear_i8: bad m=%lld", (long long)m);
    if (w->n < 1 || w->n > (int64_t(1) << 30) || w->k < 1 || w->k > BITNET_MAX_K)
        return fail(BITNET_ERR_INVALID_ARG, "linear_i8: bad sizes n=%lld k=%lld", (long long)w->n, (long long)w->k);
    if (!aligned(w->w, 16) || !aligned(x, 16))
        return fail(BITNET_ERR_INVALID_ARG, "linear_i8: weights or x not 16-byte aligned");
    bitnet_status s = check_epi(epi, 0);
    if (s != BITNET_OK) return s;
    const size_t need = bitnet_linear_i8_workspace_bytes(m, w->k);
    if (!workspace || workspace_bytes < need)
        return fail(BITNET_ERR_WORKSPACE, "linear_i8: workspace of %zu bytes needed, %zu given", need, workspace_bytes);
    if (!aligned(workspace, 256)) return fail(BITNET_ERR_INVALID_ARG, "linear_i8: workspace not 256-byte aligned");
    DevInfo dev;
    s = check_device(&dev);
    if (s != BITNET_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int8_t *xq = static_cast<int8_t *>(workspace);
    const size_t qa = (size_t(m) * size_t(128 * blocks_of(w->k)) + 255) / 256 * 256;
    float *xs = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + qa);
    cudaError_t e = launch_quant(x, m, w->k, xq, xs, d_flags, st);
    if (e != cudaSuccess) return cuda_fail(e, "quant launch");
    e = launch_gemv_i8(w->w, w->n, w->k, w->scale, xq, xs, m, epi, y, acc_out, dev.sm_count, st);
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "i8 gemv launch");
}

}  // extern "C"

// ===================================================================
// bitnet_linear_stack_noalloc: the decode stack for callers that cannot
// allocate device memory.
//
// The ordinary stack call keeps each weight tensor's TMA tensor map in a
// per-device cache that it allocates with cudaMalloc/cudaMallocHost the first
// time it meets the tensor.  This variant instead writes the maps into the
// fixed array below, which is part of the library's module image (every GPU
// that loads the library holds it until the process exits), and otherwise runs
// the same kernel.  Its limit is the array's size: kNoallocMaxLayers maps.
// ===================================================================

static constexpr int kNoallocMaxLayers = BITNET_STACK_MAX;   // 256 maps x 128 bytes = 32 KB
static __device__ __align__(256) uint8_t g_noalloc_tmaps[kNoallocMaxLayers * sizeof(CUtensorMap)];

namespace {

std::mutex g_na_mu;                        // guards everything below
void *g_na_dev_addr[64] = {nullptr};       // device address of g_noalloc_tmaps, per device
struct NaKey {
    const void *p;
    int64_t n, k;
};
NaKey g_na_copied[64][kNoallocMaxLayers];  // descriptors whose maps each device's array holds
int g_na_copied_count[64] = {0};
CUtensorMap g_na_host_maps[kNoallocMaxLayers];
LayerReq g_na_layers[kNoallocMaxLayers];
int g_na_input_of[kNoallocMaxLayers];
GemvParams g_na_params;

// Set-up, once per device, with that device current: the array's name is only
// a host-side stand-in, so its device address is looked up here.
bitnet_status noalloc_scratch(int dev, void **addr)
{
    if (!g_na_dev_addr[dev]) {
        void *a = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&a, g_noalloc_tmaps);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(noalloc tensor-map array)");
        g_na_dev_addr[dev] = a;
    }
    *addr = g_na_dev_addr[dev];
    return BITNET_OK;
}

// Same byte-balanced partition as the ordinary stack call, over fixed arrays.
bitnet_status noalloc_plan_and_launch(int count, int m, int32_t *flags, cudaStream_t st, const DevInfo &dev,
                                      const CUtensorMap *maps)
{
    GemvParams &p = g_na_params;
    const LayerReq *L = g_na_layers;
    int ninp = 0;
    int64_t max_kpad = 0;
    for (int i = 0; i < count; ++i) {
        int found = -1;
        for (int j = 0; j < ninp; ++j)
            if (p.inp[j].x == L[i].x && p.inp[j].k == int32_t(L[i].w.k)) {
                found = j;
                break;
            }
        if (found < 0) {
            found = ninp++;
            p.inp[found].x = L[i].x;
            p.inp[found].scale = nullptr;
            p.inp[found].k = int32_t(L[i].w.k);
            p.inp[found].kb = int32_t(blocks_of(L[i].w.k));
        }
        g_na_input_of[i] = found;
        const int64_t kp = 128 * blocks_of(L[i].w.k);
        if (kp > max_kpad) max_kpad = kp;
        p.lin[i].tmap = maps + i;
        p.lin[i].y = L[i].y;
        p.lin[i].acc = L[i].acc;
        p.lin[i].n = int32_t(L[i].w.n);
        p.lin[i].kb = int32_t(blocks_of(L[i].w.k));
        p.lin[i].scale = L[i].w.scale;
        p.lin[i].input = int16_t(found);
        p.lin[i].bias = nullptr;
        p.lin[i].gamma = nullptr;
        p.lin[i].res = nullptr;
        p.lin[i].relu = 0;
    }
    p.has_epi = 0;
    const int variant = pick_variant(m, max_kpad);
    if (variant < 0)
        return fail(BITNET_ERR_INVALID_ARG, "noalloc stack: m=%d x kpad=%lld exceeds the GEMV activation area", m,
                    (long long)max_kpad);
    const int64_t xcap = x_cap(kVariants[variant].nw, kVariants[variant].boxes);
    int64_t total = 0;
    for (int i = 0; i < count; ++i) total += L[i].w.n * 32 * blocks_of(L[i].w.k);
    const int64_t G = dev.sm_count;
    int nr = 0, ns = 0, cur_target = -1;
    int64_t cur_x = 0, xmax = 0, cum = 0;
    bool open = false;
    for (int i = 0; i < count; ++i) {
        const int64_t rowb = 32 * blocks_of(L[i].w.k);
        const int64_t tiles = (L[i].w.n + kTileRows - 1) / kTileRows;
        const int64_t xin = int64_t(m) * 128 * blocks_of(L[i].w.k);
        for (int64_t t = 0; t < tiles; ++t) {
            const int64_t rows = (t + 1 < tiles) ? kTileRows : L[i].w.n - t * kTileRows;
            const int64_t tb = rows * rowb;
            const int target = int((cum + tb / 2) * G / total);
            cum += tb;
            if (open && target != cur_target) {
                if (p.rng[nr].nseg > 0) {
                    xmax = cur_x > xmax ? cur_x : xmax;
                    ++nr;
                }
                open = false;
            }
            for (;;) {
                if (!open) {
                    if (nr == kMaxRanges) return fail(BITNET_ERR_INVALID_ARG, "noalloc stack needs more than %d CTAs", kMaxRanges);
                    p.rng[nr].seg0 = int16_t(ns);
                    p.rng[nr].nseg = 0;
                    p.rng[nr].nin = 0;
                    cur_x = 0;
                    cur_target = target;
                    open = true;
                }
                GemvRange &r = p.rng[nr];
                int slot = -1;
                for (int u = 0; u < r.nin; ++u)
                    if (r.in[u] == g_na_input_of[i]) slot = u;
                const bool same_seg = r.nseg > 0 && p.seg[ns - 1].lin == i && p.seg[ns - 1].tile1 == t;
                const bool need_in = slot < 0;
                if ((need_in && (r.nin == kMaxRangeInputs || cur_x + xin > xcap)) ||
                    (!same_seg && (r.nseg == kMaxRangeSegs || ns == kMaxSegs))) {
                    if (r.nseg == 0 || ns == kMaxSegs)
                        return fail(BITNET_ERR_INVALID_ARG, "noalloc stack too large for one launch");
                    xmax = cur_x > xmax ? cur_x : xmax;
                    ++nr;
                    open = false;
                    continue;
                }
                if (need_in) {
                    slot = r.nin;
                    r.in[r.nin++] = int16_t(g_na_input_of[i]);
                    cur_x += xin;
                }
                if (!same_seg) {
                    GemvSeg &sg = p.seg[ns++];
                    sg.lin = int16_t(i);
                    sg.slot = int16_t(slot);
                    sg.tile0 = int32_t(t);
                    sg.tile1 = int32_t(t + 1);
                    r.nseg++;
                } else {
                    p.seg[ns - 1].tile1 = int32_t(t + 1);
                }
                break;
            }
        }
    }
    if (open && p.rng[nr].nseg > 0) {
        xmax = cur_x > xmax ? cur_x : xmax;
        ++nr;
    }
    p.m = m;
    p.num_ranges = nr;
    p.prequant = 0;
    p.force_stall = g_force_stall;
    p.flags = flags;
    p.wait_limit = wait_limit();
    p.trace = g_trace;
    p.x_bytes = int32_t((xmax + 127) / 128 * 128);
    p.fence_maps = 1;   // the fixed array is rewritten in place between calls
    cudaError_t e = launch_gemv(p, variant, st);
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "gemv launch");
}

}  // namespace

extern "C" bitnet_status bitnet_linear_stack_noalloc(const float *const *x, int64_t m, const bitnet_tw *w,
                                                     int64_t count, float *const *y, int32_t *const *acc_out,
                                                     int32_t *d_flags, void *stream)
{
    if (!x || !w || !y) return fail(BITNET_ERR_INVALID_ARG, "noalloc stack: NULL array");
    if (count < 1 || count > kNoallocMaxLayers)
        return fail(BITNET_ERR_INVALID_ARG,
                    "noalloc stack: count=%lld exceeds the %d tensor maps its fixed device array holds",
                    (long long)count, kNoallocMaxLayers);
    if (m < 1 || m > (int64_t(1) << 31) - 1) return fail(BITNET_ERR_INVALID_ARG, "noalloc stack: bad m");
    for (int64_t i = 0; i < count; ++i) {
        bitnet_status s = check_tw(w[i], i);
        if (s != BITNET_OK) return s;
        if (!x[i] || !y[i])
            return fail(BITNET_ERR_INVALID_ARG, "noalloc stack: layer %lld has a NULL x or y", (long long)i);
        if (!aligned(x[i], 16))
            return fail(BITNET_ERR_INVALID_ARG, "noalloc stack: layer %lld x not 16-byte aligned", (long long)i);
    }
    DevInfo dev;
    bitnet_status s = check_device(&dev);
    if (s != BITNET_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    std::lock_guard<std::mutex> lock(g_na_mu);
    void *scratch = nullptr;
    s = noalloc_scratch(dev.ordinal, &scratch);
    if (s != BITNET_OK) return s;
    const int n = int(count);
    // rewrite the device array only when it does not already hold these maps
    bool same = g_na_copied_count[dev.ordinal] == n;
    for (int i = 0; same && i < n; ++i) {
        const NaKey &k = g_na_copied[dev.ordinal][i];
        same = k.p == w[i].packed && k.n == w[i].n && k.k == w[i].k;
    }
    if (!same) {
        for (int i = 0; i < n; ++i) {
            s = encode_weight_map(&g_na_host_maps[i], w[i].packed, w[i].n, blocks_of(w[i].k));
            if (s != BITNET_OK) return s;
        }
        // from pageable memory: the bytes are staged before this returns, so
        // the host array may be rewritten by the next call
        cudaError_t e = cudaMemcpyAsync(scratch, g_na_host_maps, size_t(n) * sizeof(CUtensorMap),
                                        cudaMemcpyHostToDevice, st);
        if (e != cudaSuccess) {
            g_na_copied_count[dev.ordinal] = 0;
            return cuda_fail(e, "noalloc tensor-map copy");
        }
        for (int i = 0; i < n; ++i) g_na_copied[dev.ordinal][i] = NaKey{w[i].packed, w[i].n, w[i].k};
        g_na_copied_count[dev.ordinal] = n;
    }
    const CUtensorMap *maps = static_cast<const CUtensorMap *>(scratch);
    for (int64_t m0 = 0; m0 < m; m0 += BITNET_GEMV_MAX_M) {
        const int ms = int((m - m0) < BITNET_GEMV_MAX_M ? (m - m0) : BITNET_GEMV_MAX_M);
        for (int i = 0; i < n; ++i) {
            LayerReq &r = g_na_layers[i];
            r.x = x[i] + m0 * w[i].k;
            r.xscale = nullptr;
            r.w = w[i];
            r.y = y[i] + m0 * w[i].n;
            r.acc = (acc_out && acc_out[i]) ? acc_out[i] + m0 * w[i].n : nullptr;
            r.bias = r.gamma = r.res = nullptr;
            r.relu = 0;
        }
        s = noalloc_plan_and_launch(n, ms, d_flags, st, dev, maps);
        if (s != BITNET_OK) return s;
    }
    return BITNET_OK;
}
