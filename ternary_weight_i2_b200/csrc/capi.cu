// capi.cu -- the C ABI declared in include/bitnet.h: argument checks, the
// device check, work partitioning for the streaming GEMV, and dispatch.
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <vector>

#include "common.cuh"
#include "gemv.cuh"

namespace bitnet {
cudaError_t launch_gemv(const GemvParams &p, int nw, cudaStream_t st);
cudaError_t launch_pack(const int8_t *w, int64_t n, int64_t k, uint8_t *packed, int32_t *flags, cudaStream_t st);
cudaError_t launch_unpack(const uint8_t *packed, int64_t n, int64_t k, int8_t *w, cudaStream_t st);
cudaError_t launch_quant(const float *x, int64_t m, int64_t k, int8_t *xq, float *scale, int32_t *flags,
                         cudaStream_t st);
bool gemm_available();
cudaError_t launch_gemm(const int8_t *xq, const float *act_scale, int64_t m, const bitnet_tw *w, float *y,
                        int32_t *acc, int32_t *flags, cudaStream_t st);
}  // namespace bitnet

using namespace bitnet;

namespace {

thread_local char g_err[512] = "";
uint64_t g_wait_limit = 0;   // 0: built-in bound
int g_force_stall = 0;       // test aid: kernels wait on a barrier nobody arrives at

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

uint64_t wait_limit() { return g_wait_limit ? g_wait_limit : kDefaultWaitLimit; }

// ---------------------------------------------------------------- GEMV plan

struct LayerReq {
    const void *x;         // this slice's activation rows (fp32, or int8 when prequant)
    const float *xscale;   // prequant: per-token scales
    bitnet_tw w;
    float *y;
    int32_t *acc;
};

int nw_for(int m)
{
    if (m <= 1) return 8;
    if (m <= 5) return 6;
    return 4;
}

// Split the layers' 32-row tiles into contiguous byte-balanced ranges (one CTA
// each) under the per-CTA limits: distinct inputs, segments, and the shared
// memory that holds the quantised activations.
bitnet_status plan_and_launch(const std::vector<LayerReq> &L, int m, bool prequant, int32_t *flags,
                              cudaStream_t st, const DevInfo &dev)
{
    static thread_local GemvParams p;   // host staging of the kernel parameter block
    static thread_local std::vector<int> input_of;
    const int count = int(L.size());
    // distinct inputs: same pointer and same width
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
        p.lin[i].packed = L[i].w.packed;
        p.lin[i].y = L[i].y;
        p.lin[i].acc = L[i].acc;
        p.lin[i].n = int32_t(L[i].w.n);
        p.lin[i].kb = int32_t(blocks_of(L[i].w.k));
        p.lin[i].scale = L[i].w.scale;
        p.lin[i].input = found;
    }
    int nw = nw_for(m);
    if (int64_t(m) * max_kpad > gemv_x_cap(nw)) nw = 4;
    if (int64_t(m) * max_kpad > gemv_x_cap(nw))
        return fail(BITNET_ERR_INVALID_ARG, "m=%d x kpad=%lld exceeds the GEMV activation area", m,
                    (long long)max_kpad);
    const int64_t xcap = gemv_x_cap(nw);

    int64_t total = 0;
    for (int i = 0; i < count; ++i) total += L[i].w.n * 32 * blocks_of(L[i].w.k);
    int64_t target = (total + dev.sm_count - 1) / dev.sm_count;
    for (int attempt = 0; attempt < 8; ++attempt, target += target / 2 + 1) {
        int nr = 0, ns = 0;
        bool open = false, overflow = false;
        int64_t cur_bytes = 0, cur_x = 0, xmax = 0;
        auto open_range = [&]() -> bool {
            if (nr == kMaxRanges) return false;
            GemvRange &r = p.rng[nr];
            r.seg0 = int16_t(ns);
            r.nseg = 0;
            r.nin = 0;
            cur_bytes = 0;
            cur_x = 0;
            open = true;
            return true;
        };
        auto close_range = [&]() {
            if (open && p.rng[nr].nseg > 0) {
                xmax = cur_x > xmax ? cur_x : xmax;
                ++nr;
            }
            open = false;
        };
        for (int i = 0; i < count && !overflow; ++i) {
            const int64_t rowb = 32 * blocks_of(L[i].w.k);
            const int64_t tiles = (L[i].w.n + kTileRows - 1) / kTileRows;
            const int64_t tb = kTileRows * rowb;
            const int64_t xin = int64_t(m) * 128 * blocks_of(L[i].w.k);
            int64_t t = 0;
            while (t < tiles) {
                if (!open && !open_range()) {
                    overflow = true;
                    break;
                }
                GemvRange &r = p.rng[nr];
                int slot = -1;
                for (int u = 0; u < r.nin; ++u)
                    if (r.in[u] == input_of[i]) slot = u;
                const bool need_in = slot < 0;
                if (ns == kMaxSegs) {
                    overflow = true;
                    break;
                }
                if ((need_in && (r.nin == kMaxRangeInputs || cur_x + xin > xcap)) || r.nseg == kMaxRangeSegs) {
                    close_range();   // r.nseg > 0 here: an empty range always fits one input
                    continue;
                }
                if (need_in) {
                    slot = r.nin;
                    r.in[r.nin++] = int16_t(input_of[i]);
                    cur_x += xin;
                }
                int64_t room = (target - cur_bytes + tb - 1) / tb;
                if (room < 1) room = 1;
                const int64_t take = (tiles - t) < room ? (tiles - t) : room;
                GemvSeg &sg = p.seg[ns++];
                sg.lin = int16_t(i);
                sg.slot = int16_t(slot);
                sg.tile0 = int32_t(t);
                sg.tile1 = int32_t(t + take);
                r.nseg++;
                t += take;
                cur_bytes += take * tb;
                if (cur_bytes >= target) close_range();
            }
        }
        if (overflow) continue;
        close_range();
        p.m = m;
        p.num_ranges = nr;
        p.prequant = prequant ? 1 : 0;
        p.force_stall = g_force_stall;
        p.flags = flags;
        p.wait_limit = wait_limit();
        p.x_bytes = int32_t((xmax + 127) / 128 * 128);
        cudaError_t e = launch_gemv(p, nw, st);
        if (e != cudaSuccess) return cuda_fail(e, "gemv launch");
        return BITNET_OK;
    }
    return fail(BITNET_ERR_INVALID_ARG, "could not partition %d layers into %d ranges", count, kMaxRanges);
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
                                 const bitnet_tw *w, int64_t count, float *const *y, int32_t *const *acc,
                                 int32_t *d_flags, cudaStream_t st, const DevInfo &dev)
{
    std::vector<LayerReq> L;
    L.resize(static_cast<size_t>(count));
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
        }
        bitnet_status s = plan_and_launch(L, ms, xq != nullptr, d_flags, st, dev);
        if (s != BITNET_OK) return s;
    }
    return BITNET_OK;
}

bitnet_status bitnet_linear(const float *x, int64_t m, const bitnet_tw *w, float *y, int32_t *acc_out,
                            void *workspace, size_t workspace_bytes, int32_t *d_flags, void *stream)
{
    if (!x || !w || !y) return fail(BITNET_ERR_INVALID_ARG, "linear: NULL pointer");
    if (m < 1 || m > (int64_t(1) << 31) - 1) return fail(BITNET_ERR_INVALID_ARG, "linear: bad m=%lld", (long long)m);
    bitnet_status s = check_tw(*w, 0);
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
            return gemv_slices(nullptr, xqa, xsa, m, w, 1, ya, aa, d_flags, st, dev);
        }
        const float *xa[1] = {x};
        float *ya[1] = {y};
        int32_t *aa[1] = {acc_out};
        return gemv_slices(xa, nullptr, nullptr, m, w, 1, ya, aa, d_flags, st, dev);
    }
    int8_t *xq = static_cast<int8_t *>(workspace);
    const size_t qa = (size_t(m) * size_t(128 * blocks_of(w->k)) + 255) / 256 * 256;
    float *xs = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + qa);
    cudaError_t e = launch_quant(x, m, w->k, xq, xs, d_flags, st);
    if (e != cudaSuccess) return cuda_fail(e, "quant launch");
    e = launch_gemm(xq, xs, m, w, y, acc_out, d_flags, st);
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "gemm launch");
}

bitnet_status bitnet_linear_q(const int8_t *xq, const float *act_scale, int64_t m, const bitnet_tw *w, float *y,
                              int32_t *acc_out, int32_t *d_flags, void *stream)
{
    if (!xq || !act_scale || !w || !y) return fail(BITNET_ERR_INVALID_ARG, "linear_q: NULL pointer");
    if (m < 1 || m > (int64_t(1) << 31) - 1) return fail(BITNET_ERR_INVALID_ARG, "linear_q: bad m");
    bitnet_status s = check_tw(*w, 0);
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
        return gemv_slices(nullptr, xqa, xsa, m, w, 1, ya, aa, d_flags, st, dev);
    }
    cudaError_t e = launch_gemm(xq, act_scale, m, w, y, acc_out, d_flags, st);
    return e == cudaSuccess ? BITNET_OK : cuda_fail(e, "gemm launch");
}

bitnet_status bitnet_linear_stack(const float *const *x, int64_t m, const bitnet_tw *w, int64_t count,
                                  float *const *y, int32_t *const *acc_out, int32_t *d_flags, void *stream)
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
    }
    DevInfo dev;
    bitnet_status s = check_device(&dev);
    if (s != BITNET_OK) return s;
    return gemv_slices(x, nullptr, nullptr, m, w, count, y, acc_out, d_flags, static_cast<cudaStream_t>(stream), dev);
}

}  // extern "C"
