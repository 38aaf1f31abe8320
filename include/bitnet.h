/*
 * bitnet.h -- C ABI of the B200 (sm_100a) I2_S ternary linear-layer library.
 *
 * The operation ("VibeVoice-ASR-BitNet Technical Report", §2.2.2 and §2.4.2,
 * Figure 4): a linear layer y = x W^T whose weights W [N,K] take values in
 * {-1, 0, +1} and are stored 2 bits each, grouped 128 elements per block (the
 * grouping the ARM debugging blog post "Paper 說支援 ARM，我大概是第一個真的去編譯
 * 的人" establishes in its second postscript), with one fp32 scale s_w per
 * tensor; activations x [M,K] are quantised per token to int8 by absmax/127 at
 * run time, multiplied against the ternary weights with exact int32
 * accumulation, and the sums are dequantised in fp32.
 *
 * Around it: the absmean quantiser that turns full-precision weights into
 * the ternary codes and scale (bitnet_quantize_pack), an optional fused
 * epilogue after the dequantisation (bias, ReLU, layer-scaled residual add:
 * the operator fusion of §2.4.1; the *_ex entry points), and the I8_S layer
 * with plain int8 weights (§2.2.1, §2.4.2; bitnet_linear_i8*).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers named d_* or documented "device" point to CUDA device memory of
 *   the current device; the caller owns every buffer.  Functions that take a
 *   workspace never allocate; no function allocates device memory per call.
 *   The GEMV path (bitnet_linear[_ex] and bitnet_linear_q[_ex] with m <= 8,
 *   bitnet_linear_stack[_ex]) streams each weight tensor through a TMA tensor map
 *   that the library encodes the first time it meets that tensor (same
 *   packed pointer, n and k) and keeps in a per-device cache (128 bytes of
 *   device memory per tensor, allocated 128 KB at a time, until
 *   bitnet_release_device_cache() or exit).  That first call allocates and
 *   copies synchronously, so it must not be made under CUDA stream capture;
 *   later calls with the same tensors only look the maps up.
 * - `stream` is a cudaStream_t (NULL = legacy default stream).  All GPU work is
 *   enqueued on it and the functions return without synchronising.
 * - Errors found on the host (bad argument, misaligned pointer, device that is
 *   not sm_100) are returned synchronously and nothing is enqueued.  A
 *   function never returns BITNET_OK without doing its work.
 * - Conditions found on the GPU are OR-ed as BITNET_FLAG_* bits into the
 *   int32 word *d_flags (device memory, nullable); read it after the stream
 *   has been synchronised.  bitnet_status_from_flags() maps it to a status.
 * - Layouts are row-major and dense: x [M,K] fp32, y [M,N] fp32, int32
 *   acc [M,N], int8 w [N,K], packed [N, 32*ceil(K/128)] bytes.
 *
 * Packed format (readings of points the pages leave open)
 * ---------------------------------------------------------
 * Row n of the packed matrix holds 32*ceil(K/128) bytes.  Element
 * k = 128*j + 32*g + b (g = 0..3, b = 0..31) is the 2-bit field at bits
 * [2g, 2g+1] of byte 32*j + b; the field holds w + 1 (00 = -1, 01 = 0,
 * 10 = +1); fields of positions k >= K hold 01.  The weight scale is not in the
 * buffer: it travels in bitnet_tw.  Compatibility with other I2_S files is not
 * claimed.
 *
 * Activation quantiser (per token m, fp32, no fused multiply-add)
 * ---------------------------------------------------------------
 * amax = max_k |x[m,k]|; a row holding NaN or Inf gives codes 0 and scale 0 and
 * raises BITNET_FLAG_NONFINITE; amax == 0 gives codes 0 and scale 0; otherwise
 * inv = 127/amax, q = 0 where x == 0, else clamp(rint(x*inv), -127, 127)
 * (round half to even), and scale = amax/127.  Pads k >= K of int8 rows are 0.
 *
 * Linear
 * ------
 * acc[m,n] = sum_k q[m,k] * w[n,k] (exact int32);
 * y[m,n] = ((float)acc[m,n] * s_act[m]) * s_w, two rounded fp32 products.
 */
#ifndef BITNET_H
#define BITNET_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BITNET_API __attribute__((visibility("default")))
#else
#define BITNET_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BITNET_OK = 0,
    BITNET_ERR_INVALID_ARG = 1,        /* null/negative/misaligned/oversized argument   */
    BITNET_ERR_NOT_TERNARY = 2,        /* a weight outside {-1,0,+1} (device flag)      */
    BITNET_ERR_UNSUPPORTED_DEVICE = 3, /* current device is not sm_100 (B200)           */
    BITNET_ERR_CUDA = 4,               /* a CUDA runtime call failed                    */
    BITNET_ERR_NONFINITE = 5,          /* NaN/Inf in an activation row or in a weight
                                          tensor being quantised (device flag)          */
    BITNET_ERR_TIMEOUT = 6,            /* a bounded device-side wait ran out (flag)     */
    BITNET_ERR_WORKSPACE = 7           /* the workspace given is too small              */
} bitnet_status;

/* Bits OR-ed into *d_flags by the kernels. */
#define BITNET_FLAG_NOT_TERNARY 0x1
#define BITNET_FLAG_NONFINITE   0x2
#define BITNET_FLAG_TIMEOUT     0x4

/* One ternary weight tensor as produced by bitnet_pack_ternary.
 * packed: device pointer, 16-byte aligned, [n, 32*ceil(k/128)] bytes;
 * n, k: output and input widths (1 <= k <= BITNET_MAX_K, n >= 1);
 * scale: the per-tensor fp32 weight scale s_w. */
typedef struct {
    const uint8_t *packed;
    int64_t n;
    int64_t k;
    float scale;
} bitnet_tw;

/*
 * Optional fused epilogue of a linear layer, applied to each output after
 * the dequantisation y = ((float)acc * s_act[m]) * s_w, in the order of the
 * technical report's §2.4.1 operator fusion (matrix multiply + bias + ReLU,
 * then residual addition with a layer-scale factor):
 *   h   = y + bias[c]                 (bias != NULL)
 *   h   = h > 0 ? h : +0              (relu != 0)
 *   h   = gamma[c] * h                (gamma != NULL)
 *   out = residual[r, c] + h          (residual != NULL)
 * Every step is one rounded fp32 operation (no fused multiply-add), so the
 * result equals the oracle's bit for bit.  All pointers are device memory:
 *   bias, gamma  fp32 [n], 4-byte aligned; must not overlap any output of
 *                the call (they are read through the read-only cache)
 *   residual     fp32 [m, n] row-major, 4-byte aligned; it may be the output
 *                y itself (an in-place residual add: each element is read
 *                before it is written, by the same thread), but must not
 *                overlap any other output of the same call.
 * The int32 accumulators (acc_out) are not affected.  An all-NULL, relu = 0
 * epilogue is the plain layer.
 */
typedef struct {
    const float *bias;
    const float *gamma;
    const float *residual;
    int32_t relu;
    int32_t reserved;   /* must be 0 */
} bitnet_epilogue;

#define BITNET_MAX_K 65536
/* Largest number of tokens the decode (GEMV) path takes in one pass; larger M
 * runs through the tensor-core GEMM path. */
#define BITNET_GEMV_MAX_M 8
/* Largest number of layers one bitnet_linear_stack call takes. */
#define BITNET_STACK_MAX 256
/* Largest number of layers one bitnet_linear_q_grouped call takes. */
#define BITNET_GROUP_MAX 8

/* Library version as 10000*major + 100*minor + patch. */
BITNET_API int bitnet_version(void);

/* Text of a status code (static storage). */
BITNET_API const char *bitnet_status_str(bitnet_status s);

/* Detail of the last error returned on the calling thread (static storage,
 * overwritten by the next failing call). */
BITNET_API const char *bitnet_last_error(void);

/* Map a *d_flags word read back from the device to a status
 * (TIMEOUT > NONFINITE > NOT_TERNARY > OK in priority). */
BITNET_API bitnet_status bitnet_status_from_flags(int32_t flags);

/* Bytes of a packed [n, k] tensor: n * 32 * ceil(k/128); 0 on bad sizes. */
BITNET_API size_t bitnet_packed_bytes(int64_t n, int64_t k);

/* Padded int8 row width 128 * ceil(k/128); 0 on bad sizes. */
BITNET_API int64_t bitnet_kpad(int64_t k);

/*
 * Pack int8 ternary weights into the 2-bit format (the I2_S weight storage of
 * the technical report §2.2.2; 128-element blocks per the blog post's second
 * postscript).
 *   w      device, int8 [n, k], values in {-1, 0, +1}
 *   packed device, [n, 32*ceil(k/128)] bytes, 16-byte aligned; fully written
 * A value outside {-1,0,+1} is stored as weight 0 and raises
 * BITNET_FLAG_NOT_TERNARY in *d_flags.  Load-time operation.
 */
BITNET_API bitnet_status bitnet_pack_ternary(const int8_t *w, int64_t n, int64_t k,
                                  uint8_t *packed, int32_t *d_flags, void *stream);

/* Workspace bytes bitnet_quantize_pack needs (a fixed 16384). */
BITNET_API size_t bitnet_quantize_pack_workspace_bytes(void);

/*
 * Absmean ternary quantiser fused with the pack: full-precision weights ->
 * the 2-bit format above + one per-tensor scale (the ternary weights and
 * per-tensor scale of the technical report §2.2.2; the rounding rule is
 * the absmean recipe of the BitNet b1.58 work the report builds on, taken as):
 *   scale = mean |W| over all n*k elements, summed in fp64 and rounded once
 *           to fp32;
 *   w     = clamp(rint(W / scale), -1, +1), quotient in fp32 (correctly
 *           rounded), rint half to even;
 *   an all-zero W gives scale 0 and every w = 0.
 *   w          device fp32 [n, k], 4-byte aligned
 *   packed     device, [n, 32*ceil(k/128)] bytes, 16-byte aligned; fully written
 *   d_scale    device fp32 [1], receives scale (w_scale of the linear call)
 *   workspace  device, 8-byte aligned, >= bitnet_quantize_pack_workspace_bytes()
 *              bytes, owned by the caller; must not be reused by another call
 *              until this one has completed on `stream`
 *   d_flags    device int32 or NULL
 * A non-finite element sets scale 0 and every w = 0 and raises
 * BITNET_FLAG_NONFINITE.  The result does not depend on the device or the
 * launch: the fp64 partial sums use a fixed grid and a fixed order.
 * Load-time operation (two kernel launches on `stream`).
 */
BITNET_API bitnet_status bitnet_quantize_pack(const float *w, int64_t n, int64_t k, uint8_t *packed,
                                              float *d_scale, void *workspace, size_t workspace_bytes,
                                              int32_t *d_flags, void *stream);

/* Inverse of bitnet_pack_ternary (test and inspection aid):
 *   packed device [n, 32*ceil(k/128)] -> w device int8 [n, k]. */
BITNET_API bitnet_status bitnet_unpack_ternary(const uint8_t *packed, int64_t n, int64_t k,
                                    int8_t *w, void *stream);

/*
 * Per-token int8 activation quantiser (technical report §2.2.2: activations
 * quantised to INT8 per token at run time; absmax/127 rule above).
 *   x         device fp32 [m, k], 16-byte aligned
 *   xq        device int8 [m, kpad], kpad = bitnet_kpad(k), pads written as 0
 *   act_scale device fp32 [m]
 * Non-finite rows raise BITNET_FLAG_NONFINITE.
 */
BITNET_API bitnet_status bitnet_quant_act(const float *x, int64_t m, int64_t k, int8_t *xq,
                               float *act_scale, int32_t *d_flags, void *stream);

/* Workspace bytes bitnet_linear needs for m tokens of width k: 0 when
 * m <= BITNET_GEMV_MAX_M (the quantiser is fused into the GEMV), otherwise
 * room for the int8 activations and their scales. */
BITNET_API size_t bitnet_linear_workspace_bytes(int64_t m, int64_t k);

/*
 * One ternary linear layer y = dequant(quant(x) W^T) (technical report
 * §2.2.2, §2.4.2 and Figure 4: unpack the 2-bit weights to int8, multiply-add
 * into int32, per-token and per-tensor scales in fp32).
 *   x         device fp32 [m, w->k], 16-byte aligned, m >= 1
 *   w         host pointer to the weight descriptor
 *   y         device fp32 [m, w->n]
 *   acc_out   device int32 [m, w->n] or NULL: the exact integer sums
 *   workspace device, 256-byte aligned, >= bitnet_linear_workspace_bytes(m,k)
 *             bytes (may be NULL when that is 0); owned by the caller, must not
 *             be used by another call until this one has completed on `stream`
 * m <= 8 runs the fused quantiser + streaming GEMV; larger m quantises into
 * the workspace and runs the tensor-core GEMM.
 */
BITNET_API bitnet_status bitnet_linear(const float *x, int64_t m, const bitnet_tw *w, float *y,
                            int32_t *acc_out, void *workspace, size_t workspace_bytes,
                            int32_t *d_flags, void *stream);

/*
 * The same layer on activations already quantised by bitnet_quant_act
 * (prefill on pre-quantised A).
 *   xq        device int8 [m, bitnet_kpad(w->k)], 16-byte aligned, pads 0
 *   act_scale device fp32 [m]
 */
BITNET_API bitnet_status bitnet_linear_q(const int8_t *xq, const float *act_scale, int64_t m,
                              const bitnet_tw *w, float *y, int32_t *acc_out,
                              int32_t *d_flags, void *stream);

/*
 * `count` independent layers on pre-quantised activations in one launch
 * (prefill: the token count m is shared, each layer has its own input, weight
 * and output; TR §3.2, Figure 6a).  m > 8 runs one persistent tensor-core GEMM
 * over all layers' 128-feature x 192-token output tiles, dealt to the SMs heaviest first, so
 * that layers of different K and N balance inside one launch; m <= 8 runs the
 * streaming GEMV.
 *   xq[i]        device int8 [m, bitnet_kpad(w[i].k)], 16-byte aligned, pads 0
 *   act_scale[i] device fp32 [m]
 *   y[i]         device fp32 [m, w[i].n], 16-byte aligned
 *   acc_out      NULL or host array of `count` device int32 [m, w[i].n] (entries
 *                may be NULL)
 * 1 <= count <= BITNET_GROUP_MAX.  Inputs may be shared between layers.
 */
BITNET_API bitnet_status bitnet_linear_q_grouped(const int8_t *const *xq, const float *const *act_scale, int64_t m,
                                                 const bitnet_tw *w, int64_t count, float *const *y,
                                                 int32_t *const *acc_out, int32_t *d_flags, void *stream);

/*
 * A sequence of `count` independent ternary linear layers sharing the token
 * count m, run in one launch (the decoder's linears back to back: each
 * token reads every layer's weights once, technical report §2.2.2 and §3.2,
 * Figure 6 decode).
 *   x[i]      device fp32 [m, w[i].k]; the same pointer may feed several
 *             layers (it is quantised once per use within a CTA)
 *   w         host array of `count` descriptors
 *   y[i]      device fp32 [m, w[i].n]; outputs must not overlap any input
 *   acc_out   NULL, or host array of `count` device int32 [m, w[i].n]
 *             pointers (entries may be NULL)
 * 1 <= count <= BITNET_STACK_MAX.  m > BITNET_GEMV_MAX_M is processed in
 * slices of at most BITNET_GEMV_MAX_M tokens.
 */
BITNET_API bitnet_status bitnet_linear_stack(const float *const *x, int64_t m, const bitnet_tw *w,
                                  int64_t count, float *const *y, int32_t *const *acc_out,
                                  int32_t *d_flags, void *stream);

/*
 * The entry points above with a fused epilogue (bitnet_epilogue).  Arguments,
 * layouts and errors are those of the call without the suffix; `epi` is a
 * host pointer to one descriptor (bitnet_linear_ex, bitnet_linear_q_ex) or a
 * host array of `count` descriptors, one per layer (the stack and grouped
 * calls), and may be NULL (no epilogue).  The residual of layer i is
 * [m, w[i].n]; m > BITNET_GEMV_MAX_M on the stack call is processed in
 * slices like the outputs.  A descriptor with reserved != 0 returns
 * BITNET_ERR_INVALID_ARG.
 */
BITNET_API bitnet_status bitnet_linear_ex(const float *x, int64_t m, const bitnet_tw *w, const bitnet_epilogue *epi,
                                          float *y, int32_t *acc_out, void *workspace, size_t workspace_bytes,
                                          int32_t *d_flags, void *stream);
BITNET_API bitnet_status bitnet_linear_q_ex(const int8_t *xq, const float *act_scale, int64_t m, const bitnet_tw *w,
                                            const bitnet_epilogue *epi, float *y, int32_t *acc_out,
                                            int32_t *d_flags, void *stream);
BITNET_API bitnet_status bitnet_linear_q_grouped_ex(const int8_t *const *xq, const float *const *act_scale,
                                                    int64_t m, const bitnet_tw *w, const bitnet_epilogue *epi,
                                                    int64_t count, float *const *y, int32_t *const *acc_out,
                                                    int32_t *d_flags, void *stream);
BITNET_API bitnet_status bitnet_linear_stack_ex(const float *const *x, int64_t m, const bitnet_tw *w,
                                                const bitnet_epilogue *epi, int64_t count, float *const *y,
                                                int32_t *const *acc_out, int32_t *d_flags, void *stream);

/*
 * I8_S linear layer: int8 weights x per-token int8 activations (technical
 * report §2.2.1: the full-pipeline INT8 scheme of the VAE tokenizer; §2.4.2:
 * the I8_S kernel works on blocks of Q_K = 32 elements through the same
 * multiply-add pipeline as I2_S).  Weights are plain int8 with one fp32
 * scale per tensor, each row stored as whole Q_K blocks:
 *   w->w      device int8 [n, bitnet_i8_row_bytes(k)], 16-byte aligned; the
 *             pad bytes of each row may hold anything (they meet zero
 *             activations)
 *   w->scale  s_w
 * acc[m,n] = sum_{k<K} q[m,k] * w[n,k] exactly; y = ((float)acc * s_act) *
 * s_w (the int-to-float conversion rounds to nearest even once |acc| > 2^24),
 * then the optional epilogue (NULL: none).  x, y, acc_out and d_flags as in
 * bitnet_linear.  The activations are quantised into the caller's workspace
 * (>= bitnet_linear_i8_workspace_bytes(m, k), 256-byte aligned), then the
 * GEMV streams the weight rows in slices of at most 8 tokens.
 */
typedef struct {
    const int8_t *w;
    int64_t n;
    int64_t k;
    float scale;
} bitnet_i8w;

/* Bytes of one I8_S weight row: 32 * ceil(k/32); 0 on bad k. */
BITNET_API size_t bitnet_i8_row_bytes(int64_t k);

/* Workspace of bitnet_linear_i8: int8 activations [m, bitnet_kpad(k)] and
 * their scales; 0 on bad sizes. */
BITNET_API size_t bitnet_linear_i8_workspace_bytes(int64_t m, int64_t k);

BITNET_API bitnet_status bitnet_linear_i8(const float *x, int64_t m, const bitnet_i8w *w, const bitnet_epilogue *epi,
                                          float *y, int32_t *acc_out, void *workspace, size_t workspace_bytes,
                                          int32_t *d_flags, void *stream);

/*
 * `count` I8_S layers sharing the token count m in one GEMV launch per slice
 * of at most 8 tokens (the decoder-layer pattern: several linears, some on
 * the same input).  Distinct inputs (same x pointer and k) are quantised
 * once each into the workspace, then one launch streams the rows of all the
 * layers.  Arguments as bitnet_linear_i8, per layer: x[i], w[i], y[i],
 * acc_out (NULL or an array of `count` entries that may be NULL), epi (NULL
 * or an array of `count` descriptors).  workspace >=
 * bitnet_linear_i8_grouped_workspace_bytes(x, m, w, count), 256-byte
 * aligned.  1 <= count <= BITNET_I8_GROUP_MAX.
 */
#define BITNET_I8_GROUP_MAX 64
BITNET_API size_t bitnet_linear_i8_grouped_workspace_bytes(const float *const *x, int64_t m, const bitnet_i8w *w,
                                                           int64_t count);
BITNET_API bitnet_status bitnet_linear_i8_grouped(const float *const *x, int64_t m, const bitnet_i8w *w,
                                                  const bitnet_epilogue *epi, int64_t count, float *const *y,
                                                  int32_t *const *acc_out, void *workspace, size_t workspace_bytes,
                                                  int32_t *d_flags, void *stream);

/*
 * bitnet_linear_stack with no device allocation, for callers that cannot call
 * cudaMalloc: code running where the allocator is owned by someone else (a
 * host framework with its own pooling allocator, a real-time loop that must not
 * take the allocator's locks, a process whose memory is reserved up front) or
 * that must not grow the device footprint after start-up.  The technical report
 * has no counterpart to this entry point.
 *
 * Same arguments, layouts, results and errors as bitnet_linear_stack.  The
 * per-layer TMA tensor maps, which bitnet_linear_stack keeps in an allocated
 * per-device cache, are written instead into one fixed array of 256 maps
 * (32 KB) that is part of the library's device image: every GPU that loads the
 * library holds it until the process exits.  Limit: count <= 256
 * (BITNET_STACK_MAX); a larger count returns BITNET_ERR_INVALID_ARG.
 * - No cudaMalloc, cudaFree, pinned or other allocation is made.
 * - The first call on a device looks up the array's device address; make that
 *   first call before any stream capture.
 * - The array is shared by every call and keeps the last call's maps.  A call
 *   whose weight descriptors differ from the ones the array holds rewrites it
 *   with a copy from host memory on `stream` (that copy waits for earlier work
 *   on `stream`).  Calls that overlap on the GPU (other streams, other host
 *   threads) race on the array and must not be made.
 */
BITNET_API bitnet_status bitnet_linear_stack_noalloc(const float *const *x, int64_t m, const bitnet_tw *w,
                                                     int64_t count, float *const *y, int32_t *const *acc_out,
                                                     int32_t *d_flags, void *stream);

/* Free the current device's tensor-map cache (waits for the device to be
 * idle first).  Later calls rebuild entries as needed. */
BITNET_API bitnet_status bitnet_release_device_cache(void);

/* Test aid: bound, in SM clock cycles, on every device-side wait (0 = the
 * built-in bound of about 2^31 cycles).  A wait that runs past it makes the
 * kernel raise BITNET_FLAG_TIMEOUT and return instead of hanging.
 * Process-wide; affects launches made after the call. */
BITNET_API bitnet_status bitnet_debug_set_wait_limit(uint64_t cycles);

/* Test aid: when on, the GEMV kernels of later launches first wait on a
 * barrier that nothing ever completes, so that the bounded wait expires; they
 * raise BITNET_FLAG_TIMEOUT and return without writing outputs.  Used to test
 * the timeout path without faulting or hanging a GPU.  Process-wide. */
BITNET_API bitnet_status bitnet_debug_force_stall(int on);

/* Profiling aid: when d_trace (device memory) is not NULL, GEMV launches made
 * after the call write, per CTA c and warp w of the launch, 8 uint64
 * %globaltimer stamps (ns) at d_trace[(c*warps + w)*8 + e]: e = 0 set-up done,
 * 1 first weight copies issued, 2 activations quantised, 3 first chunk landed,
 * 4 last chunk consumed (other slots unused).  The buffer must hold
 * 8 * warps * CTAs entries (at most 8 * 16 * 160).  Tensor-core GEMM launches
 * (m > 8) write SM clock (clock64) stamps of CTA 0: for its first 48 K blocks
 * it, d_trace[it*16 + e]: e = 0 TMA issued, 1/2 MMA thread saw the tile / the
 * expanded weights, 3 MMAs issued, 4+q / 8+q / 12+q expander warp of TMEM lane
 * quadrant q saw the tile / a free weight buffer / finished writing it; then
 * d_trace[768 + 0] kernel entry, [768 + 1] set-up done, [768 + 2] all roles
 * done, [768 + 3] / [768 + 4] %globaltimer (ns) at entry / at the end,
 * [768 + 8 + t] epilogue of the CTA's tile t done and [768 + 24 + t] MMA
 * thread found tile t's accumulator free (t < 16).
 * NULL turns it off. */
BITNET_API bitnet_status bitnet_debug_set_trace(void *d_trace);

#ifdef __cplusplus
}
#endif
#endif /* BITNET_H */
