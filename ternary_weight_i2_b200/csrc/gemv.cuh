// gemv.cuh -- parameters of the streaming ternary GEMV (decode path).
#pragma once

#include <cstdint>

namespace bitnet {

// A tile is 32 consecutive weight rows of one layer: one lane per row.  A
// unit is a tile's chunk of BOX tensor-map boxes; each box is 128 bytes (four
// 128-element blocks) of each of the tile's 32 rows, 4 KB, landed by one TMA
// load with the 128-byte swizzle.  A warp keeps kSlotsPerWarp units in flight.
constexpr int kTileRows = 32;
constexpr int kSlotsPerWarp = 2;
constexpr int kBoxBytes = 128 * kTileRows;   // 4096
constexpr int kBoxBlocks = 4;                // 128-element blocks per box row

constexpr int slot_bytes(int boxes) { return boxes * kBoxBytes; }

constexpr int kMaxLinears = 256;
constexpr int kMaxInputs = 256;
constexpr int kMaxSegs = 448;
constexpr int kMaxRanges = 160;
constexpr int kMaxRangeInputs = 8;   // distinct inputs one CTA quantises
constexpr int kMaxRangeSegs = 32;
constexpr int kMaxWarps = 16;
constexpr int kMetaBytes = 4096;
constexpr int kSmemLimit = 232448;   // 227 KB opt-in per CTA on sm_100

constexpr int kAlignPad = 1024;             // swizzled TMA boxes need 1024-byte alignment
constexpr int ring_bytes(int nw, int boxes) { return nw * kSlotsPerWarp * slot_bytes(boxes); }
constexpr int x_cap(int nw, int boxes) { return kSmemLimit - kAlignPad - ring_bytes(nw, boxes) - kMetaBytes; }

// Kernel shapes (warps per CTA, boxes per unit) the host chooses from.
struct GemvVariant {
    int nw;
    int boxes;
};
constexpr GemvVariant kVariants[] = {{8, 3}, {16, 1}, {6, 3}, {4, 3}};
constexpr int kNumVariants = 4;
// Largest token count each variant is instantiated for.
constexpr int kVariantMaxM[] = {2, 1, 5, 8};

struct GemvLinear {
    const void *tmap;        // device CUtensorMap of packed [n, 32*kb] bytes, box 128 x 32
    float *y;                // [m, n]
    int32_t *acc;            // [m, n] or null
    const float *bias;       // fused epilogue: [n] or null
    const float *gamma;      // [n] or null (layer scale)
    const float *res;        // [m, n] or null (residual; may be y)
    int32_t n;
    int32_t kb;              // 128-element blocks per row
    float scale;             // s_w
    int16_t input;           // index into inputs[]
    int16_t relu;            // fused epilogue: ReLU after the bias
};

struct GemvInput {
    const void *x;           // fp32 [m, k] (or int8 [m, 128*kb] when pre-quantised)
    const float *scale;      // pre-quantised mode: per-token scales [m]
    int32_t k;
    int32_t kb;
};

struct GemvSeg {
    int16_t lin;
    int16_t slot;            // range-local input slot
    int32_t tile0, tile1;    // tiles [tile0, tile1) of the layer
};

struct GemvRange {
    int16_t seg0, nseg;
    int16_t nin, pad_;
    int16_t in[kMaxRangeInputs];
};

struct GemvParams {
    int32_t m;               // tokens in this launch (== template M)
    int32_t num_ranges;
    int32_t prequant;        // inputs are int8 + scales instead of fp32
    int32_t force_stall;     // test aid: wait on a barrier nobody arrives at
    int32_t *flags;
    uint64_t wait_limit;
    int32_t x_bytes;         // bytes of the shared-memory activation area
    int32_t fence_maps;      // tensor maps may have been rewritten at a reused address
    int32_t has_epi;         // some layer of the launch has a fused-epilogue operand
    uint64_t *trace;         // optional: kTraceEvents globaltimer stamps per warp
    GemvLinear lin[kMaxLinears];
    GemvInput inp[kMaxInputs];
    GemvSeg seg[kMaxSegs];
    GemvRange rng[kMaxRanges];
};

static_assert(sizeof(GemvParams) <= 32760, "kernel parameter block too large");

// Trace events recorded per warp when GemvParams::trace is set:
// 0 set-up done, 1 first copies issued, 2 activations quantised,
// 3 first chunk landed, 4 last chunk consumed.
constexpr int kTraceEvents = 8;

}  // namespace bitnet
