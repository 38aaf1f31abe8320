// gemv.cuh -- parameters of the streaming ternary GEMV (decode path).
#pragma once

#include <cstdint>

namespace bitnet {

// A tile is 32 consecutive weight rows of one layer: one lane per row.
constexpr int kTileRows = 32;
// A chunk is up to kChunkBlocks 128-element blocks (32 bytes each) of a row.
constexpr int kChunkBlocks = 12;
constexpr int kChunkBytes = 32 * kChunkBlocks;
// Shared-memory row pitch of a staged chunk: +16 bytes so that the 32 lanes'
// 16-byte reads of one column fall in distinct bank groups.
constexpr int kSlotPitch = kChunkBytes + 16;
constexpr int kSlotBytes = kTileRows * kSlotPitch;
constexpr int kSlotsPerWarp = 2;

constexpr int kMaxLinears = 256;
constexpr int kMaxInputs = 256;
constexpr int kMaxSegs = 448;
constexpr int kMaxRanges = 160;
constexpr int kMaxRangeInputs = 8;   // distinct inputs one CTA quantises
constexpr int kMaxRangeSegs = 32;
constexpr int kMetaBytes = 4096;
constexpr int kSmemLimit = 232448;   // 227 KB opt-in per CTA on sm_100

struct GemvLinear {
    const uint8_t *packed;   // [n, 32*kb]
    float *y;                // [m, n]
    int32_t *acc;            // [m, n] or null
    int32_t n;
    int32_t kb;              // 128-element blocks per row
    float scale;             // s_w
    int32_t input;           // index into inputs[]
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
    int32_t m;               // tokens in this launch (<= template M)
    int32_t num_ranges;
    int32_t prequant;        // inputs are int8 + scales instead of fp32
    int32_t force_stall;     // test aid: wait on a barrier nobody arrives at
    int32_t *flags;
    uint64_t wait_limit;
    int32_t x_bytes;         // bytes of the shared-memory activation area
    int32_t pad_;
    GemvLinear lin[kMaxLinears];
    GemvInput inp[kMaxInputs];
    GemvSeg seg[kMaxSegs];
    GemvRange rng[kMaxRanges];
};

static_assert(sizeof(GemvParams) <= 32760, "kernel parameter block too large");

// Warps per CTA of the instantiation used for token count M (big-K variants
// use 4 warps to leave more room for activations).
constexpr int gemv_ring_bytes(int nw) { return nw * kSlotsPerWarp * kSlotBytes; }
constexpr int gemv_x_cap(int nw) { return kSmemLimit - gemv_ring_bytes(nw) - kMetaBytes; }

}  // namespace bitnet
