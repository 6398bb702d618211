// Arguments of the pipelined per-group quantizer, shared by the dispatcher
// (bq_pipe.cu) and the per-dtype kernel translation units.
#pragma once

#include <stdint.h>

#include "bq_internal.h"

namespace bq {

enum PipeKind { PK_INT_Q = 0, PK_INT_FAKE = 1, PK_FP8 = 2, PK_MX = 3, PK_NV = 4, PK_MX4 = 5 };

struct PipeArgs {
    const void* x;
    int64_t n_seg;
    int G;              // elements per group
    int P;              // groups per tile (256 / TEAM)
    int64_t n_tiles;
    int slot_bytes;     // P * G * sizeof(T)
    int stages;
    IntCfg cfg;
    uint8_t* q;         // int codes, or FP8 / FP4 codes
    void* y;            // fake-quantized output
    float* scale;       // int / FP8 1x128 scales
    uint8_t* zp;        // int zero-points, or MXFP8 / NVFP4 scale bytes
    const unsigned long long* amax_rec;
    float* global_scale;
    int static_global;  // 0: record from the range kernel before; 1: static; 2: caller's record
};

// Column groups with dynamic scales through the 2D-TMA ring (k_col_tma): x
// row-major [rows, inner], groups of gs consecutive rows at one column.
struct ColPipeArgs {
    const void* x;
    int64_t rows, inner, gs;
    IntCfg cfg;
    float* scale;       // [rows / gs, inner]
    uint8_t* zp;        // [rows / gs, inner] or null
    void* out;          // codes (quantize) or x's dtype (fake-quantize)
};

}  // namespace bq
