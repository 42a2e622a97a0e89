// rq_params.h -- kernel parameter blocks of librq, shared by host and device code.
#pragma once
#include <cstddef>
#include <cstdint>

namespace rq {

// 1.5 * 2^23: fma(y, a, kLutMagic + b0) lands in [2^23, 2^24) where the fp32
// spacing is 1, so its bit pattern minus kLutMagic's is round(y * a + b0).
constexpr float kLutMagic = 12582912.0f;
constexpr int kMaxLutCells = 128;
constexpr int kMaxLevels = 256;
constexpr size_t kMaxSmemPerBlock = 232448;   // sm_100 opt-in limit (227 KB)

// Per-call tables, passed by value as a kernel parameter (no device allocation).
struct QuantTables {
    float centroid[kMaxLevels];      // 2^bits levels, ascending
    float bound[kMaxLevels];         // K-1 decision thresholds, +inf padded to K
    float lut_t[kMaxLutCells];       // per cell: the one boundary inside it, or +inf
    uint32_t lut_k[kMaxLutCells];    // per cell: #boundaries below the cell
    uint32_t sign_words[16];         // sign diagonal bits, coordinate j -> bit j%32 of word j/32
    float lut_a;                     // cell = clamp(bits(fma(y, lut_a, lut_b)) - bits(magic))
    float lut_b;
    int lut_cells;                   // 0: use the binary search over bound[]
    int levels;                      // K = 2^bits
    // Saturating-grid LUT (one-block-per-thread kernels):
    //   cell = bits(fma(sat(fma(y, sat_a, sat_b)), sat_k, magic)) - bits(magic), in [0, sat_cells)
    // where sat() clamps to [0, 1]; no cell holds more than one boundary.
    float sat_t[kMaxLutCells];       // per cell: the one boundary inside it, or +inf
    uint32_t sat_base[kMaxLutCells]; // per cell: #boundaries below the cell
    float sat_a;
    float sat_b;
    float sat_k;                     // sat_cells - 1
    int sat_cells;                   // 0: no such grid (the caller takes another kernel)
};

}  // namespace rq
