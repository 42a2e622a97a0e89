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
};

}  // namespace rq
