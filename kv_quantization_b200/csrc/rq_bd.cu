// rq_bd.cu -- launchers of the non-power-of-two block kernels (rq_bd.cuh).
#include <cmath>

#include "rq_bd.cuh"
#include "rq_kernels.h"

namespace rq {

bool bd_size(int d) { return d > 64 && d < 512 && d % 32 == 0 && (d & (d - 1)) != 0; }

// Sub-blocks of d, largest power of two first, with the fp32 scales of the
// block-diagonal rotation.
static BdGeom bd_geom(int d)
{
    BdGeom G{};
    int o = 0;
    for (int b = 512; b >= 32; b >>= 1)
        if (d - o >= b) {
            G.k0[G.nsub] = o / 32;
            G.nk[G.nsub] = b / 32;
            G.g[G.nsub] = (float)std::sqrt((double)d / (double)b);
            G.h[G.nsub] = (float)(1.0 / std::sqrt((double)d * (double)b));
            o += b;
            ++G.nsub;
        }
    return G;
}

// Persistent grid: a warp takes W = 32 / (d / 32) consecutive blocks per
// step; at most as many CTAs as fit on the SMs at once.
static unsigned bd_grid(int64_t nblocks, int d, int num_sms, int per_sm)
{
    const int64_t W = 32 / (d / 32);
    const int64_t tasks = (nblocks + W - 1) / W;
    const int64_t want = (tasks + kBdWarps - 1) / kBdWarps;
    const int64_t cap = (int64_t)num_sms * (per_sm > 0 ? per_sm : 1);
    return (unsigned)(want < cap ? (want > 0 ? want : 1) : cap);
}

template <int PW, bool BF16>
static void run_quantize_bd(const QuantArgs &a, const BdGeom &G, cudaStream_t st)
{
    const size_t smem = 2048 + (size_t)(a.tables->sat_cells > 0 ? a.tables->sat_cells : 0) * 128;
    static const int per_sm = [] {        // at the largest table
        int n = 0;
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, quantize_bd_kernel<PW, BF16>, kBdWarps * 32,
                                                      2048 + (size_t)kMaxLutCells * 128);
        return n;
    }();
    const unsigned grid = bd_grid(a.nblocks, a.d, a.num_sms, per_sm);
    quantize_bd_kernel<PW, BF16><<<grid, kBdWarps * 32, smem, st>>>(
        static_cast<const uint16_t *>(a.x), a.nblocks, a.d, *a.tables, G, static_cast<uint8_t *>(a.codes), a.norms);
}

template <int PW, bool BF16>
static void run_dequantize_bd(const DequantArgs &a, const BdGeom &G, cudaStream_t st)
{
    static const int per_sm = [] {
        int n = 0;
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, dequantize_bd_kernel<PW, BF16>, kBdWarps * 32,
                                                      dequantize_bd_smem(PW));
        return n;
    }();
    const unsigned grid = bd_grid(a.nblocks, a.d, a.num_sms, per_sm);
    dequantize_bd_kernel<PW, BF16><<<grid, kBdWarps * 32, dequantize_bd_smem(PW), st>>>(static_cast<const uint8_t *>(a.codes), a.norms,
                                                                    a.nblocks, a.d, *a.tables, G,
                                                                    static_cast<uint16_t *>(a.out));
}

template <bool BF16>
static bool dispatch_quantize_bd(const QuantArgs &a, const BdGeom &G, cudaStream_t st)
{
    switch (a.pw) {
    case 1: run_quantize_bd<1, BF16>(a, G, st); return true;
    case 2: run_quantize_bd<2, BF16>(a, G, st); return true;
    case 3: run_quantize_bd<3, BF16>(a, G, st); return true;
    case 4: run_quantize_bd<4, BF16>(a, G, st); return true;
    case 5: run_quantize_bd<5, BF16>(a, G, st); return true;
    case 6: run_quantize_bd<6, BF16>(a, G, st); return true;
    case 7: run_quantize_bd<7, BF16>(a, G, st); return true;
    case 8: run_quantize_bd<8, BF16>(a, G, st); return true;
    default: return false;
    }
}

template <bool BF16>
static bool dispatch_dequantize_bd(const DequantArgs &a, const BdGeom &G, cudaStream_t st)
{
    switch (a.pw) {
    case 1: run_dequantize_bd<1, BF16>(a, G, st); return true;
    case 2: run_dequantize_bd<2, BF16>(a, G, st); return true;
    case 3: run_dequantize_bd<3, BF16>(a, G, st); return true;
    case 4: run_dequantize_bd<4, BF16>(a, G, st); return true;
    case 5: run_dequantize_bd<5, BF16>(a, G, st); return true;
    case 6: run_dequantize_bd<6, BF16>(a, G, st); return true;
    case 7: run_dequantize_bd<7, BF16>(a, G, st); return true;
    case 8: run_dequantize_bd<8, BF16>(a, G, st); return true;
    default: return false;
    }
}

cudaError_t launch_quantize_bd(const QuantArgs &a, cudaStream_t st)
{
    if (!bd_size(a.d)) return cudaErrorNotSupported;
    const BdGeom G = bd_geom(a.d);
    const bool ok = a.bf16 ? dispatch_quantize_bd<true>(a, G, st) : dispatch_quantize_bd<false>(a, G, st);
    if (!ok) return cudaErrorNotSupported;
    note_launch("quantize_bd_kernel");
    return cudaGetLastError();
}

cudaError_t launch_dequantize_bd(const DequantArgs &a, cudaStream_t st)
{
    if (!bd_size(a.d)) return cudaErrorNotSupported;
    const BdGeom G = bd_geom(a.d);
    const bool ok =
        a.bf16 ? dispatch_dequantize_bd<true>(a, G, st) : dispatch_dequantize_bd<false>(a, G, st);
    if (!ok) return cudaErrorNotSupported;
    note_launch("dequantize_bd_kernel");
    return cudaGetLastError();
}

}  // namespace rq
