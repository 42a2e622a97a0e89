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

static unsigned bd_grid(int64_t nblocks, int num_sms)
{
    const int64_t want = (nblocks + kBdWarps - 1) / kBdWarps;
    const int64_t cap = (int64_t)num_sms * 6;
    return (unsigned)(want < cap ? (want > 0 ? want : 1) : cap);
}

cudaError_t launch_quantize_bd(const QuantArgs &a, cudaStream_t st)
{
    if (!bd_size(a.d)) return cudaErrorNotSupported;
    const BdGeom G = bd_geom(a.d);
    const unsigned grid = bd_grid(a.nblocks, a.num_sms);
    const uint16_t *x = static_cast<const uint16_t *>(a.x);
    uint8_t *codes = static_cast<uint8_t *>(a.codes);
    if (a.bf16)
        quantize_bd_kernel<true><<<grid, kBdWarps * 32, 0, st>>>(x, a.nblocks, a.d, a.pw, *a.tables, G, codes, a.norms);
    else
        quantize_bd_kernel<false><<<grid, kBdWarps * 32, 0, st>>>(x, a.nblocks, a.d, a.pw, *a.tables, G, codes, a.norms);
    note_launch("quantize_bd_kernel");
    return cudaGetLastError();
}

cudaError_t launch_dequantize_bd(const DequantArgs &a, cudaStream_t st)
{
    if (!bd_size(a.d)) return cudaErrorNotSupported;
    const BdGeom G = bd_geom(a.d);
    const unsigned grid = bd_grid(a.nblocks, a.num_sms);
    const uint8_t *codes = static_cast<const uint8_t *>(a.codes);
    uint16_t *out = static_cast<uint16_t *>(a.out);
    if (a.bf16)
        dequantize_bd_kernel<true><<<grid, kBdWarps * 32, 0, st>>>(codes, a.norms, a.nblocks, a.d, a.pw, *a.tables, G,
                                                                   out);
    else
        dequantize_bd_kernel<false><<<grid, kBdWarps * 32, 0, st>>>(codes, a.norms, a.nblocks, a.d, a.pw, *a.tables, G,
                                                                    out);
    note_launch("dequantize_bd_kernel");
    return cudaGetLastError();
}

}  // namespace rq
