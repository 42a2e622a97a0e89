// rq_bd.cuh -- rotated scalar quantization of blocks whose size d is not a
// power of two (sm_100a).
//
// The block is transformed block-diagonally: d is decomposed into powers of
// two, largest first (GLQ README, "Bit widths": 2688 = 2048 + 512 + 128), and
// each sub-block of size b gets its own Walsh-Hadamard transform after the
// seeded sign diagonal (turbopress "Package layout": block-diagonal
// Walsh-Hadamard times Rademacher signs).  With R = blockdiag(H_b / sqrt(b)) D
// orthogonal, the coordinates are y = sqrt(d) R x / ||x|| and the
// reconstruction x^ = ||x|| R^T c / sqrt(d).  In the canonical fp32 order:
//   norm: squares, pairwise sums within each sub-block, the sub-block sums
//         added in order, correctly rounded square root;
//   y_j  = w_j * fl32(g_b * inv),  g_b = fl32(sqrt(d / b)), inv = fl32(1 / n32),
//   x^_j = s_j * (w'_j * fl32(n16 * h_b)),  h_b = fl32(1 / sqrt(d b)),
// with w = H_b D x and w' = H_b c in radix-2 stages h = 1, 2, ... b/2.
//
// One warp per block: value j = 32 k + lane sits in register k of lane
// `lane` (d / 32 registers, d a multiple of 32 and every sub-block at least
// 32).  Stages h < 32 are lane shuffles, h >= 32 pair registers of the same
// lane; the pairwise norm tree within a 32-value chunk is the xor butterfly.
// Codes go through a per-warp byte array in shared memory and are packed
// LSB-first by whole 32-bit words.
#pragma once
#include <cstdint>

#include "rq_common.cuh"

namespace rq {

constexpr int kBdWarps = 8;
constexpr int kBdMaxK = 16;          // d / 32 <= 16
constexpr int kBdMaxSub = 5;

struct BdGeom {
    int nsub;
    int k0[kBdMaxSub];               // first 32-value chunk of each sub-block
    int nk[kBdMaxSub];               // chunks in it (a power of two)
    float g[kBdMaxSub];              // fl32(sqrt(d / b))
    float h[kBdMaxSub];              // fl32(1 / sqrt(d b))
};

__device__ __forceinline__ float bd_load16(const uint16_t *p, bool bf16)
{
    const uint32_t u = (uint32_t)__ldg(p);
    return bf16 ? __uint_as_float(u << 16) : h16_to_f32((uint16_t)u);
}

// In-place block-diagonal transform of the warp's block (registers v[0 .. nk)):
// stages h = 1 ... 16 by lane shuffles, then the warp's copy of the block in
// shared memory (`sm`, d floats) takes the stages h = 32 ... b/2 of every
// sub-block, one butterfly per lane and step.
__device__ __forceinline__ void bd_fwht(float (&v)[kBdMaxK], const BdGeom &G, int nk, int lane, float *sm)
{
#pragma unroll
    for (int hs = 1; hs < 32; hs *= 2) {
#pragma unroll
        for (int k = 0; k < kBdMaxK; ++k) {
            const float p = __shfl_xor_sync(0xffffffffu, v[k], hs);
            v[k] = (lane & hs) ? __fsub_rn(p, v[k]) : __fadd_rn(v[k], p);
        }
    }
    __syncwarp();
#pragma unroll
    for (int k = 0; k < kBdMaxK; ++k)
        if (k < nk) sm[32 * k + lane] = v[k];
    __syncwarp();
    for (int i = 0; i < G.nsub; ++i) {
        const int off = 32 * G.k0[i], b = 32 * G.nk[i];
        for (int h = 32; h < b; h *= 2) {
            for (int p = lane; p < b / 2; p += 32) {
                const int j0 = off + (p / h) * 2 * h + (p % h);
                const float a = sm[j0], c = sm[j0 + h];
                sm[j0] = __fadd_rn(a, c);
                sm[j0 + h] = __fsub_rn(a, c);
            }
            __syncwarp();
        }
    }
#pragma unroll
    for (int k = 0; k < kBdMaxK; ++k)
        if (k < nk) v[k] = sm[32 * k + lane];
}

template <bool BF16>
__global__ void __launch_bounds__(kBdWarps * 32)
quantize_bd_kernel(const uint16_t *__restrict__ x, int64_t nblocks, int d, int pw,
                   const __grid_constant__ QuantTables T, const __grid_constant__ BdGeom G,
                   uint8_t *__restrict__ codes, uint16_t *__restrict__ norms)
{
    __shared__ float bnd[256];
    __shared__ __align__(16) uint8_t cbuf[kBdWarps][512];
    __shared__ float fbufq[kBdWarps][512];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) bnd[i] = i < T.levels - 1 ? T.bound[i] : INFINITY;
    __syncthreads();
    const int nk = d / 32;
    const bool int8 = pw == 8;                           // one byte per code (either layout)
    const int cb = d * pw / 8;                           // a multiple of 4
    uint32_t smask = 0;                                  // sign bits of this lane's values
#pragma unroll
    for (int k = 0; k < kBdMaxK; ++k)
        if (k < nk) smask |= ((T.sign_words[k] >> lane) & 1u) << k;
    uint8_t *cw = cbuf[warp];
    float *fsm = fbufq[warp];
    for (int64_t b = (int64_t)blockIdx.x * kBdWarps + warp; b < nblocks; b += (int64_t)gridDim.x * kBdWarps) {
        float v[kBdMaxK];
#pragma unroll
        for (int k = 0; k < kBdMaxK; ++k) v[k] = k < nk ? bd_load16(x + b * d + 32 * k + lane, BF16) : 0.0f;
        // norm: chunk sums by the xor butterfly (pairwise within 32 values), then the chunks of a
        // sub-block pairwise, then the sub-blocks in order
        __syncwarp();                                    // the previous block's use of fsm is over
#pragma unroll
        for (int k = 0; k < kBdMaxK; ++k) {
            float s = __fmul_rn(v[k], v[k]);
#pragma unroll
            for (int o = 1; o < 32; o *= 2) s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, o));
            if (lane == 0 && k < nk) fsm[k] = s;
        }
        __syncwarp();
        float tot = 0.0f;
        if (lane == 0) {
            for (int i = 0; i < G.nsub; ++i) {
                const int k0 = G.k0[i], m = G.nk[i];
                for (int hk = 1; hk < m; hk *= 2)
                    for (int r = 0; r < m; r += 2 * hk) fsm[k0 + r] = __fadd_rn(fsm[k0 + r], fsm[k0 + r + hk]);
                tot = i == 0 ? fsm[k0] : __fadd_rn(tot, fsm[k0]);
            }
        }
        tot = __shfl_sync(0xffffffffu, tot, 0);
        const float n32 = __fsqrt_rn(tot);
        // signs, transform, coordinates, codes
#pragma unroll
        for (int k = 0; k < kBdMaxK; ++k)
            if ((smask >> k) & 1u) v[k] = -v[k];
        bd_fwht(v, G, nk, lane, fsm);
        const float inv = n32 > 0.0f ? __frcp_rn(n32) : 0.0f;
        __syncwarp();                                    // the previous block's codes have been packed
        for (int i = 0; i < G.nsub; ++i) {
            const float f = __fmul_rn(G.g[i], inv);
#pragma unroll
            for (int k = 0; k < kBdMaxK; ++k) {
                const int r = k - G.k0[i];
                if (r >= 0 && r < G.nk[i]) {
                    const float y = __fmul_rn(v[k], f);
                    cw[32 * k + lane] = (uint8_t)bsearch_code(y, bnd, T.levels);
                }
            }
        }
        __syncwarp();
        uint8_t *dst = codes + b * cb;
        if (int8) {
            for (int i = lane; i < d / 4; i += 32)
                reinterpret_cast<uint32_t *>(dst)[i] = reinterpret_cast<const uint32_t *>(cw)[i];
        } else {
            for (int w = lane; w < cb / 4; w += 32) {   // field word w: bits [32 w, 32 w + 32)
                uint32_t word = 0u;
                const int j0 = (32 * w) / pw, j1 = (32 * w + 31) / pw;
                for (int j = j0; j <= j1 && j < d; ++j) {
                    const int bit = j * pw - 32 * w;    // may be negative for the first code
                    const uint32_t c = cw[j];
                    word |= bit >= 0 ? (c << bit) : (c >> (-bit));
                }
                reinterpret_cast<uint32_t *>(dst)[w] = word;
            }
        }
        if (lane == 0) norms[b] = norm_to_h16(n32);
    }
}

template <bool BF16>
__global__ void __launch_bounds__(kBdWarps * 32)
dequantize_bd_kernel(const uint8_t *__restrict__ codes, const uint16_t *__restrict__ norms, int64_t nblocks,
                     int d, int pw, const __grid_constant__ QuantTables T,
                     const __grid_constant__ BdGeom G, uint16_t *__restrict__ out)
{
    __shared__ float cent[256];
    __shared__ uint32_t fbuf[kBdWarps][128];
    __shared__ float fbufd[kBdWarps][512];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) cent[i] = i < T.levels ? T.centroid[i] : 0.0f;
    __syncthreads();
    const int nk = d / 32;
    const bool int8 = pw == 8;
    const int cb = d * pw / 8;
    const uint32_t cmask = (1u << pw) - 1u;
    uint32_t smask = 0;
#pragma unroll
    for (int k = 0; k < kBdMaxK; ++k)
        if (k < nk) smask |= ((T.sign_words[k] >> lane) & 1u) << k;
    uint32_t *fw = fbuf[warp];
    for (int64_t b = (int64_t)blockIdx.x * kBdWarps + warp; b < nblocks; b += (int64_t)gridDim.x * kBdWarps) {
        __syncwarp();                                    // the previous block's field has been read
        for (int i = lane; i < cb / 4; i += 32) fw[i] = __ldg(reinterpret_cast<const uint32_t *>(codes + b * cb) + i);
        __syncwarp();
        float v[kBdMaxK];
#pragma unroll
        for (int k = 0; k < kBdMaxK; ++k) {
            uint32_t c = 0u;
            if (k < nk) {
                const int j = 32 * k + lane;
                if (int8) {
                    c = (fw[j >> 2] >> (8 * (j & 3))) & 0xffu;
                } else {
                    const int bit = j * pw, wi = bit >> 5, sh = bit & 31;
                    c = fw[wi] >> sh;
                    if (sh + pw > 32) c |= fw[wi + 1] << (32 - sh);
                    c &= cmask;
                }
            }
            v[k] = cent[c];
        }
        bd_fwht(v, G, nk, lane, fbufd[warp]);
        const float n16 = h16_to_f32(__ldg(norms + b));
        for (int i = 0; i < G.nsub; ++i) {
            const float sc = __fmul_rn(n16, G.h[i]);
#pragma unroll
            for (int k = 0; k < kBdMaxK; ++k) {
                const int r = k - G.k0[i];
                if (r >= 0 && r < G.nk[i]) {
                    float xh = __fmul_rn(v[k], sc);
                    if ((smask >> k) & 1u) xh = -xh;
                    out[b * d + 32 * k + lane] = BF16 ? __bfloat16_as_ushort(__float2bfloat16_rn(xh))
                                                      : __half_as_ushort(__float2half_rn(xh));
                }
            }
        }
    }
}

}  // namespace rq
