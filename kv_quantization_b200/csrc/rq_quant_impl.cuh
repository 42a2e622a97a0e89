// rq_quant_impl.cuh -- fused quantize / dequantize / sketch kernels (sm_100a).
// Included once per (d, dtype) translation unit (rq_quant_d*.cu).
//
// Blockwise rotated scalar quantization (eliza quantization README, section
// "PolarQuant", "Algorithm in one paragraph"): per block of d values the fp16
// L2 norm, the seeded sign flip, the Walsh-Hadamard rotation, the nearest
// Lloyd-Max centroid and the packed index; the inverse looks the centroid up,
// rotates back and rescales.  One HBM pass each way: values are read once,
// codes and norms written once (and vice versa).
//
// Work mapping: a CTA of 128 threads owns a tile of 128 "thread rows", each
// row E = min(d, 128) contiguous values; a block of d values is TPB = d / E
// consecutive lanes.  Tiles move between HBM and a swizzled shared-memory
// buffer with 16-byte coalesced accesses (chunk c of row r sits at slot
// c ^ (r mod NCH), so both the coalesced tile copy and the per-row reads are
// free of bank conflicts); everything else happens in registers.
#pragma once
#include <cstdint>

#include "rq_common.cuh"
#include "rq_kernels.h"

namespace rq {

constexpr int kThreads = 128;   // threads per CTA = thread rows per tile

// Shared-memory tables copied from the by-value parameter block.
__device__ __forceinline__ void setup_lut(const QuantTables &T, uint2 *lut, float *bnd)
{
    if (T.lut_cells > 0) {
        for (int i = threadIdx.x; i < T.lut_cells * 16; i += blockDim.x)
            lut[i] = make_uint2(__float_as_uint(T.lut_t[i >> 4]), T.lut_k[i >> 4]);
    } else {
        for (int i = threadIdx.x; i < T.levels; i += blockDim.x) bnd[i] = T.bound[i];
    }
}

// Centroid table replicated 32 times so that lane l always reads bank l.
__device__ __forceinline__ void setup_centroids(const QuantTables &T, float *cent, int entries)
{
    for (int i = threadIdx.x; i < entries * 32; i += blockDim.x) {
        int k = i >> 5;
        cent[i] = k < T.levels ? T.centroid[k] : 0.0f;
    }
}

// Coalesced copy of rows [row0, row0 + kThreads) of a row-major array of
// NCH 16-byte chunks per row into the swizzled tile (zero past `rows_left`).
template <int NCH>
__device__ __forceinline__ void load_tile(uint4 *tile, const uint4 *__restrict__ src, int64_t rows_left)
{
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
        const int q = i * kThreads + threadIdx.x;
        const int r = q / NCH, c = q % NCH;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (r < rows_left) v = __ldg(src + q);
        tile[r * NCH + (c ^ (r % NCH))] = v;
    }
}

template <int NCH>
__device__ __forceinline__ void store_tile(const uint4 *tile, uint4 *__restrict__ dst, int64_t rows_left)
{
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
        const int q = i * kThreads + threadIdx.x;
        const int r = q / NCH, c = q % NCH;
        if (r < rows_left) dst[q] = tile[r * NCH + (c ^ (r % NCH))];
    }
}

// Read this thread's row (E values) from the tile as fp32.
template <int E, bool BF16>
__device__ __forceinline__ void read_row(const uint4 *tile, int r, float *v)
{
    constexpr int NCH = E * 2 / 16;
#pragma unroll
    for (int k = 0; k < NCH; ++k) {
        uint4 w = tile[r * NCH + (k ^ (r % NCH))];
        unpack2<BF16>(w.x, v[8 * k + 0], v[8 * k + 1]);
        unpack2<BF16>(w.y, v[8 * k + 2], v[8 * k + 3]);
        unpack2<BF16>(w.z, v[8 * k + 4], v[8 * k + 5]);
        unpack2<BF16>(w.w, v[8 * k + 6], v[8 * k + 7]);
    }
}

template <int E, bool BF16>
__device__ __forceinline__ void write_row(uint4 *tile, int r, const float *v)
{
    constexpr int NCH = E * 2 / 16;
#pragma unroll
    for (int k = 0; k < NCH; ++k) {
        uint4 w;
        w.x = pack2<BF16>(v[8 * k + 0], v[8 * k + 1]);
        w.y = pack2<BF16>(v[8 * k + 2], v[8 * k + 3]);
        w.z = pack2<BF16>(v[8 * k + 4], v[8 * k + 5]);
        w.w = pack2<BF16>(v[8 * k + 6], v[8 * k + 7]);
        tile[r * NCH + (k ^ (r % NCH))] = w;
    }
}

template <int E>
__device__ __forceinline__ void apply_signs(float *v, const uint32_t *sign_words, int part)
{
#pragma unroll
    for (int j = 0; j < E; ++j)
        v[j] = __uint_as_float(__float_as_uint(v[j]) ^ sign_mask(sign_words, part * E + j));
}

// Canonical fp32 norm of a block held as TPB parts of E values.
template <int E, int TPB>
__device__ __forceinline__ float block_norm(const float *v)
{
    float sq[E];
#pragma unroll
    for (int j = 0; j < E; ++j) sq[j] = __fmul_rn(v[j], v[j]);
    return __fsqrt_rn(combine_parts<TPB>(pairwise_sum<E>(sq)));
}


// Sign bits of S v for one vector held as TPB parts of E values (each value
// a 16-bit number widened to fp32): P_i accumulated in fp64 from exact
// products, so the bit is the sign of the exact dot product; bit i =
// (P_i >= 0), stored LSB-first, 8 per byte, when dst != nullptr.
template <int E, int TPB, bool SBF16>
__device__ __forceinline__ void sketch_signs(const float *v, const void *proj, int D, int m, int part, uint8_t *dst)
{
    constexpr int NCH = E * 2 / 16;
    const uint8_t *Sb = reinterpret_cast<const uint8_t *>(proj) + (size_t)part * E * 2;
    uint32_t word = 0u;
    for (int i = 0; i < m; ++i) {
        const uint4 *Si = reinterpret_cast<const uint4 *>(Sb + (size_t)i * D * 2);
        double acc = 0.0;
#pragma unroll
        for (int k = 0; k < NCH; ++k) {
            const uint4 s = __ldg(Si + k);
            const uint32_t sw[4] = {s.x, s.y, s.z, s.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float a0, a1;
                unpack2<SBF16>(sw[q], a0, a1);
                acc = fma((double)a0, (double)v[8 * k + 2 * q], acc);
                acc = fma((double)a1, (double)v[8 * k + 2 * q + 1], acc);
            }
        }
#pragma unroll
        for (int off = 1; off < TPB; off *= 2) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        word |= (acc >= 0.0 ? 1u : 0u) << (i & 7);
        if ((i & 7) == 7) {
            if (dst) dst[i >> 3] = (uint8_t)word;
            word = 0u;
        }
    }
}

// --------------------------------------------------------------------------
// Quantize (optionally with the fused QJL residual sketch).
// --------------------------------------------------------------------------
template <int D, int PW, bool BF16, bool QJL>
__global__ void __launch_bounds__(kThreads)
quantize_kernel(const uint8_t *__restrict__ x, int64_t nblocks, const __grid_constant__ QuantTables T,
                uint8_t *__restrict__ codes, uint16_t *__restrict__ norms,
                int m, const uint16_t *__restrict__ proj, uint8_t *__restrict__ qsigns,
                uint16_t *__restrict__ qnorms)
{
    constexpr int E = D < 128 ? D : 128;
    constexpr int TPB = D / E;
    constexpr int NCH = E * 2 / 16;
    constexpr int CB = E * PW / 8;              // code bytes per thread row
    constexpr int NW = (E * PW + 31) / 32;
    extern __shared__ __align__(16) uint8_t smem[];
    uint4 *tile = reinterpret_cast<uint4 *>(smem);
    uint2 *lut = reinterpret_cast<uint2 *>(smem + kThreads * E * 2);
    float *bnd = reinterpret_cast<float *>(lut);
    float *cent = reinterpret_cast<float *>(smem + kThreads * E * 2 + kMaxLutCells * 16 * 8);

    setup_lut(T, lut, bnd);
    if constexpr (QJL) setup_centroids(T, cent, 1 << PW);

    const int tid = threadIdx.x, lane = tid & 31, part = tid % TPB;
    const int64_t total_rows = nblocks * TPB;
    const float lut_a = T.lut_a, lut_b = T.lut_b;
    const int cells = T.lut_cells, levels = T.levels;

    for (int64_t row0 = (int64_t)blockIdx.x * kThreads; row0 < total_rows; row0 += (int64_t)gridDim.x * kThreads) {
        __syncthreads();   // tables ready / previous tile fully consumed
        load_tile<NCH>(tile, reinterpret_cast<const uint4 *>(x) + row0 * NCH, total_rows - row0);
        __syncthreads();
        const int64_t row = row0 + tid;
        const bool valid = row < total_rows;

        float v[E];
        read_row<E, BF16>(tile, tid, v);
        const float n32 = block_norm<E, TPB>(v);
        apply_signs<E>(v, T.sign_words, part);
        fwht_local<E>(v);
        fwht_cross<E, TPB>(v, part);
        const float inv = n32 > 0.0f ? __frcp_rn(n32) : 0.0f;

        uint32_t code[E];
        if (cells > 0) {
#pragma unroll
            for (int j = 0; j < E; ++j) code[j] = lut_code(__fmul_rn(v[j], inv), lut, lut_a, lut_b, cells, lane & 15);
        } else {
#pragma unroll
            for (int j = 0; j < E; ++j) code[j] = bsearch_code(__fmul_rn(v[j], inv), bnd, levels);
        }
        uint32_t w[NW];
        pack_codes<E, PW>(code, w);
        const uint16_t n16 = norm_to_h16(n32);
        if (valid) {
            store_bytes<CB>(codes + row * CB, w);
            if (part == 0) norms[row / TPB] = n16;
        }

        if constexpr (QJL) {
            // First-stage reconstruction in fp32 (canonical), then r = x - x^32.
#pragma unroll
            for (int j = 0; j < E; ++j) v[j] = cent[code[j] * 32 + lane];
            fwht_local<E>(v);
            fwht_cross<E, TPB>(v, part);
            const float scale = __fmul_rn(h16_to_f32(n16), 1.0f / (float)D);
            float xr[E];
            read_row<E, BF16>(tile, tid, xr);
#pragma unroll
            for (int j = 0; j < E; ++j) {
                float xh = __uint_as_float(__float_as_uint(__fmul_rn(v[j], scale)) ^ sign_mask(T.sign_words, part * E + j));
                v[j] = __fsub_rn(xr[j], xh);
            }
            const float rn32 = block_norm<E, TPB>(v);
            // Sketch of bf16(r): P_i = sum_j S_ij r_j (fp64 accumulation of exact products).
#pragma unroll
            for (int j = 0; j < E; ++j) v[j] = __bfloat162float(__float2bfloat16_rn(v[j]));
            const int64_t blk = row / TPB;
            sketch_signs<E, TPB, true>(v, proj, D, m, part, (valid && part == 0) ? qsigns + blk * (m / 8) : nullptr);
            if (valid && part == 0) qnorms[blk] = norm_to_h16(rn32);
        }
    }
}

// --------------------------------------------------------------------------
// Dequantize.
// --------------------------------------------------------------------------
template <int D, int PW, bool BF16>
__global__ void __launch_bounds__(kThreads)
dequantize_kernel(const uint8_t *__restrict__ codes, const uint16_t *__restrict__ norms, int64_t nblocks,
                  const __grid_constant__ QuantTables T, uint8_t *__restrict__ out)
{
    constexpr int E = D < 128 ? D : 128;
    constexpr int TPB = D / E;
    constexpr int NCH = E * 2 / 16;
    constexpr int CB = E * PW / 8;
    constexpr int NW = (E * PW + 31) / 32;
    extern __shared__ __align__(16) uint8_t smem[];
    uint4 *tile = reinterpret_cast<uint4 *>(smem);
    float *cent = reinterpret_cast<float *>(smem + kThreads * E * 2);
    setup_centroids(T, cent, 1 << PW);

    const int tid = threadIdx.x, lane = tid & 31, part = tid % TPB;
    const int64_t total_rows = nblocks * TPB;
    for (int64_t row0 = (int64_t)blockIdx.x * kThreads; row0 < total_rows; row0 += (int64_t)gridDim.x * kThreads) {
        const int64_t row = row0 + tid;
        const bool valid = row < total_rows;
        uint32_t w[NW];
        float scale = 0.0f;
        if (valid) {
            load_bytes<CB>(codes + row * CB, w);
            scale = __fmul_rn(h16_to_f32(__ldg(norms + row / TPB)), 1.0f / (float)D);
        } else {
#pragma unroll
            for (int i = 0; i < NW; ++i) w[i] = 0u;
        }
        float v[E];
#pragma unroll
        for (int j = 0; j < E; ++j) v[j] = cent[unpack_code<E, PW>(w, j) * 32 + lane];
        fwht_local<E>(v);
        fwht_cross<E, TPB>(v, part);
#pragma unroll
        for (int j = 0; j < E; ++j)
            v[j] = __uint_as_float(__float_as_uint(__fmul_rn(v[j], scale)) ^ sign_mask(T.sign_words, part * E + j));
        __syncthreads();   // previous tile stored
        write_row<E, BF16>(tile, tid, v);
        __syncthreads();
        store_tile<NCH>(tile, reinterpret_cast<uint4 *>(out) + row0 * NCH, total_rows - row0);
    }
}


// --------------------------------------------------------------------------
// QJL sketch of plain vectors (keys): signs of S x and fp16 ||x||.
// --------------------------------------------------------------------------
template <int D, bool BF16>
__global__ void __launch_bounds__(kThreads)
sketch_kernel(const uint8_t *__restrict__ x, int64_t nvec, int m, const uint16_t *__restrict__ proj,
              uint8_t *__restrict__ signs, uint16_t *__restrict__ norms)
{
    constexpr int E = D < 128 ? D : 128;
    constexpr int TPB = D / E;
    constexpr int NCH = E * 2 / 16;
    extern __shared__ __align__(16) uint8_t smem[];
    uint4 *tile = reinterpret_cast<uint4 *>(smem);
    const int tid = threadIdx.x, part = tid % TPB;
    const int64_t total_rows = nvec * TPB;
    for (int64_t row0 = (int64_t)blockIdx.x * kThreads; row0 < total_rows; row0 += (int64_t)gridDim.x * kThreads) {
        __syncthreads();
        load_tile<NCH>(tile, reinterpret_cast<const uint4 *>(x) + row0 * NCH, total_rows - row0);
        __syncthreads();
        const int64_t row = row0 + tid;
        const bool valid = row < total_rows;
        float v[E];
        read_row<E, BF16>(tile, tid, v);
        const float n32 = block_norm<E, TPB>(v);
        const int64_t vec = row / TPB;
        sketch_signs<E, TPB, BF16>(v, proj, D, m, part, (valid && part == 0) ? signs + vec * (m / 8) : nullptr);
        if (valid && part == 0) norms[vec] = norm_to_h16(n32);
    }
}

}  // namespace rq
