// rq_v2.cuh -- TMA-pipelined quantize / dequantize kernels (sm_100a).
//
// Same arithmetic as the canonical definition (rq_common.cuh): pairwise fp32
// norm, radix-2 Walsh-Hadamard stages h = 1, 2, ..., d/2, y = v * (1/n32),
// exact LUT nearest-centroid search, x^ = s * (w * (n16/d)).
//
// Mapping.  A CTA has 256 threads; thread t owns one 64-value row (128 bytes)
// of a 256-row tile, so a block of d values spans TPB = d/64 consecutive lanes.
// A row is held as 32 float2 P[i] = (v_i, v_{i+32}): the Hadamard stages
// h = 1..16 and the pairwise-norm levels below the top then run as packed
// f32x2 adds on both halves at once, stage h = 32 is the add/sub inside each
// float2, and stages h >= 64 go across lanes with shuffles (one fma per value:
// mine * (+-1) + partner's).
//
// Memory.  quantize: the input tiles stream through a 3-stage ring of 32 KB
// shared-memory buffers filled by 2-D TMA loads (128-byte swizzle, so every
// thread reads its row without bank conflicts); one thread refills a stage as
// soon as all threads have read it.  Codes (8*bits bytes per row) and norms go
// straight to global memory, coalesced across the warp.  dequantize: codes are
// loaded one tile ahead into registers; the bf16/fp16 output rows are written
// to a double-buffered swizzled staging tile and leave through 2-D TMA stores.
#pragma once
#include <cuda.h>

#include "rq_common.cuh"
#include "sm100.cuh"

namespace rq {

constexpr int kT2 = 256;            // threads per CTA = rows per tile
constexpr int kE2 = 64;             // values per row
constexpr int kStages2 = 3;         // input ring depth (quantize)
constexpr int kTileBytes2 = kT2 * kE2 * 2;

// -------------------------------------------------------------- row helpers

template <bool BF16>
__device__ __forceinline__ float half_of(uint32_t w, bool hi)
{
    if constexpr (BF16) {
        return hi ? __uint_as_float(w & 0xffff0000u) : __uint_as_float(w << 16);
    } else {
        return h16_to_f32((uint16_t)(hi ? (w >> 16) : (w & 0xffffu)));
    }
}

// Raw row words (element pairs) -> P[i] = (v_i, v_{i+32}).
template <bool BF16>
__device__ __forceinline__ void row_to_pairs(const uint32_t *u, float2 *P)
{
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        P[i].x = half_of<BF16>(u[i >> 1], i & 1);
        P[i].y = half_of<BF16>(u[16 + (i >> 1)], i & 1);
    }
}

// Pairwise fp32 sum of squares over the 64 values of the row (canonical
// leaves (2k, 2k+1)); both halves of the tree run in the float2 lanes.
__device__ __forceinline__ float row_sumsq(const float2 *P)
{
    float2 s[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) s[i] = __fmul2_rn(P[i], P[i]);
#pragma unroll
    for (int w = 1; w < 32; w *= 2) {
#pragma unroll
        for (int i = 0; i < 32; i += 2 * w) s[i] = __fadd2_rn(s[i], s[i + w]);
    }
    return __fadd_rn(s[0].x, s[0].y);
}

template <int TPB>
__device__ __forceinline__ void fwht_row(float2 *P, int part)
{
    const float2 m1 = make_float2(-1.0f, -1.0f);
#pragma unroll
    for (int h = 1; h < 32; h *= 2) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (i & h) continue;
            const float2 a = P[i], b = P[i + h];
            P[i] = __fadd2_rn(a, b);
            P[i + h] = __ffma2_rn(b, m1, a);           // a - b, one rounding
        }
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) {                      // stage h = 32
        const float a = P[i].x, b = P[i].y;
        P[i].x = __fadd_rn(a, b);
        P[i].y = __fsub_rn(a, b);
    }
#pragma unroll
    for (int s = 0; (1 << s) < TPB; ++s) {              // stages h = 64, 128, 256
        const float sg = ((part >> s) & 1) ? -1.0f : 1.0f;
        const float2 sg2 = make_float2(sg, sg);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            float2 o;
            o.x = __shfl_xor_sync(0xffffffffu, P[i].x, 1 << s);
            o.y = __shfl_xor_sync(0xffffffffu, P[i].y, 1 << s);
            P[i] = __ffma2_rn(P[i], sg2, o);            // low: mine + o; high: o - mine
        }
    }
}

// Swizzled 128-byte row r of a TMA tile (1024-byte aligned base): chunk k.
__device__ __forceinline__ uint4 *sw_row_chunk(uint8_t *tile, int r, int k)
{
    return reinterpret_cast<uint4 *>(tile + r * 128 + ((k ^ (r & 7)) << 4));
}

// Sign-pair masks of the thread's row: bit 15 / bit 31 of word w flip values
// 2w and 2w+1 (16-bit layout).
__device__ __forceinline__ void load_pair_masks(const uint32_t *pmask, int part, uint32_t *pm)
{
    const uint4 *p = reinterpret_cast<const uint4 *>(pmask + part * 32);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const uint4 v = p[k];
        pm[4 * k] = v.x; pm[4 * k + 1] = v.y; pm[4 * k + 2] = v.z; pm[4 * k + 3] = v.w;
    }
}

__device__ __forceinline__ void setup_pair_masks(const QuantTables &T, uint32_t *pmask, int d)
{
    for (int w = threadIdx.x; w < d / 2; w += blockDim.x) {
        const int j = 2 * w;
        const uint32_t b0 = (T.sign_words[j >> 5] >> (j & 31)) & 1u;
        const uint32_t b1 = (T.sign_words[(j + 1) >> 5] >> ((j + 1) & 31)) & 1u;
        pmask[w] = (b0 << 15) | (b1 << 31);
    }
}

__device__ __forceinline__ void setup_lut_v2(const QuantTables &T, uint2 *lut, float *bnd)
{
    if (T.lut_cells > 0) {
        for (int i = threadIdx.x; i < T.lut_cells * 16; i += blockDim.x)
            lut[i] = make_uint2(__float_as_uint(T.lut_t[i >> 4]), T.lut_k[i >> 4]);
    } else {
        for (int i = threadIdx.x; i < T.levels; i += blockDim.x) bnd[i] = T.bound[i];
    }
}

__host__ __device__ inline uint32_t lut_bytes_v2(const QuantTables &T)
{
    const uint32_t b = T.lut_cells > 0 ? (uint32_t)T.lut_cells * 128u : (uint32_t)T.levels * 4u;
    return (b + 127u) & ~127u;
}

// Code of one rotated coordinate (see lut_code).  Cells below 0 clamp to 0
// through the float max (which also sends NaN to cell 0), cells past the
// table to the last one through the unsigned min.
__device__ __forceinline__ uint32_t lut_code_v2(float y, float f, const uint8_t *lut_lane, uint32_t cells_m1)
{
    uint32_t cell = __float_as_uint(fmaxf(f, kLutMagic)) - __float_as_uint(kLutMagic);
    cell = min(cell, cells_m1);
    const uint2 e = *reinterpret_cast<const uint2 *>(lut_lane + cell * 128u);
    return e.y + (__uint_as_float(e.x) < y ? 1u : 0u);
}

// -------------------------------------------------------------- quantize

__host__ __device__ inline size_t quantize_v2_smem(int d, const QuantTables &T)
{
    return 1024 + (size_t)kStages2 * kTileBytes2 + lut_bytes_v2(T) + (size_t)d / 2 * 4 + 8 * kStages2;
}

template <int D, int PW, bool BF16>
__global__ void __launch_bounds__(kT2, 2)
quantize_v2_kernel(const __grid_constant__ CUtensorMap tmx, int64_t nrows, const __grid_constant__ QuantTables T,
                   uint8_t *__restrict__ codes, uint16_t *__restrict__ norms)
{
    constexpr int TPB = D / kE2;
    constexpr int CB = kE2 * PW / 8;          // code bytes per row
    constexpr int NW = kE2 * PW / 32;         // code words per row
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *lutb = base + kStages2 * kTileBytes2;
    float *bnd = reinterpret_cast<float *>(lutb);
    uint32_t *pmask = reinterpret_cast<uint32_t *>(lutb + lut_bytes_v2(T));
    uint64_t *full = reinterpret_cast<uint64_t *>(pmask + D / 2);

    const int tid = threadIdx.x, lane = tid & 31, part = tid % TPB;
    const int64_t ntiles = (nrows + kT2 - 1) / kT2;
    if (tid == 0) {
        prefetch_tmap(&tmx);
        for (int s = 0; s < kStages2; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
        for (int s = 0; s < kStages2; ++s) {
            const int64_t t = blockIdx.x + (int64_t)s * gridDim.x;
            if (t < ntiles) {
                mbar_arrive_expect_tx(&full[s], kTileBytes2);
                tma_load_2d(base + s * kTileBytes2, &tmx, 0, (int)(t * kT2), &full[s]);
            }
        }
    }
    setup_lut_v2(T, reinterpret_cast<uint2 *>(lutb), bnd);
    setup_pair_masks(T, pmask, D);
    __syncthreads();

    const float2 la = make_float2(T.lut_a, T.lut_a), lb = make_float2(T.lut_b, T.lut_b);
    const int cells = T.lut_cells, levels = T.levels;
    const uint32_t cells_m1 = (uint32_t)(cells > 0 ? cells - 1 : 0);
    const uint8_t *lut_lane = lutb + (lane & 15) * 8;
    const uint4 *pmv = reinterpret_cast<const uint4 *>(pmask + part * 32);

    for (int64_t i = 0;; ++i) {
        const int64_t t = blockIdx.x + i * gridDim.x;
        if (t >= ntiles) break;
        const int s = (int)(i % kStages2);
        const bool got = mbar_wait(&full[s], (uint32_t)((i / kStages2) & 1));
        if (__syncthreads_or(!got)) break;                 // a bounded wait expired: unwind together
        uint8_t *tile = base + s * kTileBytes2;
        uint32_t u[32];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const uint4 v = *sw_row_chunk(tile, tid, k);
            const uint4 q = pmv[k];
            u[4 * k] = v.x ^ q.x; u[4 * k + 1] = v.y ^ q.y; u[4 * k + 2] = v.z ^ q.z; u[4 * k + 3] = v.w ^ q.w;
        }
        __syncthreads();                                   // stage s consumed by every thread
        if (tid == 0) {
            const int64_t tn = t + (int64_t)kStages2 * gridDim.x;
            if (tn < ntiles) {
                mbar_arrive_expect_tx(&full[s], kTileBytes2);
                tma_load_2d(tile, &tmx, 0, (int)(tn * kT2), &full[s]);
            }
        }
        const int64_t row = t * kT2 + tid;
        const bool valid = row < nrows;

        float2 P[32];
        row_to_pairs<BF16>(u, P);
        // the norm is sign-independent: flipping signs first changes no square
        const float n32 = __fsqrt_rn(combine_parts<TPB>(row_sumsq(P)));
        fwht_row<TPB>(P, part);
        const float inv = n32 > 0.0f ? __frcp_rn(n32) : 0.0f;
        const float2 inv2 = make_float2(inv, inv);

        uint32_t w[NW];
#pragma unroll
        for (int k = 0; k < NW; ++k) w[k] = 0u;
        if (cells > 0) {
#pragma unroll
            for (int i2 = 0; i2 < 32; ++i2) {
                const float2 y = __fmul2_rn(P[i2], inv2);
                const float2 f = __ffma2_rn(y, la, lb);
                const uint32_t c0 = lut_code_v2(y.x, f.x, lut_lane, cells_m1);
                const uint32_t c1 = lut_code_v2(y.y, f.y, lut_lane, cells_m1);
                const int b0 = i2 * PW, b1 = (i2 + 32) * PW;
                w[b0 >> 5] |= c0 << (b0 & 31);
                if ((b0 & 31) + PW > 32) w[(b0 >> 5) + 1] |= c0 >> (32 - (b0 & 31));
                w[b1 >> 5] |= c1 << (b1 & 31);
                if ((b1 & 31) + PW > 32) w[(b1 >> 5) + 1] |= c1 >> (32 - (b1 & 31));
            }
        } else {
#pragma unroll
            for (int i2 = 0; i2 < 32; ++i2) {
                const float2 y = __fmul2_rn(P[i2], inv2);
                const uint32_t c0 = bsearch_code(y.x, bnd, levels);
                const uint32_t c1 = bsearch_code(y.y, bnd, levels);
                const int b0 = i2 * PW, b1 = (i2 + 32) * PW;
                w[b0 >> 5] |= c0 << (b0 & 31);
                if ((b0 & 31) + PW > 32) w[(b0 >> 5) + 1] |= c0 >> (32 - (b0 & 31));
                w[b1 >> 5] |= c1 << (b1 & 31);
                if ((b1 & 31) + PW > 32) w[(b1 >> 5) + 1] |= c1 >> (32 - (b1 & 31));
            }
        }
        if (valid) {
            store_bytes<CB>(codes + row * CB, w);
            if (part == 0) norms[row / TPB] = norm_to_h16(n32);
        }
    }
}

// -------------------------------------------------------------- dequantize

__host__ __device__ inline size_t dequantize_v2_smem(int d, int pw)
{
    return 1024 + 2 * (size_t)kTileBytes2 + ((size_t)1 << pw) * 32 * 4 + (size_t)d / 2 * 4;
}

template <int D, int PW, bool BF16>
__global__ void __launch_bounds__(kT2, 2)
dequantize_v2_kernel(const uint8_t *__restrict__ codes, const uint16_t *__restrict__ norms, int64_t nrows,
                     const __grid_constant__ QuantTables T, const __grid_constant__ CUtensorMap tmo)
{
    constexpr int TPB = D / kE2;
    constexpr int CB = kE2 * PW / 8;
    constexpr int NW = kE2 * PW / 32;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float *cent = reinterpret_cast<float *>(base + 2 * kTileBytes2);
    uint32_t *pmask = reinterpret_cast<uint32_t *>(cent + (1 << PW) * 32);

    const int tid = threadIdx.x, lane = tid & 31, part = tid % TPB;
    const int64_t ntiles = (nrows + kT2 - 1) / kT2;
    if (tid == 0) prefetch_tmap(&tmo);
    for (int i = tid; i < (1 << PW) * 32; i += kT2) {
        const int k = i >> 5;
        cent[i] = k < T.levels ? T.centroid[k] : 0.0f;
    }
    setup_pair_masks(T, pmask, D);
    __syncthreads();
    uint32_t pm[32];
    load_pair_masks(pmask, part, pm);
    const float *cent_lane = cent + lane;

    // codes and norm of the first tile
    int64_t t = blockIdx.x;
    uint32_t cw[NW];
    float nrm = 0.0f;
    auto fetch = [&](int64_t tt, uint32_t *dst, float &n) {
        const int64_t r = tt * kT2 + tid;
        if (tt < ntiles && r < nrows) {
            load_bytes<CB>(codes + r * CB, dst);
            n = h16_to_f32(__ldg(norms + r / TPB));
        } else {
#pragma unroll
            for (int k = 0; k < NW; ++k) dst[k] = 0u;
            n = 0.0f;
        }
    };
    fetch(t, cw, nrm);

    for (int64_t i = 0; t < ntiles; ++i, t += gridDim.x) {
        uint32_t cn[NW];
        float nn;
        fetch(t + gridDim.x, cn, nn);                      // next tile's codes in flight

        float2 P[32];
#pragma unroll
        for (int i2 = 0; i2 < 32; ++i2) {
            P[i2].x = cent_lane[unpack_code<kE2, PW>(cw, i2) * 32];
            P[i2].y = cent_lane[unpack_code<kE2, PW>(cw, i2 + 32) * 32];
        }
        fwht_row<TPB>(P, part);
        const float sc = __fmul_rn(nrm, 1.0f / (float)D);
        const float2 sc2 = make_float2(sc, sc);
#pragma unroll
        for (int i2 = 0; i2 < 32; ++i2) P[i2] = __fmul2_rn(P[i2], sc2);

        uint8_t *stage = base + (int)(i & 1) * kTileBytes2;
        if (tid == 0) bulk_wait_read<1>();                 // the store issued two tiles ago left this buffer
        __syncthreads();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            uint32_t o[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int wd = 4 * k + q;                  // output word = values 2wd, 2wd+1
                const float a = wd < 16 ? P[2 * wd].x : P[2 * wd - 32].y;
                const float b = wd < 16 ? P[2 * wd + 1].x : P[2 * wd - 31].y;
                o[q] = pack2<BF16>(a, b) ^ pm[wd];
            }
            *sw_row_chunk(stage, tid, k) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            tma_store_2d(&tmo, 0, (int)(t * kT2), stage);
            bulk_commit();
        }
#pragma unroll
        for (int k = 0; k < NW; ++k) cw[k] = cn[k];
        nrm = nn;
    }
    if (tid == 0) bulk_wait<0>();
}

}  // namespace rq
