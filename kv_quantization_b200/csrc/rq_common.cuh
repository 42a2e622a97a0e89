// rq_common.cuh -- shared device helpers of librq (sm_100a).
//
// Canonical fp32 arithmetic used by every kernel (so that results are
// reproducible bit for bit, independent of how coordinates map to lanes):
//   * L2 norm: squares rounded to fp32, pairwise (recursive halving) sum,
//     correctly rounded sqrt.  Within a thread the pairwise tree runs over its
//     contiguous slice; across the TPB threads of one block the xor-shuffle
//     combine (offsets 1, 2) continues the same tree because IEEE addition is
//     commutative.
//   * Walsh-Hadamard: radix-2 butterflies (a, b) -> (a + b, a - b), stages
//     h = 1, 2, ..., d/2 in that order; the stages with h < E run inside the
//     thread, the others across lanes.
// All adds and multiplies go through __fadd_rn / __fmul_rn so that nvcc cannot
// contract them into FMAs.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "rq_params.h"

namespace rq {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float h16_to_f32(uint16_t h) { return __half2float(__ushort_as_half(h)); }

// Two 16-bit values packed in a word -> fp32.
template <bool BF16>
__device__ __forceinline__ void unpack2(uint32_t w, float &a, float &b)
{
    if constexpr (BF16) {
        a = bf16_lo(w);
        b = bf16_hi(w);
    } else {
        a = h16_to_f32((uint16_t)(w & 0xffffu));
        b = h16_to_f32((uint16_t)(w >> 16));
    }
}

// x - p * s with the product and the difference each rounded to nearest
// (the canonical two roundings), written as a packed multiply feeding an FMA
// with factor -1.  ptxas (CUDA 12.9, sm_100a) was measured to contract a
// packed f32x2 multiply feeding a packed f32x2 add -- and an FMA with factor
// +1 -- into one fused multiply-add, even with explicit .rn and
// --fmad=false; this form was measured to keep both roundings.
__device__ __forceinline__ float2 sub_mul2_rn(float2 x, float2 p, float2 s)
{
    return __ffma2_rn(__fmul2_rn(p, s), make_float2(-1.0f, -1.0f), x);
}

// Two fp32 -> packed 16-bit pair, round to nearest even.
template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float a, float b)
{
    if constexpr (BF16) {
        __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t *>(&v);
    } else {
        __half2 v = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t *>(&v);
    }
}

// fp32 -> fp16 bits, saturating at the largest finite binary16 (norm storage).
__device__ __forceinline__ uint16_t norm_to_h16(float n)
{
    uint16_t h = __half_as_ushort(__float2half_rn(n));
    if ((h & 0x7fffu) == 0x7c00u) h = (uint16_t)((h & 0x8000u) | 0x7bffu);
    return h;
}

// Pairwise sum of v[0..N) held in registers (N a power of two, compile time).
template <int N>
__device__ __forceinline__ float pairwise_sum(const float *v)
{
    if constexpr (N == 1) {
        return v[0];
    } else {
        float a = pairwise_sum<N / 2>(v);
        float b = pairwise_sum<N / 2>(v + N / 2);
        return __fadd_rn(a, b);
    }
}

// In-thread Walsh-Hadamard stages h = 1 .. E/2 on a register array.
template <int E>
__device__ __forceinline__ void fwht_local(float *v)
{
#pragma unroll
    for (int h = 1; h < E; h *= 2) {
#pragma unroll
        for (int i = 0; i < E; i += 2 * h) {
#pragma unroll
            for (int j = i; j < i + h; ++j) {
                float a = v[j], b = v[j + h];
                v[j] = __fadd_rn(a, b);
                v[j + h] = __fsub_rn(a, b);
            }
        }
    }
}

// Cross-lane stages h = E, 2E, ... for TPB consecutive lanes holding one block.
// Lane part p holds coordinates [p*E, (p+1)*E); at stage s the partner is p ^ (1<<s).
template <int E, int TPB>
__device__ __forceinline__ void fwht_cross(float *v, int part)
{
#pragma unroll
    for (int s = 0; (1 << s) < TPB; ++s) {
        const bool high = (part >> s) & 1;
#pragma unroll
        for (int j = 0; j < E; ++j) {
            float o = __shfl_xor_sync(0xffffffffu, v[j], 1 << s);
            // low half: mine + partner's; high half: partner's - mine
            v[j] = high ? __fsub_rn(o, v[j]) : __fadd_rn(v[j], o);
        }
    }
}

// Combine per-thread pairwise partial sums across the TPB lanes of a block.
template <int TPB>
__device__ __forceinline__ float combine_parts(float s)
{
#pragma unroll
    for (int off = 1; off < TPB; off *= 2) s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, off));
    return s;
}

// Sign of coordinate j under the diagonal (bit set -> negate), as an fp32 sign mask.
__device__ __forceinline__ uint32_t sign_mask(const uint32_t *words, int j)
{
    return ((words[j >> 5] >> (j & 31)) & 1u) << 31;
}

// Nearest-centroid index of y: LUT cell from one IEEE fma, then one compare
// against the cell's single candidate boundary (exact: the host builds the cell
// tables from the same fma evaluated in IEEE arithmetic).  lut points at the
// CTA's replicated {threshold, base} table; copy = lane % 16.
__device__ __forceinline__ uint32_t lut_code(float y, const uint2 *lut, float a, float b, int cells, int copy)
{
    float f = __fmaf_rn(y, a, b);
    int cell = (int)(__float_as_uint(f) - __float_as_uint(kLutMagic));
    cell = min(max(cell, 0), cells - 1);
    uint2 e = lut[cell * 16 + copy];
    return e.y + (__uint_as_float(e.x) < y ? 1u : 0u);
}

// Fallback search: #{k : t_k < y} by a branch-free binary search over the K-1
// sorted boundaries padded with +inf to kpow = K entries (K a power of two).
__device__ __forceinline__ uint32_t bsearch_code(float y, const float *t, int kpow)
{
    uint32_t lo = 0;
    for (int step = kpow >> 1; step > 0; step >>= 1)
        lo += (t[lo + step - 1] < y) ? (uint32_t)step : 0u;
    return lo;
}

// Store `nbytes` (a multiple of 4, at most 256) from registers words[] to global.
template <int NBYTES>
__device__ __forceinline__ void store_bytes(uint8_t *dst, const uint32_t *w)
{
    if constexpr (NBYTES % 16 == 0) {
#pragma unroll
        for (int i = 0; i < NBYTES / 16; ++i)
            reinterpret_cast<uint4 *>(dst)[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
    } else if constexpr (NBYTES % 8 == 0) {
#pragma unroll
        for (int i = 0; i < NBYTES / 8; ++i)
            reinterpret_cast<uint2 *>(dst)[i] = make_uint2(w[2 * i], w[2 * i + 1]);
    } else {
#pragma unroll
        for (int i = 0; i < NBYTES / 4; ++i) reinterpret_cast<uint32_t *>(dst)[i] = w[i];
    }
}

template <int NBYTES>
__device__ __forceinline__ void load_bytes(const uint8_t *src, uint32_t *w)
{
    if constexpr (NBYTES % 16 == 0) {
#pragma unroll
        for (int i = 0; i < NBYTES / 16; ++i) {
            uint4 v = __ldg(reinterpret_cast<const uint4 *>(src) + i);
            w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
        }
    } else if constexpr (NBYTES % 8 == 0) {
#pragma unroll
        for (int i = 0; i < NBYTES / 8; ++i) {
            uint2 v = __ldg(reinterpret_cast<const uint2 *>(src) + i);
            w[2 * i] = v.x; w[2 * i + 1] = v.y;
        }
    } else {
#pragma unroll
        for (int i = 0; i < NBYTES / 4; ++i) w[i] = __ldg(reinterpret_cast<const uint32_t *>(src) + i);
    }
}

// Pack E codes of PW bits (PW = 8 for the int8 layout) LSB-first into words.
template <int E, int PW>
__device__ __forceinline__ void pack_codes(const uint32_t *code, uint32_t *w)
{
    constexpr int NW = (E * PW + 31) / 32;
#pragma unroll
    for (int i = 0; i < NW; ++i) w[i] = 0u;
#pragma unroll
    for (int j = 0; j < E; ++j) {
        const int bit = j * PW;
        w[bit >> 5] |= code[j] << (bit & 31);
        if ((bit & 31) + PW > 32) w[(bit >> 5) + 1] |= code[j] >> (32 - (bit & 31));
    }
}

template <int E, int PW>
__device__ __forceinline__ uint32_t unpack_code(const uint32_t *w, int j)
{
    const int bit = j * PW;
    uint32_t v = w[bit >> 5] >> (bit & 31);
    if ((bit & 31) + PW > 32) v |= w[(bit >> 5) + 1] << (32 - (bit & 31));
    return v & ((1u << PW) - 1u);
}

}  // namespace rq
