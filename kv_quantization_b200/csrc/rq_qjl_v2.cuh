// rq_qjl_v2.cuh -- tcgen05 helpers the QJL sketch kernels share: TMEM column
// counts for a double-buffered accumulator, the MMA issue loop of one
// 128 x m16 x 128 tile, the sign-word packing and a sign-pack epilogue.
//
// Epilogue (qjl_v2_epilogue): 8 warps; warp w reads TMEM lanes 32 (w mod 4)
// .. +31 (its 32 vectors) and every other 32-column chunk starting at chunk
// w / 4, packs the 32 sign bits of a chunk into one word (bit i = P_i >= 0)
// and stores it.
#pragma once
#include "rq_qjl_mma.cuh"
#include "rq_v2.cuh"

namespace rq {

constexpr int kQ2Stages = 3;

__host__ __device__ inline uint32_t qjl_v2_tmem_cols(int m)
{
    uint32_t c = 32;
    while (c < 2u * (uint32_t)qjl_mma_m16(m)) c <<= 1;
    return c;
}

// Bit i of the result = (v[i] >= 0) for 32 fp32 values.  Adding +0 maps -0
// to +0 (and leaves every other value unchanged), so the bit is the inverted
// sign bit.  The additions run on pairs; for each g = 0..7 two byte permutes
// gather the top bytes of v[g], v[g+8], v[g+16], v[g+24] into bytes 0..3 of
// one word, whose bit 7 of byte b is then the sign of v[8b+g], moved to bit
// 8b+g with one shift and one masked OR.
__device__ __forceinline__ uint32_t sign_word(const uint32_t *v)
{
    const float2 z = make_float2(0.0f, 0.0f);
    uint32_t neg = 0u;
#pragma unroll
    for (int g = 0; g < 8; ++g) {
        const float2 lo = __fadd2_rn(make_float2(__uint_as_float(v[g]), __uint_as_float(v[g + 8])), z);
        const float2 hi = __fadd2_rn(make_float2(__uint_as_float(v[g + 16]), __uint_as_float(v[g + 24])), z);
        const uint32_t top = __byte_perm(__byte_perm(__float_as_uint(lo.x), __float_as_uint(lo.y), 0x0073u),
                                         __byte_perm(__float_as_uint(hi.x), __float_as_uint(hi.y), 0x0073u),
                                         0x5410u);
        neg |= (top >> (7 - g)) & (0x01010101u << g);
    }
    return ~neg;
}

// Sign-pack epilogue of one 128-vector tile from TMEM accumulator columns
// [col0, col0 + m16).
__device__ __forceinline__ void qjl_v2_epilogue(uint32_t tmem, uint32_t col0, int m, int m16, int64_t tok0,
                                                int64_t nvec, uint8_t *__restrict__ signs, bool ok)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t tok = tok0 + (warp & 3) * 32 + lane;
    const bool tv = ok && tok < nvec;
    uint8_t *dst = signs + tok * (m / 8);
    for (int c0 = (warp >> 2) * 32; c0 < m16; c0 += 64) {
        uint32_t acc[32];
        tmem_ld32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + col0 + (uint32_t)c0, acc);
        tmem_ld_wait();
        const uint32_t word = sign_word(acc);
        if (tv && c0 < m) {
            const int nb = min(4, (m - c0) / 8);
            if (nb == 4 && (m & 31) == 0) {
                *reinterpret_cast<uint32_t *>(dst + c0 / 8) = word;
            } else {
                for (int b = 0; b < nb; ++b) dst[c0 / 8 + b] = (uint8_t)(word >> (8 * b));
            }
        }
    }
}

// One thread issues the MMAs of a 128 x m16 x 128 tile: A (2 regions of 128
// rows) x S^T (2 regions of m16 rows), into TMEM columns [col0, col0 + m16).
__device__ __forceinline__ void qjl_v2_issue(uint32_t sA, uint32_t sS, int m16, uint32_t tmem_col)
{
#pragma unroll
    for (int kc = 0; kc < 2; ++kc) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint64_t adesc = sdesc_k_sw128(sA + (uint32_t)kc * 16384u + (uint32_t)k * 32u);
            for (int n0 = 0; n0 < m16; n0 += 256) {
                const int N = min(256, m16 - n0);
                const uint64_t bdesc =
                    sdesc_k_sw128(sS + (uint32_t)kc * (uint32_t)m16 * 128u + (uint32_t)n0 * 128u + (uint32_t)k * 32u);
                mma_f16(tmem_col + (uint32_t)n0, adesc, bdesc, idesc_f16(true, 128, N), (kc | k) != 0);
            }
        }
    }
}

}  // namespace rq
