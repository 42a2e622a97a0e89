// qjl_score_v2.cuh -- inner-product scores on the tcgen05 tensor cores (sm_100a).
//
// score[g][q][t] = (n16_t/d) <H D q, C[idx_t]> + sqrt(pi/2)/m * rn16_t * <S q, sign_t>
// (eliza quantization README, section "QJL": the query is projected through
// the same matrix and the score reconstructed from the signs; the first term
// is <q, x^_t> of the rotated scalar code).
//
// Per tile of 128 key tokens of one group: the A operand is the unpacked keys
// -- fp16 centroid values for the d first-stage coordinates, fp16 +-1 for the
// m sign bits -- written by the 128 threads (thread r = token r = TMEM lane r)
// in 128-column chunks into a double-buffered 128-byte-swizzled K-major tile;
// B is the group's n_q queries [q~/||q|| ; Sq/||q||] in fp16 (from the
// prologue), resident in shared memory.  One thread issues per 64-column
// region 4 MMAs (K = 16 each) into accumulator 1 (first-stage columns) or 2
// (sign columns); the epilogue of tile i (tcgen05.ld of both accumulators,
// fp32 scaling by the per-token norms and per-query ||q||) runs while tile
// i+1's chunks are produced.
#pragma once
#include "rq_common.cuh"
#include "sm100.cuh"

namespace rq {

constexpr int kSc2Threads = 128;
constexpr int kSc2Chunk = 128;                     // A columns per chunk (2 regions)
constexpr int kSc2ChunkBytes = 128 * kSc2Chunk * 2;

__host__ __device__ inline int sc2_m64(int m) { return (m + 63) & ~63; }
// queries padded to a multiple of 32 (MMA N, and whole 32-column TMEM loads)
__host__ __device__ inline int sc2_nq16(int nq) { return (nq + 31) & ~31; }
__host__ __device__ inline int sc2_kb(int d, int m, bool two) { return (two ? d : 0) + sc2_m64(m); }

// Workspace written by the prologue: per (g, q) a row of kb fp16 values
// [q~/||q|| (d, when two-stage) ; Sq/||q|| (m, zero-padded to m64)], then per
// (g, q) the fp32 ||q||.
__host__ __device__ inline size_t sc2_ws_bytes(int64_t G, int nq, int d, int m, bool two)
{
    const size_t rows = (size_t)G * nq;
    return ((rows * sc2_kb(d, m, two) * 2 + 255) & ~(size_t)255) + rows * 4;
}

constexpr int kSc2PrologueQ = 32;
constexpr int kSc2PrologueOut = 16;                 // S q outputs per CTA (16 rows x 16 query pairs = 256 threads)

// Shared memory of score_v2_prologue: [32][d + 4] signed copy (rotated in
// place; rows padded so that 16-byte stores from 32 queries hit distinct
// banks), [d][32] transposed raw copy (the S q operand), [32] inverse norms.
__host__ __device__ inline size_t sc2_prologue_smem(int d)
{
    return ((size_t)kSc2PrologueQ * (d + 4) + (size_t)kSc2PrologueQ * d + kSc2PrologueQ) * sizeof(float);
}

// The prologue kernel is defined in one translation unit only (qjl.cu);
// other users launch it through launch_score_prologue().
#ifndef RQ_SCORE_PROLOGUE_EXTERN
__global__ void __launch_bounds__(256)
score_v2_prologue(const uint16_t *__restrict__ q, int nq, int d, int m, const uint16_t *__restrict__ proj,
                  bool proj_bf16, const __grid_constant__ QuantTables T, bool two, uint16_t *__restrict__ wsB,
                  float *__restrict__ wsN)
{
    extern __shared__ float pq[];
    const int dl = 31 - __clz(d);                   // d is a power of two
    const int pd = d + 4;                           // padded row of pr
    float *pr = pq;                                 // [32][pd]: D q, rotated in place to H D q
    float *pt = pr + kSc2PrologueQ * pd;            // [d][32]: q, transposed
    float *pinv = pt + kSc2PrologueQ * d;           // [32] 1 / ||q||
    const int64_t g = blockIdx.x;
    const int q0 = blockIdx.y * kSc2PrologueQ;
    const int zs = blockIdx.z, nz = gridDim.z;        // slice of the S q outputs (z = 0 also rotates)
    const int nqc = min(kSc2PrologueQ, nq - q0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // staging: item p = query p % 32, coordinates 8 (p / 32) .. 8 (p / 32) + 7 (one 16-byte load)
    for (int p = tid; p < kSc2PrologueQ * (d >> 3); p += blockDim.x) {
        const int qi = p & 31, j0 = (p >> 5) << 3;
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (qi < nqc) w = __ldg(reinterpret_cast<const uint4 *>(q + ((int64_t)g * nq + q0 + qi) * d + j0));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            v[e] = __uint_as_float((e & 1) ? (ws[e >> 1] & 0xffff0000u) : (ws[e >> 1] << 16));
            pt[(j0 + e) * kSc2PrologueQ + qi] = v[e];
        }
        const uint32_t sw = T.sign_words[j0 >> 5] >> (j0 & 31);    // 8 sign bits of j0 .. j0+7
        float4 lo, hi;
        lo.x = __uint_as_float(__float_as_uint(v[0]) ^ ((sw & 1u) << 31));
        lo.y = __uint_as_float(__float_as_uint(v[1]) ^ (((sw >> 1) & 1u) << 31));
        lo.z = __uint_as_float(__float_as_uint(v[2]) ^ (((sw >> 2) & 1u) << 31));
        lo.w = __uint_as_float(__float_as_uint(v[3]) ^ (((sw >> 3) & 1u) << 31));
        hi.x = __uint_as_float(__float_as_uint(v[4]) ^ (((sw >> 4) & 1u) << 31));
        hi.y = __uint_as_float(__float_as_uint(v[5]) ^ (((sw >> 5) & 1u) << 31));
        hi.z = __uint_as_float(__float_as_uint(v[6]) ^ (((sw >> 6) & 1u) << 31));
        hi.w = __uint_as_float(__float_as_uint(v[7]) ^ (((sw >> 7) & 1u) << 31));
        *reinterpret_cast<float4 *>(pr + qi * pd + j0) = lo;
        *reinterpret_cast<float4 *>(pr + qi * pd + j0 + 4) = hi;
    }
    __syncthreads();
    for (int qi = warp; qi < kSc2PrologueQ; qi += blockDim.x / 32) {
        float sum = 0.0f;
        for (int j = lane; j < d; j += 32) sum = __fmaf_rn(pr[qi * pd + j], pr[qi * pd + j], sum);
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) {
            const float qn = sqrtf(sum);
            pinv[qi] = qn > 0.0f ? 1.0f / qn : 0.0f;
            if (qi < nqc && zs == 0) wsN[(int64_t)g * nq + q0 + qi] = qn;
        }
    }
    if (two && zs == 0) {
        for (int h = 1; h < d; h *= 2) {
            __syncthreads();
            for (int p = tid; p < kSc2PrologueQ * d / 2; p += blockDim.x) {
                const int qi = p >> (dl - 1), pp = p & (d / 2 - 1);
                const int j = qi * pd + ((pp & ~(h - 1)) << 1) + (pp & (h - 1));
                const float a = pr[j], b = pr[j + h];
                pr[j] = a + b;
                pr[j + h] = a - b;
            }
        }
    }
    __syncthreads();
    const int kb = sc2_kb(d, m, two), off = two ? d : 0;
    if (two && zs == 0)
        for (int idx = tid; idx < nqc * d; idx += blockDim.x) {
            const int qi = idx >> dl, j = idx & (d - 1);
            wsB[((int64_t)g * nq + q0 + qi) * kb + j] = __half_as_ushort(__float2half_rn(pr[qi * pd + j] * pinv[qi]));
        }
    // S q: output row i = i_lo + tid / 16 of this slice, queries 2 (tid % 16) and 2 (tid % 16) + 1
    const int per = (sc2_m64(m) + nz - 1) / nz;       // <= kSc2PrologueOut (launch)
    const int i = zs * per + tid / 16, qp = 2 * (tid % 16);
    if (tid / 16 < per && i < sc2_m64(m)) {
        float2 acc = make_float2(0.0f, 0.0f);
        if (i < m) {
            const uint4 *Srow = reinterpret_cast<const uint4 *>(proj + (int64_t)i * d);
#pragma unroll 4
            for (int j8 = 0; j8 < d / 8; ++j8) {                 // d / 8 is a multiple of 8
                const uint4 w = __ldg(Srow + j8);
                const uint32_t ws4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint16_t h = (uint16_t)(ws4[e >> 1] >> (16 * (e & 1)));
                    const float sv = proj_bf16 ? __uint_as_float((uint32_t)h << 16) : h16_to_f32(h);
                    const float2 qv = *reinterpret_cast<const float2 *>(pt + (j8 * 8 + e) * kSc2PrologueQ + qp);
                    acc = __ffma2_rn(make_float2(sv, sv), qv, acc);      // one fma per query
                }
            }
        }
        if (qp < nqc)
            wsB[((int64_t)g * nq + q0 + qp) * kb + off + i] = __half_as_ushort(__float2half_rn(acc.x * pinv[qp]));
        if (qp + 1 < nqc)
            wsB[((int64_t)g * nq + q0 + qp + 1) * kb + off + i] =
                __half_as_ushort(__float2half_rn(acc.y * pinv[qp + 1]));
    }
}
#endif  // RQ_SCORE_PROLOGUE_EXTERN

}  // namespace rq
