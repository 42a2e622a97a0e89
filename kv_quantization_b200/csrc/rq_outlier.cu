// rq_outlier.cu -- the QJL key sketch's per-group outlier part (sm_100a).
//
// QJL README, "Algorithm in one paragraph", and qjl_apply.py's key hook: per
// group of 32 consecutive tokens the top-k coordinates by their norm over the
// group are outliers; they get their own sketch, with its own norm.  The key
// splits into k_in (outlier coordinates zeroed) and k_out (only those):
//   main sketch    sign(S k_in), ||k_in||   (the tensor-core key sketch, run
//                                            on the masked keys this file writes)
//   outlier sketch sign(S_o k_out), ||k_out||, S_o = rows 0 .. m_o-1 of S
// and the score adds, per token, sqrt(pi/2)/m_o ||k_out|| <S_o q_O, sign(S_o k_out)>
// with q_O the query on the group's outlier coordinates.
//
// outlier_prep_kernel: one warp per group.  The group's 32 keys are staged in
//   shared memory; lane l sums the squares of columns 4l .. 4l+3 over the 32
//   tokens in token order (fp32); the top k are taken by k rounds of a warp
//   argmax (largest sum, ties to the lower index); then lane t (a token) reads
//   its k outlier values, forms ||k_out|| (fp32 squares in stored order) and
//   the m_o sign bits of sum_r S[i][O_r] v_r (fp32, stored order), and the warp
//   writes the masked group back contiguously.
// outlier_score_kernel: one CTA per (head, group): per token the k weights
//   w[t][r] = sum_i S[i][O_r] (+1 / -1 by sign bit i), then for every query
//   lane = token adds sqrt(pi/2)/m_o * n_out16 * sum_r q[O_r] w[t][r] to the
//   scores the pure-QJL score wrote.
#include <cmath>
#include <cstdint>

#include "rq_common.cuh"
#include "rq_kernels.h"

namespace rq {

namespace {

constexpr int kOlWarps = 4;                 // groups per CTA (prep)
constexpr int kOlMaxOut = 16;
constexpr int kOlMaxMo = 256;

__device__ __forceinline__ float bf16_at(const uint16_t *p) { return __uint_as_float((uint32_t)*p << 16); }

template <int NOUT>
__global__ void __launch_bounds__(kOlWarps * 32)
outlier_prep_kernel(const uint16_t *__restrict__ keys, int64_t ngroups, int m_o,
                    const uint16_t *__restrict__ S, uint16_t *__restrict__ kin, uint8_t *__restrict__ idx_out,
                    uint8_t *__restrict__ out_signs, uint16_t *__restrict__ out_norms)
{
    constexpr int d = 128;
    extern __shared__ __align__(16) uint8_t ol_prep_smem[];
    __shared__ int sel[kOlWarps][kOlMaxOut];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // per warp: the group's keys (8 KB), then S[i][O_r] as [r][i] (NOUT * m_o floats)
    uint8_t *wb = ol_prep_smem + (size_t)warp * (32 * d * 2 + (size_t)m_o * NOUT * 4);
    uint16_t *tl = reinterpret_cast<uint16_t *>(wb);
    float *sow = reinterpret_cast<float *>(wb + 32 * d * 2);
    for (int64_t g = (int64_t)blockIdx.x * kOlWarps + warp; g < ngroups; g += (int64_t)gridDim.x * kOlWarps) {
        const uint4 *src = reinterpret_cast<const uint4 *>(keys + g * 32 * d);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 16; ++i) reinterpret_cast<uint4 *>(tl)[lane + 32 * i] = __ldg(src + lane + 32 * i);
        __syncwarp();
        // column sums of squares, token order
        float cs[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        for (int t = 0; t < 32; ++t)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float v = bf16_at(tl + t * d + 4 * lane + c);
                cs[c] = __fadd_rn(cs[c], __fmul_rn(v, v));
            }
        // top n_out: largest sum first, ties to the lower column
        uint32_t taken = 0u;
        for (int r = 0; r < NOUT; ++r) {
            float bv = -1.0f;
            int bi = 1 << 30;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if (!((taken >> c) & 1u) && cs[c] > bv) { bv = cs[c]; bi = 4 * lane + c; }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
            }
            if ((bi >> 2) == lane) taken |= 1u << (bi & 3);
            if (lane == 0) {
                sel[warp][r] = bi;
                idx_out[g * NOUT + r] = (uint8_t)bi;
            }
        }
        __syncwarp();
        // S columns of the outlier set, transposed: sow[r][i] = S[i][O_r]
        for (int e = lane; e < m_o * NOUT; e += 32) {
            const int r = e / m_o, i = e - r * m_o;
            sow[e] = bf16_at(S + (int64_t)i * d + sel[warp][r]);
        }
        // lane = token: outlier values, norm, sketch
        float v[NOUT];
        float acc = 0.0f;
#pragma unroll
        for (int r = 0; r < NOUT; ++r) {
            v[r] = bf16_at(tl + lane * d + sel[warp][r]);
            acc = __fadd_rn(acc, __fmul_rn(v[r], v[r]));
        }
        const int64_t tok = g * 32 + lane;
        out_norms[tok] = norm_to_h16(__fsqrt_rn(acc));
        __syncwarp();
        for (int w = 0; w < m_o / 32; ++w) {
            uint32_t bits = 0u;
#pragma unroll 4
            for (int b = 0; b < 32; b += 2) {              // outputs i, i + 1 as a pair
                const int i = 32 * w + b;
                float2 p = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int r = 0; r < NOUT; ++r) {
                    const float2 sv = *reinterpret_cast<const float2 *>(sow + r * m_o + i);
                    p = __fadd2_rn(p, __fmul2_rn(sv, make_float2(v[r], v[r])));
                }
                bits |= (p.x >= 0.0f ? 1u : 0u) << b;
                bits |= (p.y >= 0.0f ? 1u : 0u) << (b + 1);
            }
            reinterpret_cast<uint32_t *>(out_signs + tok * (m_o / 8))[w] = bits;
        }
        // masked group back, contiguous
        __syncwarp();
        for (int r = 0; r < NOUT; ++r) tl[lane * d + sel[warp][r]] = 0;
        __syncwarp();
        uint4 *dst = reinterpret_cast<uint4 *>(kin + g * 32 * d);
#pragma unroll
        for (int i = 0; i < 16; ++i) dst[lane + 32 * i] = reinterpret_cast<const uint4 *>(tl)[lane + 32 * i];
    }
}

__global__ void __launch_bounds__(128)
outlier_score_kernel(const uint16_t *__restrict__ q, int nq, int64_t T, int m_o, int n_out,
                     const uint16_t *__restrict__ S, const uint8_t *__restrict__ idx,
                     const uint8_t *__restrict__ out_signs, const uint16_t *__restrict__ out_norms,
                     float *__restrict__ scores)
{
    // <S_o q_O, s_t> = sum_r q[O_r] w[t][r] with w[t][r] = sum_i S[i][O_r] s_t,i:
    // the k weights of a token are formed once (m_o signed adds each), and each
    // (token, query) score then takes k multiply-adds.
    constexpr int d = 128;
    __shared__ float sct[kOlMaxOut][kOlMaxMo];          // S[i][O_r], transposed
    __shared__ float w[32][kOlMaxOut + 1];               // per token of the group
    __shared__ float qo[32][kOlMaxOut + 1];
    __shared__ int sel[kOlMaxOut];
    const int64_t ng = T / 32;
    const int64_t hg = blockIdx.x;                       // (head, group)
    const int64_t g = hg / ng, j = hg - g * ng;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid < n_out) sel[tid] = idx[hg * n_out + tid];
    __syncthreads();
    for (int e = tid; e < m_o * n_out; e += blockDim.x) {
        const int i = e / n_out, r = e - i * n_out;
        sct[r][i] = bf16_at(S + (int64_t)i * d + sel[r]);
    }
    __syncthreads();
    // weights: warp -> outlier rows r = warp, warp + 4, ...; lane -> token
    {
        const int64_t tok = g * T + j * 32 + lane;
        const uint32_t *sg = reinterpret_cast<const uint32_t *>(out_signs + tok * (m_o / 8));
        for (int r = warp; r < n_out; r += 4) {
            const float *col = sct[r];
            float2 acc = make_float2(0.0f, 0.0f);
            for (int wd = 0; wd < m_o / 32; ++wd) {
                const uint32_t bits = __ldg(sg + wd);
#pragma unroll
                for (int b = 0; b < 32; b += 2) {
                    // +S where the bit is set, -S where it is clear
                    const float x = __uint_as_float(__float_as_uint(col[32 * wd + b]) ^ ((~bits << (31 - b)) & 0x80000000u));
                    const float y =
                        __uint_as_float(__float_as_uint(col[32 * wd + b + 1]) ^ ((~bits << (30 - b)) & 0x80000000u));
                    acc = __fadd2_rn(acc, make_float2(x, y));
                }
            }
            w[lane][r] = __fadd_rn(acc.x, acc.y);
        }
    }
    const float c = (float)(1.2533141373155002512 / (double)m_o);   // sqrt(pi/2) / m_o
    const int64_t tok = g * T + j * 32 + lane;
    const float no = h16_to_f32(out_norms[tok]) * c;
    for (int q0 = 0; q0 < nq; q0 += 32) {
        const int nqc = nq - q0 < 32 ? nq - q0 : 32;
        __syncthreads();
        for (int e = tid; e < nqc * n_out; e += blockDim.x) {
            const int qq = e / n_out, r = e - qq * n_out;
            qo[qq][r] = bf16_at(q + (g * nq + q0 + qq) * d + sel[r]);
        }
        __syncthreads();
        for (int qq = warp; qq < nqc; qq += 4) {
            float dot = 0.0f;
            for (int r = 0; r < n_out; ++r) dot = __fadd_rn(dot, __fmul_rn(qo[qq][r], w[lane][r]));
            float *dst = scores + (g * nq + q0 + qq) * T + j * 32 + lane;
            *dst = __fadd_rn(*dst, __fmul_rn(no, dot));
        }
    }
}

}  // namespace


template <int NOUT>
static cudaError_t run_outlier_prep(const uint16_t *keys, int64_t ngroups, int m_o, const uint16_t *S, uint16_t *kin,
                                    uint8_t *idx, uint8_t *out_signs, uint16_t *out_norms, int num_sms, cudaStream_t st)
{
    int64_t grid = (ngroups + kOlWarps - 1) / kOlWarps;
    const int64_t cap = (int64_t)num_sms * 8;
    if (grid > cap) grid = cap;
    const size_t smem = (size_t)kOlWarps * (32 * 128 * 2 + (size_t)m_o * NOUT * 4);
    cudaError_t e = cudaFuncSetAttribute(outlier_prep_kernel<NOUT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    outlier_prep_kernel<NOUT><<<(unsigned)(grid > 0 ? grid : 1), kOlWarps * 32, smem, st>>>(keys, ngroups, m_o, S, kin,
                                                                                           idx, out_signs, out_norms);
    return cudaGetLastError();
}

cudaError_t launch_outlier_prep(const uint16_t *keys, int64_t nvec, int n_out, int m_o, const uint16_t *S,
                                uint16_t *kin, uint8_t *idx, uint8_t *out_signs, uint16_t *out_norms, int num_sms,
                                cudaStream_t st)
{
    const int64_t ng = nvec / 32;
    cudaError_t e;
    switch (n_out) {
#define RQ_OUTLIER_CASE(K) \
    case K: e = run_outlier_prep<K>(keys, ng, m_o, S, kin, idx, out_signs, out_norms, num_sms, st); break;
        RQ_OUTLIER_CASE(1) RQ_OUTLIER_CASE(2) RQ_OUTLIER_CASE(3) RQ_OUTLIER_CASE(4) RQ_OUTLIER_CASE(5)
        RQ_OUTLIER_CASE(6) RQ_OUTLIER_CASE(7) RQ_OUTLIER_CASE(8) RQ_OUTLIER_CASE(9) RQ_OUTLIER_CASE(10)
        RQ_OUTLIER_CASE(11) RQ_OUTLIER_CASE(12) RQ_OUTLIER_CASE(13) RQ_OUTLIER_CASE(14) RQ_OUTLIER_CASE(15)
        RQ_OUTLIER_CASE(16)
#undef RQ_OUTLIER_CASE
    default: return cudaErrorNotSupported;
    }
    note_launch("outlier_prep_kernel");
    return e;
}

cudaError_t launch_outlier_score(const uint16_t *q, int64_t G, int nq, int64_t T, int m_o, int n_out,
                                 const uint16_t *S, const uint8_t *idx, const uint8_t *out_signs,
                                 const uint16_t *out_norms, float *scores, cudaStream_t st)
{
    const int64_t blocks = G * (T / 32);
    outlier_score_kernel<<<(unsigned)blocks, 128, 0, st>>>(q, nq, T, m_o, n_out, S, idx, out_signs, out_norms,
                                                             scores);
    note_launch("outlier_score_kernel");
    return cudaGetLastError();
}

}  // namespace rq
