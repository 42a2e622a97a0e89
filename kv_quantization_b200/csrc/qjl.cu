// qjl.cu -- JL projection generator and inner-product score kernels (sm_100a).
//
// QJL (eliza quantization README, section "QJL", "Algorithm in one paragraph"):
// keys are stored as sign(S k) packed 8 per byte plus ||k||; at attention time
// the query is projected through the same S and the score is reconstructed as
// sqrt(pi/2)/m * ||k|| * <S q, sign(S k)>, an unbiased estimate of <q, k>.
// For two-stage keys (rotated Lloyd-Max codes plus a QJL sketch of the
// residual) the first-stage term (n16/d) <H D q, c> is added; it equals
// <q, x^> because H is symmetric with H H = d I.
#include <cstdint>

#include "rq_common.cuh"
#include "rq_kernels.h"
#include "qjl_score_v5.cuh"

namespace rq {

// SplitMix64 output k of the stream with initial state `seed`
// (Steele, Lea & Flood, OOPSLA 2014).
__device__ __forceinline__ uint64_t splitmix64(uint64_t seed, uint64_t k)
{
    uint64_t z = seed + (k + 1ull) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// S[i][j] = round16(fp32(sqrt(-2 ln u1) cos(2 pi u2))), Box-Muller over
// SplitMix64 outputs 2k and 2k+1, k = i*d + j.
__global__ void projection_kernel(uint64_t seed, int64_t count, bool bf16, uint16_t *__restrict__ S)
{
    const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= count) return;
    const double u1 = (double)((splitmix64(seed, 2ull * (uint64_t)k) >> 11) + 1ull) * 0x1p-53;
    const double u2 = (double)(splitmix64(seed, 2ull * (uint64_t)k + 1ull) >> 11) * 0x1p-53;
    const double r = sqrt(__dmul_rn(-2.0, log(u1)));
    const double z = __dmul_rn(r, cos(__dmul_rn(6.283185307179586476925286766559, u2)));
    const float zf = __double2float_rn(z);
    S[k] = bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(zf)) : __half_as_ushort(__float2half_rn(zf));
}

cudaError_t launch_projection(uint64_t seed, int m, int d, bool bf16, void *proj, cudaStream_t st)
{
    const int64_t count = (int64_t)m * d;
    const int threads = 256;
    projection_kernel<<<(unsigned)((count + threads - 1) / threads), threads, 0, st>>>(
        seed, count, bf16, static_cast<uint16_t *>(proj));
    note_launch("projection_kernel");
    return cudaGetLastError();
}

// --------------------------------------------------------------------------
// Score prologue: per (group, query) the rotated query q~ = H D q (fp32) and
// the projected query S q (fp32), written to the workspace row [d + m].
// --------------------------------------------------------------------------
__global__ void score_prologue_kernel(const uint16_t *__restrict__ q, int d, int m, const void *__restrict__ proj,
                                      bool proj_bf16, const __grid_constant__ QuantTables T, bool rotate,
                                      float *__restrict__ ws)
{
    extern __shared__ float qs[];            // [d] raw query, [d] rotated
    float *qr = qs + d;
    const int64_t row = blockIdx.x;          // g * nq + qi
    const uint16_t *qp = q + row * d;
    for (int j = threadIdx.x; j < d; j += blockDim.x) {
        const float v = __uint_as_float((uint32_t)qp[j] << 16);
        qs[j] = v;
        qr[j] = __uint_as_float(__float_as_uint(v) ^ sign_mask(T.sign_words, j));
    }
    __syncthreads();
    if (rotate) {
        for (int h = 1; h < d; h *= 2) {
            for (int p = threadIdx.x; p < d / 2; p += blockDim.x) {
                const int j = (p / h) * 2 * h + (p % h);
                const float a = qr[j], b = qr[j + h];
                qr[j] = __fadd_rn(a, b);
                qr[j + h] = __fsub_rn(a, b);
            }
            __syncthreads();
        }
    }
    float *out = ws + row * (int64_t)(d + m);
    for (int j = threadIdx.x; j < d; j += blockDim.x) out[j] = qr[j];
    const uint16_t *S = static_cast<const uint16_t *>(proj);
    for (int i = threadIdx.x; i < m; i += blockDim.x) {
        float acc = 0.0f;
        for (int j = 0; j < d; ++j) {
            const uint16_t h = S[(int64_t)i * d + j];
            const float s = proj_bf16 ? __uint_as_float((uint32_t)h << 16) : h16_to_f32(h);
            acc = __fmaf_rn(s, qs[j], acc);
        }
        out[d + i] = acc;
    }
}

// --------------------------------------------------------------------------
// Score main loop: one thread per key token, up to 32 queries per pass.  The
// group's rotated / projected queries sit in shared memory (broadcast reads).
// --------------------------------------------------------------------------
constexpr int kScoreThreads = 128;
constexpr int kScoreQ = 32;

template <int PW, bool TWO_STAGE>
__global__ void __launch_bounds__(kScoreThreads)
score_kernel(const float *__restrict__ ws, int nq, int d, int m, const uint8_t *__restrict__ signs,
             const uint16_t *__restrict__ sk_norms, int64_t T_len, const uint8_t *__restrict__ codes,
             const uint16_t *__restrict__ norms, const __grid_constant__ QuantTables T,
             float *__restrict__ scores)
{
    extern __shared__ float sh[];
    float *cent = sh;                                     // [1<<PW] (two-stage only)
    float *qw = sh + (TWO_STAGE ? (1 << PW) : 0);         // [kScoreQ][d + m]
    const int64_t g = blockIdx.y;
    const int q0 = blockIdx.z * kScoreQ;
    const int nqc = min(kScoreQ, nq - q0);
    const int w = d + m;
    if (TWO_STAGE)
        for (int k = threadIdx.x; k < (1 << PW); k += blockDim.x) cent[k] = k < T.levels ? T.centroid[k] : 0.0f;
    for (int idx = threadIdx.x; idx < nqc * w; idx += blockDim.x)
        qw[idx] = ws[((int64_t)g * nq + q0) * w + idx];
    __syncthreads();

    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T_len) return;
    const int64_t kt = g * T_len + t;
    float acc1[kScoreQ], acc2[kScoreQ];
#pragma unroll
    for (int qi = 0; qi < kScoreQ; ++qi) { acc1[qi] = 0.0f; acc2[qi] = 0.0f; }

    if (TWO_STAGE) {
        const int cb = d * PW / 8;
        const uint8_t *cp = codes + kt * cb;
        for (int j0 = 0; j0 < d; j0 += 32) {
            uint32_t cw[PW];
#pragma unroll
            for (int i = 0; i < PW; ++i) cw[i] = __ldg(reinterpret_cast<const uint32_t *>(cp + j0 * PW / 8) + i);
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
                const float c = cent[unpack_code<32, PW>(cw, jj)];
#pragma unroll
                for (int qi = 0; qi < kScoreQ; ++qi)
                    if (qi < nqc) acc1[qi] = __fmaf_rn(qw[qi * w + j0 + jj], c, acc1[qi]);
            }
        }
    }
    const uint8_t *sp = signs + kt * (m / 8);
    for (int i0 = 0; i0 < m; i0 += 8) {
        const uint32_t byte = __ldg(sp + i0 / 8);
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            const uint32_t neg = ((byte >> b) & 1u) ? 0u : 0x80000000u;
#pragma unroll
            for (int qi = 0; qi < kScoreQ; ++qi)
                if (qi < nqc) acc2[qi] = __fadd_rn(acc2[qi], __uint_as_float(__float_as_uint(qw[qi * w + d + i0 + b]) ^ neg));
        }
    }
    const float kq = 1.2533141373155002512f / (float)m;   // sqrt(pi/2) / m
    const float a2 = __fmul_rn(kq, h16_to_f32(__ldg(sk_norms + kt)));
    const float a1 = TWO_STAGE ? __fmul_rn(h16_to_f32(__ldg(norms + kt)), 1.0f / (float)d) : 0.0f;
#pragma unroll
    for (int qi = 0; qi < kScoreQ; ++qi)
        if (qi < nqc)
            scores[((int64_t)g * nq + q0 + qi) * T_len + t] = __fadd_rn(__fmul_rn(a1, acc1[qi]), __fmul_rn(a2, acc2[qi]));
}

cudaError_t launch_score_prologue(const ScoreArgs &a, bool two, uint16_t *wsB, float *wsN, cudaStream_t st)
{
    const size_t psmem = sc2_prologue_smem(a.d);
    cudaError_t e = cudaFuncSetAttribute(score_v2_prologue, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)psmem);
    if (e != cudaSuccess) return e;
    const unsigned zsl = (unsigned)((sc2_m64(a.m) + kSc2PrologueOut - 1) / kSc2PrologueOut);
    score_v2_prologue<<<dim3((unsigned)a.G, (unsigned)((a.nq + kSc2PrologueQ - 1) / kSc2PrologueQ), zsl), 256, psmem, st>>>(
        a.q, a.nq, a.d, a.m, static_cast<const uint16_t *>(a.proj), a.proj_bf16, *a.tables, two, wsB, wsN);
    note_launch("score_v2_prologue");
    return cudaGetLastError();
}

size_t score_workspace_bytes(int64_t G, int nq, int d, int m)
{
    const size_t v1 = (size_t)G * (size_t)nq * (size_t)(d + m) * sizeof(float);
    const size_t v2 = sc2_ws_bytes(G, nq, d, m, true);
    return v1 > v2 ? v1 : v2;
}

// Tensor-core score path; cudaErrorNotSupported when the shape does not fit.
template <int PW, bool TWO>
static cudaError_t launch_score_v2(const ScoreArgs &a, cudaStream_t st)
{
    if (a.nq > 128) return cudaErrorNotSupported;
    if (sc4_smem(a.nq, a.d, a.m, TWO, PW, 2, 2, 2) > kMaxSmemPerBlock) return cudaErrorNotSupported;
    uint16_t *wsB = reinterpret_cast<uint16_t *>(a.workspace);
    const size_t rows = (size_t)a.G * a.nq;
    float *wsN = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(a.workspace) +
                                           ((rows * sc2_kb(a.d, a.m, TWO) * 2 + 255) & ~(size_t)255));
    const size_t psmem = sc2_prologue_smem(a.d);
    cudaError_t e = cudaFuncSetAttribute(score_v2_prologue, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)psmem);
    if (e != cudaSuccess) return e;
    const unsigned zsl = (unsigned)((sc2_m64(a.m) + kSc2PrologueOut - 1) / kSc2PrologueOut);   // 16 S q outputs per CTA
    score_v2_prologue<<<dim3((unsigned)a.G, (unsigned)((a.nq + kSc2PrologueQ - 1) / kSc2PrologueQ), zsl), 256, psmem, st>>>(
        a.q, a.nq, a.d, a.m, static_cast<const uint16_t *>(a.proj), a.proj_bf16, *a.tables, TWO, wsB, wsN);
    note_launch("score_v2_prologue");
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // queries on M, 256 tokens on N (qjl_score_v5.cuh) when the records allow
    // aligned bulk copies: the deepest rings that fit
    if (sc5_eligible(a.nq, a.d, a.m, TWO, PW)) {
        struct Cfg5 { int ring, nrec; };
        const Cfg5 cfgs5[] = {{4, 3}, {4, 2}, {3, 2}, {2, 2}, {2, 1}};
        const int64_t items5 = a.G * ((a.T + kSc5Tok - 1) / kSc5Tok);
        const int64_t grid5 = items5 < (int64_t)a.num_sms ? items5 : (int64_t)a.num_sms;
        const bool tma = a.has_tmap_scores && a.nq <= 64;
        for (const Cfg5 &c : cfgs5) {
            const size_t smem5 = sc5_smem(a.nq, a.d, a.m, TWO, PW, c.ring, c.nrec, tma);
            if (smem5 > kMaxSmemPerBlock) continue;
            auto kern5 = score_v5_kernel<PW, TWO>;
            e = cudaFuncSetAttribute(kern5, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem5);
            if (e != cudaSuccess) return e;
            kern5<<<(unsigned)(grid5 > 0 ? grid5 : 1), kSc5Threads, smem5, st>>>(
                wsB, wsN, a.nq, a.d, a.m, a.signs, a.sk_norms, a.T, a.G, a.codes, a.norms, *a.tables, a.scores,
                c.ring, c.nrec, a.tmap_scores, tma ? 1 : 0);
            note_launch("score_v5_kernel");
            return cudaGetLastError();
        }
    }
    const int64_t items = a.G * ((a.T + 127) / 128);
    const int64_t grid = items < (int64_t)a.num_sms ? items : (int64_t)a.num_sms;
    // eight producer warps (qjl_score_v4.cuh): the deepest configuration that fits
    {
        struct Cfg { int ring, nrec, slc; };
        const Cfg cfgs[] = {{4, 3, 8}, {3, 3, 8}, {3, 2, 2}, {2, 2, 2}};
        for (const Cfg &c : cfgs) {
            const size_t smem4 = sc4_smem(a.nq, a.d, a.m, TWO, PW, c.ring, c.nrec, c.slc);
            if (smem4 > kMaxSmemPerBlock) continue;
            auto kern4 = c.nrec == 3 ? score_v4_kernel<PW, TWO, 3> : score_v4_kernel<PW, TWO, 2>;
            e = cudaFuncSetAttribute(kern4, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem4);
            if (e != cudaSuccess) return e;
            kern4<<<(unsigned)(grid > 0 ? grid : 1), kSc4Threads, smem4, st>>>(
                wsB, wsN, a.nq, a.d, a.m, a.signs, a.sk_norms, a.T, a.G, a.codes, a.norms, *a.tables, a.scores, c.ring,
                c.slc);
            note_launch("score_v4_kernel");
            return cudaGetLastError();
        }
    }
    return cudaErrorNotSupported;
}

template <int PW, bool TWO>
static cudaError_t launch_score_main(const ScoreArgs &a, cudaStream_t st)
{
    auto kern = score_kernel<PW, TWO>;
    const size_t smem = (size_t)((TWO ? (1 << PW) : 0) + kScoreQ * (a.d + a.m)) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((a.T + kScoreThreads - 1) / kScoreThreads), (unsigned)a.G,
              (unsigned)((a.nq + kScoreQ - 1) / kScoreQ));
    kern<<<grid, kScoreThreads, smem, st>>>(a.workspace, a.nq, a.d, a.m, a.signs, a.sk_norms, a.T, a.codes,
                                            a.norms, *a.tables, a.scores);
    note_launch("score_kernel");
    return cudaGetLastError();
}

cudaError_t launch_score(const ScoreArgs &a, cudaStream_t st)
{
    const bool two = a.codes != nullptr;
    {
        cudaError_t e2 = cudaErrorNotSupported;
        if (!two) {
            e2 = launch_score_v2<1, false>(a, st);
        } else {
            switch (a.pw) {
            case 1: e2 = launch_score_v2<1, true>(a, st); break;
            case 2: e2 = launch_score_v2<2, true>(a, st); break;
            case 3: e2 = launch_score_v2<3, true>(a, st); break;
            case 4: e2 = launch_score_v2<4, true>(a, st); break;
            case 5: e2 = launch_score_v2<5, true>(a, st); break;
            case 6: e2 = launch_score_v2<6, true>(a, st); break;
            case 7: e2 = launch_score_v2<7, true>(a, st); break;
            case 8: e2 = launch_score_v2<8, true>(a, st); break;
            default: break;
            }
        }
        if (e2 != cudaErrorNotSupported) return e2;
    }
    const size_t psmem = (size_t)2 * a.d * sizeof(float);
    score_prologue_kernel<<<(unsigned)(a.G * a.nq), 256, psmem, st>>>(a.q, a.d, a.m, a.proj, a.proj_bf16, *a.tables,
                                                                      two, a.workspace);
    note_launch("score_prologue_kernel");
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (!two) return launch_score_main<1, false>(a, st);
    switch (a.pw) {
    case 1: return launch_score_main<1, true>(a, st);
    case 2: return launch_score_main<2, true>(a, st);
    case 3: return launch_score_main<3, true>(a, st);
    case 4: return launch_score_main<4, true>(a, st);
    case 5: return launch_score_main<5, true>(a, st);
    case 6: return launch_score_main<6, true>(a, st);
    case 7: return launch_score_main<7, true>(a, st);
    case 8: return launch_score_main<8, true>(a, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace rq
