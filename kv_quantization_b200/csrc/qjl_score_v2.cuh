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

// Per-tile record staging: codes (128 x d*pw/8) and signs (128 x m/8), each
// section 16-byte aligned.
__host__ __device__ inline size_t sc2_rec_codes(int d, int pw, bool two) { return two ? (size_t)128 * d * pw / 8 : 0; }
__host__ __device__ inline size_t sc2_rec_signs(int m) { return ((size_t)128 * m / 8 + 15) & ~(size_t)15; }
__host__ __device__ inline size_t sc2_rec_bytes(int d, int m, bool two, int pw)
{
    return sc2_rec_codes(d, pw, two) + sc2_rec_signs(m);
}

__host__ __device__ inline size_t sc2_smem(int nq, int d, int m, bool two, int pw)
{
    const int kb = sc2_kb(d, m, two), nq16 = sc2_nq16(nq);
    size_t b = 1024;
    b += 2 * (size_t)kSc2ChunkBytes;                          // A double buffer
    b += (size_t)nq16 * kb * 2;                               // B (queries)
    b += (size_t)256 * 8 * 16;                                // sign byte -> 8 fp16, 8 copies
    if (two) b += pw <= 4 ? ((size_t)1 << (2 * pw)) * 32 * 4 : ((size_t)1 << pw) * 32 * 2;
    b += (size_t)nq16 * 4;                                    // ||q||
    b += 2 * sc2_rec_bytes(d, m, two, pw);                    // staged key records, 2 tiles
    return b + 8 * 6 + 16;
}

// Prologue: for up to 32 queries of one group per CTA, q~ = H D q (fp32
// butterfly in shared memory) and S q (fp32, each thread one row of S against
// all queries), both scaled by 1/||q|| and rounded to fp16, plus ||q|| itself.
constexpr int kSc2PrologueQ = 32;
constexpr int kSc2PrologueOut = 16;                 // S q outputs per CTA (16 rows x 16 query pairs = 256 threads)

// Shared memory of score_v2_prologue: [32][d] signed copy (rotated in place),
// [d][32] transposed raw copy (the S q operand), [32] inverse norms.
__host__ __device__ inline size_t sc2_prologue_smem(int d)
{
    return ((size_t)2 * kSc2PrologueQ * d + kSc2PrologueQ) * sizeof(float);
}

__global__ void __launch_bounds__(256)
score_v2_prologue(const uint16_t *__restrict__ q, int nq, int d, int m, const uint16_t *__restrict__ proj,
                  bool proj_bf16, const __grid_constant__ QuantTables T, bool two, uint16_t *__restrict__ wsB,
                  float *__restrict__ wsN)
{
    extern __shared__ float pq[];
    float *pr = pq;                                 // [32][d]: D q, rotated in place to H D q
    float *pt = pr + kSc2PrologueQ * d;             // [d][32]: q, transposed
    float *pinv = pt + kSc2PrologueQ * d;           // [32] 1 / ||q||
    const int64_t g = blockIdx.x;
    const int q0 = blockIdx.y * kSc2PrologueQ;
    const int zs = blockIdx.z, nz = gridDim.z;        // slice of the S q outputs (z = 0 also rotates)
    const int nqc = min(kSc2PrologueQ, nq - q0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int idx = tid; idx < kSc2PrologueQ * d; idx += blockDim.x) {
        const int qi = idx / d, j = idx % d;
        float v = 0.0f;
        if (qi < nqc) v = __uint_as_float((uint32_t)q[((int64_t)g * nq + q0 + qi) * d + j] << 16);
        pt[j * kSc2PrologueQ + qi] = v;
        pr[idx] = __uint_as_float(__float_as_uint(v) ^ sign_mask(T.sign_words, j));
    }
    __syncthreads();
    for (int qi = warp; qi < kSc2PrologueQ; qi += blockDim.x / 32) {
        float sum = 0.0f;
        for (int j = lane; j < d; j += 32) sum = __fmaf_rn(pr[qi * d + j], pr[qi * d + j], sum);
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
                const int qi = p / (d / 2), pp = p % (d / 2);
                const int j = qi * d + (pp / h) * 2 * h + (pp % h);
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
            const int qi = idx / d, j = idx % d;
            wsB[((int64_t)g * nq + q0 + qi) * kb + j] = __half_as_ushort(__float2half_rn(pr[idx] * pinv[qi]));
        }
    // S q: output row i = i_lo + tid / 16 of this slice, queries 2 (tid % 16) and 2 (tid % 16) + 1
    const int per = (sc2_m64(m) + nz - 1) / nz;       // <= kSc2PrologueOut (launch)
    const int i = zs * per + tid / 16, qp = 2 * (tid % 16);
    if (tid / 16 < per && i < sc2_m64(m)) {
        float acc0 = 0.0f, acc1 = 0.0f;
        if (i < m) {
            const uint4 *Srow = reinterpret_cast<const uint4 *>(proj + (int64_t)i * d);
            for (int j8 = 0; j8 < d / 8; ++j8) {
                const uint4 w = __ldg(Srow + j8);
                const uint32_t ws4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint16_t h = (uint16_t)(ws4[e >> 1] >> (16 * (e & 1)));
                    const float sv = proj_bf16 ? __uint_as_float((uint32_t)h << 16) : h16_to_f32(h);
                    const float2 qv = *reinterpret_cast<const float2 *>(pt + (j8 * 8 + e) * kSc2PrologueQ + qp);
                    acc0 = __fmaf_rn(sv, qv.x, acc0);
                    acc1 = __fmaf_rn(sv, qv.y, acc1);
                }
            }
        }
        if (qp < nqc)
            wsB[((int64_t)g * nq + q0 + qp) * kb + off + i] = __half_as_ushort(__float2half_rn(acc0 * pinv[qp]));
        if (qp + 1 < nqc)
            wsB[((int64_t)g * nq + q0 + qp + 1) * kb + off + i] =
                __half_as_ushort(__float2half_rn(acc1 * pinv[qp + 1]));
    }
}

template <int PW, bool TWO>
__global__ void __launch_bounds__(kSc2Threads, 1)
score_v2_kernel(const uint16_t *__restrict__ wsB, const float *__restrict__ wsN, int nq, int d, int m,
                const uint8_t *__restrict__ signs, const uint16_t *__restrict__ sk_norms, int64_t T_len,
                int64_t G, const uint8_t *__restrict__ codes, const uint16_t *__restrict__ norms,
                const __grid_constant__ QuantTables T, float *__restrict__ scores)
{
    const int nq16 = sc2_nq16(nq), m64 = sc2_m64(m), kb = sc2_kb(d, m, TWO);
    const int dreg = TWO ? d / 64 : 0;             // regions of first-stage columns
    const uint32_t ncols = 4u * (uint32_t)nq16 <= 32u ? 32u : (4u * (uint32_t)nq16 <= 64u ? 64u :
                           (4u * (uint32_t)nq16 <= 128u ? 128u : (4u * (uint32_t)nq16 <= 256u ? 256u : 512u)));
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *sA = base;                                            // 2 x 32 KB
    uint8_t *sB = sA + 2 * kSc2ChunkBytes;                         // nreg regions x nq16 rows x 128 B
    uint4 *slut = reinterpret_cast<uint4 *>(sB + (size_t)nq16 * kb * 2);  // sign byte -> 8 fp16, 8 copies
    uint32_t *clut = reinterpret_cast<uint32_t *>(slut + 256 * 8);
    const size_t clut_bytes = TWO ? (PW <= 4 ? ((size_t)1 << (2 * PW)) * 32 * 4 : ((size_t)1 << PW) * 32 * 2) : 0;
    float *sqn = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(clut) + clut_bytes);
    uint8_t *srec = reinterpret_cast<uint8_t *>(sqn + nq16);       // 2 record buffers
    const size_t rec_codes = sc2_rec_codes(d, PW, TWO), rec_signs = sc2_rec_signs(m);
    const size_t rec_bytes = sc2_rec_bytes(d, m, TWO, PW);
    uint64_t *bars = reinterpret_cast<uint64_t *>(srec + 2 * rec_bytes);  // [0,1] A, [2,3] acc, [4,5] records
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 6);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // sign byte -> eight fp16 +-1 (bit 1 -> +1), replicated 8 times
    for (int i = tid; i < 256 * 8; i += kSc2Threads) {
        const int byte = i >> 3;
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t lo = ((byte >> (2 * k)) & 1) ? 0x3C00u : 0xBC00u;
            const uint32_t hi = ((byte >> (2 * k + 1)) & 1) ? 0x3C00u : 0xBC00u;
            w[k] = lo | (hi << 16);
        }
        slut[i] = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if constexpr (TWO) {
        if constexpr (PW <= 4) {   // pair table: (code_a | code_b << PW) -> fp16 pair, 32 copies
            for (int i = tid; i < (1 << (2 * PW)) * 32; i += kSc2Threads) {
                const int e = i >> 5, ca = e & ((1 << PW) - 1), cb = e >> PW;
                const float fa = ca < T.levels ? T.centroid[ca] : 0.0f, fb = cb < T.levels ? T.centroid[cb] : 0.0f;
                clut[i] = (uint32_t)__half_as_ushort(__float2half_rn(fa)) |
                          ((uint32_t)__half_as_ushort(__float2half_rn(fb)) << 16);
            }
        } else {
            uint16_t *cl16 = reinterpret_cast<uint16_t *>(clut);
            for (int i = tid; i < (1 << PW) * 32; i += kSc2Threads) {
                const int e = i >> 5;
                cl16[i] = __half_as_ushort(__float2half_rn(e < T.levels ? T.centroid[e] : 0.0f));
            }
        }
    }
    if (tid == 0) {
        for (int b = 0; b < 6; ++b) mbar_init(&bars[b], 1);
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, ncols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t sA0 = smem_u32(sA), sB0 = smem_u32(sB);
    const uint32_t idesc = idesc_f16(false, 128, nq16);

    const int64_t tiles_per_g = (T_len + 127) / 128;
    const int64_t items = G * tiles_per_g;
    const int64_t it0 = items * blockIdx.x / gridDim.x, it1 = items * (blockIdx.x + 1) / gridDim.x;
    int64_t cur_g = -1;
    uint32_t abar_phase[2] = {0u, 0u}, accbar_phase[2] = {0u, 0u};
    bool abuf_busy[2] = {false, false};
    int chunk_ctr = 0;
    bool ok = true, pend = false;
    int64_t pend_g = 0, pend_t0 = 0;
    const float kq = 1.2533141373155002512f / (float)m;
    const int cbytes = TWO ? d * PW / 8 : 0, sbytes = m / 8;
    uint32_t rec_phase[2] = {0u, 0u};

    // Stage the records of work item `w` into buffer rb: full tiles by bulk
    // copies (thread 0), the ragged last tile of a group by plain loads.
    auto fetch = [&](int64_t w, int rb) {
        const int64_t g = w / tiles_per_g, t0 = (w % tiles_per_g) * 128;
        const int64_t ntok = min((int64_t)128, T_len - t0);
        const int64_t kt0 = g * T_len + t0;
        uint8_t *R = srec + rb * rec_bytes;
        const bool aligned = (((uintptr_t)(codes + kt0 * cbytes) | (uintptr_t)(signs + kt0 * sbytes)) & 15u) == 0;
        if (ntok == 128 && aligned) {
            if (tid == 0) {
                mbar_arrive_expect_tx(&bars[4 + rb], (uint32_t)(rec_codes + (size_t)128 * sbytes));
                if (TWO) bulk_load(R, codes + kt0 * cbytes, (uint32_t)rec_codes, &bars[4 + rb]);
                bulk_load(R + rec_codes, signs + kt0 * sbytes, (uint32_t)(128 * sbytes), &bars[4 + rb]);
            }
        } else {   // ragged or unaligned tile: plain loads; the next block-wide barrier publishes them
            for (int64_t i = tid; i < ntok * cbytes; i += kSc2Threads) R[i] = __ldg(codes + kt0 * cbytes + i);
            for (int64_t i = tid; i < ntok * sbytes; i += kSc2Threads) R[rec_codes + i] = __ldg(signs + kt0 * sbytes + i);
            if (tid == 0) mbar_arrive_expect_tx(&bars[4 + rb], 0u);
        }
    };

    auto epilogue = [&](int64_t g, int64_t t0, int accs) {
        if (ok && !mbar_wait(&bars[2 + accs], accbar_phase[accs])) ok = false;
        accbar_phase[accs] ^= 1u;
        tc_fence_after();
        const int64_t t = t0 + tid;
        const bool tv = ok && t < T_len;
        const int64_t kt = g * T_len + (tv ? t : t0);
        const float a2 = tv ? __fmul_rn(kq, h16_to_f32(__ldg(sk_norms + kt))) : 0.0f;
        const float a1 = (TWO && tv) ? __fmul_rn(h16_to_f32(__ldg(norms + kt)), 1.0f / (float)d) : 0.0f;
        const uint32_t col1 = (uint32_t)(accs * 2 * nq16), col2 = col1 + (uint32_t)nq16;
        for (int q0 = 0; q0 < nq16; q0 += 32) {
            uint32_t r1[32], r2[32];
            tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + col2 + (uint32_t)q0, r2);
            if (TWO) tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + col1 + (uint32_t)q0, r1);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int qi = q0 + i;
                if (tv && qi < nq) {
                    const float qn = sqn[qi];
                    float s = __fmul_rn(a2, __uint_as_float(r2[i]));
                    if (TWO) s = __fmaf_rn(a1, __uint_as_float(r1[i]), s);
                    scores[((int64_t)g * nq + qi) * T_len + t] = __fmul_rn(s, qn);
                }
            }
        }
        tc_fence_before();
    };

    if (it0 < it1) fetch(it0, 0);
    for (int64_t it = it0; it < it1; ++it) {
        const int64_t g = it / tiles_per_g, t0 = (it % tiles_per_g) * 128;
        const int accs = (int)((it - it0) & 1);
        const int rb = (int)((it - it0) & 1);
        if (ok && !mbar_wait(&bars[4 + rb], rec_phase[rb])) ok = false;
        rec_phase[rb] ^= 1u;
        if (it + 1 < it1) fetch(it + 1, rb ^ 1);            // next tile's records in flight
        const uint8_t *Rc = srec + rb * rec_bytes + (size_t)tid * cbytes;
        const uint8_t *Rs = srec + rb * rec_bytes + rec_codes + (size_t)tid * sbytes;
        if (g != cur_g) {
            // new group: B (queries) into shared memory, once the previous tile's MMAs are done with it
            if (pend) { epilogue(pend_g, pend_t0, (int)((it - 1 - it0) & 1)); pend = false; }
            for (int b = 0; b < 2; ++b)
                if (abuf_busy[b]) {
                    if (ok && !mbar_wait(&bars[b], abar_phase[b])) ok = false;
                    abar_phase[b] ^= 1u;
                    abuf_busy[b] = false;
                }
            __syncthreads();
            const uint16_t *src = wsB + (int64_t)g * nq * kb;
            for (int idx = tid; idx < nq16 * (kb / 8); idx += kSc2Threads) {
                const int row = idx / (kb / 8), c = idx % (kb / 8);
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (row < nq) v = __ldg(reinterpret_cast<const uint4 *>(src + (int64_t)row * kb) + c);
                *reinterpret_cast<uint4 *>(sB + (size_t)(c >> 3) * nq16 * 128 + sw128_offset(row, c & 7)) = v;
            }
            for (int i = tid; i < nq16; i += kSc2Threads) sqn[i] = i < nq ? wsN[(int64_t)g * nq + i] : 0.0f;
            fence_proxy_async_smem();
            __syncthreads();
            cur_g = g;
        }
        const bool tv = t0 + tid < T_len;
        for (int c0 = 0; c0 < kb; c0 += kSc2Chunk) {
            const int b = chunk_ctr & 1;
            ++chunk_ctr;
            if (abuf_busy[b]) {                              // the MMAs that read this buffer are done
                if (ok && !mbar_wait(&bars[b], abar_phase[b])) ok = false;
                abar_phase[b] ^= 1u;
                abuf_busy[b] = false;
            }
            uint8_t *A = sA + b * kSc2ChunkBytes;
            const int ncol = min(kSc2Chunk, kb - c0);
            for (int r = 0; r < ncol / 64; ++r) {            // one 64-column region at a time
                const int gc0 = c0 + 64 * r;                 // global K column of the region
                uint8_t *Ar = A + (size_t)r * 16384 + (size_t)tid * 128;
                if (TWO && gc0 < d) {
                    uint32_t cw[2 * PW];                     // 64 codes = 8*PW bytes, 8-byte aligned
#pragma unroll
                    for (int q = 0; q < PW; ++q) {
                        const uint2 v2 = tv ? *reinterpret_cast<const uint2 *>(Rc + gc0 * PW / 8 + 8 * q)
                                            : make_uint2(0u, 0u);
                        cw[2 * q] = v2.x;
                        cw[2 * q + 1] = v2.y;
                    }
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        uint32_t o[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const uint32_t ca = unpack_code<64, PW>(cw, 8 * k + 2 * e);
                            const uint32_t cb2 = unpack_code<64, PW>(cw, 8 * k + 2 * e + 1);
                            if constexpr (PW <= 4) {
                                o[e] = clut[((ca | (cb2 << PW)) << 5) + lane];
                            } else {
                                const uint16_t *cl16 = reinterpret_cast<const uint16_t *>(clut);
                                o[e] = (uint32_t)cl16[(ca << 5) + lane] | ((uint32_t)cl16[(cb2 << 5) + lane] << 16);
                            }
                        }
                        uint4 v = tv ? make_uint4(o[0], o[1], o[2], o[3]) : make_uint4(0u, 0u, 0u, 0u);
                        *reinterpret_cast<uint4 *>(Ar + ((k ^ (tid & 7)) << 4)) = v;
                    }
                } else {
                    const int sc0 = gc0 - (TWO ? d : 0);     // first sign column of the region
                    uint32_t sb[2] = {0u, 0u};
                    if (tv) {
                        const uint8_t *sp = Rs + sc0 / 8;
                        const int nbytes = min(8, max(0, (m - sc0) / 8));
                        if (nbytes == 8 && (((uintptr_t)sp) & 7u) == 0) {
                            const uint2 v2 = *reinterpret_cast<const uint2 *>(sp);
                            sb[0] = v2.x;
                            sb[1] = v2.y;
                        } else {
                            for (int b = 0; b < nbytes; ++b) sb[b >> 2] |= (uint32_t)sp[b] << (8 * (b & 3));
                        }
                    }
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const bool live = tv && sc0 + 8 * k < m;
                        const uint32_t byte = (sb[k >> 2] >> (8 * (k & 3))) & 0xffu;
                        const uint4 v = live ? slut[(byte << 3) + (lane & 7)] : make_uint4(0u, 0u, 0u, 0u);
                        *reinterpret_cast<uint4 *>(Ar + ((k ^ (tid & 7)) << 4)) = v;
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();
            if (tid == 0 && ok) {
                tc_fence_after();
                for (int r = 0; r < ncol / 64; ++r) {
                    const int greg = c0 / 64 + r;                 // global region
                    const bool first = greg < dreg;
                    const uint32_t dcol = (uint32_t)(accs * 2 * nq16 + (first ? 0 : nq16));
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint64_t adesc = sdesc_k_sw128(sA0 + (uint32_t)b * kSc2ChunkBytes + (uint32_t)r * 16384u + k * 32u);
                        const uint64_t bdesc = sdesc_k_sw128(sB0 + (uint32_t)greg * (uint32_t)nq16 * 128u + k * 32u);
                        const bool acc = !(k == 0 && (greg == 0 || greg == dreg));
                        mma_f16(tmem + dcol, adesc, bdesc, idesc, acc ? 1u : 0u);
                    }
                }
                mma_commit(&bars[b]);
                if (c0 + kSc2Chunk >= kb) mma_commit(&bars[2 + accs]);
            }
            abuf_busy[b] = true;
            if (c0 == 0 && pend) {                           // previous tile's scores while this tile's MMAs run
                epilogue(pend_g, pend_t0, (int)((it - 1 - it0) & 1));
                pend = false;
            }
        }
        pend = true;
        pend_g = g;
        pend_t0 = t0;
        if (!__syncthreads_and(ok)) { ok = false; break; }
    }
    if (pend) epilogue(pend_g, pend_t0, (int)((it1 - 1 - it0) & 1));
    for (int b = 0; b < 2; ++b)
        if (abuf_busy[b] && ok) {
            if (!mbar_wait(&bars[b], abar_phase[b])) ok = false;
        }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, ncols);
}

}  // namespace rq
