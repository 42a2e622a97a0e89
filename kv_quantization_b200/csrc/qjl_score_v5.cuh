// qjl_score_v5.cuh -- tensor-core score with the queries on M and 256 key
// tokens on N (sm_100a).
//
// The arithmetic is the one of qjl_score_v2.cuh: the prologue writes each
// query as [q~/||q|| ; Sq/||q||] in fp16 (q~ = H D q), the keys are unpacked
// to fp16 (centroid values for the first-stage codes, signs for the sketch),
// and the score is the fp32 dot product times per-token and per-query
// factors.  The operands are swapped: D[q][t] = A[q] . B[t] with
//   A = the group's queries, M = 64 (n_q <= 64) or 128 rows (rows >= n_q are
//   not read back),
//   B = 256 key tokens, N = 256,
// because a thread issuing tcgen05.mma kind::f16 (K = 16) gets one
// instruction through about every 150 cycles whatever its M and N (measured
// on B200): a 256-token instruction does eight times the work of a 32-query
// one in the same issue time.
//
// Per-token factors.  Pure QJL: score = ||q|| * (kq * rn_t) * D[q][t] with
// B = +-1, kq = sqrt(pi/2) / m.  Two-stage keys: the sign columns of B carry
// +-rho_t, rho_t = fp16(kq * rn_t * d / n_t), so that one accumulator holds
//   <q~/||q||, c_t> + rho_t <Sq/||q||, sign_t>
// and score = ||q|| * (n_t / d) * D[q][t].  Rounding rho_t to fp16 changes
// the sketch term by at most 2^-11 of itself.
//
// Pipeline (one CTA per SM, persistent over (group, 256-token tile) items):
//   warp 16 (loader)   : one cp.async.bulk per tile for the signs (and one
//                        for the codes) into a ring of record slots;
//   warps 0-7 (producers, thread = token row): unpack their token's bytes of
//                        each 64-column slice into a ring of 32 KB B slots
//                        (128-byte-swizzled K-major, 256 rows);
//   warp 17 (MMA)      : per slice four MMAs into one of two 256-column TMEM
//                        accumulators; reloads the group's queries (A) when
//                        the group changes, after its MMAs have drained;
//   warps 8-15 (epilogue): warp w reads TMEM lane quarter w % 4 (queries)
//                        and columns 128 ((w - 8) / 4) ... of the tile, scales
//                        them (per-token factors loaded one tile ahead) and
//                        stores them: when n_q <= 64 and T % 4 == 0 through
//                        a swizzled 16 x 32 stage and one TMA store per box
//                        (a {T, n_q, G} tensor map, so no box crosses a
//                        group), else as 16-byte runs of scores[g][q][t].
// With n_q <= 64 the MMAs are M = 64: half the A operand is read per
// instruction, and the 64 rows spread over the four lane quarters (16 each),
// so that up to four quarters' epilogue warps share the output.
#pragma once
#include <cuda.h>

#include "qjl_score_v4.cuh"

namespace rq {

constexpr int kSc5Tok = 256;                         // tokens per tile (MMA N)
constexpr int kSc5SliceBytes = kSc5Tok * 128;        // one 64-column slice of B
constexpr int kSc5Threads = 18 * 32;
constexpr int kSc5MaxRing = 6;
constexpr int kSc5MaxRec = 4;

__host__ __device__ inline int sc5_qrows(int nq) { return (nq + 7) & ~7; }

// A: one 64-column region of qrows rows per slice; the MMA reads 128 rows, the
// rows past qrows fall on whatever follows (never read back).
__host__ __device__ inline size_t sc5_a_bytes(int nq, int kb)
{
    return (size_t)(kb / 64) * sc5_qrows(nq) * 128;
}
__host__ __device__ inline size_t sc5_rec_bytes(int d, int m, bool two, int pw)
{
    return (size_t)kSc5Tok * ((size_t)m / 8 + (two ? (size_t)d * pw / 8 : 0));
}
// TMA-store stage of the epilogue: per epilogue warp two 16-row x 32-float
// boxes (128-byte swizzle), used when n_q <= 64 and T % 4 == 0.
constexpr size_t kSc5StageBytes = (size_t)8 * 2 * 16 * 128;
__host__ __device__ inline size_t sc5_smem(int nq, int d, int m, bool two, int pw, int ring, int nrec, bool tma)
{
    const int kb = sc2_kb(d, m, two);
    size_t b = 1024;
    b += (sc5_a_bytes(nq, kb) + 1023) & ~(size_t)1023;            // A (queries)
    if (tma) b += kSc5StageBytes;                                  // output stage
    b += (size_t)ring * kSc5SliceBytes;                            // B ring (also absorbs the A overrun)
    b += (size_t)nrec * ((sc5_rec_bytes(d, m, two, pw) + 127) & ~(size_t)127);   // records
    if (two) b += pw <= 4 ? ((size_t)1 << (2 * pw)) * 32 * 4 : ((size_t)1 << pw) * 32 * 2;
    b += (size_t)8 * 128 * 4;                                      // epilogue per-token factors
    return b + 8 * (2 * kSc5MaxRing + 2 * kSc5MaxRec + 5) + 16;
}

// Shapes the kernel takes: every record copy 16-byte aligned and sized.
__host__ __device__ inline bool sc5_eligible(int nq, int d, int m, bool two, int pw)
{
    if (nq < 1 || nq > 128) return false;
    if ((m / 8) % 16 != 0) return false;                 // sign bytes of a token: a multiple of 16
    if (two && (d * pw / 8) % 16 != 0) return false;     // code bytes of a token: a multiple of 16
    return true;
}

// Eight sign bits -> eight fp16 values +-mag (bit 1 -> +mag): mag2 holds the
// magnitude in both halves, the sign of value 2k (2k + 1) goes to bit 15 (31)
// of word k.  ALU only, so the shared-memory bandwidth stays with the
// tensor-core operands.
__device__ __forceinline__ uint4 signs8_to_h2x4(uint32_t byte, uint32_t mag2)
{
    const uint32_t nb = ~byte;
    uint4 v;
    v.x = mag2 | ((nb << 15) & 0x00008000u) | ((nb << 30) & 0x80000000u);
    v.y = mag2 | ((nb << 13) & 0x00008000u) | ((nb << 28) & 0x80000000u);
    v.z = mag2 | ((nb << 11) & 0x00008000u) | ((nb << 26) & 0x80000000u);
    v.w = mag2 | ((nb << 9) & 0x00008000u) | ((nb << 24) & 0x80000000u);
    return v;
}

template <int PW, bool TWO>
__global__ void __launch_bounds__(kSc5Threads, 1)
score_v5_kernel(const uint16_t *__restrict__ wsB, const float *__restrict__ wsN, int nq, int d, int m,
                const uint8_t *__restrict__ signs, const uint16_t *__restrict__ sk_norms, int64_t T_len,
                int64_t G, const uint8_t *__restrict__ codes, const uint16_t *__restrict__ norms,
                const __grid_constant__ QuantTables T, float *__restrict__ scores, int ring, int nrec,
                const __grid_constant__ CUtensorMap tmo, int use_tma)
{
    const int kb = sc2_kb(d, m, TWO);
    const int nsl = kb / 64;                         // 64-column slices per tile
    const int dsl = TWO ? d / 64 : 0;                // of which first-stage (code) slices
    const int qrows = sc5_qrows(nq);
    const uint32_t sbytes = (uint32_t)m / 8, cbytes = TWO ? (uint32_t)(d * PW / 8) : 0u;
    const size_t rec_stride = (sc5_rec_bytes(d, m, TWO, PW) + 127) & ~(size_t)127;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *sA = base;
    uint8_t *sStage = sA + ((sc5_a_bytes(nq, kb) + 1023) & ~(size_t)1023);
    uint8_t *sB = sStage + (use_tma ? kSc5StageBytes : 0);
    uint8_t *sR = sB + (size_t)ring * kSc5SliceBytes;
    uint32_t *clut = reinterpret_cast<uint32_t *>(sR + (size_t)nrec * rec_stride);
    const size_t clut_bytes = TWO ? (PW <= 4 ? ((size_t)1 << (2 * PW)) * 32 * 4 : ((size_t)1 << PW) * 32 * 2) : 0;
    float *sF = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(clut) + clut_bytes);
    uint64_t *b_full = reinterpret_cast<uint64_t *>(sF + 8 * 128);
    uint64_t *b_empty = b_full + kSc5MaxRing;
    uint64_t *r_full = b_empty + kSc5MaxRing;
    uint64_t *r_empty = r_full + kSc5MaxRec;
    uint64_t *acc_full = r_empty + kSc5MaxRec;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *mma_done = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if constexpr (TWO) {
        if constexpr (PW <= 4) {
            for (int i = tid; i < (1 << (2 * PW)) * 32; i += kSc5Threads) {
                const int e = i >> 5, ca = e & ((1 << PW) - 1), cb = e >> PW;
                const float fa = ca < T.levels ? T.centroid[ca] : 0.0f, fb = cb < T.levels ? T.centroid[cb] : 0.0f;
                clut[i] = (uint32_t)__half_as_ushort(__float2half_rn(fa)) |
                          ((uint32_t)__half_as_ushort(__float2half_rn(fb)) << 16);
            }
        } else {
            uint16_t *cl16 = reinterpret_cast<uint16_t *>(clut);
            for (int i = tid; i < (1 << PW) * 32; i += kSc5Threads) {
                const int e = i >> 5;
                cl16[i] = __half_as_ushort(__float2half_rn(e < T.levels ? T.centroid[e] : 0.0f));
            }
        }
    }
    if (tid == 0) {
        for (int b = 0; b < ring; ++b) {
            mbar_init(&b_full[b], 8);          // one arrival per producer warp
            mbar_init(&b_empty[b], 1);         // MMA commit
        }
        for (int r = 0; r < nrec; ++r) {
            mbar_init(&r_full[r], 1);          // loader arrival + transaction bytes
            mbar_init(&r_empty[r], 8);         // one arrival per producer warp
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);        // MMA commit
            mbar_init(&acc_empty[a], 8);       // one arrival per epilogue warp
        }
        mbar_init(mma_done, 1);
        fence_barrier_init();
    }
    if (warp == 17) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int64_t tiles_per_g = (T_len + kSc5Tok - 1) / kSc5Tok;
    const int64_t items = G * tiles_per_g;
    const int64_t it0 = items * blockIdx.x / gridDim.x, it1 = items * (blockIdx.x + 1) / gridDim.x;
    bool ok = true;

    if (warp == 16) {
        // ------------------------------------------------------------ record loader
        if (lane == 0) {
            for (int64_t it = it0; it < it1 && ok; ++it) {
                const int64_t k = it - it0;
                const int rs = (int)(k % nrec);
                if (k >= nrec && !mbar_wait(&r_empty[rs], (uint32_t)(((k / nrec) - 1) & 1))) { ok = false; break; }
                const int64_t g = it / tiles_per_g, t0 = (it % tiles_per_g) * kSc5Tok;
                const int64_t nt = T_len - t0 < kSc5Tok ? T_len - t0 : kSc5Tok;
                const uint32_t sb = (uint32_t)nt * sbytes, cb = (uint32_t)nt * cbytes;
                uint8_t *R = sR + (size_t)rs * rec_stride;
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(&r_full[rs], sb + cb);
                bulk_load(R, signs + (g * T_len + t0) * sbytes, sb, &r_full[rs]);
                if (TWO) bulk_load(R + (size_t)kSc5Tok * sbytes, codes + (g * T_len + t0) * cbytes, cb, &r_full[rs]);
            }
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------ producers
        const int r = tid;                           // token row of the tile, 0..255
        const float kq = 1.2533141373155002512f / (float)m;
        int64_t slice = 0;
        for (int64_t it = it0; it < it1 && ok; ++it) {
            const int64_t k = it - it0;
            const int rs = (int)(k % nrec);
            const int64_t g = it / tiles_per_g, t0 = (it % tiles_per_g) * kSc5Tok;
            const bool tv = t0 + r < T_len;
            uint32_t rho2 = 0x3C003C00u;             // +-1 for the pure sketch
            if (TWO) {
                float rho = 0.0f;
                if (tv) {
                    const float n1 = h16_to_f32(__ldg(norms + g * T_len + t0 + r));
                    const float rn = h16_to_f32(__ldg(sk_norms + g * T_len + t0 + r));
                    if (n1 > 0.0f) rho = __fdiv_rn(__fmul_rn(__fmul_rn(kq, rn), (float)d), n1);
                }
                const uint32_t h = (uint32_t)__half_as_ushort(__float2half_rn(rho));
                rho2 = h | (h << 16);
            }
            if (ok && !mbar_wait(&r_full[rs], (uint32_t)((k / nrec) & 1))) ok = false;
            const uint8_t *R = sR + (size_t)rs * rec_stride;
            const uint8_t *Rs = R + (size_t)r * sbytes;
            const uint8_t *Rc = R + (size_t)kSc5Tok * sbytes + (size_t)r * cbytes;
            for (int s = 0; s < nsl; ++s, ++slice) {
                const int b = (int)(slice % ring);
                const int64_t use = slice / ring;
                if (use > 0 && ok && !mbar_wait(&b_empty[b], (uint32_t)((use - 1) & 1))) ok = false;
                uint8_t *Br = sB + (size_t)b * kSc5SliceBytes + (size_t)(r >> 3) * 1024 + (size_t)(r & 7) * 128;
                if (TWO && s < dsl) {
                    uint32_t cw[2 * PW];
                    const uint8_t *cp = Rc + s * 8 * PW;
#pragma unroll
                    for (int q = 0; q < PW; ++q) {
                        const uint2 v2 = *reinterpret_cast<const uint2 *>(cp + 8 * q);
                        cw[2 * q] = v2.x;
                        cw[2 * q + 1] = v2.y;
                    }
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        uint32_t o[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const uint32_t ca = unpack_code<64, PW>(cw, 8 * kk + 2 * e);
                            const uint32_t cb2 = unpack_code<64, PW>(cw, 8 * kk + 2 * e + 1);
                            if constexpr (PW <= 4) {
                                o[e] = clut[((ca | (cb2 << PW)) << 5) + lane];
                            } else {
                                const uint16_t *cl16 = reinterpret_cast<const uint16_t *>(clut);
                                o[e] = (uint32_t)cl16[(ca << 5) + lane] | ((uint32_t)cl16[(cb2 << 5) + lane] << 16);
                            }
                        }
                        *reinterpret_cast<uint4 *>(Br + ((kk ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                    }
                } else {
                    const int sc0 = (s - dsl) * 64;          // first sign column of the slice
                    const uint2 v2 = *reinterpret_cast<const uint2 *>(Rs + sc0 / 8);
                    const uint32_t sb[2] = {v2.x, v2.y};
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t byte = (sb[kk >> 2] >> (8 * (kk & 3))) & 0xffu;
                        *reinterpret_cast<uint4 *>(Br + ((kk ^ (r & 7)) << 4)) = signs8_to_h2x4(byte, rho2);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&b_full[b]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&r_empty[rs]);    // this warp's reads of the record are done
        }
    } else if (warp == 17) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t sA0 = smem_u32(sA), sB0 = smem_u32(sB);
        const uint32_t idesc = idesc_f16(false, nq <= 64 ? 64 : 128, kSc5Tok);
        const uint32_t aregion = (uint32_t)qrows * 128u;
        int64_t cur_g = -1, slice = 0;
        uint32_t done_phase = 0;
        bool issued = false;
        for (int64_t it = it0; it < it1 && ok; ++it) {
            const int64_t g = it / tiles_per_g;
            const int a = (int)((it - it0) & 1);
            const int64_t ause = (it - it0) >> 1;
            if (g != cur_g) {
                if (issued) {                                   // the old queries are still being read
                    if (lane == 0) mma_commit(mma_done);
                    if (ok && !mbar_wait(mma_done, done_phase)) ok = false;
                    done_phase ^= 1u;
                }
                const uint16_t *src = wsB + (int64_t)g * nq * kb;
                for (int idx = lane; idx < qrows * (kb / 8); idx += 32) {
                    const int row = idx / (kb / 8), c = idx % (kb / 8);
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (row < nq) v = __ldg(reinterpret_cast<const uint4 *>(src + (int64_t)row * kb) + c);
                    *reinterpret_cast<uint4 *>(sA + (size_t)(c >> 3) * aregion + (size_t)(row >> 3) * 1024 +
                                               (size_t)(row & 7) * 128 + (((c & 7) ^ (row & 7)) << 4)) = v;
                }
                fence_proxy_async_smem();
                __syncwarp();
                cur_g = g;
            }
            if (ause > 0 && ok && !mbar_wait(&acc_empty[a], (uint32_t)((ause - 1) & 1))) ok = false;
            tc_fence_after();
            for (int s = 0; s < nsl; ++s, ++slice) {
                const int b = (int)(slice % ring);
                if (ok && !mbar_wait(&b_full[b], (uint32_t)((slice / ring) & 1))) ok = false;
                tc_fence_after();
                if (lane == 0 && ok) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t adesc = sdesc_k_sw128(sA0 + (uint32_t)s * aregion + kk * 32u);
                        const uint64_t bdesc = sdesc_k_sw128(sB0 + (uint32_t)b * kSc5SliceBytes + kk * 32u);
                        mma_f16(tmem + (uint32_t)(a * kSc5Tok), adesc, bdesc, idesc, (s > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(&b_empty[b]);
                    if (s == nsl - 1) mma_commit(&acc_full[a]);
                }
                __syncwarp();
                issued = true;
            }
        }
        if (issued) {
            if (lane == 0) mma_commit(mma_done);
            if (ok && !mbar_wait(mma_done, done_phase)) ok = false;
        }
    } else {
        // ------------------------------------------------------------ epilogue (warps 8-15)
        // M = 64 accumulators (n_q <= 64) keep row r in TMEM lane 32 (r / 16) + r % 16; M = 128
        // ones keep row r in lane r.
        const int quarter = warp & 3;
        const int half = (warp - 8) >> 2;
        const bool m64 = nq <= 64;
        const int qi = m64 ? quarter * 16 + lane : quarter * 32 + lane;     // query row of this thread
        const bool lane_ok = (m64 ? lane < 16 : true) && qi < nq;
        const bool live = (m64 ? quarter * 16 : quarter * 32) < nq;         // the warp has queries at all
        const float kq = 1.2533141373155002512f / (float)m;
        const float inv_d = 1.0f / (float)d;
        const uint16_t *nsrc = TWO ? norms : sk_norms;
        float *fac = sF + (warp - 8) * 128;                 // this warp's per-token factors
        uint8_t *stage = sStage + (size_t)(warp - 8) * 2 * 16 * 128;   // two 2 KB boxes (use_tma)
        int nstored = 0;                                     // boxes this warp has stored
        int64_t qn_g = -1;
        float qn = 0.0f;
        // lane l holds the factors of tokens 4 l ... 4 l + 3 of the warp's 128 columns; the next
        // tile's are loaded while this one is processed
        auto load_f = [&](int64_t it, float *f) {
            const int64_t g = it / tiles_per_g, tb = (it % tiles_per_g) * kSc5Tok + half * 128;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int64_t t = tb + 4 * lane + e;
                const float nv = t < T_len ? h16_to_f32(__ldg(nsrc + g * T_len + t)) : 0.0f;
                f[e] = TWO ? __fmul_rn(nv, inv_d) : __fmul_rn(kq, nv);
            }
        };
        float fn[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if (live && it0 < it1) load_f(it0, fn);
        for (int64_t it = it0; it < it1 && ok; ++it) {
            const int64_t g = it / tiles_per_g, t0 = (it % tiles_per_g) * kSc5Tok;
            const int a = (int)((it - it0) & 1);
            const int64_t ause = (it - it0) >> 1;
            const int64_t tb = t0 + half * 128;              // first token of this warp's 128 columns
            const float f4[4] = {fn[0], fn[1], fn[2], fn[3]};
            if (live) {
                if (it + 1 < it1) load_f(it + 1, fn);
                if (g != qn_g) {
                    qn = lane_ok ? __ldg(wsN + g * nq + qi) : 0.0f;
                    qn_g = g;
                }
            }
            if (ok && !mbar_wait(&acc_full[a], (uint32_t)(ause & 1))) ok = false;
            tc_fence_after();
            if (live && ok) {
                *reinterpret_cast<float4 *>(fac + 4 * lane) = make_float4(f4[0], f4[1], f4[2], f4[3]);
                __syncwarp();
                float *dst0 = scores + ((int64_t)g * nq + qi) * T_len;
                for (int c = 0; c < 4; ++c) {
                    uint32_t rr[32];
                    tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(a * kSc5Tok + half * 128 + c * 32),
                              rr);
                    tmem_ld_wait();
                    const int64_t tc0 = tb + c * 32;
                    if (use_tma) {
                        // rows 16 quarter ... of the box: this lane's 32 scores, 128-byte swizzled
                        uint8_t *box = stage + (size_t)(nstored & 1) * 2048;
                        if (lane == 0 && nstored >= 2) bulk_wait_read<1>();    // the box's previous store has read it
                        __syncwarp();
                        if (lane < 16) {
#pragma unroll
                            for (int i = 0; i < 32; i += 4) {
                                const float4 fv = *reinterpret_cast<const float4 *>(fac + c * 32 + i);
                                float4 v;
                                v.x = __fmul_rn(__fmul_rn(fv.x, __uint_as_float(rr[i])), qn);
                                v.y = __fmul_rn(__fmul_rn(fv.y, __uint_as_float(rr[i + 1])), qn);
                                v.z = __fmul_rn(__fmul_rn(fv.z, __uint_as_float(rr[i + 2])), qn);
                                v.w = __fmul_rn(__fmul_rn(fv.w, __uint_as_float(rr[i + 3])), qn);
                                *reinterpret_cast<float4 *>(box + sw128_offset((uint32_t)lane, (uint32_t)(i >> 2))) = v;
                            }
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {                               // boxes with no column inside T are skipped
                            if (tc0 < T_len) tma_store_3d(&tmo, (int)tc0, quarter * 16, (int)g, box);
                            bulk_commit();
                        }
                        ++nstored;
                    } else if (lane_ok) {
                        float *dst = dst0 + tc0;
                        const bool full = tc0 + 32 <= T_len && ((reinterpret_cast<uintptr_t>(dst) & 15u) == 0);
#pragma unroll
                        for (int i = 0; i < 32; i += 4) {
                            const float4 fv = *reinterpret_cast<const float4 *>(fac + c * 32 + i);
                            float4 v;
                            v.x = __fmul_rn(__fmul_rn(fv.x, __uint_as_float(rr[i])), qn);
                            v.y = __fmul_rn(__fmul_rn(fv.y, __uint_as_float(rr[i + 1])), qn);
                            v.z = __fmul_rn(__fmul_rn(fv.z, __uint_as_float(rr[i + 2])), qn);
                            v.w = __fmul_rn(__fmul_rn(fv.w, __uint_as_float(rr[i + 3])), qn);
                            if (full) {
                                *reinterpret_cast<float4 *>(dst + i) = v;
                            } else {
                                if (tc0 + i < T_len) dst[i] = v.x;
                                if (tc0 + i + 1 < T_len) dst[i + 1] = v.y;
                                if (tc0 + i + 2 < T_len) dst[i + 2] = v.z;
                                if (tc0 + i + 3 < T_len) dst[i + 3] = v.w;
                            }
                        }
                    }
                }
                __syncwarp();                                   // fac is rewritten for the next tile
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[a]);
        }
        if (use_tma && lane == 0) bulk_wait<0>();              // every store has completed before exit
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 17) tmem_dealloc(tmem, 512);
}

}  // namespace rq
