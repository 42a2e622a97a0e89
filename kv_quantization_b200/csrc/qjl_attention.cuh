// qjl_attention.cuh -- attention decode over compressed keys and values on the
// tcgen05 tensor cores (sm_100a).
//
//   out[g][q][:] = sum_t softmax_t(scale * s(q, t)) * vh_t
//
// s(q, t) is the QJL / two-stage score of qjl_score (the query is projected
// through the same S and the score rebuilt from the key's sign bits and
// norms: eliza quantization README, "QJL", "Algorithm in one paragraph"), and
// vh_t the reconstruction of value block (g, t): vh_t = D H (c[v_t] * n_t / d)
// (the PolarQuant inverse of the same README).  The values are dequantized
// inside the kernel, as the GLQ README's "Inline-dequant E8 KV" does, and the
// key range is split over the SMs with a combine step (flash-decoding).
//
// Because H and D are linear and the same for every token, the weighted sum
// is taken in the rotated domain and rotated once per query at the end:
//   out = D H ( sum_t p_t (n_t / d) c[v_t] ) / sum_t p_t,
// so the per-token work on V is a centroid lookup and a multiply, with no
// Walsh-Hadamard transform per token.
//
// Main kernel, per (group, 256-token tile), one CTA per SM over a contiguous
// range of tiles (queries on M as in qjl_score_v5.cuh):
//   producers (8 warps, thread = token): key slices as score_v5; then the
//     token's value row as fp16 V' = fp16(c[v_t]) * fp16(n_t / d) into a
//     128-token value slice (MN-major B operand: token rows, two 64-wide
//     atoms of d).  Measured: splitting the warps into key and value groups
//     made the key unpack (4 warps) the critical path, so all eight do both;
//   MMA issuer 1: S[q][t] = A_q . K_t (M = 128, N = 256) into TMEM;
//   softmax warps (4 warps of TMEM lane quarter 0: lane = query, 64 columns
//     each): a = S * g_t * (||q|| scale log2 e) (g_t the score's per-token
//     factor), running max m, p = 2^(a - m), l += p, P' = fp16(2^14 p) into
//     a K-major A operand [query][token] in shared memory;
//   MMA issuer 2: O_tile[q][j] = P' . V' (M = 128, N = d = 128, K = 256);
//   the softmax warps fold each O_tile into fp32 registers,
//     O = O * 2^(m_old - m_new) + O_tile, 32 columns of d per warp.
// At the end of a group's run of tiles the CTA writes (m, l, O) per query to
// its partial slot (CTA index + group: unique and increasing along the
// ordered (CTA, group) segments).
//
// Combine kernel, per (group, query): M = max m_s, L = sum l_s 2^(m_s - M),
// o = sum O_s 2^(m_s - M) / L (l and O both carry the factor 2^14 of the
// weights), then the fp32 radix-2 transform of o
// (stages h = 1 ... d/2) and the value sign diagonal: out = D H o.
#pragma once
#include "qjl_score_v5.cuh"

namespace rq {

constexpr int kAtTok = 256;                      // tokens per tile (MMA 1 N, MMA 2 K)
constexpr int kAtD = 128;                        // value head dimension (MMA 2 N)
constexpr int kAtThreads = 16 * 32;
constexpr int kAtKSlice = kAtTok * 128;          // 64 key columns of 256 tokens, fp16
constexpr int kAtVSlice = 128 * kAtD * 2;        // 128 tokens x 128 values, fp16
constexpr int kAtPBuf = 4 * 32 * 128;            // 4 regions of 64 tokens x 32 query rows, fp16
constexpr int kAtMaxQ = 32;
constexpr int kAtMaxKRing = 3;
constexpr int kAtMaxRec = 3;
constexpr float kAtPExp = 14.0f;                 // P' = 2^14 p keeps small weights normal in fp16

__host__ __device__ inline int at_kcopies() { return 8; }
__host__ __device__ inline size_t at_klut_bytes(bool two, int pw)
{
    return two ? (pw <= 4 ? ((size_t)1 << (2 * pw)) * 8 * 4 : ((size_t)1 << pw) * 8 * 2) : 0;
}
__host__ __device__ inline size_t at_vlut_bytes(int vpw)
{
    return vpw <= 4 ? ((size_t)1 << (2 * vpw)) * 8 * 4 : ((size_t)1 << vpw) * 8 * 2;
}
__host__ __device__ inline size_t at_smem(int d, int m, bool two, int pw, int vpw, int kring, int nrec)
{
    const int kb = sc2_kb(d, m, two);
    size_t b = 1024;
    b += (size_t)(kb / 64) * 32 * 128;                            // A (queries), 32 rows per region
    b += (size_t)kring * kAtKSlice;                                // key slices (absorb the A overrun)
    b += (size_t)2 * kAtVSlice;                                    // value slices
    b += (size_t)2 * kAtPBuf;                                      // P' (double buffer)
    b += (size_t)nrec * ((sc5_rec_bytes(d, m, two, pw) + 127) & ~(size_t)127);   // key records (absorb the P overrun)
    b += at_klut_bytes(two, pw) + at_vlut_bytes(vpw);
    b += (size_t)4 * 64 * 4 + 2 * 4 * 32 * 4 + 4 * 32 * 4;         // per-token factors, max and sum exchange
    return b + 8 * (2 * kAtMaxKRing + 2 * 2 + 2 * kAtMaxRec + 2 + 2 * 2 + 2 * 2 + 1) + 16;
}

__host__ __device__ inline bool at_eligible(int nq, int d, int m, bool two, int pw)
{
    return nq >= 1 && nq <= kAtMaxQ && d == kAtD && sc5_eligible(nq, d, m, two, pw);
}

// Partial results of one (CTA, group) segment: O [nq][d], then m [nq] and
// l [nq], padded to a multiple of four floats (16-byte aligned slots).
__host__ __device__ inline size_t at_part_floats(int nq, int d) { return ((size_t)nq * (d + 2) + 3) & ~(size_t)3; }

__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void named_sync(int id, int threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Shared-memory descriptor with explicit leading/stride byte offsets (128-byte swizzle).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3ffffu) >> 4);
    d |= (uint64_t)((lbo >> 4) & 0x3fffu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3fffu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

template <int PW, bool TWO, int VPW>
__global__ void __launch_bounds__(kAtThreads, 1)
attention_kernel(const uint16_t *__restrict__ wsB, const float *__restrict__ wsN, int nq, int d, int m,
                 const uint8_t *__restrict__ signs, const uint16_t *__restrict__ sk_norms, int64_t T_len, int64_t G,
                 const uint8_t *__restrict__ codes, const uint16_t *__restrict__ norms,
                 const uint8_t *__restrict__ vcodes, const uint16_t *__restrict__ vnorms,
                 const __grid_constant__ QuantTables TK, const __grid_constant__ QuantTables TV, float qscale,
                 float *__restrict__ part, int kring, int nrec)
{
    const int kb = sc2_kb(d, m, TWO);
    const int nsl = kb / 64;
    const int dsl = TWO ? d / 64 : 0;
    const uint32_t sbytes = (uint32_t)m / 8, cbytes = TWO ? (uint32_t)(d * PW / 8) : 0u;
    constexpr uint32_t vcb = (uint32_t)(kAtD * VPW / 8);          // value code bytes per token
    const size_t rec_stride = (sc5_rec_bytes(d, m, TWO, PW) + 127) & ~(size_t)127;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *sA = base;
    uint8_t *sK = sA + (size_t)nsl * 32 * 128;
    uint8_t *sV = sK + (size_t)kring * kAtKSlice;
    uint8_t *sP = sV + (size_t)2 * kAtVSlice;
    uint8_t *sR = sP + (size_t)2 * kAtPBuf;
    uint32_t *klut = reinterpret_cast<uint32_t *>(sR + (size_t)nrec * rec_stride);
    uint32_t *vlut = reinterpret_cast<uint32_t *>(reinterpret_cast<uint8_t *>(klut) + at_klut_bytes(TWO, PW));
    float *sG = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(vlut) + at_vlut_bytes(VPW));   // [4][64]
    float *sXM = sG + 4 * 64;                                       // [2][4][32] tile maxima
    float *sXL = sXM + 2 * 4 * 32;                                  // [4][32] sums
    uint64_t *k_full = reinterpret_cast<uint64_t *>(sXL + 4 * 32);
    uint64_t *k_empty = k_full + kAtMaxKRing;
    uint64_t *v_full = k_empty + kAtMaxKRing;
    uint64_t *v_empty = v_full + 2;
    uint64_t *r_full = v_empty + 2;
    uint64_t *r_empty = r_full + kAtMaxRec;
    uint64_t *s_full = r_empty + kAtMaxRec;
    uint64_t *s_empty = s_full + 1;
    uint64_t *p_full = s_empty + 1;
    uint64_t *p_empty = p_full + 2;
    uint64_t *o_full = p_empty + 2;
    uint64_t *o_empty = o_full + 2;
    uint64_t *mma_done = o_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // centroid pair tables (fp16), 8 copies (lane % 8)
    auto fill_pairs = [&](const QuantTables &T, uint32_t *lut, int pw) {
        if (pw <= 4) {
            for (int i = tid; i < (1 << (2 * pw)) * 8; i += kAtThreads) {
                const int e = i >> 3, ca = e & ((1 << pw) - 1), cb = e >> pw;
                const float fa = ca < T.levels ? T.centroid[ca] : 0.0f, fb = cb < T.levels ? T.centroid[cb] : 0.0f;
                lut[i] = (uint32_t)__half_as_ushort(__float2half_rn(fa)) |
                         ((uint32_t)__half_as_ushort(__float2half_rn(fb)) << 16);
            }
        } else {
            uint16_t *l16 = reinterpret_cast<uint16_t *>(lut);
            for (int i = tid; i < (1 << pw) * 8; i += kAtThreads) {
                const int e = i >> 3;
                l16[i] = __half_as_ushort(__float2half_rn(e < T.levels ? T.centroid[e] : 0.0f));
            }
        }
    };
    if (TWO) fill_pairs(TK, klut, PW);
    fill_pairs(TV, vlut, VPW);
    if (tid == 0) {
        for (int b = 0; b < kring; ++b) { mbar_init(&k_full[b], 8); mbar_init(&k_empty[b], 1); }   // 8 producer warps
        for (int b = 0; b < 2; ++b) { mbar_init(&v_full[b], 4); mbar_init(&v_empty[b], 1); }       // 4 per tile half
        for (int r = 0; r < nrec; ++r) { mbar_init(&r_full[r], 1); mbar_init(&r_empty[r], 8); }
        mbar_init(s_full, 1);
        mbar_init(s_empty, 4);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&p_full[b], 4); mbar_init(&p_empty[b], 1);
            mbar_init(&o_full[b], 1); mbar_init(&o_empty[b], 4);
        }
        mbar_init(mma_done, 1);
        fence_barrier_init();
    }
    if (warp == 11) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int64_t tiles_per_g = (T_len + kAtTok - 1) / kAtTok;
    const int64_t items = G * tiles_per_g;
    const int64_t it0 = items * blockIdx.x / gridDim.x, it1 = items * (blockIdx.x + 1) / gridDim.x;
    bool ok = true;
    const bool softmax_warp = (warp & 3) == 0;                      // warps 0, 4, 8, 12: TMEM lanes 0-31
    const int pidx = softmax_warp ? -1 : (warp < 11 ? warp - 1 - (warp >> 2) : -1);   // producers 1,2,3,5,6,7,9,10

    if (warp == 14) {
        // ------------------------------------------------------------ key record loader
        if (lane == 0) {
            for (int64_t it = it0; it < it1 && ok; ++it) {
                const int64_t k = it - it0;
                const int rs = (int)(k % nrec);
                if (k >= nrec && !mbar_wait(&r_empty[rs], (uint32_t)(((k / nrec) - 1) & 1))) { ok = false; break; }
                const int64_t g = it / tiles_per_g, t0 = (it % tiles_per_g) * kAtTok;
                const int64_t nt = T_len - t0 < kAtTok ? T_len - t0 : kAtTok;
                const uint32_t sb = (uint32_t)nt * sbytes, cb = (uint32_t)nt * cbytes;
                uint8_t *R = sR + (size_t)rs * rec_stride;
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(&r_full[rs], sb + cb);
                bulk_load(R, signs + (g * T_len + t0) * sbytes, sb, &r_full[rs]);
                if (TWO) bulk_load(R + (size_t)kAtTok * sbytes, codes + (g * T_len + t0) * cbytes, cb, &r_full[rs]);
            }
        }
    } else if (pidx >= 0) {
        // ------------------------------------------------------------ producers (thread = token row)
        const int r = pidx * 32 + lane;                           // 0..255
        const int vh = r >> 7, vr = r & 127;                      // value slice (tile half) and row in it
        const float kq = 1.2533141373155002512f / (float)m;
        const uint32_t lane8 = (uint32_t)(lane & 7);
        int64_t slice = 0;
        for (int64_t it = it0; it < it1 && ok; ++it) {
            const int64_t k = it - it0;
            const int rs = (int)(k % nrec);
            const int64_t g = it / tiles_per_g, t0 = (it % tiles_per_g) * kAtTok;
            const bool tv = t0 + r < T_len;
            const int64_t kt = g * T_len + t0 + r;
            // the value row's codes and norm (loaded early, used after the keys)
            uint32_t vw[vcb / 4];
            uint32_t vf2 = 0u;
#pragma unroll
            for (int i = 0; i < (int)(vcb / 16); ++i) {
                const uint4 v4 = tv ? __ldg(reinterpret_cast<const uint4 *>(vcodes + kt * vcb) + i) : make_uint4(0u, 0u, 0u, 0u);
                vw[4 * i] = v4.x; vw[4 * i + 1] = v4.y; vw[4 * i + 2] = v4.z; vw[4 * i + 3] = v4.w;
            }
            if (tv) {
                const float fv = __fmul_rn(h16_to_f32(__ldg(vnorms + kt)), 1.0f / (float)kAtD);
                const uint32_t h = (uint32_t)__half_as_ushort(__float2half_rn(fv));
                vf2 = h | (h << 16);
            }
            uint32_t rho2 = 0x3C003C00u;
            if (TWO) {
                float rho = 0.0f;
                if (tv) {
                    const float n1 = h16_to_f32(__ldg(norms + kt));
                    const float rn = h16_to_f32(__ldg(sk_norms + kt));
                    if (n1 > 0.0f) rho = __fdiv_rn(__fmul_rn(__fmul_rn(kq, rn), (float)d), n1);
                }
                const uint32_t h = (uint32_t)__half_as_ushort(__float2half_rn(rho));
                rho2 = h | (h << 16);
            }
            if (ok && !mbar_wait(&r_full[rs], (uint32_t)((k / nrec) & 1))) ok = false;
            const uint8_t *R = sR + (size_t)rs * rec_stride;
            const uint8_t *Rs = R + (size_t)r * sbytes;
            const uint8_t *Rc = R + (size_t)kAtTok * sbytes + (size_t)r * cbytes;
            for (int s = 0; s < nsl; ++s, ++slice) {
                const int b = (int)(slice % kring);
                const int64_t use = slice / kring;
                if (use > 0 && ok && !mbar_wait(&k_empty[b], (uint32_t)((use - 1) & 1))) ok = false;
                uint8_t *Br = sK + (size_t)b * kAtKSlice + (size_t)(r >> 3) * 1024 + (size_t)(r & 7) * 128;
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
                                o[e] = klut[((ca | (cb2 << PW)) << 3) + lane8];
                            } else {
                                const uint16_t *k16 = reinterpret_cast<const uint16_t *>(klut);
                                o[e] = (uint32_t)k16[(ca << 3) + lane8] | ((uint32_t)k16[(cb2 << 3) + lane8] << 16);
                            }
                        }
                        *reinterpret_cast<uint4 *>(Br + ((kk ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                    }
                } else {
                    const int sc0 = (s - dsl) * 64;
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
                if (lane == 0) mbar_arrive(&k_full[b]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&r_empty[rs]);
            // value row: V' = fp16(c) * fp16(n / d), rows of the MN-major B operand (two 64-wide atoms of d)
            if (k > 0 && ok && !mbar_wait(&v_empty[vh], (uint32_t)((k - 1) & 1))) ok = false;
            uint8_t *Vr = sV + (size_t)vh * kAtVSlice + (size_t)(vr >> 3) * 1024 + (size_t)(vr & 7) * 128;
#pragma unroll
            for (int ch = 0; ch < 16; ++ch) {                     // 16 chunks of 8 values: d = 8 ch ... 8 ch + 7
                uint32_t o[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = 8 * ch + 2 * e;
                    const uint32_t ca = unpack_code<kAtD, VPW>(vw, j), cb2 = unpack_code<kAtD, VPW>(vw, j + 1);
                    uint32_t pr;
                    if constexpr (VPW <= 4) {
                        pr = vlut[((ca | (cb2 << VPW)) << 3) + lane8];
                    } else {
                        const uint16_t *v16 = reinterpret_cast<const uint16_t *>(vlut);
                        pr = (uint32_t)v16[(ca << 3) + lane8] | ((uint32_t)v16[(cb2 << 3) + lane8] << 16);
                    }
                    const __half2 hv = __hmul2(*reinterpret_cast<const __half2 *>(&pr),
                                               *reinterpret_cast<const __half2 *>(&vf2));
                    o[e] = tv ? *reinterpret_cast<const uint32_t *>(&hv) : 0u;
                }
                const int atom = ch >> 3, c8 = ch & 7;
                *reinterpret_cast<uint4 *>(Vr + (size_t)atom * (kAtVSlice / 2) + ((c8 ^ (vr & 7)) << 4)) =
                    make_uint4(o[0], o[1], o[2], o[3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&v_full[vh]);
        }
    } else if (warp == 11) {
        // ------------------------------------------------------------ MMA 1: S = A_q . K
        const uint32_t sA0 = smem_u32(sA), sK0 = smem_u32(sK);
        const uint32_t idesc = idesc_f16(false, 128, kAtTok);
        int64_t cur_g = -1, slice = 0;
        uint32_t done_phase = 0;
        bool issued = false;
        for (int64_t it = it0; it < it1 && ok; ++it) {
            const int64_t g = it / tiles_per_g;
            const int64_t c = it - it0;
            if (g != cur_g) {
                if (issued) {
                    if (lane == 0) mma_commit(mma_done);
                    if (ok && !mbar_wait(mma_done, done_phase)) ok = false;
                    done_phase ^= 1u;
                }
                const uint16_t *src = wsB + (int64_t)g * nq * kb;
                for (int idx = lane; idx < 32 * (kb / 8); idx += 32) {
                    const int row = idx / (kb / 8), col = idx % (kb / 8);
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (row < nq) v = __ldg(reinterpret_cast<const uint4 *>(src + (int64_t)row * kb) + col);
                    *reinterpret_cast<uint4 *>(sA + (size_t)(col >> 3) * 4096 + (size_t)(row >> 3) * 1024 +
                                               (size_t)(row & 7) * 128 + (((col & 7) ^ (row & 7)) << 4)) = v;
                }
                fence_proxy_async_smem();
                __syncwarp();
                cur_g = g;
            }
            if (c > 0 && ok && !mbar_wait(s_empty, (uint32_t)((c - 1) & 1))) ok = false;
            tc_fence_after();
            for (int s = 0; s < nsl; ++s, ++slice) {
                const int b = (int)(slice % kring);
                if (ok && !mbar_wait(&k_full[b], (uint32_t)((slice / kring) & 1))) ok = false;
                tc_fence_after();
                if (lane == 0 && ok) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t adesc = sdesc_k_sw128(sA0 + (uint32_t)s * 4096u + kk * 32u);
                        const uint64_t bdesc = sdesc_k_sw128(sK0 + (uint32_t)b * kAtKSlice + kk * 32u);
                        mma_f16(tmem, adesc, bdesc, idesc, (s > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(&k_empty[b]);
                    if (s == nsl - 1) mma_commit(s_full);
                }
                __syncwarp();
                issued = true;
            }
        }
        if (issued) {
            if (lane == 0) mma_commit(mma_done);
            if (ok && !mbar_wait(mma_done, done_phase)) ok = false;
        }
    } else if (warp == 13) {
        // ------------------------------------------------------------ MMA 2: O_tile = P' . V'
        const uint32_t sP0 = smem_u32(sP), sV0 = smem_u32(sV);
        const uint32_t idesc = idesc_f16(false, 128, kAtD) | (1u << 16);   // B (values) MN-major
        for (int64_t it = it0; it < it1 && ok; ++it) {
            const int64_t c = it - it0;
            const int b = (int)(c & 1);
            if (ok && !mbar_wait(&p_full[b], (uint32_t)((c >> 1) & 1))) ok = false;
            if (c >= 2 && ok && !mbar_wait(&o_empty[b], (uint32_t)(((c >> 1) - 1) & 1))) ok = false;
            tc_fence_after();
            for (int vh = 0; vh < 2; ++vh) {
                if (ok && !mbar_wait(&v_full[vh], (uint32_t)(c & 1))) ok = false;
                tc_fence_after();
                if (lane == 0 && ok) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const int tok = vh * 128 + kk * 16;         // first token of this K step
                        const uint64_t adesc = sdesc_k_sw128(sP0 + (uint32_t)b * kAtPBuf + (uint32_t)(tok >> 6) * 4096u +
                                                             (uint32_t)((tok & 63) >> 3) * 16u);
                        const uint64_t bdesc = sdesc_sw128(sV0 + (uint32_t)vh * kAtVSlice + (uint32_t)kk * 2048u,
                                                           (uint32_t)(kAtVSlice / 2), 1024u);
                        mma_f16(tmem + 256u + (uint32_t)b * 128u, adesc, bdesc, idesc, (vh > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(&v_empty[vh]);
                    if (vh == 1) {
                        mma_commit(&p_empty[b]);
                        mma_commit(&o_full[b]);
                    }
                }
                __syncwarp();
            }
        }
    } else if (softmax_warp) {
        // ------------------------------------------------------------ softmax + output accumulation
        const int kw = warp >> 2;                                // column quarter: S columns 64 kw ..., O columns 32 kw ...
        const int qi = lane;
        const float kq = 1.2533141373155002512f / (float)m;
        const float inv_d = 1.0f / (float)d;
        const uint16_t *gsrc = TWO ? norms : sk_norms;
        float *gw = sG + kw * 64;
        float mrun = -INFINITY, lpart = 0.0f, cq = 0.0f, alpha_prev = 0.0f;
        float O[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) O[j] = 0.0f;
        int64_t pending = -1;                                    // tile whose O_tile is still to be folded in
        float gn0 = 0.0f, gn1 = 0.0f;                            // norms of this lane's two columns, next tile
        auto load_g = [&](int64_t it) {
            const int64_t g = it / tiles_per_g, ta = (it % tiles_per_g) * kAtTok + kw * 64 + 2 * lane;
            gn0 = ta < T_len ? h16_to_f32(__ldg(gsrc + g * T_len + ta)) : 0.0f;
            gn1 = ta + 1 < T_len ? h16_to_f32(__ldg(gsrc + g * T_len + ta + 1)) : 0.0f;
        };
        if (it0 < it1) load_g(it0);
        auto fold = [&](int64_t c, float alpha) {
            const int b = (int)(c & 1);
            if (ok && !mbar_wait(&o_full[b], (uint32_t)((c >> 1) & 1))) ok = false;
            tc_fence_after();
            uint32_t r32[32];
            tmem_ld32(tmem + 256u + (uint32_t)b * 128u + (uint32_t)(kw * 32), r32);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) O[j] = __fmaf_rn(O[j], alpha, __uint_as_float(r32[j]));
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&o_empty[b]);
        };
        // Every softmax warp runs every item and every named barrier, also
        // after a wait has expired (ok == false), so that the four stay in
        // step on barrier 1.
        for (int64_t it = it0; it < it1; ++it) {
            const int64_t c = it - it0;
            const int b = (int)(c & 1);
            const int64_t g = it / tiles_per_g, t0 = (it % tiles_per_g) * kAtTok;
            const bool seg_start = it == it0 || (it - 1) / tiles_per_g != g;
            if (seg_start) cq = qi < nq ? __fmul_rn(__ldg(wsN + g * nq + qi), qscale) : 0.0f;
            // per-token score factors of this warp's 64 columns (loaded one tile ahead)
            __syncwarp();                                        // the previous tile's reads of gw are done
            *reinterpret_cast<float2 *>(gw + 2 * lane) = make_float2(TWO ? __fmul_rn(gn0, inv_d) : __fmul_rn(kq, gn0),
                                                                     TWO ? __fmul_rn(gn1, inv_d) : __fmul_rn(kq, gn1));
            __syncwarp();
            if (it + 1 < it1) load_g(it + 1);
            if (ok && !mbar_wait(s_full, (uint32_t)(c & 1))) ok = false;
            tc_fence_after();
            uint32_t sr[64];
            tmem_ld32(tmem + (uint32_t)(kw * 64), sr);
            tmem_ld32(tmem + (uint32_t)(kw * 64 + 32), sr + 32);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(s_empty);
            const int64_t tcol = t0 + kw * 64;                   // token of column 0 of this warp
            const int nvalid = T_len - tcol >= 64 ? 64 : (T_len - tcol > 0 ? (int)(T_len - tcol) : 0);
            // a_j = S_j g_j ||q|| scale log2(e), kept in place of S_j
            float mx = -INFINITY;
#pragma unroll
            for (int j = 0; j < 64; j += 2) {
                const float2 gj = *reinterpret_cast<const float2 *>(gw + j);
                const float2 v = __fmul2_rn(__fmul2_rn(make_float2(__uint_as_float(sr[j]), __uint_as_float(sr[j + 1])), gj),
                                            make_float2(cq, cq));
                sr[j] = __float_as_uint(v.x);
                sr[j + 1] = __float_as_uint(v.y);
                if (j < nvalid) mx = fmaxf(mx, v.x);
                if (j + 1 < nvalid) mx = fmaxf(mx, v.y);
            }
            float *xm = sXM + (c & 1) * 128;
            xm[kw * 32 + lane] = mx;
            named_sync(1, 128);
            const float mt = fmaxf(fmaxf(xm[lane], xm[32 + lane]), fmaxf(xm[64 + lane], xm[96 + lane]));
            const float mnew = fmaxf(mrun, mt);
            const float alpha = ex2_approx(mrun - mnew);        // 0 for the first tile (mrun = -inf)
            // P' = 2^14 p = 2^(a - m + 14): row qi of tokens 64 kw ... 64 kw + 63, region kw of buffer b
            if (c >= 2 && ok && !mbar_wait(&p_empty[b], (uint32_t)(((c >> 1) - 1) & 1))) ok = false;
            uint8_t *Pr = sP + (size_t)b * kAtPBuf + (size_t)kw * 4096 + (size_t)(qi >> 3) * 1024 + (size_t)(qi & 7) * 128;
            const float moff = mnew - kAtPExp;
            float ls = 0.0f;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                uint32_t w4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = 8 * ch + 2 * e;
                    const float p0 = j < nvalid ? ex2_approx(__uint_as_float(sr[j]) - moff) : 0.0f;
                    const float p1 = j + 1 < nvalid ? ex2_approx(__uint_as_float(sr[j + 1]) - moff) : 0.0f;
                    ls += p0 + p1;
                    const __half2 h = __floats2half2_rn(p0, p1);
                    w4[e] = *reinterpret_cast<const uint32_t *>(&h);
                }
                *reinterpret_cast<uint4 *>(Pr + ((ch ^ (qi & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
            lpart = __fmaf_rn(lpart, alpha, ls);
            mrun = mnew;
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[b]);
            // fold the previous tile's O_tile (its P used the maximum before this tile's)
            if (pending >= 0) fold(pending, alpha_prev);
            pending = c;
            alpha_prev = alpha;
            const bool seg_end = it + 1 >= it1 || (it + 1) / tiles_per_g != g;
            if (seg_end) {
                fold(pending, alpha_prev);
                pending = -1;
                // l over the four column quarters
                sXL[kw * 32 + lane] = lpart;
                named_sync(1, 128);
                const float lt = sXL[lane] + sXL[32 + lane] + sXL[64 + lane] + sXL[96 + lane];
                float *P = part + (size_t)(blockIdx.x + g) * at_part_floats(nq, d);
                if (qi < nq) {
                    if (kw == 0) {
                        P[(size_t)nq * d + qi] = mrun;
                        P[(size_t)nq * d + nq + qi] = lt;
                    }
                    float *Po = P + (size_t)qi * d + kw * 32;
#pragma unroll
                    for (int j = 0; j < 32; j += 4) *reinterpret_cast<float4 *>(Po + j) = make_float4(O[j], O[j + 1], O[j + 2], O[j + 3]);
                }
                named_sync(1, 128);                               // sXL is rewritten by the next segment
                mrun = -INFINITY;
                lpart = 0.0f;
#pragma unroll
                for (int j = 0; j < 32; ++j) O[j] = 0.0f;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 11) tmem_dealloc(tmem, 512);
}

// Combine the partial slots of each group and rotate back: one CTA of d
// threads per (group, query).
__global__ void __launch_bounds__(kAtD)
attention_combine_kernel(const float *__restrict__ part, int nq, int d, int64_t T_len, int64_t G, int grid_main,
                         const __grid_constant__ QuantTables TV, float *__restrict__ out)
{
    __shared__ float o[kAtD];
    const int64_t g = blockIdx.x;
    const int qi = blockIdx.y;
    const int j = threadIdx.x;
    const int64_t tiles_per_g = (T_len + kAtTok - 1) / kAtTok;
    const int64_t items = G * tiles_per_g;
    const int64_t lo = g * tiles_per_g, hi = (g + 1) * tiles_per_g;   // this group's items
    // CTAs whose ranges [items c / grid, items (c + 1) / grid) meet [lo, hi)
    int c0 = (int)((lo * grid_main) / items);
    while (c0 > 0 && items * c0 / grid_main > lo) --c0;
    while (items * (c0 + 1) / grid_main <= lo) ++c0;
    float M = -INFINITY;
    for (int c = c0; c < grid_main && items * c / grid_main < hi; ++c) {
        if (items * (c + 1) / grid_main <= items * c / grid_main) continue;      // empty range
        M = fmaxf(M, part[(size_t)(c + g) * at_part_floats(nq, d) + (size_t)nq * d + qi]);
    }
    float L = 0.0f, acc = 0.0f;
    for (int c = c0; c < grid_main && items * c / grid_main < hi; ++c) {
        if (items * (c + 1) / grid_main <= items * c / grid_main) continue;
        const float *P = part + (size_t)(c + g) * at_part_floats(nq, d);
        const float w = exp2f(P[(size_t)nq * d + qi] - M);
        L = __fmaf_rn(P[(size_t)nq * d + nq + qi], w, L);
        acc = __fmaf_rn(P[(size_t)qi * d + j], w, acc);
    }
    o[j] = acc / L;                                  // O and l both carry the factor 2^14
    __syncthreads();
    for (int h = 1; h < d; h *= 2) {
        float v = 0.0f;
        const bool lo_half = (j & h) == 0;
        const float a = o[lo_half ? j : j - h], b2 = o[lo_half ? j + h : j];
        v = lo_half ? __fadd_rn(a, b2) : __fsub_rn(a, b2);
        __syncthreads();
        o[j] = v;
        __syncthreads();
    }
    const bool neg = (TV.sign_words[j >> 5] >> (j & 31)) & 1u;
    out[((size_t)g * nq + qi) * d + j] = neg ? -o[j] : o[j];
}

}  // namespace rq
