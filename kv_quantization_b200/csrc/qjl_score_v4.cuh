// qjl_score_v4.cuh -- warp-specialised tensor-core score kernel (sm_100a).
//
// Arithmetic as described in qjl_score_v2.cuh (A = unpacked keys in fp16,
// B = prologue queries in fp16, two fp32 TMEM accumulators), organised as a
// producer / MMA / epilogue pipeline that meets only at mbarriers, with the
// A-operand production split over two sets of four producer warps: set s stages only the packed bytes of the
// 64-column regions g with g % 2 == s (its own cp.async group, so no thread
// waits for another's copies) and writes only those regions of each chunk; a
// chunk is full after eight warp arrivals.  Measured on the pure-QJL KV-cache
// shape, the four-warp producer was the critical path of the pipeline (about
// 0.7 us per 32 KB chunk); the ring of chunks is 3 or 4 deep as shared memory
// allows.  Warps: 0-7 producers, 8 MMA issuer, 9-12 epilogue (TMEM lane
// quarter = warp mod 4).
#pragma once
#include "qjl_score_v2.cuh"

namespace rq {

__device__ __forceinline__ void cp_async16(void *dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(void *dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Per-thread record row: codes then signs; the row length is an odd number
// of 8-byte words so that 64-bit reads of 16 consecutive rows hit 32 distinct
// banks.
__host__ __device__ inline int sc3_row_bytes(int d, int m, bool two, int pw)
{
    const int raw = (two ? d * pw / 8 : 0) + ((m / 8 + 7) & ~7);
    int w8 = (raw + 7) / 8;
    if ((w8 & 1) == 0) ++w8;
    return 8 * w8;
}

constexpr int kSc4Threads = 13 * 32;
constexpr int kSc4MaxRing = 4;

// ring: A chunks in flight; nrec: key-record tiles staged (prefetch depth nrec - 1);
// slc: copies of the sign-byte LUT (8: conflict-free, 2: for the largest shapes)
__host__ __device__ inline size_t sc4_smem(int nq, int d, int m, bool two, int pw, int ring, int nrec, int slc)
{
    const int kb = sc2_kb(d, m, two), nq32 = sc2_nq16(nq);
    size_t b = 1024;
    b += (size_t)ring * kSc2ChunkBytes;                            // A ring
    b += (size_t)nq32 * kb * 2;                                    // B
    b += (size_t)256 * slc * 16;                                   // sign LUT
    if (two) b += pw <= 4 ? ((size_t)1 << (2 * pw)) * 32 * 4 : ((size_t)1 << pw) * 32 * 2;
    b += (size_t)nrec * 128 * sc3_row_bytes(d, m, two, pw);        // staged records
    return b + 8 * (2 * kSc4MaxRing + 5) + 16;
}

template <int PW, bool TWO, int NREC>
__global__ void __launch_bounds__(kSc4Threads, 1)
score_v4_kernel(const uint16_t *__restrict__ wsB, const float *__restrict__ wsN, int nq, int d, int m,
                const uint8_t *__restrict__ signs, const uint16_t *__restrict__ sk_norms, int64_t T_len,
                int64_t G, const uint8_t *__restrict__ codes, const uint16_t *__restrict__ norms,
                const __grid_constant__ QuantTables T, float *__restrict__ scores, int ring, int slc)
{
    const int nq32 = sc2_nq16(nq), kb = sc2_kb(d, m, TWO);
    const int dreg = TWO ? d / 64 : 0;
    const int nchunks = (kb + kSc2Chunk - 1) / kSc2Chunk;
    const int nreg = kb / 64;
    const int cbytes = TWO ? d * PW / 8 : 0, sbytes = m / 8;
    const int rowb = sc3_row_bytes(d, m, TWO, PW);
    const uint32_t ncols = 4u * (uint32_t)nq32 <= 128u ? 128u : (4u * (uint32_t)nq32 <= 256u ? 256u : 512u);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *sA = base;
    uint8_t *sB = sA + (size_t)ring * kSc2ChunkBytes;
    uint4 *slut = reinterpret_cast<uint4 *>(sB + (size_t)nq32 * kb * 2);
    uint32_t *clut = reinterpret_cast<uint32_t *>(slut + 256 * slc);
    const size_t clut_bytes = TWO ? (PW <= 4 ? ((size_t)1 << (2 * PW)) * 32 * 4 : ((size_t)1 << PW) * 32 * 2) : 0;
    uint8_t *srec = reinterpret_cast<uint8_t *>(clut) + clut_bytes;
    uint64_t *a_full = reinterpret_cast<uint64_t *>(srec + NREC * 128 * rowb);
    uint64_t *a_empty = a_full + kSc4MaxRing;
    uint64_t *acc_full = a_empty + kSc4MaxRing;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *mma_done = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slc_log2 = slc == 8 ? 3 : (slc == 4 ? 2 : (slc == 2 ? 1 : 0));   // slc is a power of two <= 8
    const uint32_t slc_lane = (uint32_t)(threadIdx.x & 31) & (uint32_t)(slc - 1);
    for (int i = tid; i < 256 * slc; i += kSc4Threads) {
        const int byte = i >> slc_log2;
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
        if constexpr (PW <= 4) {
            for (int i = tid; i < (1 << (2 * PW)) * 32; i += kSc4Threads) {
                const int e = i >> 5, ca = e & ((1 << PW) - 1), cb = e >> PW;
                const float fa = ca < T.levels ? T.centroid[ca] : 0.0f, fb = cb < T.levels ? T.centroid[cb] : 0.0f;
                clut[i] = (uint32_t)__half_as_ushort(__float2half_rn(fa)) |
                          ((uint32_t)__half_as_ushort(__float2half_rn(fb)) << 16);
            }
        } else {
            uint16_t *cl16 = reinterpret_cast<uint16_t *>(clut);
            for (int i = tid; i < (1 << PW) * 32; i += kSc4Threads) {
                const int e = i >> 5;
                cl16[i] = __half_as_ushort(__float2half_rn(e < T.levels ? T.centroid[e] : 0.0f));
            }
        }
    }
    if (tid == 0) {
        for (int b = 0; b < ring; ++b) {
            mbar_init(&a_full[b], 8);          // one arrival per producer warp
            mbar_init(&a_empty[b], 1);         // MMA commit
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);        // MMA commit
            mbar_init(&acc_empty[a], 4);       // one arrival per epilogue warp
        }
        mbar_init(mma_done, 1);
        fence_barrier_init();
    }
    if (warp == 8) tmem_alloc(tmem_slot, ncols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int64_t tiles_per_g = (T_len + 127) / 128;
    const int64_t items = G * tiles_per_g;
    const int64_t it0 = items * blockIdx.x / gridDim.x, it1 = items * (blockIdx.x + 1) / gridDim.x;
    bool ok = true;

    if (warp < 8) {
        // ------------------------------------------------------------ producers
        const int r = (warp & 3) * 32 + lane;      // token row within the tile
        const int set = warp >> 2;                 // this warp fills the regions g with g % 2 == set
        // Only the bytes of this set's regions: region g < dreg is codes
        // bytes [8 PW g, 8 PW (g+1)), region g >= dreg is sign bytes
        // [8 (g - dreg), 8 (g - dreg + 1)) clipped to m/8.
        auto prefetch = [&](int64_t it, int rb) {
            const int64_t g = it / tiles_per_g, t = (it % tiles_per_g) * 128 + r;
            if (t >= T_len) return;
            const int64_t kt = g * T_len + t;
            uint8_t *R = srec + (size_t)rb * 128 * rowb + (size_t)r * rowb;
            for (int reg = set; reg < nreg; reg += 2) {
                if (TWO && reg < dreg) {
                    const int o0 = reg * 8 * PW;
                    const uint8_t *src = codes + kt * cbytes + o0;
                    if (((uintptr_t)src & 7u) == 0 && ((smem_u32(R + o0)) & 7u) == 0) {
                        for (int o = 0; o < 8 * PW; o += 8) cp_async8(R + o0 + o, src + o);
                    } else {
                        for (int o = 0; o < 8 * PW; o += 4) cp_async4(R + o0 + o, src + o);
                    }
                } else {
                    const int s0 = (reg - dreg) * 8;
                    const int nb = min(8, sbytes - s0);
                    if (nb <= 0) continue;
                    const uint8_t *ssrc = signs + kt * sbytes + s0;
                    uint8_t *S = R + cbytes + s0;
                    if (nb == 8 && ((uintptr_t)ssrc & 7u) == 0 && (smem_u32(S) & 7u) == 0) cp_async8(S, ssrc);
                    else if (nb == 8 && ((uintptr_t)ssrc & 3u) == 0 && (smem_u32(S) & 3u) == 0) { cp_async4(S, ssrc); cp_async4(S + 4, ssrc + 4); }
                    else { for (int o = 0; o < nb; ++o) S[o] = __ldg(ssrc + o); }
                }
            }
        };
        if (it0 < it1) prefetch(it0, 0);
        cp_async_commit();
        if (NREC == 3) {
            if (it0 + 1 < it1) prefetch(it0 + 1, 1);
            cp_async_commit();
        }
        int64_t chunk = 0;
        for (int64_t it = it0; it < it1 && ok; ++it) {
            const int rb = (int)((it - it0) % NREC);
            if constexpr (NREC == 3) {
                asm volatile("cp.async.wait_group 1;" ::: "memory");   // this tile's record is in shared memory
            } else {
                asm volatile("cp.async.wait_group 0;" ::: "memory");
            }
            if (it + NREC - 1 < it1) prefetch(it + NREC - 1, (int)((it + NREC - 1 - it0) % NREC));
            cp_async_commit();
            const int64_t t = (it % tiles_per_g) * 128 + r;
            const bool tv = t < T_len;
            const uint8_t *Rc = srec + (size_t)rb * 128 * rowb + (size_t)r * rowb;
            const uint8_t *Rs = Rc + cbytes;
            for (int c = 0; c < nchunks; ++c, ++chunk) {
                const int b = (int)(chunk % ring);
                const int64_t use = chunk / ring;
                if (use > 0 && ok && !mbar_wait(&a_empty[b], (uint32_t)((use - 1) & 1))) ok = false;
                uint8_t *A = sA + (size_t)b * kSc2ChunkBytes;
                const int c0 = c * kSc2Chunk;
                const int ncol = min(kSc2Chunk, kb - c0);
                for (int rg = set; rg < ncol / 64; rg += 2) {
                    const int gc0 = c0 + 64 * rg;
                    uint8_t *Ar = A + (size_t)rg * 16384 + (size_t)r * 128;
                    if (TWO && gc0 < d) {
                        uint32_t cw[2 * PW];
#pragma unroll
                        for (int q = 0; q < 2 * PW; ++q) cw[q] = 0u;
                        if (tv) {
                            const uint8_t *cp = Rc + gc0 * PW / 8;
#pragma unroll
                            for (int q = 0; q < PW; ++q) {
                                const uint2 v2 = *reinterpret_cast<const uint2 *>(cp + 8 * q);
                                cw[2 * q] = v2.x;
                                cw[2 * q + 1] = v2.y;
                            }
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
                            const uint4 v = tv ? make_uint4(o[0], o[1], o[2], o[3]) : make_uint4(0u, 0u, 0u, 0u);
                            *reinterpret_cast<uint4 *>(Ar + ((k ^ (r & 7)) << 4)) = v;
                        }
                    } else {
                        const int sc0 = gc0 - (TWO ? d : 0);
                        uint32_t sb[2] = {0u, 0u};
                        if (tv) {
                            const uint8_t *sp = Rs + sc0 / 8;
                            const int nbytes = min(8, max(0, (m - sc0) / 8));
                            if (nbytes == 8 && (((uintptr_t)sp) & 7u) == 0) {
                                const uint2 v2 = *reinterpret_cast<const uint2 *>(sp);
                                sb[0] = v2.x;
                                sb[1] = v2.y;
                            } else {
                                for (int bb = 0; bb < nbytes; ++bb) sb[bb >> 2] |= (uint32_t)sp[bb] << (8 * (bb & 3));
                            }
                        }
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const bool live = tv && sc0 + 8 * k < m;
                            const uint32_t byte = (sb[k >> 2] >> (8 * (k & 3))) & 0xffu;
                            const uint4 v = live ? slut[(byte << slc_log2) + slc_lane] : make_uint4(0u, 0u, 0u, 0u);
                            *reinterpret_cast<uint4 *>(Ar + ((k ^ (r & 7)) << 4)) = v;
                        }
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&a_full[b]);
            }
        }
        cp_async_wait_all();
    } else if (warp == 8) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t sA0 = smem_u32(sA), sB0 = smem_u32(sB);
        const uint32_t idesc = idesc_f16(false, 128, nq32);
        int64_t cur_g = -1, chunk = 0;
        uint32_t done_phase = 0;
        bool issued = false;
        for (int64_t it = it0; it < it1 && ok; ++it) {
            const int64_t g = it / tiles_per_g;
            const int a = (int)((it - it0) & 1);
            const int64_t ause = (it - it0) >> 1;
            if (g != cur_g) {
                // all MMAs issued so far must be done before B is overwritten
                if (issued) {
                    if (lane == 0) mma_commit(mma_done);
                    if (ok && !mbar_wait(mma_done, done_phase)) ok = false;
                    done_phase ^= 1u;
                }
                const uint16_t *src = wsB + (int64_t)g * nq * kb;
                for (int idx = lane; idx < nq32 * (kb / 8); idx += 32) {
                    const int row = idx / (kb / 8), c = idx % (kb / 8);
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (row < nq) v = __ldg(reinterpret_cast<const uint4 *>(src + (int64_t)row * kb) + c);
                    *reinterpret_cast<uint4 *>(sB + (size_t)(c >> 3) * nq32 * 128 + sw128_offset(row, c & 7)) = v;
                }
                fence_proxy_async_smem();
                __syncwarp();
                cur_g = g;
            }
            if (ause > 0 && ok && !mbar_wait(&acc_empty[a], (uint32_t)((ause - 1) & 1))) ok = false;
            tc_fence_after();
            for (int c = 0; c < nchunks; ++c, ++chunk) {
                const int b = (int)(chunk % ring);
                if (ok && !mbar_wait(&a_full[b], (uint32_t)((chunk / ring) & 1))) ok = false;
                tc_fence_after();
                const int c0 = c * kSc2Chunk;
                const int ncol = min(kSc2Chunk, kb - c0);
                if (lane == 0 && ok) {
                    for (int rg = 0; rg < ncol / 64; ++rg) {
                        const int greg = c0 / 64 + rg;
                        const bool first = greg < dreg;
                        const uint32_t dcol = (uint32_t)(a * 2 * nq32 + (first ? 0 : nq32));
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint64_t adesc =
                                sdesc_k_sw128(sA0 + (uint32_t)b * kSc2ChunkBytes + (uint32_t)rg * 16384u + k * 32u);
                            const uint64_t bdesc = sdesc_k_sw128(sB0 + (uint32_t)greg * (uint32_t)nq32 * 128u + k * 32u);
                            const bool acc = !(k == 0 && (greg == 0 || greg == dreg));
                            mma_f16(tmem + dcol, adesc, bdesc, idesc, acc ? 1u : 0u);
                        }
                    }
                    mma_commit(&a_empty[b]);
                    if (c == nchunks - 1) mma_commit(&acc_full[a]);
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
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;              // TMEM lanes this warp may read
        const int r = quarter * 32 + lane;         // token row
        const float kq = 1.2533141373155002512f / (float)m;
        int64_t qn_g = -1;
        float qn_reg[4] = {0.0f, 0.0f, 0.0f, 0.0f}; // lane i holds ||q|| of queries i, 32+i, 64+i, 96+i
        for (int64_t it = it0; it < it1 && ok; ++it) {
            const int64_t g = it / tiles_per_g, t = (it % tiles_per_g) * 128 + r;
            const int a = (int)((it - it0) & 1);
            const int64_t ause = (it - it0) >> 1;
            const bool tin = t < T_len;
            const int64_t kt = g * T_len + (tin ? t : 0);
            // loads that do not depend on the accumulator go out before the wait
            const uint16_t skn = tin ? __ldg(sk_norms + kt) : (uint16_t)0;
            const uint16_t n1 = (TWO && tin) ? __ldg(norms + kt) : (uint16_t)0;
            if (g != qn_g) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int qi = 32 * k + lane;
                    qn_reg[k] = qi < nq ? __ldg(wsN + g * nq + qi) : 0.0f;
                }
                qn_g = g;
            }
            if (ok && !mbar_wait(&acc_full[a], (uint32_t)(ause & 1))) ok = false;
            tc_fence_after();
            const bool tv = ok && tin;
            const float a2 = __fmul_rn(kq, h16_to_f32(skn));
            const float a1 = TWO ? __fmul_rn(h16_to_f32(n1), 1.0f / (float)d) : 0.0f;
            const uint32_t col1 = (uint32_t)(a * 2 * nq32), col2 = col1 + (uint32_t)nq32;
            for (int q0 = 0; q0 < nq32; q0 += 32) {
                uint32_t r1[32], r2[32];
                tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + col2 + (uint32_t)q0, r2);
                if (TWO) tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + col1 + (uint32_t)q0, r1);
                tmem_ld_wait();
                const float qn_mine = qn_reg[q0 >> 5];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int qi = q0 + i;
                    const float qn = __shfl_sync(0xffffffffu, qn_mine, i);
                    if (tv && qi < nq) {
                        float sv = __fmul_rn(a2, __uint_as_float(r2[i]));
                        if (TWO) sv = __fmaf_rn(a1, __uint_as_float(r1[i]), sv);
                        scores[((int64_t)g * nq + qi) * T_len + t] = __fmul_rn(sv, qn);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[a]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 8) tmem_dealloc(tmem, ncols);
}

}  // namespace rq
