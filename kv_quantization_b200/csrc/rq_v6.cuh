// rq_v6.cuh -- fused quantize + QJL residual sketch for d = 128 with two lanes
// per block and sixteen warps per CTA (sm_100a).
//
// Arithmetic and tables as in rq_v5.cuh (saturating-grid LUT whose 16-byte
// entries also carry the two candidate centroids).  Lane j of a warp and lane j + 16 own
// the two 64-value halves of one block (values 0..63 and 64..127), each held
// as 32 float2 P[i] = (v_i, v_{i+32}) of its half: Hadamard stages h = 1..16
// are packed f32x2 operations, h = 32 is the add/sub inside each float2 and
// h = 64 exchanges the halves with one shuffle per value (xor 16).  Half the
// values per thread halves the registers and the straight-line code of the
// loop, so sixteen warps fit on an SM and the loop stays in the instruction
// cache.
//
// Two groups of eight warps each run their own 128-block tile ring (3-D TMA
// straight into the tensor-core A layout); a tile's rows are block =
// 16 * warp + (lane mod 16) and its two halves sit in the two 64-column
// regions, so a quarter-warp's 16-byte loads touch eight different bank
// groups.  The residual r' = s * r overwrites the tile in place as the bf16 A
// operand (the sign diagonal is folded into the staged projection S' = S diag(s)),
// the last of the group's eight warps to finish issues the sketch MMA
// (P = R S^T into TMEM), the sign epilogue of a tile runs after the next tile
// is computed, and the group's first warp refills a stage in the middle of the
// next tile, once the MMA that read it has completed.
#pragma once
#include "rq_v5.cuh"

namespace rq {

constexpr int kW6 = 16;                       // warps per CTA
constexpr int kGroups6 = 2;                   // groups of eight warps
constexpr int kNSG6 = 2;                      // tile ring depth per group
constexpr uint32_t kTileBytes6 = 128u * 256u;  // 128 blocks x 2 regions x 128 B

// S (m16 rows x D columns, 16-bit) into the tcgen05 B layout by 2-D TMA, one
// box of min(m16, 256) rows per 64-column region (rows >= m are zero-filled);
// issued by one thread, completion counted on `bar`.
template <int D>
__device__ __forceinline__ void tma_stage_projection(const CUtensorMap *tms, uint8_t *s_S, int m16, uint64_t *bar)
{
    mbar_arrive_expect_tx(bar, (uint32_t)m16 * 128u * (uint32_t)(D / 64));
    for (int kc = 0; kc < D / 64; ++kc)
        for (int r0 = 0; r0 < m16; r0 += 256)
            tma_load_2d(s_S + (size_t)kc * m16 * 128 + (size_t)r0 * 128, tms, 64 * kc, r0, bar);
}

// S' = S diag(s) in place (the sign diagonal folded into the projection's
// columns: a bf16 sign flip is exact, so P = r' S'^T = r S^T bit for bit with
// r' = s * r the residual before its final sign flip): every 16-byte chunk
// (8 columns of one row) XORed with the pair masks of its columns.
template <int D>
__device__ __forceinline__ void sign_fold_projection(uint8_t *s_S, int m16, const uint32_t *pmask)
{
    for (int idx = threadIdx.x; idx < m16 * (D / 8); idx += blockDim.x) {
        const int i = idx / (D / 8), c = idx % (D / 8);
        uint4 *p = reinterpret_cast<uint4 *>(s_S + (size_t)(c >> 3) * m16 * 128 + sw128_offset(i, c & 7));
        const uint4 q = *reinterpret_cast<const uint4 *>(pmask + 4 * c);
        uint4 v = *p;
        v.x ^= q.x; v.y ^= q.y; v.z ^= q.z; v.w ^= q.w;
        *p = v;
    }
}

template <bool BF16, bool SIGNS>
__device__ __forceinline__ void load_half64(uint32_t row_base, int blk, uint32_t pmask_half, float2 *P)
{
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        uint4 a = lds128_fresh(row_base + sw128_offset(blk, k));
        uint4 b = lds128_fresh(row_base + sw128_offset(blk, k + 4));
        if constexpr (SIGNS) {
            const uint4 ma = lds128_fresh(pmask_half + 16u * k);
            const uint4 mb = lds128_fresh(pmask_half + 16u * (k + 4));
            a.x ^= ma.x; a.y ^= ma.y; a.z ^= ma.z; a.w ^= ma.w;
            b.x ^= mb.x; b.y ^= mb.y; b.z ^= mb.z; b.w ^= mb.w;
        }
        const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            P[8 * k + e].x = half_of<BF16>(wa[e >> 1], e & 1);
            P[8 * k + e].y = half_of<BF16>(wb[e >> 1], e & 1);
        }
    }
}

// P <- x - P * sc for the lane's half of the input row (two roundings).
template <bool BF16, bool SIGNS>
__device__ __forceinline__ void residual_half64(uint32_t row_base, int blk, uint32_t pmask_half, float2 sc2,
                                                float2 *P)
{
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        uint4 a = lds128_fresh(row_base + sw128_offset(blk, k));
        uint4 b = lds128_fresh(row_base + sw128_offset(blk, k + 4));
        if constexpr (SIGNS) {
            const uint4 ma = lds128_fresh(pmask_half + 16u * k);
            const uint4 mb = lds128_fresh(pmask_half + 16u * (k + 4));
            a.x ^= ma.x; a.y ^= ma.y; a.z ^= ma.z; a.w ^= ma.w;
            b.x ^= mb.x; b.y ^= mb.y; b.z ^= mb.z; b.w ^= mb.w;
        }
        const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float2 x = make_float2(half_of<BF16>(wa[e >> 1], e & 1), half_of<BF16>(wb[e >> 1], e & 1));
            P[8 * k + e] = sub_mul2_rn(x, P[8 * k + e], sc2);
        }
    }
}

template <bool SIGNS>
__device__ __forceinline__ void store_half64(uint32_t row_base, int blk, uint32_t pmask_half, const float2 *P)
{
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        uint4 a, b;
        a.x = pack2<true>(P[8 * k + 0].x, P[8 * k + 1].x);
        a.y = pack2<true>(P[8 * k + 2].x, P[8 * k + 3].x);
        a.z = pack2<true>(P[8 * k + 4].x, P[8 * k + 5].x);
        a.w = pack2<true>(P[8 * k + 6].x, P[8 * k + 7].x);
        b.x = pack2<true>(P[8 * k + 0].y, P[8 * k + 1].y);
        b.y = pack2<true>(P[8 * k + 2].y, P[8 * k + 3].y);
        b.z = pack2<true>(P[8 * k + 4].y, P[8 * k + 5].y);
        b.w = pack2<true>(P[8 * k + 6].y, P[8 * k + 7].y);
        if constexpr (SIGNS) {
            const uint4 ma = lds128_fresh(pmask_half + 16u * k);
            const uint4 mb = lds128_fresh(pmask_half + 16u * (k + 4));
            a.x ^= ma.x; a.y ^= ma.y; a.z ^= ma.z; a.w ^= ma.w;
            b.x ^= mb.x; b.y ^= mb.y; b.z ^= mb.z; b.w ^= mb.w;
        }
        sts128(row_base + sw128_offset(blk, k), a);
        sts128(row_base + sw128_offset(blk, k + 4), b);
    }
}

// Canonical pairwise sum of squares of the whole block: the lane's 64-value
// part (aligned 8-leaf subtrees), then the parts of the block's LANES lanes
// (lane strides STRIDE, 2*STRIDE, ...: adjacent 64-value parts first).
template <int LANES = 2, int STRIDE = 16>
__device__ __forceinline__ float sumsq_half64(const float2 *P)
{
    float2 t[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float2 s[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) s[i] = __fmul2_rn(P[8 * j + i], P[8 * j + i]);
#pragma unroll
        for (int w = 1; w < 8; w *= 2) {
#pragma unroll
            for (int i = 0; i < 8; i += 2 * w) s[i] = __fadd2_rn(s[i], s[i + w]);
        }
        t[j] = s[0];
    }
    t[0] = __fadd2_rn(t[0], t[1]);
    t[2] = __fadd2_rn(t[2], t[3]);
    t[0] = __fadd2_rn(t[0], t[2]);
    float part = __fadd_rn(t[0].x, t[0].y);
#pragma unroll
    for (int l = 1; l < LANES; l *= 2) part = __fadd_rn(part, __shfl_xor_sync(0xffffffffu, part, STRIDE * l));
    return part;
}

// Stages h = 1..32 in the lane, then h = 64, 128, ... across the block's
// LANES lanes (partner lane ^ STRIDE*l for stage 64*l); `q` = the lane's
// 64-value part index within the block.
template <int LANES = 2, int STRIDE = 16>
__device__ __forceinline__ void fwht_half64(float2 *P, int q)
{
    const float2 m1 = make_float2(-1.0f, -1.0f);
#pragma unroll
    for (int h = 1; h < 32; h *= 2) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (i & h) continue;
            const float2 a = P[i], b = P[i + h];
            P[i] = __fadd2_rn(a, b);
            P[i + h] = __ffma2_rn(b, m1, a);
        }
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) {                      // stage h = 32
        const float a = P[i].x, b = P[i].y;
        P[i].x = __fadd_rn(a, b);
        P[i].y = __fsub_rn(a, b);
    }
#pragma unroll
    for (int l = 1; l < LANES; l *= 2) {                // stages h = 64 l
        const float sg = (q & l) ? -1.0f : 1.0f;
        const float2 sg2 = make_float2(sg, sg);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            float2 o;
            o.x = __shfl_xor_sync(0xffffffffu, P[i].x, STRIDE * l);
            o.y = __shfl_xor_sync(0xffffffffu, P[i].y, STRIDE * l);
            P[i] = __ffma2_rn(P[i], sg2, o);            // lower: mine + other; upper: other - mine
        }
    }
}

// Codes of the lane's 64 values of P * inv (value j of the half at bit j*PW),
// and P replaced by the chosen centroids.
template <int PW>
__device__ __forceinline__ void codes_half64(float2 *P, float inv, const SatGrid &G, uint32_t *w)
{
    const float2 inv2 = make_float2(inv, inv);
#pragma unroll
    for (int k = 0; k < 2 * PW; ++k) w[k] = 0u;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const float2 y = __fmul2_rn(P[i], inv2);
        uint32_t a0, a1;
        sat_addr(G, y, a0, a1);
        const uint4 e0 = lds128(a0), e1 = lds128(a1);
        const bool p0 = y.x > __uint_as_float(e0.x), p1 = y.y > __uint_as_float(e1.x);
        put_code<PW>(w, i, e0.y + (p0 ? 1u : 0u));
        put_code<PW>(w, i + 32, e1.y + (p1 ? 1u : 0u));
        P[i].x = __uint_as_float(p0 ? e0.w : e0.z);
        P[i].y = __uint_as_float(p1 ? e1.w : e1.z);
    }
}

__host__ __device__ inline int qjl_v6_nacc(int m) { return 2 * kGroups6 * qjl_mma_m16(m) <= 512 ? 2 : 1; }

__host__ __device__ inline uint32_t qjl_v6_tmem_cols(int m)
{
    const uint32_t need = (uint32_t)(kGroups6 * qjl_v6_nacc(m) * qjl_mma_m16(m));
    uint32_t c = 32;
    while (c < need) c <<= 1;
    return c;
}

__host__ __device__ inline size_t qjl_v6_smem(int m, const QuantTables &T)
{
    return 1024 + (size_t)qjl_mma_m16(m) * 256 + (size_t)kGroups6 * kNSG6 * kTileBytes6 +
           (size_t)T.sat_cells * 128 + 256 + 8 * (kGroups6 * (2 * kNSG6 + 2) + 1) + 16 + 8 * kGroups6;
}

template <int PW, bool BF16, bool SIGNS>
__global__ void __launch_bounds__(kW6 * 32, 1)
qjl_v6_quant_kernel(const __grid_constant__ CUtensorMap tmx, int64_t nblocks, const __grid_constant__ QuantTables T,
                    uint8_t *__restrict__ codes, uint16_t *__restrict__ norms, int m,
                    const __grid_constant__ CUtensorMap tms, uint8_t *__restrict__ qsigns, uint16_t *__restrict__ qnorms)
{
    constexpr int CB = 16 * PW;                     // code bytes per block
    constexpr int HB = 8 * PW;                      // code bytes per half block
    const int m16 = qjl_mma_m16(m);
    const int nacc = qjl_v6_nacc(m);
    const uint32_t ncols = qjl_v6_tmem_cols(m);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *s_S = base;
    uint8_t *ring = s_S + (size_t)m16 * 256;
    uint8_t *lutb = ring + (size_t)kGroups6 * kNSG6 * kTileBytes6;
    uint32_t *pmask = reinterpret_cast<uint32_t *>(lutb + (size_t)T.sat_cells * 128);
    uint64_t *full = reinterpret_cast<uint64_t *>(pmask + 64);
    uint64_t *mma_done = full + kGroups6 * kNSG6;
    uint64_t *acc_full = mma_done + kGroups6 * kNSG6;
    uint64_t *s_ready = acc_full + kGroups6 * 2;
    uint32_t *ready = reinterpret_cast<uint32_t *>(s_ready + 1);
    uint32_t *tmem_slot = ready + kGroups6;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = warp >> 3, lw = warp & 7;         // group, warp within the group
    const int blk_row = lw * 16 + (lane & 15);      // block within the tile
    const int hf = lane >> 4;                       // which 64-value half
    const int64_t ntiles = (nblocks + 127) / 128;
    const int64_t t0 = ntiles * (int64_t)blockIdx.x / gridDim.x, t1 = ntiles * (int64_t)(blockIdx.x + 1) / gridDim.x;
    auto tile_of = [&](int64_t k) { return t0 + g + 2 * k; };
    auto load_tile = [&](int64_t k) {
        const int slot = g * kNSG6 + (int)(k % kNSG6);
        uint8_t *dst = ring + (size_t)slot * kTileBytes6;
        mbar_arrive_expect_tx(&full[slot], kTileBytes6);
        tma_load_3d(dst, &tmx, 0, 0, (int)(tile_of(k) * 128), &full[slot]);
        tma_load_3d(dst + kTileBytes6 / 2, &tmx, 0, 1, (int)(tile_of(k) * 128), &full[slot]);
    };
    if (threadIdx.x == 0) {
        prefetch_tmap(&tmx);
        for (int i = 0; i < kGroups6 * kNSG6; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&mma_done[i], 1);
        }
        for (int i = 0; i < kGroups6 * 2; ++i) mbar_init(&acc_full[i], 1);
        mbar_init(s_ready, 1);
        for (int i = 0; i < kGroups6; ++i) ready[i] = 0u;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        prefetch_tmap(&tms);
        tma_stage_projection<128>(&tms, s_S, m16, s_ready);
    }
    if (lw == 0 && lane == 0)
        for (int k = 0; k < kNSG6; ++k)
            if (tile_of(k) < t1) load_tile(k);
    setup_sat_lut16(T, reinterpret_cast<uint4 *>(lutb));
    setup_pair_masks(T, pmask, 128);
    if (warp == 0) tmem_alloc(tmem_slot, ncols);
    __syncthreads();                                // masks written
    bool ok = mbar_wait(s_ready, 0u);               // S landed
    if (SIGNS) sign_fold_projection<128>(s_S, m16, pmask);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const SatGrid G = sat_grid(T, smem_u32(lutb), (uint32_t)(lane & 7) * 16u);
    const uint32_t pmh = smem_u32(pmask) + (uint32_t)hf * 128u;
    const uint32_t sS = smem_u32(s_S);
    const int eq = lw & 3, ech = lw >> 2;           // epilogue: TMEM lane quarter, column-chunk parity

    auto epilogue = [&](int64_t kk) {
        const int a = nacc == 2 ? (int)(kk & 1) : 0;
        const uint32_t par = (uint32_t)((nacc == 2 ? kk >> 1 : kk) & 1);
        if (ok && !mbar_wait(&acc_full[g * 2 + a], par)) ok = false;
        tc_fence_after();
        const int64_t blk = tile_of(kk) * 128 + eq * 32 + lane;
        const uint32_t col0 = (uint32_t)((g * nacc + a) * m16);
        uint8_t *dst = qsigns + blk * (m / 8);
        for (int c0 = 32 * ech; c0 < m16; c0 += 64) {
            uint32_t acc[32];
            tmem_ld32(tmem + ((uint32_t)(eq * 32) << 16) + col0 + (uint32_t)c0, acc);
            tmem_ld_wait();
            const uint32_t word = sign_word(acc);
            if (ok && blk < nblocks && c0 < m) {
                const int nb = min(4, (m - c0) / 8);
                if (nb == 4 && (m & 31) == 0) {
                    *reinterpret_cast<uint32_t *>(dst + c0 / 8) = word;
                } else {
                    for (int b = 0; b < nb; ++b) dst[c0 / 8 + b] = (uint8_t)(word >> (8 * b));
                }
            }
        }
        tc_fence_before();
    };

    int64_t k = 0;
    for (;; ++k) {
        const int64_t t = tile_of(k);
        if (t >= t1) break;
        const int slot = g * kNSG6 + (int)(k % kNSG6);
        if (!mbar_wait(&full[slot], (uint32_t)((k / kNSG6) & 1))) { ok = false; break; }
        const uint32_t tile = smem_u32(ring + (size_t)slot * kTileBytes6);
        const uint32_t rbase = tile + (uint32_t)hf * (kTileBytes6 / 2);
        const int64_t blk = t * 128 + blk_row;
        const bool valid = blk < nblocks;

        float2 P[32];
        load_half64<BF16, SIGNS>(rbase, blk_row, pmh, P);
        const float n32 = __fsqrt_rn(sumsq_half64(P));
        fwht_half64(P, hf);
        const float inv = n32 > 0.0f ? __frcp_rn(n32) : 0.0f;
        uint32_t w[2 * PW];
        codes_half64<PW>(P, inv, G, w);
        const uint16_t n16 = norm_to_h16(n32);
        if (valid) {
            store_bytes<HB>(codes + blk * CB + hf * HB, w);
            if (hf == 0) norms[blk] = n16;
        }
        if (lw == 0 && lane == 0 && k >= 1 && ok) {
            const int pslot = g * kNSG6 + (int)((k - 1) % kNSG6);
            if (!mbar_wait(&mma_done[pslot], (uint32_t)(((k - 1) / kNSG6) & 1))) ok = false;
            else if (tile_of(k - 1 + kNSG6) < t1) load_tile(k - 1 + kNSG6);
        }
        fwht_half64(P, hf);
        const float sc = __fmul_rn(h16_to_f32(n16), 1.0f / 128.0f);
        residual_half64<BF16, SIGNS>(rbase, blk_row, pmh, make_float2(sc, sc), P);
        const float rn32 = __fsqrt_rn(sumsq_half64(P));
        if (valid && hf == 0) qnorms[blk] = norm_to_h16(rn32);
        store_half64<false>(rbase, blk_row, pmh, P);     // r' (signs live in S')
        fence_proxy_async_smem();
        if (k >= 1) epilogue(k - 1);
        if (!__all_sync(0xffffffffu, ok)) break;
        if (lane == 0) {
            __threadfence_block();
            const uint32_t old = atomicAdd(&ready[g], 1u);
            if ((old & 7u) == 7u) {                      // last of the eight warps: issue the MMA
                __threadfence_block();
                tc_fence_after();
                const int a = nacc == 2 ? (int)(k & 1) : 0;
                const uint32_t dcol = tmem + (uint32_t)((g * nacc + a) * m16);
#pragma unroll 1
                for (int kc = 0; kc < 2; ++kc) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t adesc =
                            sdesc_k_sw128(tile + (uint32_t)kc * (kTileBytes6 / 2) + (uint32_t)kk * 32u);
                        for (int n0 = 0; n0 < m16; n0 += 256) {
                            const int N = min(256, m16 - n0);
                            const uint64_t bdesc = sdesc_k_sw128(sS + (uint32_t)kc * (uint32_t)m16 * 128u +
                                                                 (uint32_t)n0 * 128u + (uint32_t)kk * 32u);
                            mma_f16(dcol + (uint32_t)n0, adesc, bdesc, idesc_f16(true, 128, N), (kc | kk) != 0);
                        }
                    }
                }
                mma_commit(&mma_done[slot]);
                mma_commit(&acc_full[g * 2 + a]);
            }
        }
        __syncwarp();
    }
    if (k >= 1) epilogue(k - 1);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, ncols);
}

}  // namespace rq
