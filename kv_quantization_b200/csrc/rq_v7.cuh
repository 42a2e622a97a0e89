// rq_v7.cuh -- fused quantize + QJL residual sketch for d = 256 (sm_100a).
//
// The d = 128 kernel of rq_v6.cuh widened to four lanes per block: lanes
// j, j+8, j+16, j+24 of a warp own the four 64-value parts of block j (values
// 64q .. 64q+63 for part q), each as 32 float2 (v_i, v_{i+32}); Hadamard
// stages h = 1..32 run in the lane, h = 64 and h = 128 across lanes (xor 8,
// xor 16), the pairwise norm adds the parts in the same order.  Sixteen warps
// cover one 128-block tile, whose four 64-column regions are the tcgen05 A
// operand (K = 256) after the residual r' = s * r overwrites them in place
// (the sign diagonal is folded into the staged projection, as in rq_v6.cuh).
//
// The projection S (m x 256 bf16) takes up to 128 KB of shared memory, which
// leaves room for one tile: the tile's buffer is refilled as soon as the MMA
// that read it has completed, and the sign epilogue of a tile runs after the
// next tile has been computed (double-buffered TMEM accumulators).
#pragma once
#include "rq_v6.cuh"

namespace rq {

constexpr int kW7 = 16;
constexpr uint32_t kTileBytes7 = 128u * 512u;   // 128 blocks x 4 regions x 128 B

__host__ __device__ inline int qjl_v7_nacc(int m) { return 2 * qjl_mma_m16(m) <= 512 ? 2 : 1; }

__host__ __device__ inline uint32_t qjl_v7_tmem_cols(int m)
{
    const uint32_t need = (uint32_t)(qjl_v7_nacc(m) * qjl_mma_m16(m));
    uint32_t c = 32;
    while (c < need) c <<= 1;
    return c;
}

__host__ __device__ inline size_t qjl_v7_smem(int m, const QuantTables &T)
{
    return 1024 + (size_t)qjl_mma_m16(m) * 512 + kTileBytes7 + (size_t)T.sat_cells * 128 + 512 + 8 * 5 + 16;
}

template <int PW, bool BF16, bool SIGNS>
__global__ void __launch_bounds__(kW7 * 32, 1)
qjl_v7_quant_kernel(const __grid_constant__ CUtensorMap tmx, int64_t nblocks, const __grid_constant__ QuantTables T,
                    uint8_t *__restrict__ codes, uint16_t *__restrict__ norms, int m,
                    const __grid_constant__ CUtensorMap tms, uint8_t *__restrict__ qsigns, uint16_t *__restrict__ qnorms)
{
    constexpr int CB = 32 * PW;                     // code bytes per block
    constexpr int QB = 8 * PW;                      // code bytes per 64-value part
    const int m16 = qjl_mma_m16(m);
    const int nacc = qjl_v7_nacc(m);
    const uint32_t ncols = qjl_v7_tmem_cols(m);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *s_S = base;                                            // 4 regions x m16 rows x 128 B
    uint8_t *tile_b = s_S + (size_t)m16 * 512;
    uint8_t *lutb = tile_b + kTileBytes7;
    uint32_t *pmask = reinterpret_cast<uint32_t *>(lutb + (size_t)T.sat_cells * 128);
    uint64_t *full = reinterpret_cast<uint64_t *>(pmask + 128);
    uint64_t *mma_done = full + 1;
    uint64_t *acc_full = mma_done + 1;                              // [2]
    uint64_t *s_ready = acc_full + 2;
    uint32_t *ready = reinterpret_cast<uint32_t *>(s_ready + 1);
    uint32_t *tmem_slot = ready + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int blk_row = warp * 8 + (lane & 7);      // block within the tile
    const int q = lane >> 3;                        // 64-value part
    const int64_t ntiles = (nblocks + 127) / 128;
    const int64_t t0 = ntiles * (int64_t)blockIdx.x / gridDim.x, t1 = ntiles * (int64_t)(blockIdx.x + 1) / gridDim.x;
    auto load_tile = [&](int64_t t) {
        mbar_arrive_expect_tx(full, kTileBytes7);
        for (int kc = 0; kc < 4; ++kc) tma_load_3d(tile_b + (size_t)kc * 16384, &tmx, 0, kc, (int)(t * 128), full);
    };
    if (threadIdx.x == 0) {
        prefetch_tmap(&tmx);
        mbar_init(full, 1);
        mbar_init(mma_done, 1);
        mbar_init(&acc_full[0], 1);
        mbar_init(&acc_full[1], 1);
        mbar_init(s_ready, 1);
        *ready = 0u;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        prefetch_tmap(&tms);
        tma_stage_projection<256>(&tms, s_S, m16, s_ready);
        if (t0 < t1) load_tile(t0);
    }
    setup_sat_lut16(T, reinterpret_cast<uint4 *>(lutb));
    setup_pair_masks(T, pmask, 256);
    if (warp == 0) tmem_alloc(tmem_slot, ncols);
    __syncthreads();                                // masks written
    bool ok = mbar_wait(s_ready, 0u);               // S landed
    if (SIGNS) sign_fold_projection<256>(s_S, m16, pmask);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const SatGrid G = sat_grid(T, smem_u32(lutb), (uint32_t)(lane & 7) * 16u);
    const uint32_t pmq = smem_u32(pmask) + (uint32_t)q * 128u;
    const uint32_t sS = smem_u32(s_S);
    const uint32_t tile = smem_u32(tile_b);
    const uint32_t rbase = tile + (uint32_t)q * 16384u;
    const int eq = warp & 3, ech = warp >> 2;       // epilogue: TMEM lane quarter, first 32-column chunk

    auto epilogue = [&](int64_t kk) {
        const int a = nacc == 2 ? (int)(kk & 1) : 0;
        const uint32_t par = (uint32_t)((nacc == 2 ? kk >> 1 : kk) & 1);
        if (ok && !mbar_wait(&acc_full[a], par)) ok = false;
        tc_fence_after();
        const int64_t blk = (t0 + kk) * 128 + eq * 32 + lane;
        const uint32_t col0 = (uint32_t)(a * m16);
        uint8_t *dst = qsigns + blk * (m / 8);
        for (int c0 = 32 * ech; c0 < m16; c0 += 128) {
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
        const int64_t t = t0 + k;
        if (t >= t1) break;
        if (!mbar_wait(full, (uint32_t)(k & 1))) { ok = false; break; }
        const int64_t blk = t * 128 + blk_row;
        const bool valid = blk < nblocks;

        float2 P[32];
        load_half64<BF16, SIGNS>(rbase, blk_row, pmq, P);
        const float n32 = __fsqrt_rn(sumsq_half64<4, 8>(P));
        fwht_half64<4, 8>(P, q);
        const float inv = n32 > 0.0f ? __frcp_rn(n32) : 0.0f;
        uint32_t w[2 * PW];
        codes_half64<PW>(P, inv, G, w);
        const uint16_t n16 = norm_to_h16(n32);
        if (valid) {
            store_bytes<QB>(codes + blk * CB + q * QB, w);
            if (q == 0) norms[blk] = n16;
        }
        fwht_half64<4, 8>(P, q);
        const float sc = __fmul_rn(h16_to_f32(n16), 1.0f / 256.0f);
        residual_half64<BF16, SIGNS>(rbase, blk_row, pmq, make_float2(sc, sc), P);
        const float rn32 = __fsqrt_rn(sumsq_half64<4, 8>(P));
        if (valid && q == 0) qnorms[blk] = norm_to_h16(rn32);
        store_half64<false>(rbase, blk_row, pmq, P);     // r' (signs live in S')
        fence_proxy_async_smem();
        if (k >= 1) epilogue(k - 1);
        if (!__all_sync(0xffffffffu, ok)) break;
        if (lane == 0) {
            __threadfence_block();
            const uint32_t old = atomicAdd(ready, 1u);
            if ((old & 15u) == 15u) {                    // last of the sixteen warps: issue the MMA
                __threadfence_block();
                tc_fence_after();
                const int a = nacc == 2 ? (int)(k & 1) : 0;
                const uint32_t dcol = tmem + (uint32_t)(a * m16);
#pragma unroll 1
                for (int kc = 0; kc < 4; ++kc) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t adesc = sdesc_k_sw128(tile + (uint32_t)kc * 16384u + (uint32_t)kk * 32u);
                        for (int n0 = 0; n0 < m16; n0 += 256) {
                            const int N = min(256, m16 - n0);
                            const uint64_t bdesc = sdesc_k_sw128(sS + (uint32_t)kc * (uint32_t)m16 * 128u +
                                                                 (uint32_t)n0 * 128u + (uint32_t)kk * 32u);
                            mma_f16(dcol + (uint32_t)n0, adesc, bdesc, idesc_f16(true, 128, N), (kc | kk) != 0);
                        }
                    }
                }
                mma_commit(mma_done);
                mma_commit(&acc_full[a]);
            }
            if (warp == 0 && ok) {                       // the MMA has read the tile: load the next one
                if (!mbar_wait(mma_done, (uint32_t)(k & 1))) ok = false;
                else if (t + 1 < t1) load_tile(t + 1);
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
