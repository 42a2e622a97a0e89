// rq_v8.cuh -- fused quantize + QJL residual sketch for d = 512 (sm_100a).
//
// The rq_v7.cuh kernel widened to eight lanes per block (lanes j + 4q, q =
// 0..7, of a warp own the eight 64-value parts of block j; Hadamard stages
// h = 64, 128, 256 go across lanes with xor 4, 8, 16).  Sixteen warps take a
// 128-block tile in two passes of 64 blocks; the tile's eight 64-column
// regions (128 KB) become the tcgen05 A operand (K = 512) once the residual
// has overwritten them.
//
// The projection S (up to 512 x 512 bf16 = 512 KB) does not fit in shared
// memory next to the tile, so it is streamed: chunks of up to 256 rows x 64
// columns (32 KB, the B operand of one K-region of one N-half) pass through a
// two-slot ring filled by 2-D TMA; the thread that issues the tile's MMAs
// (the last warp to finish the tile) waits for each chunk, issues its four
// MMAs, commits the slot and refills it.  The accumulator takes up to all 512
// TMEM columns, so the sign epilogue of tile i runs after tile i+1 has been
// computed and before its MMAs are issued; the tile buffer is reloaded once
// the tile's MMAs have read it.  The sign diagonal is applied to the residual
// (r = s * r') before it is stored, since S is not staged as a whole.
#pragma once
#include "rq_v7.cuh"

namespace rq {

constexpr int kW8 = 16;
constexpr uint32_t kTileBytes8 = 128u * 1024u;  // 128 blocks x 8 regions x 128 B
constexpr uint32_t kSChunk8 = 256u * 128u;      // 256 S rows x 64 columns

__host__ __device__ inline int qjl_v8_nchunk_rows(int m) { return qjl_mma_m16(m) < 256 ? qjl_mma_m16(m) : 256; }

__host__ __device__ inline uint32_t qjl_v8_tmem_cols(int m)
{
    const uint32_t need = (uint32_t)qjl_mma_m16(m);
    uint32_t c = 32;
    while (c < need) c <<= 1;
    return c;
}

__host__ __device__ inline size_t qjl_v8_smem(const QuantTables &T)
{
    return 1024 + kTileBytes8 + 2 * (size_t)kSChunk8 + (size_t)T.sat_cells * 128 + 1024 + 8 * 7 + 16;
}

template <int PW, bool BF16, bool SIGNS>
__global__ void __launch_bounds__(kW8 * 32, 1)
qjl_v8_quant_kernel(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tms, int64_t nblocks,
                    const __grid_constant__ QuantTables T, uint8_t *__restrict__ codes, uint16_t *__restrict__ norms,
                    int m, uint8_t *__restrict__ qsigns, uint16_t *__restrict__ qnorms)
{
    constexpr int CB = 64 * PW;                     // code bytes per block
    constexpr int QB = 8 * PW;                      // code bytes per 64-value part
    const int m16 = qjl_mma_m16(m);
    const int crow = qjl_v8_nchunk_rows(m);         // S rows per chunk (the TMA box)
    const int nhalf = (m16 + 255) / 256;            // N pieces of at most 256 columns
    const int nchunk = nhalf * 8;                   // S chunks per tile
    const uint32_t ncols = qjl_v8_tmem_cols(m);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *tile_b = base;                                         // 8 regions x 128 rows x 128 B
    uint8_t *sring = tile_b + kTileBytes8;                          // 2 S chunks
    uint8_t *lutb = sring + 2 * kSChunk8;
    uint32_t *pmask = reinterpret_cast<uint32_t *>(lutb + (size_t)T.sat_cells * 128);
    uint64_t *full = reinterpret_cast<uint64_t *>(pmask + 256);
    uint64_t *mma_done = full + 1;
    uint64_t *acc_full = mma_done + 1;
    uint64_t *s_full = acc_full + 1;                                // [2]
    uint64_t *s_empty = s_full + 2;                                 // [2]
    uint32_t *ready = reinterpret_cast<uint32_t *>(s_empty + 2);
    uint32_t *tmem_slot = ready + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = lane >> 2;                        // 64-value part
    const int64_t ntiles = (nblocks + 127) / 128;
    const int64_t t0 = ntiles * (int64_t)blockIdx.x / gridDim.x, t1 = ntiles * (int64_t)(blockIdx.x + 1) / gridDim.x;
    auto load_tile = [&](int64_t t) {
        mbar_arrive_expect_tx(full, kTileBytes8);
        for (int kc = 0; kc < 8; ++kc) tma_load_3d(tile_b + (size_t)kc * 16384, &tmx, 0, kc, (int)(t * 128), full);
    };
    // S chunk c: N piece c / 8 (rows 256 (c / 8) ...), K region c % 8
    auto load_s = [&](int c, int slot) {
        mbar_arrive_expect_tx(&s_full[slot], (uint32_t)crow * 128u);
        tma_load_2d(sring + (size_t)slot * kSChunk8, &tms, 64 * (c % 8), 256 * (c / 8), &s_full[slot]);
    };
    if (threadIdx.x == 0) {
        prefetch_tmap(&tmx);
        prefetch_tmap(&tms);
        mbar_init(full, 1);
        mbar_init(mma_done, 1);
        mbar_init(acc_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_empty[i], 1);
        }
        *ready = 0u;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && t0 < t1) {
        load_tile(t0);
        load_s(0, 0);
        if (nchunk > 1) load_s(1, 1);
    }
    setup_sat_lut16(T, reinterpret_cast<uint4 *>(lutb));
    setup_pair_masks(T, pmask, 512);
    if (warp == 0) tmem_alloc(tmem_slot, ncols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const SatGrid G = sat_grid(T, smem_u32(lutb), (uint32_t)(lane & 7) * 16u);
    const uint32_t pmq = smem_u32(pmask) + (uint32_t)q * 128u;
    const uint32_t tile = smem_u32(tile_b);
    const uint32_t sring_a = smem_u32(sring);
    const uint32_t rbase = tile + (uint32_t)q * 16384u;
    const int eq = warp & 3, ech = warp >> 2;       // epilogue: TMEM lane quarter, first 32-column chunk
    bool ok = true;

    auto epilogue = [&](int64_t kk) {
        if (ok && !mbar_wait(acc_full, (uint32_t)(kk & 1))) ok = false;
        tc_fence_after();
        const int64_t blk = (t0 + kk) * 128 + eq * 32 + lane;
        uint8_t *dst = qsigns + blk * (m / 8);
        for (int c0 = 32 * ech; c0 < m16; c0 += 128) {
            uint32_t acc[32];
            tmem_ld32(tmem + ((uint32_t)(eq * 32) << 16) + (uint32_t)c0, acc);
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
#pragma unroll 1
        for (int pass = 0; pass < 2; ++pass) {
            const int blk_row = pass * 64 + warp * 4 + (lane & 3);
            const int64_t blk = t * 128 + blk_row;
            const bool valid = blk < nblocks;
            float2 P[32];
            load_half64<BF16, SIGNS>(rbase, blk_row, pmq, P);
            const float n32 = __fsqrt_rn(sumsq_half64<8, 4>(P));
            fwht_half64<8, 4>(P, q);
            const float inv = n32 > 0.0f ? __frcp_rn(n32) : 0.0f;
            uint32_t w[2 * PW];
            codes_half64<PW>(P, inv, G, w);
            const uint16_t n16 = norm_to_h16(n32);
            if (valid) {
                store_bytes<QB>(codes + blk * CB + q * QB, w);
                if (q == 0) norms[blk] = n16;
            }
            fwht_half64<8, 4>(P, q);
            const float sc = __fmul_rn(h16_to_f32(n16), 1.0f / 512.0f);
            residual_half64<BF16, SIGNS>(rbase, blk_row, pmq, make_float2(sc, sc), P);
            const float rn32 = __fsqrt_rn(sumsq_half64<8, 4>(P));
            if (valid && q == 0) qnorms[blk] = norm_to_h16(rn32);
            store_half64<SIGNS>(rbase, blk_row, pmq, P);
        }
        fence_proxy_async_smem();
        if (k >= 1) epilogue(k - 1);
        if (!__all_sync(0xffffffffu, ok)) break;
        if (lane == 0) {
            __threadfence_block();
            const uint32_t old = atomicAdd(ready, 1u);
            if ((old & 15u) == 15u) {                    // last of the sixteen warps: issue the tile's MMAs
                __threadfence_block();
                tc_fence_after();
                // global S chunk u = k * nchunk + c uses slot u % 2 for the (u / 2)-th time; after
                // issuing chunk u, wait for chunk u - 1's MMAs and refill its slot with chunk u + 1
                const int64_t total = (t1 - t0) * (int64_t)nchunk;
                for (int c = 0; c < nchunk && ok; ++c) {
                    const int64_t u = k * (int64_t)nchunk + c;
                    const int slot = (int)(u & 1);
                    if (!mbar_wait(&s_full[slot], (uint32_t)((u >> 1) & 1))) { ok = false; break; }
                    tc_fence_after();
                    const int kc = c % 8, n0 = 256 * (c / 8);
                    const int N = min(256, m16 - n0);
                    const uint32_t sb = sring_a + (uint32_t)slot * kSChunk8;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t adesc = sdesc_k_sw128(tile + (uint32_t)kc * 16384u + (uint32_t)kk * 32u);
                        const uint64_t bdesc = sdesc_k_sw128(sb + (uint32_t)kk * 32u);
                        mma_f16(tmem + (uint32_t)n0, adesc, bdesc, idesc_f16(true, 128, N), (kc | kk) != 0);
                    }
                    mma_commit(&s_empty[slot]);
                    if (u >= 1 && u + 1 < total) {
                        const int64_t up = u - 1;
                        if (!mbar_wait(&s_empty[up & 1], (uint32_t)((up >> 1) & 1))) { ok = false; break; }
                        load_s((int)((u + 1) % nchunk), (int)(up & 1));
                    }
                }
                mma_commit(mma_done);
                mma_commit(acc_full);
            }
        }
        __syncwarp();
        if (warp == 0 && lane == 0 && ok) {          // the MMAs have read the tile: load the next one
            if (!mbar_wait(mma_done, (uint32_t)(k & 1))) ok = false;
            else if (t + 1 < t1) load_tile(t + 1);
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
