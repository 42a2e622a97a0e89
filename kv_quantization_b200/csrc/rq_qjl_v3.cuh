// rq_qjl_v3.cuh -- fused quantize + QJL residual sketch, in place (sm_100a).
//
// The 128-block tile is loaded by 3-D TMA ({64 values, d/64 regions, blocks},
// 128-byte swizzle) straight into the tensor-core A layout: region k holds
// values [64k, 64k+64) of the 128 blocks, one 128-byte row per block.  Each
// of the 256 threads owns one such row (block tid/TPB, region tid%TPB; d = 256
// runs two sub-passes of 64 blocks), reads it, quantizes it exactly as
// quantize_v2_kernel does (codes and fp16 norms to global memory), rebuilds
// the fp32 reconstruction, and overwrites its own row with bf16 of the
// residual r = x - x^32 (the canonical residual; sign applied on the packed
// pair).  The tile is then the A operand of the sketch MMA P = R S^T (S, m x d
// bf16, resident in shared memory), issued by one thread into TMEM; the
// sign-packing epilogue of tile i runs after the threads have processed tile
// i+1, and the stage of tile i returns to the TMA ring once its MMA is done.
#pragma once
#include "rq_qjl_v2.cuh"

namespace rq {

__host__ __device__ inline size_t qjl_v3_smem(int D, int pw, int m, const QuantTables &T, int stages)
{
    size_t b = 1024;
    b += (size_t)qjl_mma_m16(m) * D * 2;                           // S, D/64 regions of m16 rows
    b += (size_t)stages * 128 * D * 2;                             // A ring (input, then residual)
    b += lut_bytes_v2(T) + ((size_t)1 << pw) * 32 * 4 + (size_t)D / 2 * 4;
    return b + 8 * (stages + 2) + 16;
}

template <int D>
__device__ __forceinline__ void stage_projection_d(const uint16_t *__restrict__ proj, uint8_t *s_S, int m, int m16)
{
    for (int idx = threadIdx.x; idx < m16 * (D / 8); idx += blockDim.x) {
        const int i = idx / (D / 8), c = idx % (D / 8);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (i < m) v = __ldg(reinterpret_cast<const uint4 *>(proj + (size_t)i * D) + c);
        *reinterpret_cast<uint4 *>(s_S + (size_t)(c >> 3) * m16 * 128 + sw128_offset(i, c & 7)) = v;
    }
}

template <int D, int PW, bool BF16, int NS>
__global__ void __launch_bounds__(kT2, 1)
qjl_v3_quant_kernel(const __grid_constant__ CUtensorMap tmv, int64_t nblocks, const __grid_constant__ QuantTables T,
                    uint8_t *__restrict__ codes, uint16_t *__restrict__ norms, int m,
                    const uint16_t *__restrict__ proj, uint8_t *__restrict__ qsigns, uint16_t *__restrict__ qnorms)
{
    constexpr int TPB = D / kE2;                  // threads (regions) per block
    constexpr int KC = D / 64;
    constexpr int SUB = TPB / 2;                  // sub-passes per 128-block tile (256 threads)
    constexpr int TOK_SUB = kT2 / TPB;            // blocks per sub-pass
    constexpr int CB = kE2 * PW / 8;
    constexpr int NW = kE2 * PW / 32;
    constexpr uint32_t STAGE_BYTES = 128u * D * 2u;
    const int m16 = qjl_mma_m16(m);
    const uint32_t ncols = qjl_v2_tmem_cols(m);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *s_S = base;
    uint8_t *ring = s_S + (size_t)m16 * D * 2;
    uint8_t *lutb = ring + (size_t)NS * STAGE_BYTES;
    float *bnd = reinterpret_cast<float *>(lutb);
    float *cent = reinterpret_cast<float *>(lutb + lut_bytes_v2(T));
    uint32_t *pmask = reinterpret_cast<uint32_t *>(cent + (1 << PW) * 32);
    uint64_t *full = reinterpret_cast<uint64_t *>(pmask + D / 2);
    uint64_t *mma_bar = full + NS;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_bar + 2);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, part = tid % TPB;
    const int64_t ntiles = (nblocks + 127) / 128;
    auto load_tile = [&](int64_t t, int s) {
        mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
        for (int kc = 0; kc < KC; ++kc)
            tma_load_3d(ring + (size_t)s * STAGE_BYTES + (size_t)kc * 16384, &tmv, 0, kc, (int)(t * 128), &full[s]);
    };
    if (tid == 0) {
        prefetch_tmap(&tmv);
        for (int s = 0; s < NS; ++s) mbar_init(&full[s], 1);
        mbar_init(&mma_bar[0], 1);
        mbar_init(&mma_bar[1], 1);
        fence_barrier_init();
        for (int s = 0; s < NS; ++s) {
            const int64_t t = blockIdx.x + (int64_t)s * gridDim.x;
            if (t < ntiles) load_tile(t, s);
        }
    }
    stage_projection_d<D>(proj, s_S, m, m16);
    setup_lut_v2(T, reinterpret_cast<uint2 *>(lutb), bnd);
    for (int i = tid; i < (1 << PW) * 32; i += kT2) {
        const int k = i >> 5;
        cent[i] = k < T.levels ? T.centroid[k] : 0.0f;
    }
    setup_pair_masks(T, pmask, D);
    if (warp == 0) tmem_alloc(tmem_slot, ncols);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t sS = smem_u32(s_S), sR = smem_u32(ring);

    const float2 la = make_float2(T.lut_a, T.lut_a), lb = make_float2(T.lut_b, T.lut_b);
    const int cells = T.lut_cells, levels = T.levels;
    const uint32_t cells_m1 = (uint32_t)(cells > 0 ? cells - 1 : 0);
    const uint8_t *lut_lane = lutb + (lane & 15) * 8;
    const float *cent_lane = cent + lane;
    const uint4 *pmv = reinterpret_cast<const uint4 *>(pmask + part * 32);
    bool ok = true;
    uint32_t mma_phase[2] = {0u, 0u};
    int64_t i = 0;

    // sign epilogue + stage recycling of the tile processed `lag` iterations ago
    auto retire = [&](int64_t j) {
        const int a = (int)(j & 1);
        if (ok && !mbar_wait(&mma_bar[a], mma_phase[a])) ok = false;
        mma_phase[a] ^= 1u;
        tc_fence_after();
        const int64_t tj = blockIdx.x + j * (int64_t)gridDim.x;
        qjl_v2_epilogue(tmem, (uint32_t)(a * m16), m, m16, tj * 128, nblocks, qsigns, ok);
        tc_fence_before();
        if (tid == 0 && ok) {                         // stage of tile j is free again
            const int64_t tn = tj + (int64_t)NS * gridDim.x;
            if (tn < ntiles) load_tile(tn, (int)(j % NS));
        }
    };

    for (;; ++i) {
        const int64_t t = blockIdx.x + i * gridDim.x;
        if (t >= ntiles) break;
        if (NS == 1 && i >= 1) retire(i - 1);              // single stage: refill before the next wait
        const int s = (int)(i % NS);
        const bool got = mbar_wait(&full[s], (uint32_t)((i / NS) & 1));
        if (__syncthreads_or(!got)) { ok = false; break; }
        uint8_t *stage = ring + (size_t)s * STAGE_BYTES;
#pragma unroll 1
        for (int sp = 0; sp < SUB; ++sp) {
            const int blk = sp * TOK_SUB + tid / TPB;            // block within the tile
            const int64_t gblk = t * 128 + blk;
            const bool valid = gblk < nblocks;
            uint8_t *rowp = stage + (size_t)part * 16384 + (size_t)blk * 128;
            uint32_t u[32];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint4 v = *reinterpret_cast<const uint4 *>(rowp + ((k ^ (blk & 7)) << 4));
                const uint4 q = pmv[k];
                u[4 * k] = v.x ^ q.x; u[4 * k + 1] = v.y ^ q.y; u[4 * k + 2] = v.z ^ q.z; u[4 * k + 3] = v.w ^ q.w;
            }
            float2 P[32];
            row_to_pairs<BF16>(u, P);
            const float n32 = __fsqrt_rn(combine_parts<TPB>(row_sumsq(P)));
            fwht_row<TPB>(P, part);
            const float inv = n32 > 0.0f ? __frcp_rn(n32) : 0.0f;
            const float2 inv2 = make_float2(inv, inv);
            uint32_t w[NW];
#pragma unroll
            for (int k = 0; k < NW; ++k) w[k] = 0u;
#pragma unroll
            for (int i2 = 0; i2 < 32; ++i2) {
                const float2 y = __fmul2_rn(P[i2], inv2);
                uint32_t c0, c1;
                if (cells > 0) {
                    const float2 f = __ffma2_rn(y, la, lb);
                    c0 = lut_code_v2(y.x, f.x, lut_lane, cells_m1);
                    c1 = lut_code_v2(y.y, f.y, lut_lane, cells_m1);
                } else {
                    c0 = bsearch_code(y.x, bnd, levels);
                    c1 = bsearch_code(y.y, bnd, levels);
                }
                const int b0 = i2 * PW, b1 = (i2 + 32) * PW;
                w[b0 >> 5] |= c0 << (b0 & 31);
                if ((b0 & 31) + PW > 32) w[(b0 >> 5) + 1] |= c0 >> (32 - (b0 & 31));
                w[b1 >> 5] |= c1 << (b1 & 31);
                if ((b1 & 31) + PW > 32) w[(b1 >> 5) + 1] |= c1 >> (32 - (b1 & 31));
            }
            const uint16_t n16 = norm_to_h16(n32);
            const int64_t grow = gblk * TPB + part;             // global 64-value row
            if (valid) {
                store_bytes<CB>(codes + grow * CB, w);
                if (part == 0) norms[gblk] = n16;
            }
            // residual r' = s*x - w*scale (canonical fp32), r = s * r'
#pragma unroll
            for (int i2 = 0; i2 < 32; ++i2) {
                P[i2].x = cent_lane[unpack_code<kE2, PW>(w, i2) * 32];
                P[i2].y = cent_lane[unpack_code<kE2, PW>(w, i2 + 32) * 32];
            }
            fwht_row<TPB>(P, part);
            const float sc = __fmul_rn(h16_to_f32(n16), 1.0f / (float)D);
            const float2 sc2 = make_float2(sc, sc);
#pragma unroll
            for (int i2 = 0; i2 < 32; ++i2) {
                float2 x;
                x.x = half_of<BF16>(u[i2 >> 1], i2 & 1);
                x.y = half_of<BF16>(u[16 + (i2 >> 1)], i2 & 1);
                P[i2] = sub_mul2_rn(x, P[i2], sc2);
            }
            const float rn32 = __fsqrt_rn(combine_parts<TPB>(row_sumsq(P)));
            if (valid && part == 0) qnorms[gblk] = norm_to_h16(rn32);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                uint32_t o[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int wd = 4 * k + q;
                    const float va = wd < 16 ? P[2 * wd].x : P[2 * wd - 32].y;
                    const float vb = wd < 16 ? P[2 * wd + 1].x : P[2 * wd - 31].y;
                    o[q] = pack2<true>(va, vb);
                }
                const uint4 q = pmv[k];
                *reinterpret_cast<uint4 *>(rowp + ((k ^ (blk & 7)) << 4)) =
                    make_uint4(o[0] ^ q.x, o[1] ^ q.y, o[2] ^ q.z, o[3] ^ q.w);
            }
        }
        // the previous tile's MMA has had this tile's compute time to finish
        if (NS > 1 && i >= 1) retire(i - 1);
        fence_proxy_async_smem();
        tc_fence_before();
        if (!__syncthreads_and(ok)) { ok = false; break; }
        if (tid == 0) {
            tc_fence_after();
            const int a = (int)(i & 1);
            const uint32_t sA = sR + (uint32_t)s * STAGE_BYTES;
#pragma unroll 1
            for (int kc = 0; kc < KC; ++kc) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint64_t adesc = sdesc_k_sw128(sA + (uint32_t)kc * 16384u + (uint32_t)k * 32u);
                    for (int n0 = 0; n0 < m16; n0 += 256) {
                        const int N = min(256, m16 - n0);
                        const uint64_t bdesc = sdesc_k_sw128(sS + (uint32_t)kc * (uint32_t)m16 * 128u +
                                                             (uint32_t)n0 * 128u + (uint32_t)k * 32u);
                        mma_f16(tmem + (uint32_t)(a * m16 + n0), adesc, bdesc, idesc_f16(true, 128, N), (kc | k) != 0);
                    }
                }
            }
            mma_commit(&mma_bar[a]);
        }
    }
    if (i >= 1) retire(i - 1);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, ncols);
}

}  // namespace rq
