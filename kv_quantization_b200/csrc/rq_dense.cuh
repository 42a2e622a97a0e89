// rq_dense.cuh -- quantization with a dense orthogonal rotation Pi for blocks
// of d = 128 (sm_100a, tcgen05).
//
// TurboQuant README, "Algorithm in one paragraph": store ||x||, rotate x / ||x||
// by a fixed random orthogonal Pi, bucketize each coordinate against the
// Lloyd-Max centroids of the coordinate law of a uniform unit vector (the Beta
// law, rq_beta_lloyd_max), pack; inverse x^ = ||x|| Pi^T c.  The rotation is a
// dense 128 x 128 contraction per block, so it runs on the tensor cores:
//
// quantize (14 warps, one CTA per SM over a strided run of 128-block tiles)
//   warp 0    TMA: each tile of 128 blocks straight into the K-major A layout
//             (two 64-column regions, 128-byte swizzle), a ring of NS stages;
//   warp 1    MMA: Y = X Pi^T (M = 128 blocks, N = 128 coordinates, K = 128,
//             kind::f16 with fp32 accumulation) into one of two TMEM buffers;
//   warps 2-5 norms: thread = block, the canonical fp32 pairwise norm from
//             the stage; the fp16 norm to global, n32 to shared memory for
//             the epilogue;
//   warps 6-13 epilogue: TMEM lane quarter (warp mod 4) = 32 blocks, two of
//             the four 32-column chunks each: z = y * fl32(1 / n32), code =
//             #{t_k < z} (saturating-grid table, else binary search), packed
//             LSB-first and stored.
// dequantize (13 warps)
//   warps 0-3 producers: thread = block, its codes -> 16-bit centroid pairs
//             (a table of packed pairs for codes of up to 4 bits) written as
//             the K-major A operand C of the tile;
//   warp 4    MMA: X^ = C Pi (B = Pi read MN-major: row j of Pi is K step j,
//             its columns the 128 outputs) into one of two TMEM buffers;
//   warps 5-12 epilogue: x^ = acc * n16, rounded to the output dtype, staged
//             in the swizzled output layout, stored by TMA.
// Pi stays in shared memory for the CTA's whole run.  Every wait is bounded
// (mbar_wait); an expired wait sets the device error word and the roles stop.
#pragma once
#include <cuda.h>

#include "rq_qjl_v2.cuh"
#include "rq_sketch_v3.cuh"
#include "rq_v5.cuh"

namespace rq {

constexpr int kDnQWarps = 14;
constexpr int kDnDWarps = 13;
constexpr uint32_t kDnTile = 128u * 128u * 2u;            // one 128 x 128 16-bit operand tile

// Shared-memory descriptor of a 128-byte-swizzled operand with explicit
// leading (between 64-element MN atoms) and stride (between 8-row groups)
// byte offsets; sm_100 descriptor version bit 46, swizzle mode 2 (128 B).
__device__ __forceinline__ uint64_t dense_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3ffffu) >> 4);
    d |= (uint64_t)((lbo >> 4) & 0x3fffu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3fffu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

__device__ __forceinline__ void named_barrier_sync(int id, int threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__host__ __device__ inline size_t quantize_dense_smem(int stages, int lut_cells)
{
    return 1024 + kDnTile + (size_t)stages * kDnTile + 2 * 128 * 4 + 1024 + (size_t)lut_cells * 128 +
           8 * (2 * stages + 8) + 16;
}

template <bool BF16, int PW, int NS>
__global__ void __launch_bounds__(kDnQWarps * 32, 1)
quantize_dense_kernel(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmp, int64_t nvec,
                      const __grid_constant__ QuantTables T, uint8_t *__restrict__ codes,
                      uint16_t *__restrict__ norms)
{
    constexpr int CB = 16 * PW;                             // code bytes per block
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *s_P = base;                                    // Pi: 2 regions x 128 rows x 128 B
    uint8_t *ring = s_P + kDnTile;
    float *nrm = reinterpret_cast<float *>(ring + (size_t)NS * kDnTile);      // [2][128]
    float *bnd = nrm + 256;                                                   // [256]
    uint2 *lut = reinterpret_cast<uint2 *>(bnd + 256);                        // sat_cells x 16
    uint64_t *stage_full = reinterpret_cast<uint64_t *>(lut + (size_t)T.sat_cells * 16);
    uint64_t *stage_free = stage_full + NS;
    uint64_t *p_ready = stage_free + NS;
    uint64_t *acc_full = p_ready + 2;
    uint64_t *acc_free = acc_full + 2;
    uint64_t *norm_full = acc_free + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(norm_full + 2);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t ntiles = (nvec + 127) / 128;
    const int64_t my_tiles = blockIdx.x < ntiles ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    for (int i = tid; i < 256; i += blockDim.x) bnd[i] = i < T.levels - 1 ? T.bound[i] : INFINITY;
    const bool sat = T.sat_cells > 0;
    if (sat) setup_sat_lut8(T, lut);
    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&stage_full[s], 1);
            mbar_init(&stage_free[s], 5);                   // 4 norm warps + 1 MMA commit
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_free[a], 8);                     // 8 epilogue warps
            mbar_init(&norm_full[a], 4);                    // 4 norm warps
        }
        mbar_init(&p_ready[0], 1);
        fence_barrier_init();
        prefetch_tmap(&tmx);
        prefetch_tmap(&tmp);
        mbar_arrive_expect_tx(&p_ready[0], kDnTile);
        for (int kc = 0; kc < 2; ++kc) tma_load_2d(s_P + (size_t)kc * 16384, &tmp, 64 * kc, 0, &p_ready[0]);
    }
    if (warp == 1) tmem_alloc(tmem_slot, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            for (int64_t i = 0; i < my_tiles && ok; ++i) {
                const int s = (int)(i % NS);
                const int64_t use = i / NS;
                if (use > 0 && !mbar_wait(&stage_free[s], (uint32_t)((use - 1) & 1))) { ok = false; break; }
                const int64_t t = blockIdx.x + i * gridDim.x;
                mbar_arrive_expect_tx(&stage_full[s], kDnTile);
                tma_load_3d(ring + (size_t)s * kDnTile, &tmx, 0, 0, (int)(t * 128), &stage_full[s]);
                tma_load_3d(ring + (size_t)s * kDnTile + 16384, &tmx, 0, 1, (int)(t * 128), &stage_full[s]);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer: Y = X Pi^T
        if (!mbar_wait(&p_ready[0], 0u)) ok = false;
        const uint32_t sP = smem_u32(s_P), sR = smem_u32(ring);
        const uint32_t idesc = idesc_f16(BF16, 128, 128);
        for (int64_t i = 0; i < my_tiles && ok; ++i) {
            const int s = (int)(i % NS);
            const int a = (int)(i & 1);
            const int64_t ause = i >> 1;
            if (ause > 0 && !mbar_wait(&acc_free[a], (uint32_t)((ause - 1) & 1))) { ok = false; break; }
            if (!mbar_wait(&stage_full[s], (uint32_t)((i / NS) & 1))) { ok = false; break; }
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int kc = 0; kc < 2; ++kc)
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint64_t adesc = sdesc_k_sw128(sR + (uint32_t)s * kDnTile + (uint32_t)kc * 16384u + k * 32u);
                        const uint64_t bdesc = sdesc_k_sw128(sP + (uint32_t)kc * 16384u + k * 32u);
                        mma_f16(tmem + (uint32_t)(a * 128), adesc, bdesc, idesc, (kc | k) != 0);
                    }
                mma_commit(&stage_free[s]);                 // operand reads done -> one of the 5 arrivals
                mma_commit(&acc_full[a]);
            }
            __syncwarp();
        }
    } else if (warp < 6) {
        // ------------------------------------------------------------ norms
        const int r = tid - 64;                             // block within the tile
        for (int64_t i = 0; i < my_tiles && ok; ++i) {
            const int s = (int)(i % NS);
            const int a = (int)(i & 1);
            if (!mbar_wait(&stage_full[s], (uint32_t)((i / NS) & 1))) { ok = false; break; }
            const uint8_t *A = ring + (size_t)s * kDnTile;
            float sums[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t u[32];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint4 v = lds128_fresh(smem_u32(A + h * 16384 + sw128_offset(r, k)));   // TMA-written
                    u[4 * k] = v.x; u[4 * k + 1] = v.y; u[4 * k + 2] = v.z; u[4 * k + 3] = v.w;
                }
                float2 P[32];
                row_to_pairs<BF16>(u, P);
                sums[h] = row_sumsq(P);
            }
            const float n32 = __fsqrt_rn(__fadd_rn(sums[0], sums[1]));
            __syncwarp();
            if (lane == 0) mbar_arrive_cta(&stage_free[s]);
            // the epilogue of tile i - 2 has finished reading this buffer's norms
            if (i >= 2 && !mbar_wait(&acc_free[a], (uint32_t)(((i >> 1) - 1) & 1))) { ok = false; break; }
            nrm[a * 128 + r] = n32;
            __syncwarp();
            if (lane == 0) mbar_arrive_cta(&norm_full[a]);
            const int64_t tok = (blockIdx.x + i * gridDim.x) * 128 + r;
            if (tok < nvec) norms[tok] = norm_to_h16(n32);
        }
    } else {
        // ------------------------------------------------------------ epilogue: codes
        const int quarter = warp & 3;
        const int part = (warp - 6) >> 2;                   // chunks 2 part, 2 part + 1
        const SatGrid SG = sat_grid(T, smem_u32(lut), (uint32_t)(lane & 15) * 8u);
        for (int64_t i = 0; i < my_tiles && ok; ++i) {
            const int a = (int)(i & 1);
            if (!mbar_wait(&acc_full[a], (uint32_t)((i >> 1) & 1))) { ok = false; break; }
            if (!mbar_wait(&norm_full[a], (uint32_t)((i >> 1) & 1))) { ok = false; break; }
            tc_fence_after();
            const int row = quarter * 32 + lane;
            const int64_t tok = (blockIdx.x + i * gridDim.x) * 128 + row;
            const float n32 = *reinterpret_cast<volatile float *>(&nrm[a * 128 + row]);
            const float inv = n32 > 0.0f ? __frcp_rn(n32) : 0.0f;
            const float2 inv2 = make_float2(inv, inv);
            uint32_t acc[2][32];
#pragma unroll
            for (int q = 0; q < 2; ++q)
                tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(a * 128 + 32 * (2 * part + q)), acc[q]);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cta(&acc_free[a]);   // accumulator (and the norms) consumed
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                uint32_t w[PW];
#pragma unroll
                for (int k = 0; k < PW; ++k) w[k] = 0u;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float2 z = __fmul2_rn(make_float2(__uint_as_float(acc[q][2 * j]), __uint_as_float(acc[q][2 * j + 1])),
                                                inv2);
                    if (sat) {
                        uint32_t a0, a1;
                        sat_addr(SG, z, a0, a1);
                        const uint2 e0 = lds64(a0), e1 = lds64(a1);
                        put_code_cmp<PW>(w, 2 * j, e0.y, z.x, __uint_as_float(e0.x));
                        put_code_cmp<PW>(w, 2 * j + 1, e1.y, z.y, __uint_as_float(e1.x));
                    } else {
                        put_code<PW>(w, 2 * j, bsearch_code(z.x, bnd, T.levels));
                        put_code<PW>(w, 2 * j + 1, bsearch_code(z.y, bnd, T.levels));
                    }
                }
                if (tok < nvec) store_bytes<4 * PW>(codes + tok * CB + (2 * part + q) * 4 * PW, w);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 256);
}

// ------------------------------------------------------------------ dequantize

__host__ __device__ inline size_t dequantize_dense_smem(int stages, int pw)
{
    const size_t tab = pw <= 4 ? ((size_t)1 << (2 * pw)) * 16 * 4 : 256 * 2;
    return 1024 + 2 * kDnTile + (size_t)stages * kDnTile + tab + 8 * (2 * stages + 8) + 16;
}

template <bool BF16, int PW, int NS>
__global__ void __launch_bounds__(kDnDWarps * 32, 1)
dequantize_dense_kernel(const __grid_constant__ CUtensorMap tmp, const __grid_constant__ CUtensorMap tmo,
                        const uint8_t *__restrict__ codes, const uint16_t *__restrict__ norms, int64_t nvec,
                        const __grid_constant__ QuantTables T)
{
    constexpr int CB = 16 * PW;
    constexpr bool kPairs = PW <= 4;
    constexpr int NE = kPairs ? 1 << (2 * PW) : 256;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *s_P = base;                                    // Pi rows (K) x two 64-wide column atoms (N)
    uint8_t *s_O = s_P + kDnTile;                           // output tile staged for the TMA store
    uint8_t *ring = s_O + kDnTile;                          // A stages: C, K-major
    uint32_t *ptab = reinterpret_cast<uint32_t *>(ring + (size_t)NS * kDnTile);   // pairs x 16 copies
    uint16_t *ctab = reinterpret_cast<uint16_t *>(ptab);                          // or single levels
    const size_t tab_bytes = kPairs ? (size_t)NE * 16 * 4 : 256 * 2;
    uint64_t *a_full = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(ptab) + tab_bytes);
    uint64_t *a_free = a_full + NS;
    uint64_t *p_ready = a_free + NS;
    uint64_t *acc_full = p_ready + 2;
    uint64_t *acc_free = acc_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_free + 2);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t ntiles = (nvec + 127) / 128;
    const int64_t my_tiles = blockIdx.x < ntiles ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    // the centroid operand: each level rounded once to the 16-bit dtype
    auto c16 = [&](int k) -> uint32_t {
        const float c = k < T.levels ? T.centroid[k] : 0.0f;
        return BF16 ? (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(c)) : (uint32_t)__half_as_ushort(__float2half_rn(c));
    };
    if constexpr (kPairs) {
        for (int i = tid; i < NE * 16; i += blockDim.x) {
            const int e = i >> 4;
            ptab[i] = c16(e & ((1 << PW) - 1)) | (c16(e >> PW) << 16);
        }
    } else {
        for (int i = tid; i < 256; i += blockDim.x) ctab[i] = (uint16_t)c16(i);
    }
    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&a_full[s], 4);                       // 4 producer warps
            mbar_init(&a_free[s], 1);                       // MMA commit
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_free[a], 8);
        }
        mbar_init(&p_ready[0], 1);
        fence_barrier_init();
        prefetch_tmap(&tmp);
        prefetch_tmap(&tmo);
        mbar_arrive_expect_tx(&p_ready[0], kDnTile);
        for (int kc = 0; kc < 2; ++kc) tma_load_2d(s_P + (size_t)kc * 16384, &tmp, 64 * kc, 0, &p_ready[0]);
    }
    if (warp == 4) tmem_alloc(tmem_slot, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    if (warp < 4) {
        // ------------------------------------------------------------ producers: C tile
        const int r = tid;                                  // block within the tile
        const uint32_t ptab_lane = smem_u32(ptab) + (uint32_t)(lane & 15) * 4u;
        // the codes of tile i + 1 are loaded while tile i is unpacked
        auto load_codes = [&](int64_t i, uint32_t *w) {
            const int64_t tok = (blockIdx.x + i * gridDim.x) * 128 + r;
            if (i < my_tiles && tok < nvec) {
                load_bytes<CB>(codes + tok * CB, w);
            } else {
#pragma unroll
                for (int k = 0; k < 4 * PW; ++k) w[k] = 0u;
            }
        };
        uint32_t wn[4 * PW];
        load_codes(0, wn);
        for (int64_t i = 0; i < my_tiles && ok; ++i) {
            const int s = (int)(i % NS);
            const int64_t use = i / NS;
            uint32_t w[4 * PW];
#pragma unroll
            for (int k = 0; k < 4 * PW; ++k) w[k] = wn[k];
            load_codes(i + 1, wn);
            if (use > 0 && !mbar_wait(&a_free[s], (uint32_t)((use - 1) & 1))) { ok = false; break; }
            const uint32_t A = smem_u32(ring + (size_t)s * kDnTile);
#pragma unroll
            for (int k = 0; k < 16; ++k) {                  // 16-byte chunk k: values 8k .. 8k+7
                uint32_t o[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int p = 4 * k + q;                // value pair (2p, 2p+1)
                    if constexpr (kPairs) {
                        const uint32_t e = unpack_code<64, 2 * PW>(w, p);
                        asm("ld.shared.u32 %0, [%1];" : "=r"(o[q]) : "r"(ptab_lane + e * 64u));
                    } else {
                        const uint32_t e0 = unpack_code<128, PW>(w, 2 * p) & 0xffu;
                        const uint32_t e1 = unpack_code<128, PW>(w, 2 * p + 1) & 0xffu;
                        o[q] = (uint32_t)ctab[e0] | ((uint32_t)ctab[e1] << 16);
                    }
                }
                sts128(A + (uint32_t)(k >> 3) * 16384u + sw128_offset(r, k & 7), make_uint4(o[0], o[1], o[2], o[3]));
            }
            fence_proxy_async_smem();                       // generic writes -> visible to the MMA
            __syncwarp();
            if (lane == 0) mbar_arrive_cta(&a_full[s]);
        }
    } else if (warp == 4) {
        // ------------------------------------------------------------ MMA issuer: X^ = C Pi
        if (!mbar_wait(&p_ready[0], 0u)) ok = false;
        const uint32_t sP = smem_u32(s_P), sR = smem_u32(ring);
        const uint32_t idesc = idesc_f16(BF16, 128, 128) | (1u << 16);     // B (Pi) MN-major
        for (int64_t i = 0; i < my_tiles && ok; ++i) {
            const int s = (int)(i % NS);
            const int a = (int)(i & 1);
            const int64_t ause = i >> 1;
            if (ause > 0 && !mbar_wait(&acc_free[a], (uint32_t)((ause - 1) & 1))) { ok = false; break; }
            if (!mbar_wait(&a_full[s], (uint32_t)((i / NS) & 1))) { ok = false; break; }
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {            // K step kk: rows j = 16 kk .. 16 kk + 15 of Pi
                    const uint64_t adesc =
                        sdesc_k_sw128(sR + (uint32_t)s * kDnTile + (uint32_t)(kk >> 2) * 16384u + (uint32_t)(kk & 3) * 32u);
                    const uint64_t bdesc = dense_desc_sw128(sP + (uint32_t)kk * 2048u, 16384u, 1024u);
                    mma_f16(tmem + (uint32_t)(a * 128), adesc, bdesc, idesc, kk != 0);
                }
                mma_commit(&a_free[s]);
                mma_commit(&acc_full[a]);
            }
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------------ epilogue: x^ = acc * n16
        // The 8 warps stage the tile in s_O (the TMA layout of the output:
        // two 64-column regions, 128-byte swizzle) and one thread stores it.
        // Every warp takes both named barriers of every tile, also after an
        // expired wait (it then skips the work), so none can wait forever.
        const int quarter = warp & 3;
        const int part = (warp - 5) >> 2;                   // chunks 2 part, 2 part + 1
        const bool leader = warp == 5 && lane == 0;
        const uint32_t sO = smem_u32(s_O);
        for (int64_t i = 0; i < my_tiles; ++i) {
            const int a = (int)(i & 1);
            const int row = quarter * 32 + lane;
            const int64_t t = blockIdx.x + i * gridDim.x;
            const int64_t tok = t * 128 + row;
            const float n16 = tok < nvec ? h16_to_f32(__ldg(norms + tok)) : 0.0f;
            if (ok && !mbar_wait(&acc_full[a], (uint32_t)((i >> 1) & 1))) ok = false;
            tc_fence_after();
            uint32_t acc[2][32];
            if (ok) {
#pragma unroll
                for (int q = 0; q < 2; ++q)
                    tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(a * 128 + 32 * (2 * part + q)), acc[q]);
                tmem_ld_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0 && ok) mbar_arrive_cta(&acc_free[a]);
            if (leader) bulk_wait_read<0>();                 // the previous tile's store has read s_O
            named_barrier_sync(1, 256);
            if (ok) {
                const float2 n2 = make_float2(n16, n16);
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int col0 = 32 * (2 * part + q);
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8) {        // 8 values = one 16-byte chunk of the row
                        uint32_t o[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int e = 8 * c8 + 2 * j;
                            const float2 v = __fmul2_rn(make_float2(__uint_as_float(acc[q][e]), __uint_as_float(acc[q][e + 1])), n2);
                            o[j] = pack2<BF16>(v.x, v.y);
                        }
                        const int col = col0 + 8 * c8;
                        sts128(sO + (uint32_t)(col >> 6) * 16384u + sw128_offset(row, (col & 63) >> 3),
                               make_uint4(o[0], o[1], o[2], o[3]));
                    }
                }
            }
            fence_proxy_async_smem();                       // generic writes -> visible to the TMA store
            named_barrier_sync(1, 256);
            if (leader && ok) {
                tma_store_3d(&tmo, 0, 0, (int)(t * 128), s_O);
                tma_store_3d(&tmo, 0, 1, (int)(t * 128), s_O + 16384);
                bulk_commit();
            }
        }
        if (leader) bulk_wait<0>();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 4) tmem_dealloc(tmem, 256);
}

}  // namespace rq
