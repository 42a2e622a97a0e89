// rq_sketch_v3.cuh -- warp-specialised QJL key sketch for d = 128 (sm_100a).
//
// P = K S^T for 128 keys per tile (tcgen05.mma kind::f16, fp32 in TMEM), sign
// bits packed from the accumulator, fp16 key norms from shared memory.  The
// roles run concurrently and meet only at mbarriers:
//   warp 0   TMA: 3-D loads of each tile straight into the A layout (two
//            64-column regions), a ring of NS stages; waits stage_free;
//   warp 1   MMA: waits stage_full and acc_free, issues d/16 MMAs per N-half,
//            commits stage_mma (the stage's operand reads are done) and
//            acc_full;
//   warps 2-5 norms: thread = key, canonical fp32 pairwise norm of its 128
//            values read from the stage, arrive stage_free;
//   warps 6-13 epilogue: TMEM lane quarter (warp mod 4) = 32 keys, half of
//            the 32-column chunks each (two warps per quarter), loaded two at
//            a time, sign words stored, arrive acc_free.
// A stage returns to the TMA warp when both its MMA and its norm pass are done
// (stage_free counts 4 norm-warp arrivals + 1 MMA commit).
#pragma once
#include "rq_qjl_v2.cuh"

namespace rq {

constexpr int kSk3Warps = 14;

__device__ __forceinline__ void mbar_arrive_cta(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__host__ __device__ inline size_t sketch_v3_smem(int m, int stages)
{
    return 1024 + (size_t)qjl_mma_m16(m) * 256 + (size_t)stages * 32768 + 8 * (3 * stages + 4) + 16;
}

template <bool BF16, int NS>
__global__ void __launch_bounds__(kSk3Warps * 32, 1)
sketch_v3_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tms, int64_t nvec,
                 int m, uint8_t *__restrict__ signs, uint16_t *__restrict__ norms)
{
    constexpr uint32_t ATILE = 128 * 128 * 2;
    const int m16 = qjl_mma_m16(m);
    const uint32_t ncols = qjl_v2_tmem_cols(m);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *s_S = base;                                    // 2 regions x m16 rows x 128 B
    uint8_t *ring = s_S + (size_t)m16 * 256;
    uint64_t *stage_full = reinterpret_cast<uint64_t *>(ring + (size_t)NS * ATILE);
    uint64_t *stage_free = stage_full + NS;
    uint64_t *s_ready = stage_free + NS;                    // S staged ([0]; the rest is padding)
    uint64_t *acc_full = s_ready + NS;
    uint64_t *acc_free = acc_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_free + 2);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t ntiles = (nvec + 127) / 128;
    const int64_t my_tiles = blockIdx.x < ntiles ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&stage_full[s], 1);
            mbar_init(&stage_free[s], 5);                   // 4 norm warps + 1 MMA commit
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_free[a], 8);                     // 8 epilogue warps
        }
        mbar_init(&s_ready[0], 1);
        fence_barrier_init();
        prefetch_tmap(&tmk);
        prefetch_tmap(&tms);
        // S: two 64-column boxes of up to 256 rows each, straight into the B layout
        const uint32_t sbytes = (uint32_t)m16 * 256u;
        mbar_arrive_expect_tx(&s_ready[0], sbytes);
        for (int kc = 0; kc < 2; ++kc)
            for (int r0 = 0; r0 < m16; r0 += 256)
                tma_load_2d(s_S + (size_t)kc * m16 * 128 + (size_t)r0 * 128, &tms, 64 * kc, r0, &s_ready[0]);
    }
    if (warp == 1) tmem_alloc(tmem_slot, ncols);
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
                mbar_arrive_expect_tx(&stage_full[s], ATILE);
                tma_load_3d(ring + (size_t)s * ATILE, &tmk, 0, 0, (int)(t * 128), &stage_full[s]);
                tma_load_3d(ring + (size_t)s * ATILE + 16384, &tmk, 0, 1, (int)(t * 128), &stage_full[s]);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (!mbar_wait(&s_ready[0], 0u)) ok = false;     // S landed
        const uint32_t sS = smem_u32(s_S), sR = smem_u32(ring);
        for (int64_t i = 0; i < my_tiles && ok; ++i) {
            const int s = (int)(i % NS);
            const int a = (int)(i & 1);
            const int64_t ause = i >> 1;
            if (ause > 0 && !mbar_wait(&acc_free[a], (uint32_t)((ause - 1) & 1))) { ok = false; break; }
            if (!mbar_wait(&stage_full[s], (uint32_t)((i / NS) & 1))) { ok = false; break; }
            tc_fence_after();
            if (lane == 0) {
                qjl_v2_issue(sR + (uint32_t)s * ATILE, sS, m16, tmem + (uint32_t)(a * m16));
                mma_commit(&stage_free[s]);                 // operand reads done -> one of the 5 arrivals
                mma_commit(&acc_full[a]);
            }
            __syncwarp();
        }
    } else if (warp < 6) {
        // ------------------------------------------------------------ norms
        const int r = tid - 64;                             // key within the tile
        for (int64_t i = 0; i < my_tiles && ok; ++i) {
            const int s = (int)(i % NS);
            if (!mbar_wait(&stage_full[s], (uint32_t)((i / NS) & 1))) { ok = false; break; }
            const uint8_t *A = ring + (size_t)s * ATILE;
            float sums[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t u[32];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(A + h * 16384 + sw128_offset(r, k));
                    u[4 * k] = v.x; u[4 * k + 1] = v.y; u[4 * k + 2] = v.z; u[4 * k + 3] = v.w;
                }
                float2 P[32];
                row_to_pairs<BF16>(u, P);
                sums[h] = row_sumsq(P);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive_cta(&stage_free[s]);
            const int64_t tok = (blockIdx.x + i * gridDim.x) * 128 + r;
            if (tok < nvec) norms[tok] = norm_to_h16(__fsqrt_rn(__fadd_rn(sums[0], sums[1])));
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;
        const int part = (warp - 6) >> 2;                   // which half of the column chunks
        const int nchk = (m16 + 31) / 32, half = (nchk + 1) / 2;
        const int ch0 = part * half, ch1 = min(nchk, ch0 + half);
        for (int64_t i = 0; i < my_tiles && ok; ++i) {
            const int a = (int)(i & 1);
            if (!mbar_wait(&acc_full[a], (uint32_t)((i >> 1) & 1))) { ok = false; break; }
            tc_fence_after();
            const int64_t tok = (blockIdx.x + i * gridDim.x) * 128 + quarter * 32 + lane;
            uint8_t *dst = signs + tok * (m / 8);
            for (int ch = ch0; ch < ch1; ch += 2) {
                uint32_t acc[2][32];
                const int nch = min(2, ch1 - ch);
#pragma unroll
                for (int q = 0; q < 2; ++q)
                    if (q < nch)
                        tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(a * m16 + 32 * (ch + q)), acc[q]);
                tmem_ld_wait();
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int cc = 32 * (ch + q);
                    if (q < nch && tok < nvec && cc < m) {
                        const uint32_t word = sign_word(acc[q]);
                        const int nb = min(4, (m - cc) / 8);
                        if (nb == 4 && (m & 31) == 0) {
                            *reinterpret_cast<uint32_t *>(dst + cc / 8) = word;
                        } else {
                            for (int bb = 0; bb < nb; ++bb) dst[cc / 8 + bb] = (uint8_t)(word >> (8 * bb));
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cta(&acc_free[a]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, ncols);
}

}  // namespace rq
