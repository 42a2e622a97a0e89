// rq_qjl_v2.cuh -- pipelined QJL key sketch for d = 128 (sm_100a), and the
// tcgen05 helpers the later sketch kernels share (TMEM column counts, the
// MMA issue loop, the sign-word packing).
//
// qjl_v2_sketch_kernel (qjl_sketch; the fallback of rq_sketch_v3.cuh): 3-D
// TMA loads put 128 keys straight into the A layout (one 64-column region per
// load); the threads only compute the canonical fp32 norms from shared
// memory; MMA of tile i overlaps the norm pass of tile i+1 and the epilogue
// of tile i-1.
//
// Epilogue: 8 warps; warp w reads TMEM lanes 32 (w mod 4) .. +31 (its 32
// vectors) and every other 32-column chunk starting at chunk w / 4, packs the
// 32 sign bits of a chunk into one word (bit i = P_i >= 0) and stores it.
#pragma once
#include "rq_qjl_mma.cuh"
#include "rq_v2.cuh"

namespace rq {

constexpr int kQ2Stages = 3;

__host__ __device__ inline uint32_t qjl_v2_tmem_cols(int m)
{
    uint32_t c = 32;
    while (c < 2u * (uint32_t)qjl_mma_m16(m)) c <<= 1;
    return c;
}

// Shared memory (bytes, with 1024-byte alignment slack).
__host__ __device__ inline size_t qjl_v2_smem(int mode, int pw, int m, const QuantTables &T, int stages)
{
    const size_t S = (size_t)qjl_mma_m16(m) * 128 * 2;            // m16 rows x 128 bf16, 2 regions
    size_t b = 1024 + S;
    if (mode == 0) {
        b += (size_t)stages * kTileBytes2;                        // input ring
        b += 2 * (size_t)128 * 128 * 2;                           // A double buffer
        b += lut_bytes_v2(T) + ((size_t)1 << pw) * 32 * 4 + 64 * 4;
    } else {
        b += (size_t)stages * 128 * 128 * 2;                      // A ring (TMA targets)
    }
    return b + 8 * (stages + 2) + 16;
}

// Bit i of the result = (v[i] >= 0) for 32 fp32 values.  Adding +0 maps -0
// to +0 (and leaves every other value unchanged), so the bit is the inverted
// sign bit.  The additions run on pairs; for each g = 0..7 two byte permutes
// gather the top bytes of v[g], v[g+8], v[g+16], v[g+24] into bytes 0..3 of
// one word, whose bit 7 of byte b is then the sign of v[8b+g], moved to bit
// 8b+g with one shift and one masked OR.
__device__ __forceinline__ uint32_t sign_word(const uint32_t *v)
{
    const float2 z = make_float2(0.0f, 0.0f);
    uint32_t neg = 0u;
#pragma unroll
    for (int g = 0; g < 8; ++g) {
        const float2 lo = __fadd2_rn(make_float2(__uint_as_float(v[g]), __uint_as_float(v[g + 8])), z);
        const float2 hi = __fadd2_rn(make_float2(__uint_as_float(v[g + 16]), __uint_as_float(v[g + 24])), z);
        const uint32_t top = __byte_perm(__byte_perm(__float_as_uint(lo.x), __float_as_uint(lo.y), 0x0073u),
                                         __byte_perm(__float_as_uint(hi.x), __float_as_uint(hi.y), 0x0073u),
                                         0x5410u);
        neg |= (top >> (7 - g)) & (0x01010101u << g);
    }
    return ~neg;
}

// Sign-pack epilogue of one 128-vector tile from TMEM accumulator columns
// [col0, col0 + m16).
__device__ __forceinline__ void qjl_v2_epilogue(uint32_t tmem, uint32_t col0, int m, int m16, int64_t tok0,
                                                int64_t nvec, uint8_t *__restrict__ signs, bool ok)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t tok = tok0 + (warp & 3) * 32 + lane;
    const bool tv = ok && tok < nvec;
    uint8_t *dst = signs + tok * (m / 8);
    for (int c0 = (warp >> 2) * 32; c0 < m16; c0 += 64) {
        uint32_t acc[32];
        tmem_ld32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + col0 + (uint32_t)c0, acc);
        tmem_ld_wait();
        const uint32_t word = sign_word(acc);
        if (tv && c0 < m) {
            const int nb = min(4, (m - c0) / 8);
            if (nb == 4 && (m & 31) == 0) {
                *reinterpret_cast<uint32_t *>(dst + c0 / 8) = word;
            } else {
                for (int b = 0; b < nb; ++b) dst[c0 / 8 + b] = (uint8_t)(word >> (8 * b));
            }
        }
    }
}

// One thread issues the MMAs of a 128 x m16 x 128 tile: A (2 regions of 128
// rows) x S^T (2 regions of m16 rows), into TMEM columns [col0, col0 + m16).
__device__ __forceinline__ void qjl_v2_issue(uint32_t sA, uint32_t sS, int m16, uint32_t tmem_col)
{
#pragma unroll
    for (int kc = 0; kc < 2; ++kc) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint64_t adesc = sdesc_k_sw128(sA + (uint32_t)kc * 16384u + (uint32_t)k * 32u);
            for (int n0 = 0; n0 < m16; n0 += 256) {
                const int N = min(256, m16 - n0);
                const uint64_t bdesc =
                    sdesc_k_sw128(sS + (uint32_t)kc * (uint32_t)m16 * 128u + (uint32_t)n0 * 128u + (uint32_t)k * 32u);
                mma_f16(tmem_col + (uint32_t)n0, adesc, bdesc, idesc_f16(true, 128, N), (kc | k) != 0);
            }
        }
    }
}

template <bool SBF16>
__device__ __forceinline__ void stage_projection(const uint16_t *__restrict__ proj, uint8_t *s_S, int m, int m16)
{
    for (int idx = threadIdx.x; idx < m16 * 16; idx += blockDim.x) {
        const int i = idx >> 4, c = idx & 15;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (i < m) v = __ldg(reinterpret_cast<const uint4 *>(proj + (size_t)i * 128) + c);
        *reinterpret_cast<uint4 *>(s_S + (size_t)(c >> 3) * m16 * 128 + sw128_offset(i, c & 7)) = v;
    }
}


// -------------------------------------------------------------- key sketch

// 3-D view of the keys: {64 values, 2 chunks, n tokens}; box {64, 1, 128}.
template <bool BF16, int STAGES>
__global__ void __launch_bounds__(kT2, 1)
qjl_v2_sketch_kernel(const __grid_constant__ CUtensorMap tmk, int64_t nvec, int m, const uint16_t *__restrict__ proj,
                     uint8_t *__restrict__ signs, uint16_t *__restrict__ norms)
{
    constexpr int ATILE = 128 * 128 * 2;
    const int m16 = qjl_mma_m16(m);
    const uint32_t ncols = qjl_v2_tmem_cols(m);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *s_S = base;
    uint8_t *ring = s_S + (size_t)m16 * 256;
    uint64_t *full = reinterpret_cast<uint64_t *>(ring + (size_t)STAGES * ATILE);
    uint64_t *mma_bar = full + STAGES;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_bar + 2);

    const int tid = threadIdx.x, warp = tid >> 5, part = tid & 1;
    const int64_t ntiles = (nvec + 127) / 128;
    if (tid == 0) {
        prefetch_tmap(&tmk);
        for (int s = 0; s < STAGES; ++s) mbar_init(&full[s], 1);
        mbar_init(&mma_bar[0], 1);
        mbar_init(&mma_bar[1], 1);
        fence_barrier_init();
        for (int s = 0; s < STAGES; ++s) {
            const int64_t t = blockIdx.x + (int64_t)s * gridDim.x;
            if (t < ntiles) {
                mbar_arrive_expect_tx(&full[s], ATILE);
                tma_load_3d(ring + s * ATILE, &tmk, 0, 0, (int)(t * 128), &full[s]);
                tma_load_3d(ring + s * ATILE + 16384, &tmk, 0, 1, (int)(t * 128), &full[s]);
            }
        }
    }
    stage_projection<BF16>(proj, s_S, m, m16);
    if (warp == 0) tmem_alloc(tmem_slot, ncols);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t sS = smem_u32(s_S), sR = smem_u32(ring);
    bool ok = true;
    uint32_t mma_phase[2] = {0u, 0u};
    int64_t i = 0;

    for (;; ++i) {
        const int64_t t = blockIdx.x + i * gridDim.x;
        if (t >= ntiles) break;
        const int s = (int)(i % STAGES);
        const bool got = mbar_wait(&full[s], (uint32_t)((i / STAGES) & 1));
        if (__syncthreads_or(!got)) { ok = false; break; }
        // MMA of tile i as soon as its keys have landed
        if (tid == 0) {
            tc_fence_after();
            qjl_v2_issue(sR + (uint32_t)s * ATILE, sS, m16, tmem + (uint32_t)((i & 1) * m16));
            mma_commit(&mma_bar[i & 1]);
        }
        // canonical fp32 norm of each key: thread = (key tid/2, half tid%2)
        {
            const uint8_t *Ar = ring + s * ATILE + part * 16384;
            const int r = tid >> 1;
            uint32_t u[32];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint4 v = *reinterpret_cast<const uint4 *>(Ar + sw128_offset(r, k));
                u[4 * k] = v.x; u[4 * k + 1] = v.y; u[4 * k + 2] = v.z; u[4 * k + 3] = v.w;
            }
            float2 P[32];
            row_to_pairs<BF16>(u, P);
            const float n32 = __fsqrt_rn(combine_parts<2>(row_sumsq(P)));
            const int64_t tok = t * 128 + r;
            if (part == 0 && tok < nvec) norms[tok] = norm_to_h16(n32);
        }
        // tile i-1: accumulator ready -> signs; its A stage returns to the TMA ring
        if (i >= 1) {
            const int a = (int)((i - 1) & 1);
            if (ok && !mbar_wait(&mma_bar[a], mma_phase[a])) ok = false;
            mma_phase[a] ^= 1u;
            tc_fence_after();
            const int64_t tp = t - gridDim.x;
            qjl_v2_epilogue(tmem, (uint32_t)(a * m16), m, m16, tp * 128, nvec, signs, ok);
            tc_fence_before();
            if (tid == 0) {
                const int sp = (int)((i - 1) % STAGES);
                const int64_t tn = tp + (int64_t)STAGES * gridDim.x;
                if (tn < ntiles) {
                    mbar_arrive_expect_tx(&full[sp], ATILE);
                    tma_load_3d(ring + sp * ATILE, &tmk, 0, 0, (int)(tn * 128), &full[sp]);
                    tma_load_3d(ring + sp * ATILE + 16384, &tmk, 0, 1, (int)(tn * 128), &full[sp]);
                }
            }
        }
        if (!__syncthreads_and(ok)) { ok = false; break; }
    }
    if (i >= 1) {
        const int a = (int)((i - 1) & 1);
        if (ok && !mbar_wait(&mma_bar[a], mma_phase[a])) ok = false;
        mma_phase[a] ^= 1u;
        tc_fence_after();
        qjl_v2_epilogue(tmem, (uint32_t)(a * m16), m, m16, (blockIdx.x + (i - 1) * (int64_t)gridDim.x) * 128, nvec,
                        signs, ok);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, ncols);
}

}  // namespace rq
