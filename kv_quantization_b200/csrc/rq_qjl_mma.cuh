// rq_qjl_mma.cuh -- QJL sketch on the tcgen05 tensor cores (sm_100a).
//
// The sketch P = V S^T (V: 128 vectors x d per tile, S: m x d) is a dense
// contraction, so it runs as tcgen05.mma kind::f16 (bf16/fp16 operands from
// shared memory, fp32 accumulator in TMEM); the epilogue reads the accumulator
// with tcgen05.ld and packs sign bits straight from it (QJL paragraph of the
// eliza quantization README: sign of each sketch coordinate, 8 per byte).
//
// MODE 0 (rq_quantize_qjl): each thread quantizes its block slice exactly as
//   quantize_kernel does, rebuilds the fp32 reconstruction, and writes the
//   residual r = x - x^32 (rounded to bf16) into the tile's A operand; the
//   residual's fp16 norm is stored beside the codes.
// MODE 1 (qjl_sketch): the A operand is the input vectors themselves.
//
// Per CTA (persistent, one per SM): S is staged once into shared memory in the
// 128-byte-swizzled K-major layout; per tile of 128 vectors the threads fill
// the A tile (TPB sub-tiles of 128/TPB vectors when d > 128), one thread
// issues d/16 MMAs (two N-halves when m > 256) and commits to an mbarrier; the
// epilogue of tile i runs after the threads have already loaded and processed
// the first sub-tile of tile i+1, so the MMA overlaps the next tile's HBM reads.
#pragma once
#include "rq_quant_impl.cuh"
#include "sm100.cuh"

namespace rq {

__host__ __device__ constexpr int qjl_mma_m16(int m) { return (m + 15) & ~15; }

__host__ __device__ inline uint32_t qjl_mma_tmem_cols(int m)
{
    uint32_t c = 32;
    while (c < (uint32_t)qjl_mma_m16(m)) c <<= 1;
    return c;
}

__host__ __device__ inline uint32_t qjl_lut_bytes(const QuantTables &T, int mode)
{
    if (mode != 0) return 0;
    uint32_t b = T.lut_cells > 0 ? (uint32_t)T.lut_cells * 16u * 8u : (uint32_t)T.levels * 4u;
    return (b + 15u) & ~15u;
}

// Dynamic shared memory of qjl_mma_kernel (bytes), including alignment slack.
__host__ __device__ inline size_t qjl_mma_smem_bytes(int D, int pw, int m, const QuantTables &T, int mode)
{
    const int E = D < 128 ? D : 128;
    const size_t kc = (size_t)D / 64;
    size_t b = 1024;                                      // 1024-byte alignment slack
    b += kc * (size_t)qjl_mma_m16(m) * 128;               // S
    b += kc * 128 * 128;                                  // A tile (128 vectors)
    b += (size_t)kThreads * E * 2;                        // input sub-tile
    b += qjl_lut_bytes(T, mode);
    b += mode == 0 ? ((size_t)1 << pw) * 32 * 4 : 0;      // replicated centroids
    b += 16;                                              // mbarrier + TMEM address
    return b;
}

template <int D, int PW, bool BF16, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
qjl_mma_kernel(const uint8_t *__restrict__ x, int64_t nvec, const __grid_constant__ QuantTables T,
               uint8_t *__restrict__ codes, uint16_t *__restrict__ norms, int m, const uint16_t *__restrict__ proj,
               uint8_t *__restrict__ signs, uint16_t *__restrict__ snorms)
{
    constexpr int E = D < 128 ? D : 128;
    constexpr int TPB = D / E;
    constexpr int NCH = E * 2 / 16;          // 16-byte chunks per thread row
    constexpr int KC = D / 64;               // 64-element K regions
    constexpr int TOK_SUB = kThreads / TPB;  // vectors per sub-tile
    constexpr int CB = E * PW / 8;
    constexpr int NW = (E * PW + 31) / 32;
    constexpr bool OP_BF16 = MODE == 0 ? true : BF16;
    const int m16 = qjl_mma_m16(m);
    const uint32_t ncols = qjl_mma_tmem_cols(m);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *s_S = base;
    uint8_t *s_A = s_S + (size_t)KC * m16 * 128;
    uint4 *tile = reinterpret_cast<uint4 *>(s_A + (size_t)KC * 128 * 128);
    uint8_t *p = reinterpret_cast<uint8_t *>(tile) + kThreads * E * 2;
    uint2 *lut = reinterpret_cast<uint2 *>(p);
    float *bnd = reinterpret_cast<float *>(p);
    p += qjl_lut_bytes(T, MODE);
    float *cent = reinterpret_cast<float *>(p);
    p += MODE == 0 ? (1 << PW) * 32 * 4 : 0;
    uint64_t *mbar = reinterpret_cast<uint64_t *>(p);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(p + 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, part = tid % TPB;

    // ---- one-time setup: S (zero rows m..m16), tables, barrier, TMEM
    for (int idx = tid; idx < m16 * (D / 8); idx += kThreads) {
        const int i = idx / (D / 8), c = idx % (D / 8);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (i < m) v = __ldg(reinterpret_cast<const uint4 *>(proj + (size_t)i * D) + c);
        *reinterpret_cast<uint4 *>(s_S + (size_t)(c >> 3) * m16 * 128 + sw128_offset(i, c & 7)) = v;
    }
    if constexpr (MODE == 0) {
        setup_lut(T, lut, bnd);
        setup_centroids(T, cent, 1 << PW);
    }
    if (tid == 0) {
        mbar_init(mbar, 1);
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, ncols);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const uint32_t sA = smem_u32(s_A), sS = smem_u32(s_S);
    const int64_t total_rows = nvec * TPB;
    const float lut_a = T.lut_a, lut_b = T.lut_b;
    const int cells = T.lut_cells, levels = T.levels;
    uint32_t phase = 0;
    bool pending = false, ok = true;
    int64_t pend_base = 0;

    auto epilogue = [&](int64_t tb) {
        if (ok && !mbar_wait(mbar, phase)) ok = false;
        phase ^= 1u;
        tc_fence_after();
        const int64_t tok = tb + warp * 32 + lane;
        const bool tv = ok && tok < nvec;
        uint8_t *dst = signs + tok * (m / 8);
        for (int c0 = 0; c0 < m16; c0 += 32) {
            uint32_t acc[32];
            tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, acc);
            tmem_ld_wait();
            uint32_t word = 0u;
#pragma unroll
            for (int i = 0; i < 32; ++i) word |= (__uint_as_float(acc[i]) >= 0.0f ? 1u : 0u) << i;
            if (tv && c0 < m) {
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

    for (int64_t tb = (int64_t)blockIdx.x * 128; tb < nvec; tb += (int64_t)gridDim.x * 128) {
#pragma unroll 1
        for (int sub = 0; sub < TPB; ++sub) {
            const int64_t row0 = (tb + (int64_t)sub * TOK_SUB) * TPB;
            __syncthreads();   // input sub-tile free
            load_tile<NCH>(tile, reinterpret_cast<const uint4 *>(x) + row0 * NCH, total_rows - row0);
            __syncthreads();
            const int64_t row = row0 + tid;
            const bool valid = row < total_rows;
            float v[E];
            read_row<E, BF16>(tile, tid, v);
            float vn;
            if constexpr (MODE == 0) {
                const float n32 = block_norm<E, TPB>(v);
                apply_signs<E>(v, T.sign_words, part);
                fwht_local<E>(v);
                fwht_cross<E, TPB>(v, part);
                const float inv = n32 > 0.0f ? __frcp_rn(n32) : 0.0f;
                uint32_t w[NW];
#pragma unroll
                for (int i = 0; i < NW; ++i) w[i] = 0u;
#pragma unroll
                for (int j = 0; j < E; ++j) {
                    const float y = __fmul_rn(v[j], inv);
                    const uint32_t c = cells > 0 ? lut_code(y, lut, lut_a, lut_b, cells, lane & 15)
                                                 : bsearch_code(y, bnd, levels);
                    const int bit = j * PW;
                    w[bit >> 5] |= c << (bit & 31);
                    if ((bit & 31) + PW > 32) w[(bit >> 5) + 1] |= c >> (32 - (bit & 31));
                }
                const uint16_t n16 = norm_to_h16(n32);
                if (valid) {
                    store_bytes<CB>(codes + row * CB, w);
                    if (part == 0) norms[row / TPB] = n16;
                }
                // fp32 reconstruction and residual r = x - x^32
#pragma unroll
                for (int j = 0; j < E; ++j) v[j] = cent[unpack_code<E, PW>(w, j) * 32 + lane];
                fwht_local<E>(v);
                fwht_cross<E, TPB>(v, part);
                const float scale = __fmul_rn(h16_to_f32(n16), 1.0f / (float)D);
#pragma unroll
                for (int k = 0; k < NCH; ++k) {
                    const uint4 xw = tile[tid * NCH + (k ^ (tid % NCH))];
                    float xr[8];
                    unpack2<BF16>(xw.x, xr[0], xr[1]);
                    unpack2<BF16>(xw.y, xr[2], xr[3]);
                    unpack2<BF16>(xw.z, xr[4], xr[5]);
                    unpack2<BF16>(xw.w, xr[6], xr[7]);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int j = 8 * k + i;
                        const float xh = __uint_as_float(__float_as_uint(__fmul_rn(v[j], scale)) ^
                                                         sign_mask(T.sign_words, part * E + j));
                        v[j] = __fsub_rn(xr[i], xh);
                    }
                }
                vn = block_norm<E, TPB>(v);
            } else {
                vn = block_norm<E, TPB>(v);
            }
            if (valid && part == 0) snorms[row / TPB] = norm_to_h16(vn);

            // the previous tile's MMA must be complete before the A tile is rewritten
            if (sub == 0 && pending) {
                epilogue(pend_base);
                pending = false;
            }
            const int arow = sub * TOK_SUB + tid / TPB;
#pragma unroll
            for (int k = 0; k < NCH; ++k) {
                const int gc = part * NCH + k;             // 16-byte chunk index within the vector
                uint4 w;
                if constexpr (MODE == 0) {
                    w.x = pack2<true>(v[8 * k + 0], v[8 * k + 1]);
                    w.y = pack2<true>(v[8 * k + 2], v[8 * k + 3]);
                    w.z = pack2<true>(v[8 * k + 4], v[8 * k + 5]);
                    w.w = pack2<true>(v[8 * k + 6], v[8 * k + 7]);
                } else {
                    w = tile[tid * NCH + (k ^ (tid % NCH))];
                }
                *reinterpret_cast<uint4 *>(s_A + (size_t)(gc >> 3) * 128 * 128 + sw128_offset(arow, gc & 7)) = w;
            }
        }
        // ---- A tile complete: issue the MMAs for this tile
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && ok) {
            tc_fence_after();
#pragma unroll 1
            for (int kc = 0; kc < KC; ++kc) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint64_t adesc = sdesc_k_sw128(sA + (uint32_t)kc * 16384u + (uint32_t)k * 32u);
                    for (int n0 = 0; n0 < m16; n0 += 256) {
                        const int N = min(256, m16 - n0);
                        const uint64_t bdesc =
                            sdesc_k_sw128(sS + (uint32_t)kc * (uint32_t)m16 * 128u + (uint32_t)n0 * 128u + (uint32_t)k * 32u);
                        mma_f16(tmem + (uint32_t)n0, adesc, bdesc, idesc_f16(OP_BF16, 128, N), (kc | k) != 0);
                    }
                }
            }
            mma_commit(mbar);
        }
        pending = true;
        pend_base = tb;
        if (!__syncthreads_and(ok)) break;   // a bounded wait expired: unwind
    }
    if (pending) epilogue(pend_base);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, ncols);
}

}  // namespace rq
