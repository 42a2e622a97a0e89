// rq_bd.cuh -- rotated scalar quantization of blocks whose size d is not a
// power of two (sm_100a).
//
// The block is transformed block-diagonally: d is decomposed into powers of
// two, largest first (GLQ README, "Bit widths": 2688 = 2048 + 512 + 128), and
// each sub-block of size b gets its own Walsh-Hadamard transform after the
// seeded sign diagonal (turbopress "Package layout": block-diagonal
// Walsh-Hadamard times Rademacher signs).  With R = blockdiag(H_b / sqrt(b)) D
// orthogonal, the coordinates are y = sqrt(d) R x / ||x|| and the
// reconstruction x^ = ||x|| R^T c / sqrt(d).  In the canonical fp32 order:
//   norm: squares, pairwise sums within each sub-block, the sub-block sums
//         added in order, correctly rounded square root;
//   y_j  = w_j * fl32(g_b * inv),  g_b = fl32(sqrt(d / b)), inv = fl32(1 / n32),
//   x^_j = s_j * (w'_j * fl32(n16 * h_b)),  h_b = fl32(1 / sqrt(d b)),
// with w = H_b D x and w' = H_b c in radix-2 stages h = 1, 2, ... b/2.
//
// Mapping.  d is a multiple of 32 and every sub-block holds at least 32
// values, so a block is C = d / 32 chunks of 32 and a chunk never straddles
// two sub-blocks.  A thread owns one chunk, held as 16 float2
// P[k] = (v_2k, v_2k+1) -- exactly the bf16/fp16 pairs of its input or
// output words, so the sign diagonal is one XOR per word -- and a warp owns
// W = 32 / C consecutive blocks (lane l -> block l / C, chunk l % C), so its
// loads and stores are one contiguous range.  Inside a chunk everything is
// register arithmetic: Hadamard stage h = 1 inside each float2, h = 2..16 as
// packed f32x2 operations on the pair index.  Stages h >= 32 pair two chunks
// of one sub-block (lanes l and l +- h/32) through lane shuffles, as one
// packed multiply-add each (a + b, or a - b, or the value kept), and so do
// the upper levels of the norm tree and the in-order sum over sub-blocks.
//
// Nearest centroid: the saturating-grid table of the power-of-two kernels
// when the codebook has one (an exact count of boundaries below y), else a
// binary search over the boundaries.  Dequantize reads codes of up to 4 bits
// as value pairs from a table of centroid pairs.
#pragma once
#include <cstdint>

#include "rq_common.cuh"
#include "rq_v5.cuh"

namespace rq {

constexpr int kBdWarps = 8;
constexpr int kBdMaxSub = 5;

struct BdGeom {
    int nsub;
    int k0[kBdMaxSub];               // first 32-value chunk of each sub-block
    int nk[kBdMaxSub];               // chunks in it (a power of two)
    float g[kBdMaxSub];              // fl32(sqrt(d / b))
    float h[kBdMaxSub];              // fl32(1 / sqrt(d b))
};

// Where chunk c of a block sits: its sub-block s, its index r inside it and
// the sub-block's chunk count.
struct BdChunk {
    int s, r, nk;
};

__device__ __forceinline__ BdChunk bd_chunk(const BdGeom &G, int c)
{
    BdChunk q{0, c, G.nk[0]};
#pragma unroll
    for (int i = 1; i < kBdMaxSub; ++i)
        if (i < G.nsub && c >= G.k0[i]) q = BdChunk{i, c - G.k0[i], G.nk[i]};
    return q;
}

// Hadamard stages h = 1 ... 16 of the thread's chunk.
__device__ __forceinline__ void bd_fwht32(float2 *P)
{
#pragma unroll
    for (int k = 0; k < 16; ++k) {                         // stage h = 1
        const float a = P[k].x, b = P[k].y;
        P[k] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
    }
    const float2 m1 = make_float2(-1.0f, -1.0f);
#pragma unroll
    for (int h = 1; h < 16; h *= 2) {                      // stages 2h = 2 .. 16 on the pair index
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            if (k & h) continue;
            const float2 a = P[k], b = P[k + h];
            P[k] = __fadd2_rn(a, b);
            P[k + h] = __ffma2_rn(b, m1, a);               // a - b, one rounding
        }
    }
}

// Stages h = 32, 64, ... of every sub-block: the chunk with index r pairs
// with r ^ (h / 32) (lane `lane - r + (r ^ (h / 32))`); the lower chunk keeps
// a + b = fma(a, 1, b), the upper a - b = fma(b, -1, a); a lane outside the
// stage reads itself and keeps fma(v, 0, v) = v.
__device__ __forceinline__ void bd_fwht_cross(float2 *P, const BdChunk &q, int nk_max, int lane, bool on)
{
    for (int hk = 1; hk < nk_max; hk *= 2) {
        const bool part = on && hk < q.nk;
        const int src = part ? lane - q.r + (q.r ^ hk) : lane;
        const float sg = part ? ((q.r & hk) ? -1.0f : 1.0f) : 0.0f;
        const float2 sg2 = make_float2(sg, sg);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float2 p = make_float2(__shfl_sync(0xffffffffu, P[k].x, src), __shfl_sync(0xffffffffu, P[k].y, src));
            P[k] = __ffma2_rn(P[k], sg2, p);
        }
    }
}

// Bring bytes [begin, end) after p (p 16-byte aligned) into L2, trimmed to
// whole 16-byte units inside the range.
__device__ __forceinline__ void bd_prefetch_l2(const void *p, int64_t begin, int64_t end)
{
    begin = (begin + 15) & ~(int64_t)15;
    end &= ~(int64_t)15;
    if (end > begin)
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(static_cast<const uint8_t *>(p) + begin),
                     "r"((uint32_t)(end - begin))
                     : "memory");
}

template <int PW, bool BF16>
__global__ void __launch_bounds__(kBdWarps * 32, 2)
quantize_bd_kernel(const uint16_t *__restrict__ x, int64_t nblocks, int d, const __grid_constant__ QuantTables T,
                   const __grid_constant__ BdGeom G, uint8_t *__restrict__ codes, uint16_t *__restrict__ norms)
{
    extern __shared__ __align__(16) uint8_t bd_smem[];
    float *bnd = reinterpret_cast<float *>(bd_smem);                 // 256 floats
    uint32_t *pmask = reinterpret_cast<uint32_t *>(bd_smem + 1024);  // d / 2 sign words of value pairs
    uint2 *lut = reinterpret_cast<uint2 *>(bd_smem + 2048);         // sat_cells * 16 entries
    for (int i = threadIdx.x; i < 256; i += blockDim.x) bnd[i] = i < T.levels - 1 ? T.bound[i] : INFINITY;
    setup_pair_masks(T, pmask, d);
    const bool sat = T.sat_cells > 0;
    if (sat) setup_sat_lut8(T, lut);
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = d >> 5, W = 32 / C;
    const int bi = lane / C, c = lane - bi * C;
    const bool lane_on = bi < W;
    const BdChunk q = bd_chunk(G, lane_on ? c : 0);
    const int nk_max = G.nk[0];
    const float gs = G.g[q.s];
    const SatGrid SG = sat_grid(T, smem_u32(lut), (uint32_t)(lane & 15) * 8u);
    const uint32_t pm = smem_u32(pmask) + (uint32_t)(lane_on ? c : 0) * 64u;

    const int64_t ntask = (nblocks + W - 1) / W;
    const int64_t stride = (int64_t)gridDim.x * kBdWarps;
    // the warp's task t is the contiguous input range of blocks [t W, t W + W):
    // keep the next two in flight to L2
    auto prefetch = [&](int64_t tp) {
        if (lane == 0 && tp < ntask) {
            const int64_t b0 = tp * W, b1 = b0 + W < nblocks ? b0 + W : nblocks;
            bd_prefetch_l2(x, b0 * d * 2, b1 * d * 2);
        }
    };
    prefetch((int64_t)blockIdx.x * kBdWarps + warp + stride);
    for (int64_t t = (int64_t)blockIdx.x * kBdWarps + warp; t < ntask; t += stride) {
        prefetch(t + 2 * stride);
        const int64_t blk = t * W + bi;
        const bool on = lane_on && blk < nblocks;
        uint32_t raw[16];
        if (on) {
            load_bytes<64>(reinterpret_cast<const uint8_t *>(x + blk * d + 32 * c), raw);
        } else {
#pragma unroll
            for (int k = 0; k < 16; ++k) raw[k] = 0u;
        }
        // signs on the input pairs (negation is exact and leaves the squares alone)
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
            const uint4 m = lds128(pm + 16u * k4);
            raw[4 * k4] ^= m.x; raw[4 * k4 + 1] ^= m.y; raw[4 * k4 + 2] ^= m.z; raw[4 * k4 + 3] ^= m.w;
        }
        float2 P[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) unpack2<BF16>(raw[k], P[k].x, P[k].y);

        // norm: the pairwise tree within the chunk (leaves (2k, 2k+1)), the
        // chunks of the sub-block pairwise, the sub-blocks in order
        float l1[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float2 sq = __fmul2_rn(P[k], P[k]);
            l1[k] = __fadd_rn(sq.x, sq.y);
        }
#pragma unroll
        for (int w = 1; w < 16; w *= 2)
#pragma unroll
            for (int k = 0; k < 16; k += 2 * w) l1[k] = __fadd_rn(l1[k], l1[k + w]);
        float s = l1[0];
        for (int hk = 1; hk < nk_max; hk *= 2) {
            const float p = __shfl_down_sync(0xffffffffu, s, hk);
            if (hk < q.nk && (q.r & (2 * hk - 1)) == 0) s = __fadd_rn(s, p);
        }
        const int first = bi * C;
        float tot = __shfl_sync(0xffffffffu, s, lane_on ? first + G.k0[0] : lane);
        for (int i = 1; i < G.nsub; ++i) {
            const float p = __shfl_sync(0xffffffffu, s, lane_on ? first + G.k0[i] : lane);
            tot = __fadd_rn(tot, p);
        }
        const float n32 = __fsqrt_rn(tot);

        // transform
        bd_fwht32(P);
        bd_fwht_cross(P, q, nk_max, lane, on);

        // coordinates and codes
        const float inv = n32 > 0.0f ? __frcp_rn(n32) : 0.0f;
        const float f = __fmul_rn(gs, inv);
        const float2 f2 = make_float2(f, f);
        uint32_t w[PW];
#pragma unroll
        for (int k = 0; k < PW; ++k) w[k] = 0u;
        if (sat) {
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float2 y = __fmul2_rn(P[k], f2);
                uint32_t a0, a1;
                sat_addr(SG, y, a0, a1);
                const uint2 e0 = lds64(a0), e1 = lds64(a1);
                put_code_cmp<PW>(w, 2 * k, e0.y, y.x, __uint_as_float(e0.x));
                put_code_cmp<PW>(w, 2 * k + 1, e1.y, y.y, __uint_as_float(e1.x));
            }
        } else {
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float2 y = __fmul2_rn(P[k], f2);
                put_code<PW>(w, 2 * k, bsearch_code(y.x, bnd, T.levels));
                put_code<PW>(w, 2 * k + 1, bsearch_code(y.y, bnd, T.levels));
            }
        }
        if (on) {
            store_bytes<4 * PW>(codes + (blk * C + c) * (4 * PW), w);
            if (c == 0) norms[blk] = norm_to_h16(n32);
        }
    }
}

__host__ __device__ inline size_t dequantize_bd_smem(int pw)
{
    return 2048 + (pw <= 4 ? ((size_t)1 << (2 * pw)) * 16 * 8 : 0);
}

template <int PW, bool BF16>
__global__ void __launch_bounds__(kBdWarps * 32, 2)
dequantize_bd_kernel(const uint8_t *__restrict__ codes, const uint16_t *__restrict__ norms, int64_t nblocks, int d,
                     const __grid_constant__ QuantTables T, const __grid_constant__ BdGeom G,
                     uint16_t *__restrict__ out)
{
    constexpr bool kPairs = PW <= 4;                                 // centroid-pair table
    constexpr int NE = kPairs ? 1 << (2 * PW) : 0;
    constexpr uint32_t kMask = PW == 8 ? 0xffu : ((1u << PW) - 1u);
    extern __shared__ __align__(16) uint8_t bd_smem[];
    float *cent = reinterpret_cast<float *>(bd_smem);                // 256 floats
    uint32_t *pmask = reinterpret_cast<uint32_t *>(bd_smem + 1024);  // d / 2 sign words of value pairs
    float2 *ptab = reinterpret_cast<float2 *>(bd_smem + 2048);      // NE pairs x 16 copies
    for (int i = threadIdx.x; i < 256; i += blockDim.x) cent[i] = i < T.levels ? T.centroid[i] : 0.0f;
    setup_pair_masks(T, pmask, d);
    if constexpr (kPairs)
        for (int i = threadIdx.x; i < NE * 16; i += blockDim.x) {
            const int e = i >> 4;
            ptab[i] = make_float2(T.centroid[e & ((1 << PW) - 1)], T.centroid[e >> PW]);
        }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = d >> 5, W = 32 / C;
    const int bi = lane / C, c = lane - bi * C;
    const bool lane_on = bi < W;
    const BdChunk q = bd_chunk(G, lane_on ? c : 0);
    const int nk_max = G.nk[0];
    const float hs = G.h[q.s];
    const uint32_t pm = smem_u32(pmask) + (uint32_t)(lane_on ? c : 0) * 64u;
    const uint32_t ptab_lane = smem_u32(ptab) + (uint32_t)(lane & 15) * 8u;

    const int64_t ntask = (nblocks + W - 1) / W;
    const int64_t stride = (int64_t)gridDim.x * kBdWarps;
    const int64_t cb = (int64_t)C * 4 * PW;                          // code bytes per block
    auto prefetch = [&](int64_t tp) {
        if (lane == 0 && tp < ntask) {
            const int64_t b0 = tp * W, b1 = b0 + W < nblocks ? b0 + W : nblocks;
            bd_prefetch_l2(codes, b0 * cb, b1 * cb);
        }
    };
    prefetch((int64_t)blockIdx.x * kBdWarps + warp + stride);
    for (int64_t t = (int64_t)blockIdx.x * kBdWarps + warp; t < ntask; t += stride) {
        prefetch(t + 2 * stride);
        const int64_t blk = t * W + bi;
        const bool on = lane_on && blk < nblocks;
        uint32_t w[PW];
        float n16 = 0.0f;
        if (on) {
            load_bytes<4 * PW>(codes + (blk * C + c) * (4 * PW), w);
            n16 = h16_to_f32(__ldg(norms + blk));
        } else {
#pragma unroll
            for (int k = 0; k < PW; ++k) w[k] = 0u;
        }
        float2 P[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            if constexpr (kPairs) {
                const uint32_t e = unpack_code<32, 2 * PW>(w, k);     // codes of values 2k (low) and 2k+1
                const uint2 v = lds64(ptab_lane + e * 128u);
                P[k] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
            } else {
                const int b0 = 2 * k * PW, b1 = b0 + PW;
                uint32_t c0 = w[b0 >> 5] >> (b0 & 31), c1 = w[b1 >> 5] >> (b1 & 31);
                if ((b0 & 31) + PW > 32) c0 |= w[(b0 >> 5) + 1] << (32 - (b0 & 31));
                if ((b1 & 31) + PW > 32) c1 |= w[(b1 >> 5) + 1] << (32 - (b1 & 31));
                P[k] = make_float2(cent[c0 & kMask], cent[c1 & kMask]);
            }
        }
        bd_fwht32(P);
        bd_fwht_cross(P, q, nk_max, lane, on);
        const float sc = __fmul_rn(n16, hs);
        const float2 sc2 = make_float2(sc, sc);
        uint32_t o[16];
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
            const uint4 m = lds128(pm + 16u * k4);                   // signs after rounding: negation is exact
            const uint32_t mm[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 xh = __fmul2_rn(P[4 * k4 + j], sc2);
                o[4 * k4 + j] = pack2<BF16>(xh.x, xh.y) ^ mm[j];
            }
        }
        if (on) store_bytes<64>(reinterpret_cast<uint8_t *>(out + blk * d + 32 * c), o);
    }
}

}  // namespace rq
