// rq_v5.cuh -- one-block-per-thread quantize / dequantize kernels for d = 128
// (sm_100a), and the saturating-grid LUT the d = 128 kernels share.
//
// Arithmetic is the canonical definition (rq_common.cuh): pairwise fp32 norm,
// radix-2 Walsh-Hadamard stages h = 1, 2, ..., 64 in that order, y = v * (1/n32),
// nearest centroid = #{t_k < y}, x^ = s * (w * (n16/d)), residual r = x - x^32.
//
// Mapping.  A thread owns a whole block of 128 values, held as 64 float2
// P[i] = (v_i, v_{i+64}): Hadamard stages h = 1..32 and all but the top level
// of the pairwise norm are packed f32x2 operations on both halves, stage 64 is
// the add/sub inside each float2, and no value ever crosses a lane.
//
// Nearest centroid.  A saturating grid over the boundary range: fs = sat(y*a+b)
// (one fma.sat), cell = round(fs*k) read from the low mantissa bits of
// fs*k + 1.5*2^23 (one packed fma), a shared-memory entry {boundary inside the
// cell or +inf, #boundaries below the cell} at cell*128 + copy (one integer
// multiply-add), code = base + (y > boundary).  The host checked every cell's
// exact y-interval, so this is the exact count, not an approximation.
//
// Memory.  The 128-value rows of a 32-block chunk arrive by 3-D TMA
// ({64 values, 2 halves, 32 blocks}, 128-byte swizzle: lane r reads row r
// without bank conflicts); every warp runs its own ring of chunks, with no
// barrier shared with other warps; twelve warps per CTA at 168 registers.  (The fused quantize+QJL kernel for d = 128
// is in rq_v6.cuh: with a whole block per thread its loop outgrew the
// instruction cache, so it splits each block over two lanes.)
#pragma once
#include <cuda.h>

#include "rq_qjl_v3.cuh"
#include "rq_v2.cuh"

namespace rq {

constexpr int kW5 = 12;                     // warps per CTA (168 registers each)
constexpr int kNSW5 = 2;                    // per-warp ring depth (quantize)
constexpr uint32_t kChunkBytes5 = 32u * 256u;   // 32 rows x 2 halves x 128 B

__device__ __forceinline__ float fma_sat(float a, float b, float c)
{
    float r;
    asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr)
{
    uint2 v;
    asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr)
{
    uint4 v;
    asm("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

// A shared-memory load the compiler keeps in program order relative to the
// other volatile asm (the mbarrier waits) and never merges with an earlier
// load of the same address: every read of smem that a bulk copy or TMA
// writes asynchronously goes through it, so it cannot be hoisted above the
// wait that guards the data (the plain lds64 / lds128 above are for tables
// written before a __syncthreads, or for addresses computed from such data).
__device__ __forceinline__ uint4 lds128_fresh(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v)
{
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// ------------------------------------------------------------------ LUT

// Plain entries {boundary, base}, 16 copies of each cell (lane % 16 reads its
// own copy, so a half-warp never conflicts).
__device__ __forceinline__ void setup_sat_lut8(const QuantTables &T, uint2 *lut)
{
    for (int i = threadIdx.x; i < T.sat_cells * 16; i += blockDim.x)
        lut[i] = make_uint2(__float_as_uint(T.sat_t[i >> 4]), T.sat_base[i >> 4]);
}

// Fused entries {boundary, base, c[base], c[base + 1]}, 8 copies of each cell
// (an 8-lane quarter-warp never conflicts on a 16-byte load).
__device__ __forceinline__ void setup_sat_lut16(const QuantTables &T, uint4 *lut)
{
    for (int i = threadIdx.x; i < T.sat_cells * 8; i += blockDim.x) {
        const uint32_t base = T.sat_base[i >> 3];
        const uint32_t hi = base + 1 < (uint32_t)T.levels ? base + 1 : base;
        lut[i] = make_uint4(__float_as_uint(T.sat_t[i >> 3]), base, __float_as_uint(T.centroid[base]),
                            __float_as_uint(T.centroid[hi]));
    }
}

struct SatGrid {
    float a, b;
    float2 k2, m2;
    uint32_t off;     // lut + copy offset - bits(magic) * 128 (mod 2^32)
};

__device__ __forceinline__ SatGrid sat_grid(const QuantTables &T, uint32_t lut_smem, uint32_t copy_off)
{
    SatGrid g;
    g.a = T.sat_a;
    g.b = T.sat_b;
    g.k2 = make_float2(T.sat_k, T.sat_k);
    g.m2 = make_float2(kLutMagic, kLutMagic);
    g.off = lut_smem + copy_off - (__float_as_uint(kLutMagic) << 7);
    return g;
}

// Entry addresses of the two coordinates of y.
__device__ __forceinline__ void sat_addr(const SatGrid &G, float2 y, uint32_t &a0, uint32_t &a1)
{
    const float2 fs = make_float2(fma_sat(y.x, G.a, G.b), fma_sat(y.y, G.a, G.b));
    const float2 g = __ffma2_rn(fs, G.k2, G.m2);
    a0 = __float_as_uint(g.x) * 128u + G.off;
    a1 = __float_as_uint(g.y) * 128u + G.off;
}

template <int PW>
__device__ __forceinline__ void put_code(uint32_t *w, int j, uint32_t c)
{
    const int b = j * PW;
    w[b >> 5] |= c << (b & 31);
    if ((b & 31) + PW > 32) w[(b >> 5) + 1] |= c >> (32 - (b & 31));
}

// put_code of base + (y > t) into zeroed fields: the base is added at its
// offset (fields never carry into each other, base + 1 < 2^PW when a
// boundary sits in the cell) and the comparison becomes one predicated add.
template <int PW>
__device__ __forceinline__ void put_code_cmp(uint32_t *w, int j, uint32_t base, float y, float t)
{
    const int b = j * PW;
    if ((b & 31) + PW > 32) {
        put_code<PW>(w, j, base + (y > t ? 1u : 0u));
    } else {
        uint32_t v = w[b >> 5] + (base << (b & 31));
        asm("{\n\t.reg .pred p;\n\t"
            "setp.gt.f32 p, %1, %2;\n\t"
            "@p add.u32 %0, %0, %3;\n\t}"
            : "+r"(v)
            : "f"(y), "f"(t), "r"(1u << (b & 31)));
        w[b >> 5] = v;
    }
}

// ------------------------------------------------------------------ row of 128

// Row `r` of a chunk/tile whose two 64-value halves are regions `half_bytes`
// apart: P[i] = (v_i, v_{i+64}), signs applied on the packed pairs.
template <bool BF16, bool SIGNS>
__device__ __forceinline__ void load_row128(uint32_t tile, uint32_t half_bytes, int r, uint32_t pmask_smem,
                                            float2 *P)
{
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        uint4 lo = lds128_fresh(tile + sw128_offset(r, k));
        uint4 hi = lds128_fresh(tile + half_bytes + sw128_offset(r, k));
        if constexpr (SIGNS) {
            const uint4 ml = lds128_fresh(pmask_smem + 16u * k);
            const uint4 mh = lds128_fresh(pmask_smem + 128u + 16u * k);
            lo.x ^= ml.x; lo.y ^= ml.y; lo.z ^= ml.z; lo.w ^= ml.w;
            hi.x ^= mh.x; hi.y ^= mh.y; hi.z ^= mh.z; hi.w ^= mh.w;
        }
        const uint32_t wl[4] = {lo.x, lo.y, lo.z, lo.w}, wh[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            P[8 * k + e].x = half_of<BF16>(wl[e >> 1], e & 1);
            P[8 * k + e].y = half_of<BF16>(wh[e >> 1], e & 1);
        }
    }
}

// Write bf16/fp16 of P back as row r (signs re-applied on the packed pairs).
template <bool OUT_BF16, bool SIGNS>
__device__ __forceinline__ void store_row128(uint32_t tile, uint32_t half_bytes, int r, uint32_t pmask_smem,
                                             const float2 *P)
{
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        uint4 lo, hi;
        lo.x = pack2<OUT_BF16>(P[8 * k + 0].x, P[8 * k + 1].x);
        lo.y = pack2<OUT_BF16>(P[8 * k + 2].x, P[8 * k + 3].x);
        lo.z = pack2<OUT_BF16>(P[8 * k + 4].x, P[8 * k + 5].x);
        lo.w = pack2<OUT_BF16>(P[8 * k + 6].x, P[8 * k + 7].x);
        hi.x = pack2<OUT_BF16>(P[8 * k + 0].y, P[8 * k + 1].y);
        hi.y = pack2<OUT_BF16>(P[8 * k + 2].y, P[8 * k + 3].y);
        hi.z = pack2<OUT_BF16>(P[8 * k + 4].y, P[8 * k + 5].y);
        hi.w = pack2<OUT_BF16>(P[8 * k + 6].y, P[8 * k + 7].y);
        if constexpr (SIGNS) {
            const uint4 ml = lds128_fresh(pmask_smem + 16u * k);
            const uint4 mh = lds128_fresh(pmask_smem + 128u + 16u * k);
            lo.x ^= ml.x; lo.y ^= ml.y; lo.z ^= ml.z; lo.w ^= ml.w;
            hi.x ^= mh.x; hi.y ^= mh.y; hi.z ^= mh.z; hi.w ^= mh.w;
        }
        sts128(tile + sw128_offset(r, k), lo);
        sts128(tile + half_bytes + sw128_offset(r, k), hi);
    }
}

// Canonical pairwise sum of squares of the 128 values (leaves (2k, 2k+1)),
// reduced as eight aligned 8-leaf subtrees (the same tree, fewer live values).
__device__ __forceinline__ float sumsq128(const float2 *P)
{
    float2 t[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
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
#pragma unroll
    for (int w = 1; w < 8; w *= 2) {
#pragma unroll
        for (int i = 0; i < 8; i += 2 * w) t[i] = __fadd2_rn(t[i], t[i + w]);
    }
    return __fadd_rn(t[0].x, t[0].y);
}

__device__ __forceinline__ void fwht128(float2 *P)
{
    const float2 m1 = make_float2(-1.0f, -1.0f);
#pragma unroll
    for (int h = 1; h < 64; h *= 2) {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            if (i & h) continue;
            const float2 a = P[i], b = P[i + h];
            P[i] = __fadd2_rn(a, b);
            P[i + h] = __ffma2_rn(b, m1, a);
        }
    }
#pragma unroll
    for (int i = 0; i < 64; ++i) {                      // stage h = 64
        const float a = P[i].x, b = P[i].y;
        P[i].x = __fadd_rn(a, b);
        P[i].y = __fsub_rn(a, b);
    }
}

// Codes of P * inv (the plain 8-byte LUT).
template <int PW>
__device__ __forceinline__ void codes128(const float2 *P, float inv, const SatGrid &G, uint32_t *w)
{
    const float2 inv2 = make_float2(inv, inv);
#pragma unroll
    for (int k = 0; k < 4 * PW; ++k) w[k] = 0u;
#pragma unroll
    for (int i = 0; i < 64; ++i) {
        const float2 y = __fmul2_rn(P[i], inv2);
        uint32_t a0, a1;
        sat_addr(G, y, a0, a1);
        const uint2 e0 = lds64(a0), e1 = lds64(a1);
        put_code_cmp<PW>(w, i, e0.y, y.x, __uint_as_float(e0.x));
        put_code_cmp<PW>(w, i + 64, e1.y, y.y, __uint_as_float(e1.x));
    }
}

// Balanced contiguous range of 32-block chunks for this CTA.
__device__ __forceinline__ void cta_chunks(int64_t nchunks, int64_t &c0, int64_t &c1)
{
    c0 = nchunks * (int64_t)blockIdx.x / gridDim.x;
    c1 = nchunks * (int64_t)(blockIdx.x + 1) / gridDim.x;
}

// ------------------------------------------------------------------ quantize

__host__ __device__ inline size_t quantize_v5_smem(const QuantTables &T)
{
    return 1024 + (size_t)kW5 * kNSW5 * kChunkBytes5 + (size_t)T.sat_cells * 128 + 256 + 8 * kW5 * kNSW5;
}

template <int PW, bool BF16, bool SIGNS>
__global__ void __launch_bounds__(kW5 * 32, 1)
quantize_v5_kernel(const __grid_constant__ CUtensorMap tmx, int64_t nblocks, const __grid_constant__ QuantTables T,
                   uint8_t *__restrict__ codes, uint16_t *__restrict__ norms)
{
    constexpr int CB = 16 * PW;                   // code bytes per block
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *ring = base;
    uint8_t *lutb = ring + (size_t)kW5 * kNSW5 * kChunkBytes5;
    uint32_t *pmask = reinterpret_cast<uint32_t *>(lutb + (size_t)T.sat_cells * 128);
    uint64_t *full = reinterpret_cast<uint64_t *>(pmask + 64);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t nchunks = (nblocks + 31) / 32;
    int64_t c0, c1;
    cta_chunks(nchunks, c0, c1);
    if (threadIdx.x == 0) {
        prefetch_tmap(&tmx);
        for (int s = 0; s < kW5 * kNSW5; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
    }
    setup_sat_lut8(T, reinterpret_cast<uint2 *>(lutb));
    setup_pair_masks(T, pmask, 128);
    __syncthreads();

    uint8_t *wring = ring + (size_t)warp * kNSW5 * kChunkBytes5;
    uint64_t *wfull = full + warp * kNSW5;
    auto issue = [&](int64_t j, int s) {
        fence_proxy_async_smem();                   // the slot's earlier generic reads precede the copy
        mbar_arrive_expect_tx(&wfull[s], kChunkBytes5);
        uint8_t *dst = wring + (size_t)s * kChunkBytes5;
        tma_load_3d(dst, &tmx, 0, 0, (int)(j * 32), &wfull[s]);
        tma_load_3d(dst + kChunkBytes5 / 2, &tmx, 0, 1, (int)(j * 32), &wfull[s]);
    };
    if (lane == 0)
        for (int s = 0; s < kNSW5; ++s) {
            const int64_t j = c0 + warp + (int64_t)s * kW5;
            if (j < c1) issue(j, s);
        }
    const SatGrid G = sat_grid(T, smem_u32(lutb), (uint32_t)(lane & 15) * 8u);
    const uint32_t pm = smem_u32(pmask);

    for (int64_t k = 0;; ++k) {
        const int64_t j = c0 + warp + k * kW5;
        if (j >= c1) break;
        const int s = (int)(k % kNSW5);
        if (!mbar_wait(&wfull[s], (uint32_t)((k / kNSW5) & 1))) break;
        float2 P[64];
        load_row128<BF16, SIGNS>(smem_u32(wring + (size_t)s * kChunkBytes5), kChunkBytes5 / 2, lane, pm, P);
        const float n32 = __fsqrt_rn(sumsq128(P));       // every load has been consumed
        __syncwarp();
        if (lane == 0 && j + (int64_t)kNSW5 * kW5 < c1) issue(j + (int64_t)kNSW5 * kW5, s);
        fwht128(P);
        const float inv = n32 > 0.0f ? __frcp_rn(n32) : 0.0f;
        uint32_t w[4 * PW];
        codes128<PW>(P, inv, G, w);
        const int64_t blk = j * 32 + lane;
        if (blk < nblocks) {
            store_bytes<CB>(codes + blk * CB, w);
            norms[blk] = norm_to_h16(n32);
        }
    }
}

// ------------------------------------------------------------------ dequantize

constexpr int kNSD5 = 2;                      // per-warp code ring depth

__host__ __device__ inline int cent_copies5(int levels) { return levels <= 32 ? 32 : 1024 / levels; }

__host__ __device__ inline size_t dequantize_v5_smem(int pw, int levels)
{
    return 1024 + (size_t)kW5 * kChunkBytes5 + (size_t)kW5 * kNSD5 * (512 * pw + 64) +
           (size_t)levels * cent_copies5(levels) * 4 + 256 + 8 * kW5 * kNSD5;
}

template <int PW, bool BF16, bool SIGNS>
__global__ void __launch_bounds__(kW5 * 32, 1)
dequantize_v5_kernel(const uint8_t *__restrict__ codes, const uint16_t *__restrict__ norms, int64_t nblocks,
                     const __grid_constant__ QuantTables T, const __grid_constant__ CUtensorMap tmo)
{
    constexpr int CB = 16 * PW;
    constexpr uint32_t RING = 512u * PW;              // one chunk's codes
    constexpr uint32_t SLOT = RING + 64u;             // ... and its 32 fp16 norms
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *outb = base;                                         // kW5 staging chunks
    uint8_t *cring = outb + (size_t)kW5 * kChunkBytes5;           // kW5 x kNSD5 code chunks
    float *cent = reinterpret_cast<float *>(cring + (size_t)kW5 * kNSD5 * SLOT);
    const int copies = cent_copies5(T.levels);
    uint32_t *pmask = reinterpret_cast<uint32_t *>(cent + T.levels * copies);
    uint64_t *full = reinterpret_cast<uint64_t *>(pmask + 64);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t nchunks = (nblocks + 31) / 32;
    int64_t c0, c1;
    cta_chunks(nchunks, c0, c1);
    if (threadIdx.x == 0) {
        prefetch_tmap(&tmo);
        for (int s = 0; s < kW5 * kNSD5; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
    }
    for (int i = threadIdx.x; i < T.levels * copies; i += blockDim.x) cent[i] = T.centroid[i / copies];
    setup_pair_masks(T, pmask, 128);
    __syncthreads();

    uint8_t *wring = cring + (size_t)warp * kNSD5 * SLOT;
    uint8_t *wout = outb + (size_t)warp * kChunkBytes5;
    uint64_t *wfull = full + warp * kNSD5;
    // the chunk's codes and the whole 16-byte groups of its norms (the norms
    // of a ragged last chunk's remaining blocks are read from global memory)
    auto norm_bytes = [&](int64_t j) -> uint32_t {
        const int64_t nb = nblocks - j * 32 < 32 ? nblocks - j * 32 : 32;
        return (uint32_t)(nb * 2) & ~15u;
    };
    auto issue = [&](int64_t j, int s) {
        const int64_t nb = nblocks - j * 32 < 32 ? nblocks - j * 32 : 32;
        const uint32_t nbytes = norm_bytes(j);
        fence_proxy_async_smem();                   // the slot's earlier generic reads precede the copy
        mbar_arrive_expect_tx(&wfull[s], (uint32_t)(nb * CB) + nbytes);
        bulk_load(wring + (size_t)s * SLOT, codes + j * 32 * CB, (uint32_t)(nb * CB), &wfull[s]);
        if (nbytes) bulk_load(wring + (size_t)s * SLOT + RING, norms + j * 32, nbytes, &wfull[s]);
    };
    if (lane == 0)
        for (int s = 0; s < kNSD5; ++s) {
            const int64_t j = c0 + warp + (int64_t)s * kW5;
            if (j < c1) issue(j, s);
        }
    const uint32_t cent_lane = smem_u32(cent) + (uint32_t)(lane % copies) * 4u;
    const uint32_t cstride = (uint32_t)copies * 4u;
    // An int8-layout byte may exceed the 2^bits table (corrupt input, or the
    // unused lanes of a ragged last chunk): read it modulo 2^bits so that no
    // code can address outside the table.
    const uint32_t cmask = PW == 8 ? (uint32_t)T.levels - 1u : 0xffffffffu;
    const uint32_t pm = smem_u32(pmask);

    for (int64_t k = 0;; ++k) {
        const int64_t j = c0 + warp + k * kW5;
        if (j >= c1) break;
        const int s = (int)(k % kNSD5);
        if (!mbar_wait(&wfull[s], (uint32_t)((k / kNSD5) & 1))) break;
        float nrm;
        {
            const int64_t blk = j * 32 + lane;
            uint16_t h = 0;
            if ((uint32_t)lane * 2u < norm_bytes(j)) {
                asm volatile("ld.shared.u16 %0, [%1];"
                             : "=h"(h)
                             : "r"(smem_u32(wring + (size_t)s * SLOT + RING) + (uint32_t)lane * 2u));
            } else if (blk < nblocks) {
                h = __ldg(norms + blk);
            }
            nrm = h16_to_f32(h);
        }
        uint32_t cw[4 * PW];
        const uint32_t src = smem_u32(wring + (size_t)s * SLOT) + (uint32_t)lane * CB;
#pragma unroll
        for (int q = 0; q < PW; ++q) {
            const uint4 v = lds128_fresh(src + 16u * q);
            cw[4 * q] = v.x; cw[4 * q + 1] = v.y; cw[4 * q + 2] = v.z; cw[4 * q + 3] = v.w;
        }
        float2 P[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            float cx, cy;
            const uint32_t ix = PW == 8 ? unpack_code<128, PW>(cw, i) & cmask : unpack_code<128, PW>(cw, i);
            const uint32_t iy = PW == 8 ? unpack_code<128, PW>(cw, i + 64) & cmask : unpack_code<128, PW>(cw, i + 64);
            asm("ld.shared.f32 %0, [%1];" : "=f"(cx) : "r"(cent_lane + ix * cstride));
            asm("ld.shared.f32 %0, [%1];" : "=f"(cy) : "r"(cent_lane + iy * cstride));
            P[i] = make_float2(cx, cy);
        }
        fwht128(P);
        const float sc = __fmul_rn(nrm, 1.0f / 128.0f);
        const float2 sc2 = make_float2(sc, sc);
#pragma unroll
        for (int i = 0; i < 64; ++i) P[i] = __fmul2_rn(P[i], sc2);
        uint8_t *ob = wout;
        if (lane == 0) bulk_wait_read<0>();              // the previous chunk's store has left ob
        __syncwarp();
        store_row128<BF16, SIGNS>(smem_u32(ob), kChunkBytes5 / 2, lane, pm, P);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_3d(&tmo, 0, 0, (int)(j * 32), ob);
            tma_store_3d(&tmo, 0, 1, (int)(j * 32), ob + kChunkBytes5 / 2);
            bulk_commit();
            // every code and norm read from the slot has been consumed (the
            // staged output depends on them): refill it
            if (j + (int64_t)kNSD5 * kW5 < c1) issue(j + (int64_t)kNSD5 * kW5, s);
        }
    }
    if (lane == 0) bulk_wait<0>();
}

// ------------------------------------------------------------------ dequantize, pair layout
//
// For codes of up to 3 bits (where it measured faster: the 4- and 5-bit pair
// tables are 32 KB and lose more to latency and bank conflicts than the halved
// lookups save) the block is held as 64 float2 Q[i] = (v_2i, v_2i+1):
// the 2*PW-bit field of a value pair indexes a table of centroid pairs (one
// 8-byte load and one field extraction per two values), the Hadamard stage
// h = 1 is the add/sub inside each float2 and h = 2..64 are packed operations
// on the pair index, and the bf16/fp16 output words are the pairs themselves.
// The arithmetic (stage order, roundings) is the canonical one, as above.

__host__ __device__ inline int pair_copies5(int pw) { return pw <= 3 ? 16 : (pw == 4 ? 16 : 4); }

__host__ __device__ inline size_t dequantize_v5p_smem(int pw)
{
    return 1024 + (size_t)kW5 * kChunkBytes5 + (size_t)kW5 * kNSD5 * (512 * pw + 64) +
           ((size_t)1 << (2 * pw)) * pair_copies5(pw) * 8 + 256 + 8 * kW5 * kNSD5;
}

__device__ __forceinline__ void fwht128_pairs(float2 *Q)
{
#pragma unroll
    for (int i = 0; i < 64; ++i) {                      // stage h = 1
        const float a = Q[i].x, b = Q[i].y;
        Q[i].x = __fadd_rn(a, b);
        Q[i].y = __fsub_rn(a, b);
    }
    const float2 m1 = make_float2(-1.0f, -1.0f);
#pragma unroll
    for (int h = 1; h < 64; h *= 2) {                   // stages 2h = 2 .. 64 on the pair index
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            if (i & h) continue;
            const float2 a = Q[i], b = Q[i + h];
            Q[i] = __fadd2_rn(a, b);
            Q[i + h] = __ffma2_rn(b, m1, a);
        }
    }
}

template <bool OUT_BF16, bool SIGNS>
__device__ __forceinline__ void store_row128_pairs(uint32_t tile, uint32_t half_bytes, int r, uint32_t pmask_smem,
                                                   const float2 *Q)
{
#pragma unroll
    for (int k = 0; k < 16; ++k) {                      // 16-byte chunk k = values 8k .. 8k+7
        uint4 v;
        v.x = pack2<OUT_BF16>(Q[4 * k + 0].x, Q[4 * k + 0].y);
        v.y = pack2<OUT_BF16>(Q[4 * k + 1].x, Q[4 * k + 1].y);
        v.z = pack2<OUT_BF16>(Q[4 * k + 2].x, Q[4 * k + 2].y);
        v.w = pack2<OUT_BF16>(Q[4 * k + 3].x, Q[4 * k + 3].y);
        if constexpr (SIGNS) {
            const uint4 mk = lds128_fresh(pmask_smem + 16u * k);
            v.x ^= mk.x; v.y ^= mk.y; v.z ^= mk.z; v.w ^= mk.w;
        }
        sts128(tile + (uint32_t)(k >> 3) * half_bytes + sw128_offset(r, k & 7), v);
    }
}

template <int PW, bool BF16, bool SIGNS>
__global__ void __launch_bounds__(kW5 * 32, 1)
dequantize_v5p_kernel(const uint8_t *__restrict__ codes, const uint16_t *__restrict__ norms, int64_t nblocks,
                      const __grid_constant__ QuantTables T, const __grid_constant__ CUtensorMap tmo)
{
    static_assert(PW <= 5, "pair table of 2^(2 PW) entries");
    constexpr int CB = 16 * PW;
    constexpr uint32_t RING = 512u * PW;              // one chunk's codes
    constexpr uint32_t SLOT = RING + 64u;             // ... and its 32 fp16 norms
    constexpr int NE = 1 << (2 * PW);               // centroid pairs
    constexpr int CP = PW <= 4 ? 16 : 4;            // copies (lane % CP reads its own)
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *outb = base;
    uint8_t *cring = outb + (size_t)kW5 * kChunkBytes5;
    float2 *ptab = reinterpret_cast<float2 *>(cring + (size_t)kW5 * kNSD5 * SLOT);
    uint32_t *pmask = reinterpret_cast<uint32_t *>(ptab + NE * CP);
    uint64_t *full = reinterpret_cast<uint64_t *>(pmask + 64);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t nchunks = (nblocks + 31) / 32;
    int64_t c0, c1;
    cta_chunks(nchunks, c0, c1);
    if (threadIdx.x == 0) {
        prefetch_tmap(&tmo);
        for (int s = 0; s < kW5 * kNSD5; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
    }
    for (int i = threadIdx.x; i < NE * CP; i += blockDim.x) {
        const int e = i / CP;
        ptab[i] = make_float2(T.centroid[e & ((1 << PW) - 1)], T.centroid[e >> PW]);
    }
    setup_pair_masks(T, pmask, 128);
    __syncthreads();

    uint8_t *wring = cring + (size_t)warp * kNSD5 * SLOT;
    uint8_t *wout = outb + (size_t)warp * kChunkBytes5;
    uint64_t *wfull = full + warp * kNSD5;
    // the chunk's codes and the whole 16-byte groups of its norms (the norms
    // of a ragged last chunk's remaining blocks are read from global memory)
    auto norm_bytes = [&](int64_t j) -> uint32_t {
        const int64_t nb = nblocks - j * 32 < 32 ? nblocks - j * 32 : 32;
        return (uint32_t)(nb * 2) & ~15u;
    };
    auto issue = [&](int64_t j, int s) {
        const int64_t nb = nblocks - j * 32 < 32 ? nblocks - j * 32 : 32;
        const uint32_t nbytes = norm_bytes(j);
        fence_proxy_async_smem();                   // the slot's earlier generic reads precede the copy
        mbar_arrive_expect_tx(&wfull[s], (uint32_t)(nb * CB) + nbytes);
        bulk_load(wring + (size_t)s * SLOT, codes + j * 32 * CB, (uint32_t)(nb * CB), &wfull[s]);
        if (nbytes) bulk_load(wring + (size_t)s * SLOT + RING, norms + j * 32, nbytes, &wfull[s]);
    };
    if (lane == 0)
        for (int s = 0; s < kNSD5; ++s) {
            const int64_t j = c0 + warp + (int64_t)s * kW5;
            if (j < c1) issue(j, s);
        }
    const uint32_t ptab_lane = smem_u32(ptab) + (uint32_t)(lane & (CP - 1)) * 8u;
    const uint32_t pm = smem_u32(pmask);

    for (int64_t k = 0;; ++k) {
        const int64_t j = c0 + warp + k * kW5;
        if (j >= c1) break;
        const int s = (int)(k % kNSD5);
        if (!mbar_wait(&wfull[s], (uint32_t)((k / kNSD5) & 1))) break;
        float nrm;
        {
            const int64_t blk = j * 32 + lane;
            uint16_t h = 0;
            if ((uint32_t)lane * 2u < norm_bytes(j)) {
                asm volatile("ld.shared.u16 %0, [%1];"
                             : "=h"(h)
                             : "r"(smem_u32(wring + (size_t)s * SLOT + RING) + (uint32_t)lane * 2u));
            } else if (blk < nblocks) {
                h = __ldg(norms + blk);
            }
            nrm = h16_to_f32(h);
        }
        uint32_t cw[4 * PW];
        const uint32_t src = smem_u32(wring + (size_t)s * SLOT) + (uint32_t)lane * CB;
#pragma unroll
        for (int q = 0; q < PW; ++q) {
            const uint4 v = lds128_fresh(src + 16u * q);
            cw[4 * q] = v.x; cw[4 * q + 1] = v.y; cw[4 * q + 2] = v.z; cw[4 * q + 3] = v.w;
        }
        float2 Q[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            const uint32_t e = unpack_code<64, 2 * PW>(cw, i);         // codes of values 2i (low) and 2i+1
            uint2 v;
            asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(ptab_lane + e * (uint32_t)(CP * 8)));
            Q[i] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
        }
        fwht128_pairs(Q);
        const float sc = __fmul_rn(nrm, 1.0f / 128.0f);
        const float2 sc2 = make_float2(sc, sc);
#pragma unroll
        for (int i = 0; i < 64; ++i) Q[i] = __fmul2_rn(Q[i], sc2);
        uint8_t *ob = wout;
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
        store_row128_pairs<BF16, SIGNS>(smem_u32(ob), kChunkBytes5 / 2, lane, pm, Q);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_3d(&tmo, 0, 0, (int)(j * 32), ob);
            tma_store_3d(&tmo, 0, 1, (int)(j * 32), ob + kChunkBytes5 / 2);
            bulk_commit();
            // every code and norm read from the slot has been consumed (the
            // staged output depends on them): refill it
            if (j + (int64_t)kNSD5 * kW5 < c1) issue(j + (int64_t)kNSD5 * kW5, s);
        }
    }
    if (lane == 0) bulk_wait<0>();
}

}  // namespace rq
