// rq_quant_inst.cuh -- instantiates the quantize / dequantize / sketch kernels
// for one block size RQ_D and one dtype RQ_BF16 (set by the including file),
// so that the heavy fully unrolled kernels compile in parallel units.
#include "rq_quant_impl.cuh"
#include "rq_qjl_mma.cuh"
#include "rq_v2.cuh"
#include "rq_qjl_v2.cuh"
#include "rq_qjl_v3.cuh"
#include "rq_v5.cuh"
#include "rq_v6.cuh"
#include "rq_v7.cuh"
#include "rq_v8.cuh"
#include "rq_sketch_v3.cuh"

namespace rq {

template <int D, int PW, bool BF16, bool QJL>
static cudaError_t launch_q(const QuantArgs &a, cudaStream_t st)
{
    auto kern = quantize_kernel<D, PW, BF16, QJL>;
    const size_t smem = quantize_smem_bytes(D, QJL);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    constexpr int E = D < 128 ? D : 128;
    const int64_t rows = a.nblocks * (D / E);
    const int64_t tiles = (rows + kThreads - 1) / kThreads;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
    if (e != cudaSuccess) return e;
    const int64_t cap = (int64_t)a.num_sms * (per_sm > 0 ? per_sm : 1);
    const int64_t grid = tiles < cap ? tiles : cap;
    kern<<<(unsigned)(grid > 0 ? grid : 1), kThreads, smem, st>>>(
        static_cast<const uint8_t *>(a.x), a.nblocks, *a.tables, static_cast<uint8_t *>(a.codes), a.norms,
        a.m, static_cast<const uint16_t *>(a.proj), a.qsigns, a.qnorms);
    note_launch("quantize_kernel");
    return cudaGetLastError();
}

// Tensor-core sketch path when S and the tiles fit in shared memory; returns
// cudaErrorNotSupported when they do not (the caller then takes the SIMT path).
template <int D, int PW, bool BF16, int MODE>
static cudaError_t launch_mma(const QuantTables &T, const void *x, int64_t nvec, void *codes, uint16_t *norms,
                              int m, const void *proj, uint8_t *signs, uint16_t *snorms, int num_sms, cudaStream_t st)
{
    const size_t smem = qjl_mma_smem_bytes(D, PW, m, T, MODE);
    if (smem > kMaxSmemPerBlock) return cudaErrorNotSupported;
    auto kern = qjl_mma_kernel<D, PW, BF16, MODE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (nvec + 127) / 128;
    const int64_t grid = tiles < (int64_t)num_sms ? tiles : (int64_t)num_sms;
    kern<<<(unsigned)(grid > 0 ? grid : 1), kThreads, smem, st>>>(
        static_cast<const uint8_t *>(x), nvec, T, static_cast<uint8_t *>(codes), norms, m,
        static_cast<const uint16_t *>(proj), signs, snorms);
    note_launch(MODE == 0 ? "qjl_mma_kernel<fused>" : "qjl_mma_kernel<sketch>");
    return cudaGetLastError();
}

// In-place pipelined fused quantize + sketch (rq_qjl_v3.cuh) for d = 128 / 256;
// NotSupported when the shape or the shared memory does not fit.
template <int D, int PW, bool BF16, int NS>
static cudaError_t launch_qjl_v3_ns(const QuantArgs &a, size_t smem, cudaStream_t st)
{
    auto kern = qjl_v3_quant_kernel<D, PW, BF16, NS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (a.nblocks + 127) / 128;
    const int64_t grid = tiles < (int64_t)a.num_sms ? tiles : (int64_t)a.num_sms;
    kern<<<(unsigned)(grid > 0 ? grid : 1), kT2, smem, st>>>(a.tmap_v, a.nblocks, *a.tables,
                                                            static_cast<uint8_t *>(a.codes), a.norms, a.m,
                                                            static_cast<const uint16_t *>(a.proj), a.qsigns, a.qnorms);
    note_launch("qjl_v3_quant_kernel");
    return cudaGetLastError();
}

template <int D, int PW, bool BF16>
static cudaError_t launch_qjl_v3(const QuantArgs &a, cudaStream_t st)
{
    if constexpr (D != 128 && D != 256) {
        return cudaErrorNotSupported;
    } else {
        if (!a.has_tmap_v || 2 * qjl_mma_m16(a.m) > 512) return cudaErrorNotSupported;
        size_t smem = qjl_v3_smem(D, PW, a.m, *a.tables, 5);
        if (smem <= kMaxSmemPerBlock) return launch_qjl_v3_ns<D, PW, BF16, 5>(a, smem, st);
        smem = qjl_v3_smem(D, PW, a.m, *a.tables, 3);
        if (smem <= kMaxSmemPerBlock) return launch_qjl_v3_ns<D, PW, BF16, 3>(a, smem, st);
        smem = qjl_v3_smem(D, PW, a.m, *a.tables, 1);
        if (smem <= kMaxSmemPerBlock) return launch_qjl_v3_ns<D, PW, BF16, 1>(a, smem, st);
        return cudaErrorNotSupported;
    }
}

template <bool BF16>
static cudaError_t launch_sketch_v3(const SketchArgs &a, cudaStream_t st)
{
    if (!a.has_tmap_k || !a.has_tmap_s || 2 * qjl_mma_m16(a.m) > 512) return cudaErrorNotSupported;
    const int64_t tiles = (a.nvec + 127) / 128;
    const int64_t grid = tiles < (int64_t)a.num_sms ? tiles : (int64_t)a.num_sms;
    size_t smem = sketch_v3_smem(a.m, 5);
    auto kern = sketch_v3_kernel<BF16, 5>;
    if (smem > kMaxSmemPerBlock) {
        smem = sketch_v3_smem(a.m, 3);
        kern = sketch_v3_kernel<BF16, 3>;
    }
    if (smem > kMaxSmemPerBlock) return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(grid > 0 ? grid : 1), kSk3Warps * 32, smem, st>>>(a.tmap_k, a.tmap_s, a.nvec, a.m, a.signs,
                                                                        a.norms);
    note_launch("sketch_v3_kernel");
    return cudaGetLastError();
}

template <int D, int PW, bool BF16>
static cudaError_t launch_q2(const QuantArgs &a, cudaStream_t st)
{
    auto kern = quantize_v2_kernel<D, PW, BF16>;
    const size_t smem = quantize_v2_smem(D, *a.tables);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t rows = a.nblocks * (D / kE2);
    const int64_t tiles = (rows + kT2 - 1) / kT2;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kT2, smem);
    if (e != cudaSuccess) return e;
    const int64_t cap = (int64_t)a.num_sms * (per_sm > 0 ? per_sm : 1);
    const int64_t grid = tiles < cap ? tiles : cap;
    kern<<<(unsigned)(grid > 0 ? grid : 1), kT2, smem, st>>>(a.tmap_x, rows, *a.tables,
                                                            static_cast<uint8_t *>(a.codes), a.norms);
    note_launch("quantize_v2_kernel");
    return cudaGetLastError();
}

template <int D, int PW, bool BF16>
static cudaError_t launch_dq2(const DequantArgs &a, cudaStream_t st)
{
    auto kern = dequantize_v2_kernel<D, PW, BF16>;
    const size_t smem = dequantize_v2_smem(D, PW);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t rows = a.nblocks * (D / kE2);
    const int64_t tiles = (rows + kT2 - 1) / kT2;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kT2, smem);
    if (e != cudaSuccess) return e;
    const int64_t cap = (int64_t)a.num_sms * (per_sm > 0 ? per_sm : 1);
    const int64_t grid = tiles < cap ? tiles : cap;
    kern<<<(unsigned)(grid > 0 ? grid : 1), kT2, smem, st>>>(static_cast<const uint8_t *>(a.codes), a.norms, rows,
                                                            *a.tables, a.tmap_out);
    note_launch("dequantize_v2_kernel");
    return cudaGetLastError();
}

template <int D, bool BF16>
static cudaError_t launch_sk(const SketchArgs &a, cudaStream_t st)
{
    auto kern = sketch_kernel<D, BF16>;
    constexpr int E = D < 128 ? D : 128;
    const size_t smem = (size_t)kThreads * E * 2;
    const int64_t rows = a.nvec * (D / E);
    const int64_t tiles = (rows + kThreads - 1) / kThreads;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
    if (e != cudaSuccess) return e;
    const int64_t cap = (int64_t)a.num_sms * (per_sm > 0 ? per_sm : 1);
    const int64_t grid = tiles < cap ? tiles : cap;
    kern<<<(unsigned)(grid > 0 ? grid : 1), kThreads, smem, st>>>(
        static_cast<const uint8_t *>(a.x), a.nvec, a.m, static_cast<const uint16_t *>(a.proj), a.signs, a.norms);
    note_launch("sketch_kernel");
    return cudaGetLastError();
}

// d = 128 kernels of rq_v5.cuh / rq_v6.cuh; NotSupported when the saturating
// grid or the shared memory does not fit (the caller then takes the older
// general-d kernels).

template <int D, int PW, bool BF16>
static cudaError_t launch_q5(const QuantArgs &a, cudaStream_t st)
{
    if constexpr (D != 128) {
        return cudaErrorNotSupported;
    } else {
        if (!a.has_tmap_v32 || a.tables->sat_cells <= 0) return cudaErrorNotSupported;
        const size_t smem = quantize_v5_smem(*a.tables);
        if (smem > kMaxSmemPerBlock) return cudaErrorNotSupported;
        const bool signs = a.tables->sign_words[0] | a.tables->sign_words[1] | a.tables->sign_words[2] |
                           a.tables->sign_words[3];
        auto kern = signs ? quantize_v5_kernel<PW, BF16, true> : quantize_v5_kernel<PW, BF16, false>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        const int64_t chunks = (a.nblocks + 31) / 32;
        const int64_t want = (chunks + kW5 - 1) / kW5;
        const int64_t grid = want < (int64_t)a.num_sms ? want : (int64_t)a.num_sms;
        kern<<<(unsigned)(grid > 0 ? grid : 1), kW5 * 32, smem, st>>>(a.tmap_v32, a.nblocks, *a.tables,
                                                                     static_cast<uint8_t *>(a.codes), a.norms);
        note_launch("quantize_v5_kernel");
        return cudaGetLastError();
    }
}

template <int D, int PW, bool BF16>
static cudaError_t launch_dq5(const DequantArgs &a, cudaStream_t st)
{
    if constexpr (D != 128) {
        return cudaErrorNotSupported;
    } else {
        if (!a.has_tmap_out32) return cudaErrorNotSupported;
        const bool signs = a.tables->sign_words[0] | a.tables->sign_words[1] | a.tables->sign_words[2] |
                           a.tables->sign_words[3];
        if constexpr (PW <= 4) {                    // pair layout (rq_v5.cuh): measured faster up to 4 bits
            const size_t smemp = dequantize_v5p_smem(PW);
            if (smemp <= kMaxSmemPerBlock && a.tables->levels == (1 << PW)) {
                auto kp = signs ? dequantize_v5p_kernel<PW, BF16, true> : dequantize_v5p_kernel<PW, BF16, false>;
                cudaError_t e = cudaFuncSetAttribute(kp, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smemp);
                if (e != cudaSuccess) return e;
                const int64_t chunks = (a.nblocks + 31) / 32;
                const int64_t want = (chunks + kW5 - 1) / kW5;
                const int64_t grid = want < (int64_t)a.num_sms ? want : (int64_t)a.num_sms;
                kp<<<(unsigned)(grid > 0 ? grid : 1), kW5 * 32, smemp, st>>>(
                    static_cast<const uint8_t *>(a.codes), a.norms, a.nblocks, *a.tables, a.tmap_out32);
                note_launch("dequantize_v5p_kernel");
                return cudaGetLastError();
            }
        }
        const size_t smem = dequantize_v5_smem(PW, a.tables->levels);
        if (smem > kMaxSmemPerBlock) return cudaErrorNotSupported;
        auto kern = signs ? dequantize_v5_kernel<PW, BF16, true> : dequantize_v5_kernel<PW, BF16, false>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        const int64_t chunks = (a.nblocks + 31) / 32;
        const int64_t want = (chunks + kW5 - 1) / kW5;
        const int64_t grid = want < (int64_t)a.num_sms ? want : (int64_t)a.num_sms;
        kern<<<(unsigned)(grid > 0 ? grid : 1), kW5 * 32, smem, st>>>(static_cast<const uint8_t *>(a.codes),
                                                                     a.norms, a.nblocks, *a.tables, a.tmap_out32);
        note_launch("dequantize_v5_kernel");
        return cudaGetLastError();
    }
}

template <int D, int PW, bool BF16>
static cudaError_t launch_qjl8(const QuantArgs &a, cudaStream_t st)
{
    if constexpr (D != 512) {
        return cudaErrorNotSupported;
    } else {
        if (!a.has_tmap_v || !a.has_tmap_s || a.tables->sat_cells <= 0 || qjl_mma_m16(a.m) > 512)
            return cudaErrorNotSupported;
        const size_t smem = qjl_v8_smem(*a.tables);
        if (smem > kMaxSmemPerBlock) return cudaErrorNotSupported;
        bool signs = false;
        for (int i = 0; i < 16; ++i) signs = signs || a.tables->sign_words[i] != 0u;
        auto kern = signs ? qjl_v8_quant_kernel<PW, BF16, true> : qjl_v8_quant_kernel<PW, BF16, false>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        const int64_t tiles = (a.nblocks + 127) / 128;
        const int64_t grid = tiles < (int64_t)a.num_sms ? tiles : (int64_t)a.num_sms;
        kern<<<(unsigned)(grid > 0 ? grid : 1), kW8 * 32, smem, st>>>(
            a.tmap_v, a.tmap_s, a.nblocks, *a.tables, static_cast<uint8_t *>(a.codes), a.norms, a.m, a.qsigns,
            a.qnorms);
        note_launch("qjl_v8_quant_kernel");
        return cudaGetLastError();
    }
}

template <int D, int PW, bool BF16>
static cudaError_t launch_qjl7(const QuantArgs &a, cudaStream_t st)
{
    if constexpr (D != 256) {
        return cudaErrorNotSupported;
    } else {
        if (!a.has_tmap_v || !a.has_tmap_s || a.tables->sat_cells <= 0) return cudaErrorNotSupported;
        if ((size_t)qjl_v7_nacc(a.m) * qjl_mma_m16(a.m) > 512) return cudaErrorNotSupported;
        const size_t smem = qjl_v7_smem(a.m, *a.tables);
        if (smem > kMaxSmemPerBlock) return cudaErrorNotSupported;
        bool signs = false;
        for (int i = 0; i < 8; ++i) signs = signs || a.tables->sign_words[i] != 0u;
        auto kern = signs ? qjl_v7_quant_kernel<PW, BF16, true> : qjl_v7_quant_kernel<PW, BF16, false>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        const int64_t tiles = (a.nblocks + 127) / 128;
        const int64_t grid = tiles < (int64_t)a.num_sms ? tiles : (int64_t)a.num_sms;
        kern<<<(unsigned)(grid > 0 ? grid : 1), kW7 * 32, smem, st>>>(
            a.tmap_v, a.nblocks, *a.tables, static_cast<uint8_t *>(a.codes), a.norms, a.m,
            a.tmap_s, a.qsigns, a.qnorms);
        note_launch("qjl_v7_quant_kernel");
        return cudaGetLastError();
    }
}

template <int D, int PW, bool BF16>
static cudaError_t launch_qjl6(const QuantArgs &a, cudaStream_t st)
{
    if constexpr (D != 128) {
        return cudaErrorNotSupported;
    } else {
        if (!a.has_tmap_v || !a.has_tmap_s || a.tables->sat_cells <= 0) return cudaErrorNotSupported;
        if ((size_t)kGroups6 * qjl_v6_nacc(a.m) * qjl_mma_m16(a.m) > 512) return cudaErrorNotSupported;
        const size_t smem = qjl_v6_smem(a.m, *a.tables);
        if (smem > kMaxSmemPerBlock) return cudaErrorNotSupported;
        const bool signs = a.tables->sign_words[0] | a.tables->sign_words[1] | a.tables->sign_words[2] |
                           a.tables->sign_words[3];
        auto kern = signs ? qjl_v6_quant_kernel<PW, BF16, true> : qjl_v6_quant_kernel<PW, BF16, false>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        const int64_t tiles = (a.nblocks + 127) / 128;
        const int64_t want = (tiles + kGroups6 - 1) / kGroups6;
        const int64_t grid = want < (int64_t)a.num_sms ? want : (int64_t)a.num_sms;
        kern<<<(unsigned)(grid > 0 ? grid : 1), kW6 * 32, smem, st>>>(
            a.tmap_v, a.nblocks, *a.tables, static_cast<uint8_t *>(a.codes), a.norms, a.m,
            a.tmap_s, a.qsigns, a.qnorms);
        note_launch("qjl_v6_quant_kernel");
        return cudaGetLastError();
    }
}

#define RQ_CAT2(a, b, c) a##_d##b##_##c
#define RQ_CAT(a, b, c) RQ_CAT2(a, b, c)
#if RQ_BF16
#define RQ_DT bf16
#else
#define RQ_DT f16
#endif

cudaError_t RQ_CAT(launch_quantize, RQ_D, RQ_DT)(const QuantArgs &a, cudaStream_t st)
{
    const bool qjl = a.qsigns != nullptr;
#define RQ_CASE(PW)                                                                                       \
    case PW:                                                                                              \
        if (qjl) {                                                                                        \
            {                                                                                             \
                cudaError_t e8 = launch_qjl8<RQ_D, PW, RQ_BF16>(a, st);                                   \
                if (e8 != cudaErrorNotSupported) return e8;                                               \
                cudaError_t e7 = launch_qjl7<RQ_D, PW, RQ_BF16>(a, st);                                   \
                if (e7 != cudaErrorNotSupported) return e7;                                               \
                cudaError_t e6 = launch_qjl6<RQ_D, PW, RQ_BF16>(a, st);                                   \
                if (e6 != cudaErrorNotSupported) return e6;                                               \
                cudaError_t e2 = launch_qjl_v3<RQ_D, PW, RQ_BF16>(a, st);                                 \
                if (e2 != cudaErrorNotSupported) return e2;                                               \
            }                                                                                             \
            cudaError_t e = launch_mma<RQ_D, PW, RQ_BF16, 0>(*a.tables, a.x, a.nblocks, a.codes, a.norms, a.m, \
                                                             a.proj, a.qsigns, a.qnorms, a.num_sms, st);  \
            if (e != cudaErrorNotSupported) return e;                                                     \
            return launch_q<RQ_D, PW, RQ_BF16, true>(a, st);                                               \
        }                                                                                                 \
        {                                                                                                 \
            cudaError_t e5 = launch_q5<RQ_D, PW, RQ_BF16>(a, st);                                         \
            if (e5 != cudaErrorNotSupported) return e5;                                                   \
        }                                                                                                 \
        return launch_q2<RQ_D, PW, RQ_BF16>(a, st);
    switch (a.pw) {
    RQ_CASE(1) RQ_CASE(2) RQ_CASE(3) RQ_CASE(4) RQ_CASE(5) RQ_CASE(6) RQ_CASE(7) RQ_CASE(8)
    default: return cudaErrorInvalidValue;
    }
#undef RQ_CASE
}

cudaError_t RQ_CAT(launch_dequantize, RQ_D, RQ_DT)(const DequantArgs &a, cudaStream_t st)
{
#define RQ_CASE(PW)                                                                                       \
    case PW: {                                                                                            \
        cudaError_t e5 = launch_dq5<RQ_D, PW, RQ_BF16>(a, st);                                            \
        if (e5 != cudaErrorNotSupported) return e5;                                                       \
        return launch_dq2<RQ_D, PW, RQ_BF16>(a, st);                                                      \
    }
    switch (a.pw) {
    RQ_CASE(1) RQ_CASE(2) RQ_CASE(3) RQ_CASE(4) RQ_CASE(5) RQ_CASE(6) RQ_CASE(7) RQ_CASE(8)
    default: return cudaErrorInvalidValue;
    }
#undef RQ_CASE
}

cudaError_t RQ_CAT(launch_sketch, RQ_D, RQ_DT)(const SketchArgs &a, cudaStream_t st)
{
    if (RQ_D == 128) {
        cudaError_t e3 = launch_sketch_v3<RQ_BF16>(a, st);
        if (e3 != cudaErrorNotSupported) return e3;
    }
    QuantTables T{};
    cudaError_t e = launch_mma<RQ_D, 1, RQ_BF16, 1>(T, a.x, a.nvec, nullptr, nullptr, a.m, a.proj, a.signs, a.norms,
                                                    a.num_sms, st);
    if (e != cudaErrorNotSupported) return e;
    return launch_sk<RQ_D, RQ_BF16>(a, st);
}

}  // namespace rq
