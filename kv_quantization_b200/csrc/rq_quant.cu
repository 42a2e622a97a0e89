// rq_quant.cu -- dispatch of quantize / dequantize / sketch launches to the
// per-(block size, dtype) instantiation units rq_quant_d*_*.cu.
#include "rq_kernels.h"
#include "rq_quant_impl.cuh"

namespace rq {

#define RQ_DECL(D, DT)                                                              \
    cudaError_t launch_quantize_d##D##_##DT(const QuantArgs &, cudaStream_t);       \
    cudaError_t launch_dequantize_d##D##_##DT(const DequantArgs &, cudaStream_t);   \
    cudaError_t launch_sketch_d##D##_##DT(const SketchArgs &, cudaStream_t);
RQ_DECL(64, f16) RQ_DECL(64, bf16) RQ_DECL(128, f16) RQ_DECL(128, bf16)
RQ_DECL(256, f16) RQ_DECL(256, bf16) RQ_DECL(512, f16) RQ_DECL(512, bf16)
#undef RQ_DECL

#define RQ_DISPATCH(FN, a, st)                                                      \
    switch (a.d) {                                                                  \
    case 64: return a.bf16 ? FN##_d64_bf16(a, st) : FN##_d64_f16(a, st);            \
    case 128: return a.bf16 ? FN##_d128_bf16(a, st) : FN##_d128_f16(a, st);         \
    case 256: return a.bf16 ? FN##_d256_bf16(a, st) : FN##_d256_f16(a, st);         \
    case 512: return a.bf16 ? FN##_d512_bf16(a, st) : FN##_d512_f16(a, st);         \
    default: return cudaErrorInvalidValue;                                          \
    }

cudaError_t launch_quantize(const QuantArgs &a, cudaStream_t st) { RQ_DISPATCH(launch_quantize, a, st) }
cudaError_t launch_dequantize(const DequantArgs &a, cudaStream_t st) { RQ_DISPATCH(launch_dequantize, a, st) }
cudaError_t launch_sketch(const SketchArgs &a, cudaStream_t st) { RQ_DISPATCH(launch_sketch, a, st) }

size_t quantize_smem_bytes(int d, bool qjl)
{
    const int E = d < 128 ? d : 128;
    return (size_t)kThreads * E * 2 + (size_t)kMaxLutCells * 16 * 8 + (qjl ? (size_t)kMaxLevels * 32 * 4 : 0);
}

size_t dequantize_smem_bytes(int d)
{
    const int E = d < 128 ? d : 128;
    return (size_t)kThreads * E * 2 + (size_t)kMaxLevels * 32 * 4;
}

}  // namespace rq
