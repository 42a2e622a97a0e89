// rq_dense.cu -- launchers of the dense-rotation kernels (rq_dense.cuh).
#include "rq_dense.cuh"
#include "rq_kernels.h"

namespace rq {

namespace {

template <bool BF16, int PW, int NS>
cudaError_t run_quantize_dense(const DenseArgs &a, cudaStream_t st)
{
    auto kern = quantize_dense_kernel<BF16, PW, NS>;
    const size_t smem = quantize_dense_smem(NS, a.tables->sat_cells);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (a.nvec + 127) / 128;
    const int64_t grid = tiles < (int64_t)a.num_sms ? tiles : (int64_t)a.num_sms;
    kern<<<(unsigned)(grid > 0 ? grid : 1), kDnQWarps * 32, smem, st>>>(a.tmap_x, a.tmap_pi, a.nvec, *a.tables,
                                                                        a.codes, a.norms);
    note_launch("quantize_dense_kernel");
    return cudaGetLastError();
}

template <bool BF16, int PW, int NS>
cudaError_t run_dequantize_dense(const DenseArgs &a, cudaStream_t st)
{
    auto kern = dequantize_dense_kernel<BF16, PW, NS>;
    const size_t smem = dequantize_dense_smem(NS, PW);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (a.nvec + 127) / 128;
    const int64_t grid = tiles < (int64_t)a.num_sms ? tiles : (int64_t)a.num_sms;
    kern<<<(unsigned)(grid > 0 ? grid : 1), kDnDWarps * 32, smem, st>>>(a.tmap_pi, a.tmap_out, a.codes_in, a.norms_in,
                                                                        a.nvec, *a.tables);
    note_launch("dequantize_dense_kernel");
    return cudaGetLastError();
}

template <bool BF16>
cudaError_t quantize_dense_pw(const DenseArgs &a, cudaStream_t st)
{
    switch (a.pw) {
    case 1: return run_quantize_dense<BF16, 1, 4>(a, st);
    case 2: return run_quantize_dense<BF16, 2, 4>(a, st);
    case 3: return run_quantize_dense<BF16, 3, 4>(a, st);
    case 4: return run_quantize_dense<BF16, 4, 4>(a, st);
    case 5: return run_quantize_dense<BF16, 5, 4>(a, st);
    case 6: return run_quantize_dense<BF16, 6, 4>(a, st);
    case 7: return run_quantize_dense<BF16, 7, 4>(a, st);
    case 8: return run_quantize_dense<BF16, 8, 4>(a, st);
    default: return cudaErrorNotSupported;
    }
}

template <bool BF16>
cudaError_t dequantize_dense_pw(const DenseArgs &a, cudaStream_t st)
{
    switch (a.pw) {
    case 1: return run_dequantize_dense<BF16, 1, 3>(a, st);
    case 2: return run_dequantize_dense<BF16, 2, 3>(a, st);
    case 3: return run_dequantize_dense<BF16, 3, 3>(a, st);
    case 4: return run_dequantize_dense<BF16, 4, 3>(a, st);
    case 5: return run_dequantize_dense<BF16, 5, 3>(a, st);
    case 6: return run_dequantize_dense<BF16, 6, 3>(a, st);
    case 7: return run_dequantize_dense<BF16, 7, 3>(a, st);
    case 8: return run_dequantize_dense<BF16, 8, 3>(a, st);
    default: return cudaErrorNotSupported;
    }
}

}  // namespace

cudaError_t launch_quantize_dense(const DenseArgs &a, cudaStream_t st)
{
    return a.bf16 ? quantize_dense_pw<true>(a, st) : quantize_dense_pw<false>(a, st);
}

cudaError_t launch_dequantize_dense(const DenseArgs &a, cudaStream_t st)
{
    return a.bf16 ? dequantize_dense_pw<true>(a, st) : dequantize_dense_pw<false>(a, st);
}

}  // namespace rq
