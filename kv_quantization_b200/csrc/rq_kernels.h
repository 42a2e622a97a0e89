// rq_kernels.h -- internal launch interface between the C-ABI layer and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "rq_params.h"

namespace rq {

struct QuantArgs {
    const void *x;
    int64_t nblocks;
    int d, pw;                 // block size, bits per stored code (8 for the int8 layout)
    bool bf16;
    const QuantTables *tables;
    void *codes;
    uint16_t *norms;
    int m;                     // fused QJL residual sketch (qsigns != nullptr)
    const void *proj;
    uint8_t *qsigns;
    uint16_t *qnorms;
    int num_sms;
};

struct DequantArgs {
    const void *codes;
    const uint16_t *norms;
    int64_t nblocks;
    int d, pw;
    bool bf16;                 // output dtype
    const QuantTables *tables;
    void *out;
    int num_sms;
};

struct SketchArgs {
    const void *x;
    int64_t nvec;
    int d, m;
    bool bf16;
    const void *proj;
    uint8_t *signs;
    uint16_t *norms;
    int num_sms;
};

struct ScoreArgs {
    const uint16_t *q;         // bf16 [G][nq][d]
    int64_t G;
    int nq, d, m;
    const void *proj;
    bool proj_bf16;
    const uint8_t *signs;      // [G][T][m/8]
    const uint16_t *sk_norms;  // [G][T]
    int64_t T;
    const uint8_t *codes;      // [G][T] blocks, or nullptr
    const uint16_t *norms;
    int pw;
    const QuantTables *tables;
    float *scores;             // [G][nq][T]
    float *workspace;          // [G][nq][d + m] fp32
    int num_sms;
};

cudaError_t launch_quantize(const QuantArgs &a, cudaStream_t st);
cudaError_t launch_dequantize(const DequantArgs &a, cudaStream_t st);
cudaError_t launch_projection(uint64_t seed, int m, int d, bool bf16, void *proj, cudaStream_t st);
cudaError_t launch_sketch(const SketchArgs &a, cudaStream_t st);
cudaError_t launch_score(const ScoreArgs &a, cudaStream_t st);
size_t score_workspace_bytes(int64_t G, int nq, int d, int m);
size_t quantize_smem_bytes(int d, bool qjl);
size_t dequantize_smem_bytes(int d);

}  // namespace rq
