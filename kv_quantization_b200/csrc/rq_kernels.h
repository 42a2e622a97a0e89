// rq_kernels.h -- internal launch interface between the C-ABI layer and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
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
    CUtensorMap tmap_x;        // input as [n/64][64] 16-bit rows, 256-row boxes, 128-byte swizzle
    CUtensorMap tmap_v;        // input as {64, d/64, n/d} blocks, {64, 1, 128} boxes (tensor-core A layout)
    bool has_tmap_v;
    CUtensorMap tmap_v32;      // the same view with {64, 1, 32} boxes (one warp's 32-block chunk)
    bool has_tmap_v32;
    CUtensorMap tmap_s;        // S [m][d] 16-bit with {64, min(256, m16)} boxes (d = 512: S streamed)
    bool has_tmap_s;
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
    CUtensorMap tmap_out;      // output as [n/64][64] 16-bit rows, 256-row boxes, 128-byte swizzle
    CUtensorMap tmap_out32;    // output as {64, d/64, n/d} blocks, {64, 1, 32} boxes
    bool has_tmap_out32;
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
    CUtensorMap tmap_k;        // keys as {64, d/64, n_vec} 16-bit, {64, 1, 128} boxes, 128-byte swizzle
    bool has_tmap_k;
    CUtensorMap tmap_s;        // S as [m][d] 16-bit, {64, rows} boxes, 128-byte swizzle (B layout)
    bool has_tmap_s;
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
    CUtensorMap tmap_scores;   // make_scores_tmap, when has_tmap_scores
    bool has_tmap_scores;
    float *workspace;          // [G][nq][d + m] fp32
    int num_sms;
};

// Launch trace of the calling host thread (rq_last_launch): begin_call()
// empties it at the start of every entry point, note_launch() appends the
// name of a kernel just enqueued.
void begin_call();
void note_launch(const char *kernel);

cudaError_t launch_quantize(const QuantArgs &a, cudaStream_t st);
// Blocks of a size d that is not a power of two (rq_bd.cuh): 64 < d < 512, d % 32 == 0.
// Dense-rotation quantization (rq_dense.cuh), d = 128.
struct DenseArgs {
    int64_t nvec;
    bool bf16;
    int pw;                    // bits per stored code (8 for the int8 layout)
    const QuantTables *tables;
    const uint8_t *codes_in;   // dequantize
    uint8_t *codes;            // quantize
    uint16_t *norms;
    const uint16_t *norms_in;
    uint16_t *out;
    int num_sms;
    CUtensorMap tmap_x;        // blocks as {64, 2, nvec}, {64, 1, 128} boxes (quantize)
    CUtensorMap tmap_pi;       // Pi as [128][128], {64, 128} boxes
    CUtensorMap tmap_out;      // output blocks as {64, 2, nvec}, {64, 1, 128} boxes (dequantize)
};
cudaError_t launch_quantize_dense(const DenseArgs &a, cudaStream_t st);
cudaError_t launch_dequantize_dense(const DenseArgs &a, cudaStream_t st);

// QJL outlier sketch (rq_outlier.cu), d = 128, groups of 32 consecutive vectors.
cudaError_t launch_outlier_prep(const uint16_t *keys, int64_t nvec, int n_out, int m_o, const uint16_t *S,
                                uint16_t *kin, uint8_t *idx, uint8_t *out_signs, uint16_t *out_norms, int num_sms,
                                cudaStream_t st);
cudaError_t launch_outlier_score(const uint16_t *q, int64_t G, int nq, int64_t T, int m_o, int n_out,
                                 const uint16_t *S, const uint8_t *idx, const uint8_t *out_signs,
                                 const uint16_t *out_norms, float *scores, cudaStream_t st);

bool bd_size(int d);
cudaError_t launch_quantize_bd(const QuantArgs &a, cudaStream_t st);
cudaError_t launch_dequantize_bd(const DequantArgs &a, cudaStream_t st);
cudaError_t launch_dequantize(const DequantArgs &a, cudaStream_t st);
cudaError_t launch_projection(uint64_t seed, int m, int d, bool bf16, void *proj, cudaStream_t st);
cudaError_t launch_sketch(const SketchArgs &a, cudaStream_t st);
cudaError_t launch_score(const ScoreArgs &a, cudaStream_t st);
// The tensor-core score prologue alone (workspace rows [q~/||q|| ; Sq/||q||]
// in fp16 and ||q|| in fp32, qjl_score_v2.cuh) for another kernel to consume.
cudaError_t launch_score_prologue(const ScoreArgs &a, bool two, uint16_t *wsB, float *wsN, cudaStream_t st);

// Attention decode over compressed keys and values (qjl_attention.cuh).
struct AttnArgs {
    ScoreArgs k;               // queries, projection, keys (scores / workspace unused)
    const uint8_t *vcodes;     // value codes [G][T] blocks of d
    const uint16_t *vnorms;    // fp16 [G][T]
    int vpw;                   // value code field width (bits, or 8 for int8)
    const QuantTables *vtables;
    float softmax_scale;
    float *out;                // fp32 [G][nq][d]
    void *workspace;
    int num_sms;
};
bool attention_supported(int nq, int d, int m, bool two, int pw, int vpw);
size_t attention_workspace_bytes(int64_t G, int nq, int d, int m, int64_t T, int num_sms);
cudaError_t launch_attention(const AttnArgs &a, cudaStream_t st);
size_t score_workspace_bytes(int64_t G, int nq, int d, int m);
size_t quantize_smem_bytes(int d, bool qjl);
// Encode the [rows][64] 16-bit row view of `ptr` as a TMA map (256-row boxes,
// 128-byte swizzle); false if the driver refuses it.
bool make_rows64_tmap(CUtensorMap *map, const void *ptr, int64_t rows);
// Encode vectors[n][d] (16-bit) as {64, d/64, n} with {64, 1, box_rows} boxes:
// one box is one 64-column region of box_rows vectors (box_rows = 128: the
// tensor-core A layout).
bool make_vectors_tmap(CUtensorMap *map, const void *ptr, int64_t n, int d, int box_rows = 128);
// Encode S[m][d] (16-bit) with {64 columns, box_rows rows} boxes (B operand layout).
bool make_proj_tmap(CUtensorMap *map, const void *ptr, int m, int d, int box_rows);
// fp32 scores [G][nq][T] as a {T, nq, G} map with 32 x 16 x 1 boxes (128-byte
// swizzle), for TMA stores that never cross a group; needs T % 4 == 0.
bool make_scores_tmap(CUtensorMap *map, const void *ptr, int64_t T, int nq, int64_t G);
size_t dequantize_smem_bytes(int d);
// One CTA that waits, at most `polls` times, on an mbarrier nothing arrives
// on, then unwinds as the tensor-core kernels do (rq_probe_bounded_wait).
constexpr uint32_t kProbeMaxPolls = 1u << 20;
cudaError_t launch_wait_probe(uint32_t polls, cudaStream_t st);

}  // namespace rq
