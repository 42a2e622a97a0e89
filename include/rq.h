/*
 * rq.h -- C ABI of librq: blockwise rotated scalar quantization and the QJL
 * 1-bit sketch on NVIDIA B200 (sm_100a).
 *
 * Operations (sources: the eliza quantization README, sections "PolarQuant",
 * "TurboQuant" and "QJL", each "Algorithm in one paragraph"; the qjl_apply.py
 * source text, `_build_jl_projections` and `_qjl_decode_keys`; the turbopress
 * 0.4.2 project description, "Package layout" and "Findings"):
 *
 *   quantize    x (blocks of d contiguous values) -> per-block fp16 L2 norm and
 *               per-coordinate index of the nearest centroid of
 *               y = H D x / ||x||, H the d x d Sylvester Hadamard matrix (unnormalised,
 *               so y is the orthonormal rotation of x/||x|| scaled by sqrt(d)), D an
 *               optional seeded +-1 diagonal.
 *   dequantize  codes, norms -> x^ = n16 * D * H c / d, c_j = centroid[code_j]
 *               (centroid lookup, divide by sqrt(d), inverse rotation, rescale).
 *   QJL sketch  v -> sign(S v) packed 8 per byte and fp16 ||v||, S an m x d
 *               seeded Gaussian matrix.
 *   QJL score   <q, k> ~ (n16/d) <H D q, c> + sqrt(pi/2)/m * ||r|| * <S q, sign(S r)>
 *               (first term only when the key carries a first-stage code).
 *
 * Conventions shared by every entry point
 *   - Pointers named x, codes, norms, out, proj, signs, scores, q and workspace
 *     are DEVICE pointers owned by the caller; `centroids` is a HOST pointer.
 *     The library keeps no pointer after a call returns and allocates no
 *     device memory.  Its only global state: one device error word
 *     (rq_device_error), the fixed scratch array of qjl_score_noalloc, and a
 *     mutex-guarded host cache of the last few per-call lookup tables (a pure
 *     function of centroids, bits, d and the sign seed).
 *   - Every call validates its arguments on the host, then enqueues its
 *     kernels asynchronously on `stream` (0 = legacy default stream) and
 *     returns.  Kernel faults surface at the caller's next synchronisation.
 *   - Return value: RQ_OK or a negative rq_status; on error nothing is enqueued.
 *   - Device pointers must be 16-byte aligned.
 *   - d (block size / head dim) is a power of two in {64, 128, 256, 512}: the
 *     PolarQuant section's knob list restricts its block size to powers of two,
 *     and the Fused TurboQuant section's compatibility constraints restrict the
 *     butterfly Hadamard to power-of-two head dims.  n must be a multiple of d.
 *   - Arithmetic is fp32 in one canonical order so results are reproducible
 *     bit for bit: the norm is the pairwise (recursive halving) fp32 sum of
 *     fp32 squares with a correctly rounded sqrt; the Hadamard transform runs
 *     radix-2 stages h = 1, 2, ..., d/2; y_j = v_j * (1/n32) (y = 0 when n32 = 0);
 *     code = #{k : t_k < y} with t_k = fl32(0.5 * fl32(c_k + c_k+1)) (ties go to
 *     the lower index); x^_j = s_j * (w_j * (n16 / d)), output rounded to
 *     nearest even.  Norms round to fp16 and saturate at 65504.
 *   - Code storage, one field of rq_code_bytes(d, bits, layout) bytes per block:
 *     RQ_CODES_INT8: one byte per coordinate; RQ_CODES_PACKED: code j of the
 *     block occupies bits [j*bits, (j+1)*bits) of the field, least significant
 *     bit first (two codes per byte at 4 bits, four at 2 bits).
 *   - Sign diagonal: s_j = -1 iff bit (j mod 64) of output floor(j/64) of the
 *     SplitMix64 stream with initial state sign_seed is set; one diagonal per
 *     call, shared by every block.
 *   - Sign sketch storage: m/8 bytes per vector; coordinate i is bit (i mod 8)
 *     of byte i/8; bit 1 <-> P_i >= 0 (sign +1).
 */
#ifndef RQ_H
#define RQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *rq_stream_t;   /* the same handle as cudaStream_t */

typedef enum {
    RQ_OK = 0,
    RQ_EINVAL = -1,        /* bad size, NULL pointer, unsorted/non-finite table, ... */
    RQ_EALIGN = -2,        /* a device pointer is not 16-byte aligned */
    RQ_ESIZE = -3,         /* a size does not fit the kernels' index arithmetic */
    RQ_EUNSUPPORTED = -4,  /* valid but not implemented (d, bits, m, dtype combination) */
    RQ_ECUDA = -5,         /* a CUDA runtime call failed (launch error, ...) */
    RQ_EDEVICE = -6        /* a kernel's bounded wait expired (see rq_device_error) */
} rq_status;

typedef enum { RQ_F16 = 0, RQ_BF16 = 1 } rq_dtype;
typedef enum { RQ_CODES_PACKED = 0, RQ_CODES_INT8 = 1 } rq_layout;

/* Human-readable name of a status code (static string). */
const char *rq_status_string(int status);

/* Device-side error word of the current device: RQ_EDEVICE if a kernel since
 * the last clear gave up a bounded wait on the tensor core (its outputs are
 * invalid; the kernel freed its resources and returned instead of hanging),
 * else RQ_OK.  Synchronous (waits for the device); clear != 0 resets the word.
 * Returns RQ_ECUDA if the word cannot be read. */
rq_status rq_device_error(int clear);

/* Launch trace: the names of the kernels that the last librq call made on
 * the calling host thread enqueued, comma-separated in launch order (e.g.
 * "score_v2_prologue,score_v4_kernel"), or "" when that call returned an error
 * before enqueuing anything.  Thread-local storage owned by the library, valid
 * until the thread's next librq call.  Which kernel runs is chosen from the
 * shape (d, bits, m, n_q, shared-memory fit); this lets a caller or a test see
 * the choice. */
const char *rq_last_launch(void);

/* Self-test of the bounded-wait failure path (no counterpart on the pages; it
 * exercises the loud-failure behaviour the entry points promise).  Enqueues
 * one CTA that allocates tensor memory, waits at most `polls` times (1 ..
 * 2^20) on an mbarrier that nothing ever arrives on, then unwinds exactly as
 * the tensor-core kernels do after an expired wait: it records RQ_EDEVICE in
 * the device error word, frees its tensor memory and returns.  No copy or MMA
 * is in flight while it waits.  After it completes, rq_device_error() reports
 * RQ_EDEVICE until cleared; the device stays usable.  RQ_EINVAL for polls out
 * of range. */
rq_status rq_probe_bounded_wait(uint32_t polls, rq_stream_t stream);

/* Bytes of code storage for n values in blocks of d: (n/d) * (d*bits/8) packed,
 * n for int8.  Returns -1 on invalid arguments. */
int64_t rq_code_bytes(int64_t n, int d, int bits, rq_layout layout);

/* Lloyd-Max reconstruction levels for N(0,1) at `bits` (1..8), ascending,
 * written to the HOST array centroids_out[2^bits] as fp32.  Computed by the
 * conditional-expectation fixed point in fp64 (the PolarQuant paragraph's
 * optimal N(0,1) levels found by iterating conditional means), made exactly
 * odd-symmetric, then rounded to fp32. */
rq_status rq_lloyd_max(int bits, float *centroids_out);

/* Quantize n values of x (dtype fp16/bf16, n % d == 0, blocks contiguous).
 *   bits 1..8 (int8 layout) or 1..8 (packed); centroids: HOST, 2^bits finite
 *   strictly ascending fp32 values.
 *   codes: rq_code_bytes(n, d, bits, layout) bytes; norms: n/d fp16.
 *   use_signs = 0 means D = I (sign_seed ignored). */
rq_status rq_quantize(const void *x, rq_dtype dtype, int64_t n, int d, int bits, rq_layout layout,
                      int use_signs, uint64_t sign_seed, const float *centroids,
                      void *codes, uint16_t *norms, rq_stream_t stream);

/* Reconstruct n values into out (out_dtype) from codes and fp16 norms written
 * by rq_quantize with the same d, bits, layout, signs and centroids.  An
 * int8-layout byte >= 2^bits is not a code rq_quantize writes: the values of
 * its block are then unspecified, but no memory outside the arguments is read. */
rq_status rq_dequantize(const void *codes, const uint16_t *norms, int64_t n, int d, int bits,
                        rq_layout layout, int use_signs, uint64_t sign_seed, const float *centroids,
                        void *out, rq_dtype out_dtype, rq_stream_t stream);

/* ---- QJL key sketch with a per-group outlier sketch ------------------------
 * QJL README, "Algorithm in one paragraph" (outlier coordinates get a top-k
 * sketch per group of group_size consecutive tokens, with its own projection
 * dimension), and qjl_apply.py's key hook (per group, the norm of every
 * coordinate over the group's tokens; the top outlier_count of them as uint8
 * indices; one projection and the outlier dimension handed to the quantizer).
 * Groups are 32 consecutive key vectors (a head's token count must be a
 * multiple of 32).  Per group the outlier set O = the n_out coordinates with
 * the largest fp32 sum of squares over the group's tokens (summed in token
 * order; ties to the lower coordinate), stored largest first.  Each key splits
 * into k_in (O zeroed) and k_out (only O):
 *   signs / norms          = sign bits of S k_in and fp16(||k_in||) (as qjl_sketch);
 *   out_signs / out_norms  = sign bits of S_o k_out, S_o = rows 0 .. m_o-1 of S,
 *                            and fp16(||k_out||) (fp32 squares in stored order);
 * and the score is  sqrt(pi/2)/m ||k_in|| <S q, sign(S k_in)>
 *                 + sqrt(pi/2)/m_o ||k_out|| <S_o q_O, sign(S_o k_out)>,
 * q_O the query on O: the sum of the two QJL estimators of <q, k_in> and
 * <q, k_out>, unbiased for <q, k>. */

/* Bytes of scratch qjl_sketch_outlier needs: the masked keys (n_vec * d bf16). */
size_t qjl_sketch_outlier_workspace_bytes(int64_t n_vec, int d);

/* keys: bf16 [n_vec][d], n_vec % 32 == 0, d = 128 (other powers of two:
 * RQ_EUNSUPPORTED); proj: bf16 [m][d], m % 8 == 0, 8 <= m <= 512; 32 <= m_o <=
 * min(m, 256), m_o % 32 == 0; 1 <= n_out <= 16.  Outputs (device, 16-byte
 * aligned): signs [n_vec][m/8], norms [n_vec] fp16, out_idx [n_vec/32][n_out]
 * uint8, out_signs [n_vec][m_o/8], out_norms [n_vec] fp16.  Sign bit = (P >= 0),
 * bit j of byte b <-> coordinate 8b + j. */
rq_status qjl_sketch_outlier(const void *keys, int64_t n_vec, int d, int m, const void *proj, int m_o, int n_out,
                             uint8_t *signs, uint16_t *norms, uint8_t *out_idx, uint8_t *out_signs,
                             uint16_t *out_norms, void *workspace, size_t workspace_bytes, rq_stream_t stream);

/* Scores [G][n_q][T] (fp32) of bf16 queries q [G][n_q][d] against G * T keys
 * sketched by qjl_sketch_outlier (T % 32 == 0; the same m, m_o, n_out, proj):
 * the pure-QJL score of the main sketch (qjl_score) plus the outlier term.
 * workspace: qjl_score_workspace_bytes(G, n_q, d, m). */
rq_status qjl_score_outlier(const void *q, int64_t G, int n_q, int d, int m, const void *proj, const uint8_t *signs,
                            const uint16_t *norms, int64_t T, int m_o, int n_out, const uint8_t *out_idx,
                            const uint8_t *out_signs, const uint16_t *out_norms, float *scores, void *workspace,
                            size_t workspace_bytes, rq_stream_t stream);

/* ---- Dense random orthogonal rotation with the Beta-law codebook ----------
 * TurboQuant README, "Algorithm in one paragraph": store ||x||, rotate the
 * unit vector x / ||x|| by a fixed random orthogonal Pi drawn by the QR
 * decomposition of a Gaussian matrix with the sign fix, bucketize every
 * coordinate against the Lloyd-Max centroids of the law of one coordinate of
 * a uniform unit vector (t^2 ~ Beta(1/2, (d-1)/2)), bit-pack; the inverse is
 * x^ = ||x|| Pi^T c.  The rotation runs as a 16-bit tensor-core GEMM with
 * fp32 accumulation, so a code next to a boundary may differ from an exact
 * evaluation by one level. */

/* Lloyd-Max centroids of f_d(t) ~ (1 - t^2)^((d-3)/2) on [-1, 1] at `bits`
 * (1..8), 3 <= d <= 65536, ascending, exactly odd-symmetric, written to the
 * HOST array centroids_out[2^bits] as fp32 (a float64 fixed point: cell
 * means by Gauss-Legendre quadrature and the closed-form first moment).
 * Host only; well under a second up to 4 bits, about half a minute at 8. */
rq_status rq_beta_lloyd_max(int d, int bits, float *centroids_out);

/* The seeded rotation Pi (d x d, row-major fp32) into the HOST array pi_out:
 * G[i][j] = Box-Muller normal k = i*d + j over SplitMix64(seed) outputs 2k
 * and 2k+1 (the stream qjl_make_projection uses), Householder QR in float64,
 * Pi = Q diag(sign(diag R)).  1 <= d <= 4096.  Host only, O(d^3). */
rq_status rq_make_rotation(int d, uint64_t seed, float *pi_out);

/* Quantize n values of x (dtype fp16/bf16, blocks of d contiguous, d = 128)
 * with the rotation pi (DEVICE, d x d row-major, the same dtype as x):
 *   norms[b] = fp16(||x_b||) (the canonical fp32 pairwise norm),
 *   codes[b] = #{t_k < z_j}, z = (Pi x_b) * (1 / ||x_b||) in fp32,
 *   t_k = fl32((c_k + c_k+1) / 2); centroids: HOST, 2^bits ascending fp32
 *   (rq_beta_lloyd_max(d, bits) for the method's codebook).
 * codes: rq_code_bytes(n, d, bits, layout) bytes.  All device pointers
 * 16-byte aligned (RQ_EALIGN); other d return RQ_EUNSUPPORTED. */
rq_status rq_quantize_dense(const void *x, rq_dtype dtype, int64_t n, int d, const void *pi, int bits,
                            rq_layout layout, const float *centroids, void *codes, uint16_t *norms,
                            rq_stream_t stream);

/* x^_b = n16_b * Pi^T c_b into out (dtype, also the dtype of pi), where c_b
 * holds the centroids of the codes, each rounded once to dtype (the GEMM
 * operand), accumulated in fp32 and rounded once to dtype. */
rq_status rq_dequantize_dense(const void *codes, const uint16_t *norms, int64_t n, int d, const void *pi, int bits,
                              rq_layout layout, const float *centroids, void *out, rq_dtype dtype,
                              rq_stream_t stream);

/* Quantize (as rq_quantize) and sketch the first-stage residual in the same
 * pass (the optional 1-bit QJL residual correction of the PolarQuant
 * paragraph; the two-stage TurboQuant-style key code):
 *   r = x - x^32 (fp32, x^32 the reconstruction before output rounding),
 *   qjl_norms[b] = fp16(||r||) (canonical fp32 norm),
 *   qjl_signs[b][m/8] = sign bits of S r_bf16, r_bf16 = bf16(r), S = proj.
 *   proj: m x d bf16 row-major (qjl_make_projection); m % 8 == 0, 8 <= m <= 512. */
rq_status rq_quantize_qjl(const void *x, rq_dtype dtype, int64_t n, int d, int bits, rq_layout layout,
                          int use_signs, uint64_t sign_seed, const float *centroids,
                          int m, const void *proj, void *codes, uint16_t *norms,
                          uint8_t *qjl_signs, uint16_t *qjl_norms, rq_stream_t stream);

/* Write the m x d JL matrix S[i][j] = round16(fp32(gauss(seed, i*d + j))) to
 * proj (dtype bf16 or fp16, row-major).  gauss(seed, k) is the Box-Muller
 * normal sqrt(-2 ln u1) cos(2 pi u2) with u1 = (w_2k >> 11 + 1) 2^-53,
 * u2 = (w_2k+1 >> 11) 2^-53, w_i output i of SplitMix64 seeded with `seed`
 * (qjl_apply.py `_build_jl_projections`: plain N(0,1) entries, no QR). */
rq_status qjl_make_projection(uint64_t seed, int m, int d, rq_dtype dtype, void *proj, rq_stream_t stream);

/* QJL sketch of n_vec vectors x[n_vec][d] (dtype = proj dtype):
 * signs[n_vec][m/8] of S x, norms[n_vec] = fp16(||x||) (the QJL paragraph:
 * the key's norm is kept, and the sign of every sketch coordinate is stored
 * as one bit, eight to a byte). */
rq_status qjl_sketch(const void *x, rq_dtype dtype, int64_t n_vec, int d, int m, const void *proj,
                     uint8_t *signs, uint16_t *norms, rq_stream_t stream);

/* Device workspace qjl_score needs for G groups of n_q queries (bytes). */
size_t qjl_score_workspace_bytes(int64_t G, int n_q, int d, int m);

/* Inner-product scores of n_q queries against T compressed keys per group
 * (group = batch x kv-head; the n_q queries of a group share its keys, the
 * grouped-query shape):
 *   q: bf16 [G][n_q][d]; proj: m x d (proj_dtype); signs [G][T][m/8];
 *   sk_norms fp16 [G][T] (the norm the sketch was taken of);
 *   codes/norms: first-stage codes [G][T] blocks of d and fp16 norms, or
 *   codes == NULL for the pure QJL score;
 *   scores: fp32 [G][n_q][T];
 *   workspace: qjl_score_workspace_bytes(G, n_q, d, m) bytes of device memory
 *   (overwritten). */
rq_status qjl_score(const void *q, int64_t G, int n_q, int d, int m, const void *proj, rq_dtype proj_dtype,
                    const uint8_t *signs, const uint16_t *sk_norms, int64_t T,
                    const void *codes, const uint16_t *norms, int bits, rq_layout layout,
                    int use_signs, uint64_t sign_seed, const float *centroids,
                    float *scores, void *workspace, size_t workspace_bytes, rq_stream_t stream);

/* Device workspace qjl_attention needs (bytes), for the current device. */
size_t qjl_attention_workspace_bytes(int64_t G, int n_q, int d, int m, int64_t T);

/* Attention decode over compressed keys and values.  The QJL page ("QJL",
 * "What this is -- and what it is NOT") pairs 1-bit JL keys with 4-bit
 * TurboQuant values and ("Algorithm in one paragraph") rebuilds each
 * query-key score at attention time from the same projection; the GLQ page
 * ("KV cache compression", "Inline-dequant E8 KV") dequantizes K/V inside the
 * attention kernel, with the inverse Hadamard and a split of the key range for
 * long contexts.  For every group g and query i:
 *   out[g][i][:] = sum_t p_t vh_t,  p_t = softmax over t of softmax_scale * s(i, t),
 * s the qjl_score estimator of the keys (pure QJL when codes == NULL, else
 * two-stage) and vh_t the reconstruction of value block (g, t) that
 * rq_dequantize computes before its 16-bit rounding:
 *   vh_t = D_v H (c_v[v_codes_t] * v_norms_t / d).
 *   q, proj, signs, sk_norms, codes, norms, bits, layout, use_signs,
 *   sign_seed, centroids: as qjl_score;
 *   v_codes [G][T] blocks of d (v_layout), v_norms fp16 [G][T], with their
 *   own v_bits, v_use_signs, v_sign_seed and v_centroids (rq_quantize's
 *   arguments for the values);
 *   out: fp32 [G][n_q][d] (caller-owned);
 *   workspace: qjl_attention_workspace_bytes(G, n_q, d, m, T) bytes of device
 *   memory (overwritten).
 * Computed in fp32 with fp16 tensor-core operands: the scores as qjl_score,
 * 2^x by the hardware approximation, the weights 2^14 p and the values
 * c * (n / d) rounded to fp16 for the weighted sum.
 * Supported: d = 128, n_q <= 32, m % 128 == 0, two-stage keys of 1, 2, 3, 4
 * bits packed or int8 codes with d * width / 8 % 16 == 0, values of 2, 3, 4
 * bits packed or int8; other valid shapes return RQ_EUNSUPPORTED.  T >= 1. */
rq_status qjl_attention(const void *q, int64_t G, int n_q, int d, int m, const void *proj, rq_dtype proj_dtype,
                        const uint8_t *signs, const uint16_t *sk_norms, int64_t T,
                        const void *codes, const uint16_t *norms, int bits, rq_layout layout,
                        int use_signs, uint64_t sign_seed, const float *centroids,
                        const void *v_codes, const uint16_t *v_norms, int v_bits, rq_layout v_layout,
                        int v_use_signs, uint64_t v_sign_seed, const float *v_centroids,
                        float softmax_scale, float *out, void *workspace, size_t workspace_bytes,
                        rq_stream_t stream);

/* qjl_score without a caller-provided workspace.  The pages have no
 * counterpart to this entry point; it exists for callers that cannot allocate
 * device memory -- a serving engine that reserved all of its HBM for the KV
 * cache at start-up and forbids later allocations, or a host that reaches this
 * library through a plain-C plugin interface that passes device pointers but
 * no allocator.  It computes exactly what qjl_score computes (same arguments
 * minus workspace / workspace_bytes) and allocates nothing: its scratch is an
 * 8 MiB array inside the library's own device image, which every GPU that
 * loads the library holds until the process exits.
 *   - Returns RQ_ESIZE when qjl_score_workspace_bytes(G, n_q, d, m) exceeds
 *     8 MiB (8388608 bytes), before touching the GPU.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and remembers it together with the device's
 *     current context; make that first call before any stream capture.  After
 *     a device reset the next call sees a new context and looks the address up
 *     again (that call, too, belongs before any capture).  RQ_ECUDA if the
 *     lookup fails.
 *   - Every call on a device shares the one array and it keeps the last
 *     call's contents (nothing in it needs to start at zero).  Calls whose
 *     work overlaps on the GPU -- e.g. on two streams without ordering between
 *     them -- race on it; order them on one stream or with events. */
rq_status qjl_score_noalloc(const void *q, int64_t G, int n_q, int d, int m, const void *proj, rq_dtype proj_dtype,
                            const uint8_t *signs, const uint16_t *sk_norms, int64_t T,
                            const void *codes, const uint16_t *norms, int bits, rq_layout layout,
                            int use_signs, uint64_t sign_seed, const float *centroids,
                            float *scores, rq_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* RQ_H */
