/*
 * rq_oracle.c -- plain, slow, single-threaded CPU oracle for blockwise rotated
 * scalar quantization and the QJL 1-bit sketch.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant generator with the CUDA library; neither includes
 * nor links the other.
 *
 * Sources followed (web pages on KV-cache / weight quantization):
 *   [PQ]  eliza "scripts/quantization" README, section "PolarQuant",
 *         "Algorithm in one paragraph": power-of-two blocks (default 128),
 *         per-block L2 norm stored fp16, normalise, Walsh-Hadamard rotation,
 *         coordinates ~N(0,1) after scaling by sqrt(d), nearest Lloyd-Max
 *         N(0,1) centroid (iterative conditional expectation), index stored;
 *         inverse: centroid lookup, divide by sqrt(d), inverse Hadamard,
 *         rescale by the norm.
 *   [TQ]  same README, section "TurboQuant", "Algorithm in one paragraph":
 *         bucketize against sorted centroids, bit-pack indices (two per byte
 *         at 4 bits, four per byte at 2 bits).
 *   [QJL] same README, section "QJL", "Algorithm in one paragraph": Gaussian
 *         JL projection, keep sign bits (8 per byte) and the vector norm; the
 *         query is projected through the same matrix for an unbiased
 *         inner-product estimate.
 *   [QA]  qjl_apply.py source text, `_build_jl_projections` (plain N(0,1)
 *         entries) and `_qjl_decode_keys` (bit j of a byte is (byte>>j)&1,
 *         mapped to sign 2*bit-1).
 *   [TP]  turbopress 0.4.2 project description, "Package layout" (Rademacher
 *         signs times block Walsh-Hadamard; Lloyd-Max N(0,1) codebooks to a
 *         float64 fixed point) and "Findings" (QJL noise std
 *         sqrt(pi/2)*||r||*||x||/sqrt(k), unbiased).
 *
 * Readings where the pages leave a step open (each one is listed in the
 * project design notes):
 *   - Arithmetic precision.  The pages fix none.  The code decision
 *     (nearest centroid) is taken in fp32, the precision the GPU path uses,
 *     and every fp32 quantity that feeds it is computed in one canonical
 *     order: the norm is the pairwise (recursive halving) fp32 sum of fp32
 *     squares; the Hadamard transform is the radix-2 butterfly with stages
 *     h = 1, 2, 4, ..., d/2 on (a, b) -> (a + b, a - b).  fp64 twins of the
 *     same quantities (orc_rotate_f64) bound the fp32 rounding in the tests.
 *   - y = (H D x) * (1 / ||x||) with the unnormalised Sylvester H: this is
 *     sqrt(d) * H_orthonormal * D * x / ||x||, i.e. the normalise, rotate,
 *     scale-by-sqrt(d) chain with the two sqrt(d) factors cancelled.
 *   - Nearest centroid = #{k : t_k < y}, t_k = fl32(0.5 * fl32(c_k + c_k+1)):
 *     ties go to the lower index.
 *   - Reconstruction x^_j = s_j * (w_j * (n16 / d)), w = H c (fp32, same
 *     stages): n16 * D * H_orth^T * (c / sqrt(d)) with exact power-of-two
 *     scaling.
 *   - Sign diagonal: s_j = -1 when bit (j mod 64) of SplitMix64 output
 *     floor(j / 64) of the stream seeded with sign_seed is set.
 *   - Projection S[i][j] = round(gauss(seed, i*d + j)) with Box-Muller over
 *     SplitMix64 outputs 2k and 2k+1; rounded to fp32 then to bf16/fp16.
 *   - Sign bit = (P >= 0); LSB-first packing, bit 1 <-> +1.
 *   - Norms saturate at the largest finite fp16 (65504).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F16 0
#define ORC_BF16 1
#define ORC_PACKED 0
#define ORC_INT8 1

/* ------------------------------------------------------------------ */
/* 16-bit float formats, written out from the IEEE-754 binary16 and the */
/* bfloat16 (truncated binary32) definitions.  Round to nearest even.   */
/* ------------------------------------------------------------------ */

static uint32_t f32_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float bits_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

float orc_bf16_to_f32(uint16_t h) { return bits_f32((uint32_t)h << 16); }

uint16_t orc_f32_to_bf16(float f)
{
    uint32_t u = f32_bits(f);
    if ((u & 0x7fffffffu) > 0x7f800000u)           /* NaN: keep it quiet */
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t keep = u >> 16, rest = u & 0xffffu;
    if (rest > 0x8000u || (rest == 0x8000u && (keep & 1u))) keep += 1u;
    return (uint16_t)keep;
}

float orc_f16_to_f32(uint16_t h)
{
    uint32_t sign = (uint32_t)(h >> 15) & 1u, e = (h >> 10) & 0x1fu, m = h & 0x3ffu;
    double v;
    if (e == 0x1f) return bits_f32((sign << 31) | 0x7f800000u | (m << 13));
    if (e == 0) v = ldexp((double)m, -24);               /* subnormal */
    else v = ldexp((double)(m | 0x400u), (int)e - 25);
    return (float)(sign ? -v : v);
}

/* Round an fp32 value to binary16 (nearest, ties to even); past the largest
 * finite value (65504 + half an ulp) the result is infinity. */
uint16_t orc_f32_to_f16(float f)
{
    uint32_t u = f32_bits(f);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t a = u & 0x7fffffffu;
    if (a > 0x7f800000u) return (uint16_t)(sign | 0x7e00u);       /* NaN */
    if (a >= 0x477ff000u) return (uint16_t)(sign | 0x7c00u);      /* |f| >= 65520 */
    if (a < 0x38800000u) {                                        /* |f| < 2^-14: subnormal */
        double scaled = (double)bits_f32(a) * 16777216.0;         /* |f| / 2^-24, exact */
        double fl = floor(scaled), fr = scaled - fl;
        uint32_t qi = (uint32_t)fl;
        if (fr > 0.5 || (fr == 0.5 && (qi & 1u))) qi += 1u;        /* 1024 = smallest normal */
        return (uint16_t)(sign | qi);
    }
    uint32_t h = ((a >> 23) - 112u) << 10 | ((a & 0x7fffffu) >> 13);
    uint32_t rest = a & 0x1fffu;
    if (rest > 0x1000u || (rest == 0x1000u && (h & 1u))) h += 1u;  /* carry may bump the exponent */
    return (uint16_t)(sign | h);
}

/* fp16 norm store: largest finite binary16 when the value rounds past it. */
static uint16_t norm_to_f16(float n)
{
    uint16_t h = orc_f32_to_f16(n);
    if ((h & 0x7fffu) == 0x7c00u) h = (uint16_t)((h & 0x8000u) | 0x7bffu);
    return h;
}

static float load_elem(const uint16_t *x, int dtype, int64_t i)
{
    return dtype == ORC_BF16 ? orc_bf16_to_f32(x[i]) : orc_f16_to_f32(x[i]);
}

static uint16_t store_elem(float v, int dtype)
{
    return dtype == ORC_BF16 ? orc_f32_to_bf16(v) : orc_f32_to_f16(v);
}

/* ------------------------------------------------------------------ */
/* SplitMix64 (Steele, Lea & Flood, OOPSLA 2014): state advances by the  */
/* golden-ratio increment; each output is the state passed through the  */
/* published variant-13 finaliser.  orc_splitmix64(seed, k) is output k  */
/* (0-based) of the stream whose initial state is `seed`.               */
/* ------------------------------------------------------------------ */

uint64_t orc_splitmix64(uint64_t seed, uint64_t k)
{
    uint64_t z = seed + (k + 1u) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* Rademacher sign diagonal s in {+1,-1}^d shared by every block of a tensor. */
void orc_sign_diagonal(uint64_t seed, int d, int8_t *s)
{
    for (int j = 0; j < d; ++j) {
        uint64_t w = orc_splitmix64(seed, (uint64_t)(j / 64));
        s[j] = ((w >> (j % 64)) & 1u) ? (int8_t)-1 : (int8_t)1;
    }
}

/* One standard normal draw by the Box-Muller transform (Box & Muller 1958)
 * from two uniforms built from 53 high bits of SplitMix64 outputs 2k, 2k+1. */
double orc_gauss(uint64_t seed, uint64_t k)
{
    double u1 = (double)((orc_splitmix64(seed, 2u * k) >> 11) + 1u) * 0x1p-53;  /* (0,1] */
    double u2 = (double)(orc_splitmix64(seed, 2u * k + 1u) >> 11) * 0x1p-53;    /* [0,1) */
    double two_pi = 6.283185307179586476925286766559;
    return sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
}

/* JL projection S (m x d, row-major), entries N(0,1) rounded to the 16-bit
 * dtype through fp32 ([QA] `_build_jl_projections`: plain N(0,1), no QR). */
void orc_projection(uint64_t seed, int m, int d, int dtype, uint16_t *S)
{
    for (int i = 0; i < m; ++i)
        for (int j = 0; j < d; ++j) {
            float z = (float)orc_gauss(seed, (uint64_t)i * (uint64_t)d + (uint64_t)j);
            S[(int64_t)i * d + j] = store_elem(z, dtype);
        }
}

/* ------------------------------------------------------------------ */
/* Lloyd-Max optimal scalar quantizer for N(0,1) ([PQ]; [TP] codebooks): */
/* alternate centroid = conditional mean of each cell and boundary =    */
/* midpoint of neighbouring centroids until a float64 fixed point.      */
/* ------------------------------------------------------------------ */

static double phi(double t) { return isinf(t) ? 0.0 : exp(-0.5 * t * t) / sqrt(2.0 * 3.14159265358979323846); }

/* P(a < Z <= b) for Z ~ N(0,1), computed on the tail side for accuracy. */
static double prob_between(double a, double b)
{
    if (a >= 0.0) return 0.5 * (erfc(a / sqrt(2.0)) - erfc(b / sqrt(2.0)));
    if (b <= 0.0) return 0.5 * (erfc(-b / sqrt(2.0)) - erfc(-a / sqrt(2.0)));
    return 1.0 - 0.5 * erfc(-a / sqrt(2.0)) - 0.5 * erfc(b / sqrt(2.0));
}

/* Returns the iteration count; c[0..2^bits) ascending, exactly symmetric. */
int orc_lloyd_max(int bits, double *c)
{
    int K = 1 << bits;
    double *t = (double *)malloc(sizeof(double) * (size_t)(K + 1));
    for (int i = 0; i < K; ++i) c[i] = -3.0 + 6.0 * (i + 0.5) / K;   /* any sorted start */
    int it;
    for (it = 1; it <= 1000000; ++it) {
        t[0] = -INFINITY; t[K] = INFINITY;
        for (int i = 1; i < K; ++i) t[i] = 0.5 * (c[i - 1] + c[i]);
        double delta = 0.0;
        for (int i = 0; i < K; ++i) {
            double p = prob_between(t[i], t[i + 1]);
            double nc = (phi(t[i]) - phi(t[i + 1])) / p;   /* E[Z | t_i < Z <= t_i+1] */
            double dd = fabs(nc - c[i]);
            if (dd > delta) delta = dd;
            c[i] = nc;
        }
        if (delta < 1e-13) break;
    }
    for (int i = 0; i < K / 2; ++i) {                  /* the N(0,1) optimum is odd-symmetric */
        double a = 0.5 * (c[K - 1 - i] - c[i]);
        c[i] = -a; c[K - 1 - i] = a;
    }
    free(t);
    return it;
}

/* Mean squared error E[(Z - Q(Z))^2] of a table under N(0,1), nearest rule. */
double orc_table_mse(int K, const double *c)
{
    double mse = 0.0;
    for (int i = 0; i < K; ++i) {
        double a = i == 0 ? -INFINITY : 0.5 * (c[i - 1] + c[i]);
        double b = i == K - 1 ? INFINITY : 0.5 * (c[i] + c[i + 1]);
        /* E[(Z-c)^2; a<Z<=b] = (1+c^2)P + ... via moments of the truncated normal */
        double p = prob_between(a, b);
        double m1 = phi(a) - phi(b);                               /* E[Z; cell] */
        double ta = isinf(a) ? 0.0 : a * phi(a), tb = isinf(b) ? 0.0 : b * phi(b);
        double m2 = p + ta - tb;                                   /* E[Z^2; cell] */
        mse += m2 - 2.0 * c[i] * m1 + c[i] * c[i] * p;
    }
    return mse;
}

/* Decision thresholds in fp32: t_k = fl32(0.5 * fl32(c_k + c_k+1)). */
void orc_boundaries(const float *c, int K, float *t)
{
    for (int k = 0; k + 1 < K; ++k) {
        float s = c[k] + c[k + 1];
        t[k] = 0.5f * s;
    }
}

/* ------------------------------------------------------------------ */
/* Canonical fp32 building blocks.                                      */
/* ------------------------------------------------------------------ */

/* Pairwise (recursive halving) fp32 sum of v[0..n), n a power of two. */
static float pairwise_sum(const float *v, int n)
{
    if (n == 1) return v[0];
    float a = pairwise_sum(v, n / 2);
    float b = pairwise_sum(v + n / 2, n / 2);
    return a + b;
}

/* Sub-blocks of a block of d values: the binary decomposition of d, largest
 * power of two first (GLQ README, "Bit widths": a non-power-of-two size such as
 * 2688 is decomposed as 2048 + 512 + 128 and transformed block-diagonally;
 * turbopress "Package layout": block-diagonal Walsh-Hadamard times Rademacher
 * signs, an orthogonal transform).  A power of two is one sub-block.
 * Returns the count; off[] and sz[] receive offsets and sizes (at most 31). */
int orc_sub_blocks(int d, int *off, int *sz)
{
    int n = 0, o = 0;
    for (int b = 1 << 30; b >= 1; b >>= 1)
        if (d - o >= b) { off[n] = o; sz[n] = b; o += b; ++n; }
    return n;
}

/* fp32 L2 norm: squares rounded to fp32, pairwise sum within each sub-block,
 * the sub-block sums added in order, correctly rounded sqrt. */
static float norm_f32(const float *v, int d, float *tmp)
{
    int off[31], sz[31];
    int nb = orc_sub_blocks(d, off, sz);
    for (int j = 0; j < d; ++j) tmp[j] = v[j] * v[j];
    float acc = pairwise_sum(tmp + off[0], sz[0]);
    for (int i = 1; i < nb; ++i) acc = acc + pairwise_sum(tmp + off[i], sz[i]);
    return sqrtf(acc);
}

/* Unnormalised Walsh-Hadamard transform, Sylvester (natural) order, in place:
 * stage h pairs j and j+h for every j with (j & h) == 0. */
static void fwht_f32(float *v, int d)
{
    for (int h = 1; h < d; h *= 2)
        for (int i = 0; i < d; i += 2 * h)
            for (int j = i; j < i + h; ++j) {
                float a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
}

static void fwht_f64(double *v, int d)
{
    for (int h = 1; h < d; h *= 2)
        for (int i = 0; i < d; i += 2 * h)
            for (int j = i; j < i + h; ++j) {
                double a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
}

/* Block-diagonal transform of a block of d values: fwht of every sub-block. */
static void rotate_f32(float *v, int d)
{
    int off[31], sz[31];
    int nb = orc_sub_blocks(d, off, sz);
    for (int i = 0; i < nb; ++i) fwht_f32(v + off[i], sz[i]);
}

/* Per-sub-block scales of the block-diagonal rotation.  With R the orthogonal
 * blockdiag(H_b / sqrt(b)) D, the quantized coordinates are
 * y = sqrt(d) R x / ||x|| and the reconstruction x^ = ||x|| R^T c / sqrt(d):
 *   y_j  = w_j * fl32(g_b * inv),   g_b = fl32(sqrt(d / b)),
 *   x^_j = s_j * (w'_j * fl32(n16 * h_b)),   h_b = fl32(1 / sqrt(d b)),
 * w = H_b D x and w' = H_b c in fp32 stages.  For a power-of-two d (one
 * sub-block) g = 1 and h = 1/d exactly: the plain path. */
static float sub_g(int d, int b) { return (float)sqrt((double)d / (double)b); }
static float sub_h(int d, int b) { return (float)(1.0 / sqrt((double)d * (double)b)); }

/* ------------------------------------------------------------------ */
/* Code storage ([PQ] int8 index; [TQ] packed, low bits first).         */
/* ------------------------------------------------------------------ */

static int64_t block_code_bytes(int d, int bits, int layout)
{
    return layout == ORC_INT8 ? (int64_t)d : (int64_t)d * bits / 8;
}

static void put_code(uint8_t *field, int j, int bits, int layout, unsigned code)
{
    if (layout == ORC_INT8) { field[j] = (uint8_t)code; return; }
    for (int b = 0; b < bits; ++b) {
        int64_t bit = (int64_t)j * bits + b;
        if ((code >> b) & 1u) field[bit / 8] |= (uint8_t)(1u << (bit % 8));
    }
}

static unsigned get_code(const uint8_t *field, int j, int bits, int layout)
{
    if (layout == ORC_INT8) return field[j];
    unsigned code = 0;
    for (int b = 0; b < bits; ++b) {
        int64_t bit = (int64_t)j * bits + b;
        code |= (unsigned)((field[bit / 8] >> (bit % 8)) & 1u) << b;
    }
    return code;
}

/* Unpack every code of `nblocks` blocks into one byte per coordinate. */
void orc_unpack_codes(const uint8_t *codes, int64_t nblocks, int d, int bits, int layout, uint8_t *out)
{
    int64_t cb = block_code_bytes(d, bits, layout);
    for (int64_t b = 0; b < nblocks; ++b)
        for (int j = 0; j < d; ++j)
            out[b * d + j] = (uint8_t)get_code(codes + b * cb, j, bits, layout);
}

void orc_pack_codes(const uint8_t *idx, int64_t nblocks, int d, int bits, int layout, uint8_t *codes)
{
    int64_t cb = block_code_bytes(d, bits, layout);
    memset(codes, 0, (size_t)(cb * nblocks));
    for (int64_t b = 0; b < nblocks; ++b)
        for (int j = 0; j < d; ++j)
            put_code(codes + b * cb, j, bits, layout, idx[b * d + j]);
}

/* ------------------------------------------------------------------ */
/* Quantize / dequantize ([PQ] algorithm paragraph).                    */
/* ------------------------------------------------------------------ */

/* x: nblocks*d 16-bit values; s: d signs or NULL; c: 2^bits fp32 centroids.
 * Writes packed/int8 codes, fp16 norm bits; optional y (fp32 rotated coords)
 * and n32 (fp32 norms) for diagnostics. */
int orc_quantize(const uint16_t *x, int dtype, int64_t nblocks, int d, int bits, int layout,
                 const int8_t *s, const float *c, uint8_t *codes, uint16_t *norms,
                 float *y_out, float *n32_out)
{
    int K = 1 << bits;
    float *t = (float *)malloc(sizeof(float) * (size_t)K);
    float *v = (float *)malloc(sizeof(float) * (size_t)d);
    float *tmp = (float *)malloc(sizeof(float) * (size_t)d);
    orc_boundaries(c, K, t);
    int64_t cb = block_code_bytes(d, bits, layout);
    memset(codes, 0, (size_t)(cb * nblocks));
    for (int64_t b = 0; b < nblocks; ++b) {
        for (int j = 0; j < d; ++j) v[j] = load_elem(x, dtype, b * d + j);
        float n32 = norm_f32(v, d, tmp);
        norms[b] = norm_to_f16(n32);
        if (n32_out) n32_out[b] = n32;
        if (s) for (int j = 0; j < d; ++j) if (s[j] < 0) v[j] = -v[j];
        rotate_f32(v, d);
        float inv = n32 > 0.0f ? 1.0f / n32 : 0.0f;
        int off[31], sz[31];
        int nsb = orc_sub_blocks(d, off, sz), sb = 0;
        float f = sub_g(d, sz[0]) * inv;
        for (int j = 0; j < d; ++j) {
            if (sb + 1 < nsb && j == off[sb + 1]) { ++sb; f = sub_g(d, sz[sb]) * inv; }
            float y = v[j] * f;
            unsigned code = 0;
            for (int k = 0; k + 1 < K; ++k) code += (t[k] < y) ? 1u : 0u;
            put_code(codes + b * cb, j, bits, layout, code);
            if (y_out) y_out[b * d + j] = y;
        }
    }
    free(t); free(v); free(tmp);
    return 0;
}

/* fp64 rotated coordinates y = sqrt(d) R x / ||x|| (the exact-arithmetic value
 * the fp32 canonical y approximates; R as above, H D x / ||x|| for a power of
 * two); used to count near-boundary coordinates. */
int orc_rotate_f64(const uint16_t *x, int dtype, int64_t nblocks, int d, const int8_t *s, double *y_out)
{
    double *v = (double *)malloc(sizeof(double) * (size_t)d);
    int off[31], sz[31];
    int nsb = orc_sub_blocks(d, off, sz);
    for (int64_t b = 0; b < nblocks; ++b) {
        double ss = 0.0;
        for (int j = 0; j < d; ++j) {
            v[j] = (double)load_elem(x, dtype, b * d + j);
            ss += v[j] * v[j];
            if (s && s[j] < 0) v[j] = -v[j];
        }
        double n = sqrt(ss);
        for (int i = 0; i < nsb; ++i) {
            fwht_f64(v + off[i], sz[i]);
            double g = sqrt((double)d / (double)sz[i]);
            for (int j = off[i]; j < off[i] + sz[i]; ++j) y_out[b * d + j] = n > 0.0 ? v[j] * g / n : 0.0;
        }
    }
    free(v);
    return 0;
}

/* fp32 reconstruction before output rounding (xh32) for every element. */
static void dequant_block_f32(const uint8_t *field, uint16_t norm16, int d, int bits, int layout,
                              const int8_t *s, const float *c, float *w)
{
    for (int j = 0; j < d; ++j) w[j] = c[get_code(field, j, bits, layout)];
    rotate_f32(w, d);
    int off[31], sz[31];
    int nsb = orc_sub_blocks(d, off, sz);
    for (int i = 0; i < nsb; ++i) {
        float scale = orc_f16_to_f32(norm16) * sub_h(d, sz[i]);   /* n16 / d exactly for a power of two */
        for (int j = off[i]; j < off[i] + sz[i]; ++j) {
            float xh = w[j] * scale;
            w[j] = (s && s[j] < 0) ? -xh : xh;
        }
    }
}

int orc_dequantize(const uint8_t *codes, const uint16_t *norms, int64_t nblocks, int d, int bits,
                   int layout, const int8_t *s, const float *c, int out_dtype, uint16_t *out,
                   float *xh32_out)
{
    float *w = (float *)malloc(sizeof(float) * (size_t)d);
    int64_t cb = block_code_bytes(d, bits, layout);
    for (int64_t b = 0; b < nblocks; ++b) {
        dequant_block_f32(codes + b * cb, norms[b], d, bits, layout, s, c, w);
        for (int j = 0; j < d; ++j) {
            if (out) out[b * d + j] = store_elem(w[j], out_dtype);
            if (xh32_out) xh32_out[b * d + j] = w[j];
        }
    }
    free(w);
    return 0;
}

/* fp64 reconstruction n16 * D * H c / d, used to bound fp32 rounding. */
int orc_dequantize_f64(const uint8_t *codes, const uint16_t *norms, int64_t nblocks, int d, int bits,
                       int layout, const int8_t *s, const float *c, double *out)
{
    double *w = (double *)malloc(sizeof(double) * (size_t)d);
    int64_t cb = block_code_bytes(d, bits, layout);
    int off[31], sz[31];
    int nsb = orc_sub_blocks(d, off, sz);
    for (int64_t b = 0; b < nblocks; ++b) {
        for (int j = 0; j < d; ++j) w[j] = c[get_code(codes + b * cb, j, bits, layout)];
        double n = orc_f16_to_f32(norms[b]);
        for (int i = 0; i < nsb; ++i) {
            fwht_f64(w + off[i], sz[i]);
            for (int j = off[i]; j < off[i] + sz[i]; ++j) {
                double xh = w[j] * n / sqrt((double)d * (double)sz[i]);
                out[b * d + j] = (s && s[j] < 0) ? -xh : xh;
            }
        }
    }
    free(w);
    return 0;
}

/* QJL residual of the first stage ([PQ] "optionally append a 1-bit QJL
 * residual"): r = x - xh32 in fp32, its fp16 norm (canonical fp32 norm) and
 * r rounded to bf16, the operand the projection multiplies. */
int orc_residual(const uint16_t *x, int dtype, const uint8_t *codes, const uint16_t *norms,
                 int64_t nblocks, int d, int bits, int layout, const int8_t *s, const float *c,
                 uint16_t *r_bf16, uint16_t *rnorms)
{
    float *w = (float *)malloc(sizeof(float) * (size_t)d);
    float *r = (float *)malloc(sizeof(float) * (size_t)d);
    float *tmp = (float *)malloc(sizeof(float) * (size_t)d);
    int64_t cb = block_code_bytes(d, bits, layout);
    for (int64_t b = 0; b < nblocks; ++b) {
        dequant_block_f32(codes + b * cb, norms[b], d, bits, layout, s, c, w);
        for (int j = 0; j < d; ++j) {
            r[j] = load_elem(x, dtype, b * d + j) - w[j];
            r_bf16[b * d + j] = orc_f32_to_bf16(r[j]);
        }
        rnorms[b] = norm_to_f16(norm_f32(r, d, tmp));
    }
    free(w); free(r); free(tmp);
    return 0;
}

/* fp16 norms of 16-bit vectors (canonical fp32 norm). */
int orc_vec_norms(const uint16_t *v, int dtype, int64_t nvec, int d, uint16_t *norms)
{
    float *a = (float *)malloc(sizeof(float) * (size_t)d);
    float *tmp = (float *)malloc(sizeof(float) * (size_t)d);
    for (int64_t i = 0; i < nvec; ++i) {
        for (int j = 0; j < d; ++j) a[j] = load_elem(v, dtype, i * d + j);
        norms[i] = norm_to_f16(norm_f32(a, d, tmp));
    }
    free(a); free(tmp);
    return 0;
}

/* QJL sketch ([QJL] steps 2-3): P = S v in fp64 from the 16-bit operands,
 * bit i = (P_i >= 0), 8 bits per byte, coordinate i -> byte i/8 bit i%8.
 * Optional p_rel = P_i / ||v|| (fp64) for boundary-window accounting. */
int orc_sketch(const uint16_t *v, int dtype, int64_t nvec, int d, int m, const uint16_t *S,
               uint8_t *signs, double *p_rel)
{
    double *a = (double *)malloc(sizeof(double) * (size_t)d);
    double *Sd = (double *)malloc(sizeof(double) * (size_t)m * (size_t)d);
    for (int64_t k = 0; k < (int64_t)m * d; ++k) Sd[k] = load_elem(S, dtype, k);
    int mb = m / 8;
    for (int64_t t = 0; t < nvec; ++t) {
        double nn = 0.0;
        for (int j = 0; j < d; ++j) { a[j] = load_elem(v, dtype, t * d + j); nn += a[j] * a[j]; }
        nn = sqrt(nn);
        memset(signs + t * mb, 0, (size_t)mb);
        for (int i = 0; i < m; ++i) {
            double p = 0.0;
            for (int j = 0; j < d; ++j) p += Sd[(int64_t)i * d + j] * a[j];
            if (p >= 0.0) signs[t * mb + i / 8] |= (uint8_t)(1u << (i % 8));
            if (p_rel) p_rel[t * m + i] = nn > 0.0 ? p / nn : 0.0;
        }
    }
    free(a); free(Sd);
    return 0;
}

/* Inner-product scores ([QJL] estimator; [TP] sqrt(pi/2)/k scaling), fp64:
 *   score[g][q][t] = (n16_t / d) * <H D q, C[idx_t]>                (first stage, when codes)
 *                  + sqrt(pi/2) / m * rn16_t * <S q, 2*bits_t - 1>   (QJL term)
 * q: bf16 [G][nq][d]; signs [G][T][m/8]; sk_norms fp16 [G][T]; codes/norms
 * [G][T] blocks of d (or NULL for the pure-QJL score). */
int orc_score(const uint16_t *q, int64_t G, int nq, int d, int m, const uint16_t *S, int sdtype,
              const uint8_t *signs, const uint16_t *sk_norms, int64_t T,
              const uint8_t *codes, const uint16_t *norms, int bits, int layout,
              const int8_t *s, const float *c, double *scores)
{
    if (codes && (d & (d - 1))) return -1;     /* two-stage scores: power-of-two blocks only */
    double *qv = (double *)malloc(sizeof(double) * (size_t)d);
    double *qt = (double *)malloc(sizeof(double) * (size_t)d);
    double *sq = (double *)malloc(sizeof(double) * (size_t)m);
    int64_t cb = codes ? block_code_bytes(d, bits, layout) : 0;
    int mb = m / 8;
    double kq = sqrt(3.14159265358979323846 / 2.0) / m;
    for (int64_t g = 0; g < G; ++g)
        for (int qi = 0; qi < nq; ++qi) {
            for (int j = 0; j < d; ++j) {
                qv[j] = orc_bf16_to_f32(q[(g * nq + qi) * d + j]);
                qt[j] = (s && s[j] < 0) ? -qv[j] : qv[j];
            }
            fwht_f64(qt, d);
            for (int i = 0; i < m; ++i) {
                double acc = 0.0;
                for (int j = 0; j < d; ++j) acc += (double)load_elem(S, sdtype, (int64_t)i * d + j) * qv[j];
                sq[i] = acc;
            }
            for (int64_t t = 0; t < T; ++t) {
                int64_t kt = g * T + t;
                double sc = 0.0;
                if (codes) {
                    double dot = 0.0;
                    for (int j = 0; j < d; ++j) dot += qt[j] * (double)c[get_code(codes + kt * cb, j, bits, layout)];
                    sc += (double)orc_f16_to_f32(norms[kt]) / d * dot;
                }
                double sd = 0.0;
                for (int i = 0; i < m; ++i) {
                    int bit = (signs[kt * mb + i / 8] >> (i % 8)) & 1;
                    sd += bit ? sq[i] : -sq[i];
                }
                sc += kq * (double)orc_f16_to_f32(sk_norms[kt]) * sd;
                scores[(g * nq + qi) * T + t] = sc;
            }
        }
    free(qv); free(qt); free(sq);
    return 0;
}

/* Explicit d x d Sylvester Hadamard matrix (entries +-1), for tests. */
/* Attention decode over compressed keys and values.  The QJL page ("QJL",
 * "What this is -- and what it is NOT" and "Algorithm in one paragraph")
 * pairs 1-bit JL keys with TurboQuant 4-bit values and reconstructs each
 * query-key score at attention time; the GLQ page ("KV cache compression",
 * "Inline-dequant E8 KV") dequantizes K/V inside the attention kernel with
 * the inverse Hadamard and splits the key range for long contexts.  The
 * attention itself is the standard one:
 *   out[g][q][:] = sum_t p_t * vh_t,  p_t = exp(a_t - max_u a_u) / sum_u exp(a_u - max_u a_u),
 *   a_t = softmax_scale * score[g][q][t]
 * with score the estimator of orc_score and vh_t the fp64 reconstruction of
 * value block (g, t) (orc_dequantize_f64).  fp64 throughout.  Arguments as
 * orc_score for the keys; vcodes/vnorms [G][T] blocks of d with their own
 * bits, layout, sign diagonal and table; out fp64 [G][nq][d]. */
int orc_attention(const uint16_t *q, int64_t G, int nq, int d, int m, const uint16_t *S, int sdtype,
                  const uint8_t *signs, const uint16_t *sk_norms, int64_t T,
                  const uint8_t *codes, const uint16_t *norms, int bits, int layout,
                  const int8_t *s, const float *c,
                  const uint8_t *vcodes, const uint16_t *vnorms, int vbits, int vlayout,
                  const int8_t *vs, const float *vc, double softmax_scale, double *out)
{
    if (T <= 0) return -1;
    double *sc = (double *)malloc(sizeof(double) * (size_t)nq * (size_t)T);
    double *vh = (double *)malloc(sizeof(double) * (size_t)T * (size_t)d);
    int64_t cb = codes ? block_code_bytes(d, bits, layout) : 0;
    int64_t vcb = block_code_bytes(d, vbits, vlayout);
    int mb = m / 8;
    for (int64_t g = 0; g < G; ++g) {
        orc_score(q + g * nq * d, 1, nq, d, m, S, sdtype, signs + g * T * mb, sk_norms + g * T, T,
                  codes ? codes + g * T * cb : NULL, norms ? norms + g * T : NULL, bits, layout, s, c, sc);
        orc_dequantize_f64(vcodes + g * T * vcb, vnorms + g * T, T, d, vbits, vlayout, vs, vc, vh);
        for (int qi = 0; qi < nq; ++qi) {
            const double *a = sc + (int64_t)qi * T;
            double mx = -INFINITY;
            for (int64_t t = 0; t < T; ++t) if (softmax_scale * a[t] > mx) mx = softmax_scale * a[t];
            double l = 0.0;
            for (int64_t t = 0; t < T; ++t) l += exp(softmax_scale * a[t] - mx);
            double *o = out + (g * nq + qi) * d;
            for (int j = 0; j < d; ++j) o[j] = 0.0;
            for (int64_t t = 0; t < T; ++t) {
                double p = exp(softmax_scale * a[t] - mx) / l;
                for (int j = 0; j < d; ++j) o[j] += p * vh[t * d + j];
            }
        }
    }
    free(sc); free(vh);
    return 0;
}

void orc_hadamard_matrix(int d, double *H)
{
    for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j)
            H[(int64_t)i * d + j] = (__builtin_popcount((unsigned)(i & j)) & 1) ? -1.0 : 1.0;
}

/* Apply the fp32 / fp64 FWHT to n vectors of length d (tests). */
void orc_fwht_f32(float *v, int64_t n, int d) { for (int64_t i = 0; i < n; ++i) fwht_f32(v + i * d, d); }
void orc_fwht_f64(double *v, int64_t n, int d) { for (int64_t i = 0; i < n; ++i) fwht_f64(v + i * d, d); }
float orc_pairwise_sum(const float *v, int n) { return pairwise_sum(v, n); }
