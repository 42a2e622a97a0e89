// rq_api.cu -- the C ABI of librq (declared in include/rq.h): argument
// validation, per-call tables (Lloyd-Max levels, decision thresholds, the
// exact search LUT, the sign diagonal) and kernel launches.  No device memory
// is allocated here; every table travels to the kernels as a by-value
// parameter block.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <mutex>
#include <vector>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "rq.h"
#include "rq_kernels.h"

using rq::QuantTables;

namespace rq {
// Set (bitwise OR) by a kernel whose bounded wait on the tensor core expired.
__device__ unsigned int g_device_error = 0;

// Names of the kernels the calling thread's last entry-point call enqueued,
// comma-separated (rq_last_launch).
namespace {
constexpr size_t kTraceBytes = 256;
thread_local char g_trace[kTraceBytes];
}  // namespace

void begin_call() { g_trace[0] = '\0'; }

void note_launch(const char *kernel)
{
    size_t n = std::strlen(g_trace);
    const size_t k = std::strlen(kernel);
    if (n + k + 2 > kTraceBytes) return;
    if (n) g_trace[n++] = ',';
    std::memcpy(g_trace + n, kernel, k + 1);
}
}  // namespace rq

namespace {

bool pow2_d(int d) { return d == 64 || d == 128 || d == 256 || d == 512; }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_sms()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

uint64_t splitmix64(uint64_t seed, uint64_t k)
{
    uint64_t z = seed + (k + 1ull) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// Total order on finite floats as integers (for searching the float line).
int64_t fkey(float f)
{
    int32_t i;
    std::memcpy(&i, &f, 4);
    return i >= 0 ? (int64_t)i : (int64_t)INT32_MIN - (int64_t)i;
}
float keyf(int64_t k)
{
    int32_t i = k >= 0 ? (int32_t)k : (int32_t)((int64_t)INT32_MIN - k);
    float f;
    std::memcpy(&f, &i, 4);
    return f;
}

// The device's cell function, evaluated with the same IEEE fma.
int lut_cell(float y, float a, float b, int cells)
{
    const float f = std::fmaf(y, a, b);
    uint32_t fb, mb;
    const float magic = rq::kLutMagic;
    std::memcpy(&fb, &f, 4);
    std::memcpy(&mb, &magic, 4);
    int c = (int)(fb - mb);
    return c < 0 ? 0 : (c > cells - 1 ? cells - 1 : c);
}

// Build the exact LUT: each cell's set of y values is an interval; a cell may
// hold at most one decision threshold.  Returns false when no grid of at most
// kMaxLutCells cells separates the thresholds (the kernels then binary-search).
bool build_lut(const float *t, int nb, QuantTables &T)
{
    if (nb < 1) return false;
    double min_gap = INFINITY;
    for (int k = 0; k + 1 < nb; ++k) min_gap = std::fmin(min_gap, (double)t[k + 1] - (double)t[k]);
    if (!(min_gap > 0)) return false;
    if (!std::isfinite(min_gap)) min_gap = 1.0;
    const double span = (double)t[nb - 1] - (double)t[0];
    const float lo_lim = -1.0e5f, hi_lim = 1.0e5f;   // |y| <= sqrt(d) for finite input
    for (int attempt = 0; attempt < 64; ++attempt) {
        const float a = (float)((1.0 + 0.125 * attempt) / min_gap);
        const int cells = (int)std::ceil(span * (double)a) + 4;
        if (cells > rq::kMaxLutCells || !(a > 0) || !std::isfinite(a)) return false;
        const float b0 = (float)(2.0 - std::floor((double)t[0] * (double)a));
        const float b = rq::kLutMagic + b0;
        if (std::fabs((double)b0) + std::fabs((double)a) * 1.0e5 > 4.0e6) return false;
        // ylo[j]: smallest float y in [lo_lim, hi_lim] with cell(y) >= j.
        std::vector<float> ylo(cells + 1);
        ylo[0] = -INFINITY;
        ylo[cells] = INFINITY;
        for (int j = 1; j < cells; ++j) {
            int64_t lo = fkey(lo_lim), hi = fkey(hi_lim);
            if (lut_cell(keyf(hi), a, b, cells) < j) { ylo[j] = INFINITY; continue; }
            while (lo < hi) {
                const int64_t mid = lo + (hi - lo) / 2;
                if (lut_cell(keyf(mid), a, b, cells) >= j) hi = mid; else lo = mid + 1;
            }
            ylo[j] = keyf(lo);
        }
        bool ok = true;
        for (int j = 0; j < cells && ok; ++j) {
            int below = 0, inside = 0;
            float cand = INFINITY;
            for (int k = 0; k < nb; ++k) {
                if (t[k] < ylo[j]) ++below;
                else if (t[k] < ylo[j + 1]) { ++inside; cand = t[k]; }
            }
            if (inside > 1) ok = false;
            T.lut_k[j] = (uint32_t)below;
            T.lut_t[j] = inside ? cand : INFINITY;
        }
        if (ok) {
            T.lut_a = a;
            T.lut_b = b;
            T.lut_cells = cells;
            return true;
        }
    }
    return false;
}

// The device's saturating-grid cell function: fma.rn.sat (clamp to [0, 1],
// NaN to 0) then an fma that rounds fs * k to an integer in the low mantissa
// bits of kLutMagic.
int sat_cell(float y, float a, float b, float k)
{
    float f = std::fmaf(y, a, b);
    f = f > 0.0f ? (f < 1.0f ? f : 1.0f) : 0.0f;
    const float g = std::fmaf(f, k, rq::kLutMagic);
    uint32_t gb, mb;
    const float magic = rq::kLutMagic;
    std::memcpy(&gb, &g, 4);
    std::memcpy(&mb, &magic, 4);
    return (int)(gb - mb);
}

// Saturating-grid LUT over [t_0 - w, t_last + w] with cell width w below the
// smallest boundary gap; every cell's y-interval is found by bisection on the
// float line and checked to hold at most one boundary.
bool build_sat_lut(const float *t, int nb, QuantTables &T)
{
    if (nb < 1) return false;
    double min_gap = INFINITY;
    for (int k = 0; k + 1 < nb; ++k) min_gap = std::fmin(min_gap, (double)t[k + 1] - (double)t[k]);
    if (!(min_gap > 0)) return false;
    if (!std::isfinite(min_gap)) min_gap = 1.0;
    const float lo_lim = -1.0e5f, hi_lim = 1.0e5f;
    for (int attempt = 0; attempt < 64; ++attempt) {
        const double w = min_gap / (1.25 + 0.125 * attempt);
        const double ylo = (double)t[0] - w, yhi = (double)t[nb - 1] + w;
        const int kcells = (int)std::ceil((yhi - ylo) / w);
        if (kcells + 1 > rq::kMaxLutCells) return false;
        const float a = (float)(1.0 / (yhi - ylo));
        const float b = (float)(-ylo / (yhi - ylo));
        const float k = (float)kcells;
        const int cells = kcells + 1;
        if (!(a > 0) || !std::isfinite(a) || !std::isfinite(b)) return false;
        std::vector<float> lo(cells + 1);
        lo[0] = -INFINITY;
        lo[cells] = INFINITY;
        for (int j = 1; j < cells; ++j) {
            int64_t l = fkey(lo_lim), h = fkey(hi_lim);
            if (sat_cell(keyf(h), a, b, k) < j) { lo[j] = INFINITY; continue; }
            while (l < h) {
                const int64_t mid = l + (h - l) / 2;
                if (sat_cell(keyf(mid), a, b, k) >= j) h = mid; else l = mid + 1;
            }
            lo[j] = keyf(l);
        }
        bool ok = sat_cell(keyf(fkey(lo_lim)), a, b, k) == 0 && sat_cell(keyf(fkey(hi_lim)), a, b, k) == cells - 1;
        for (int j = 0; j < cells && ok; ++j) {
            int below = 0, inside = 0;
            float cand = INFINITY;
            for (int q = 0; q < nb; ++q) {
                if (t[q] < lo[j]) ++below;
                else if (t[q] < lo[j + 1]) { ++inside; cand = t[q]; }
            }
            if (inside > 1) ok = false;
            T.sat_base[j] = (uint32_t)below;
            T.sat_t[j] = inside ? cand : INFINITY;
        }
        if (ok) {
            T.sat_a = a;
            T.sat_b = b;
            T.sat_k = k;
            T.sat_cells = cells;
            return true;
        }
    }
    return false;
}

// Validate a host centroid table and fill the per-call tables.
rq_status make_tables(const float *centroids, int bits, int d, int use_signs, uint64_t sign_seed,
                      QuantTables &T)
{
    std::memset(&T, 0, sizeof(T));
    const int K = 1 << bits;
    if (!centroids) return RQ_EINVAL;
    for (int k = 0; k < K; ++k) {
        if (!std::isfinite(centroids[k]) || std::fabs(centroids[k]) > 1.0e4f) return RQ_EINVAL;
        if (k > 0 && !(centroids[k] > centroids[k - 1])) return RQ_EINVAL;
        T.centroid[k] = centroids[k];
    }
    T.levels = K;
    for (int k = 0; k + 1 < K; ++k) {
        const float s = centroids[k] + centroids[k + 1];
        T.bound[k] = 0.5f * s;
    }
    T.bound[K - 1] = INFINITY;
    if (!build_lut(T.bound, K - 1, T)) T.lut_cells = 0;
    if (!build_sat_lut(T.bound, K - 1, T)) T.sat_cells = 0;
    if (use_signs) {
        for (int w = 0; w < (d + 63) / 64; ++w) {          // one SplitMix64 output per 64 coordinates
            const uint64_t r = splitmix64(sign_seed, (uint64_t)w);
            T.sign_words[2 * w] = (uint32_t)(r & 0xffffffffu);
            T.sign_words[2 * w + 1] = (uint32_t)(r >> 32);
        }
    }
    return RQ_OK;
}

// The tables depend only on (centroids, bits, d, signs, seed) and take tens of
// microseconds of host time to build (the LUT grids are verified by bisection
// on the float line), so the last few are kept: a caller that quantizes
// layer after layer with one configuration pays for them once.
struct TableCacheEntry {
    bool valid;
    int bits, d, use_signs;
    uint64_t seed;
    float centroids[rq::kMaxLevels];
    QuantTables T;
};
constexpr int kTableCache = 8;
std::mutex g_table_mutex;
TableCacheEntry g_table_cache[kTableCache];
int g_table_next = 0;

rq_status tables_for(const float *centroids, int bits, int d, int use_signs, uint64_t sign_seed, QuantTables &T)
{
    if (!centroids || bits < 1 || bits > 8) return RQ_EINVAL;
    const int K = 1 << bits;
    const uint64_t seed = use_signs ? sign_seed : 0;
    {
        std::lock_guard<std::mutex> lock(g_table_mutex);
        for (const TableCacheEntry &e : g_table_cache)
            if (e.valid && e.bits == bits && e.d == d && e.use_signs == (use_signs != 0) && e.seed == seed &&
                std::memcmp(e.centroids, centroids, sizeof(float) * K) == 0) {
                T = e.T;
                return RQ_OK;
            }
    }
    const rq_status s = make_tables(centroids, bits, d, use_signs, sign_seed, T);
    if (s) return s;
    std::lock_guard<std::mutex> lock(g_table_mutex);
    TableCacheEntry &e = g_table_cache[g_table_next];
    g_table_next = (g_table_next + 1) % kTableCache;
    e.valid = true;
    e.bits = bits;
    e.d = d;
    e.use_signs = use_signs != 0;
    e.seed = seed;
    std::memcpy(e.centroids, centroids, sizeof(float) * K);
    e.T = T;
    return RQ_OK;
}

rq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? RQ_OK : RQ_ECUDA; }

PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;   // driver entry point, looked up once
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// Lloyd-Max iteration for N(0,1): levels are conditional means of their cells,
// thresholds are midpoints.  phi / Phi differences on the tail side.
double npdf(double t) { return std::isinf(t) ? 0.0 : std::exp(-0.5 * t * t) * 0.39894228040143267794; }
double cell_mass(double a, double b)
{
    const double r = 0.70710678118654752440;
    if (a >= 0.0) return 0.5 * (std::erfc(a * r) - std::erfc(b * r));
    if (b <= 0.0) return 0.5 * (std::erfc(-b * r) - std::erfc(-a * r));
    return 1.0 - 0.5 * std::erfc(-a * r) - 0.5 * std::erfc(b * r);
}

}  // namespace

bool rq::make_rows64_tmap(CUtensorMap *map, const void *ptr, int64_t rows)
{
    auto enc = tmap_encoder();
    if (!enc || rows <= 0 || rows >= ((int64_t)1 << 31)) return false;
    const cuuint64_t dims[2] = {64, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {128};
    const cuuint32_t box[2] = {64, 256};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool rq::make_vectors_tmap(CUtensorMap *map, const void *ptr, int64_t n, int d, int box_rows)
{
    auto enc = tmap_encoder();
    if (!enc || n <= 0 || n >= ((int64_t)1 << 31) || d % 64 || box_rows <= 0 || box_rows > 256) return false;
    const cuuint64_t dims[3] = {64, (cuuint64_t)(d / 64), (cuuint64_t)n};
    const cuuint64_t strides[2] = {128, (cuuint64_t)d * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool rq::make_proj_tmap(CUtensorMap *map, const void *ptr, int m, int d, int box_rows)
{
    auto enc = tmap_encoder();
    if (!enc || m <= 0 || d % 64 || box_rows <= 0 || box_rows > 256) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)m};
    const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool rq::make_scores_tmap(CUtensorMap *map, const void *ptr, int64_t T, int nq, int64_t G)
{
    auto enc = tmap_encoder();
    if (!enc || T <= 0 || T % 4 || T >= ((int64_t)1 << 31) || nq <= 0 || G <= 0) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)T, (cuuint64_t)nq, (cuuint64_t)G};
    const cuuint64_t strides[2] = {(cuuint64_t)T * 4, (cuuint64_t)T * 4 * (cuuint64_t)nq};
    const cuuint32_t box[3] = {32, 16, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

extern "C" {

const char *rq_status_string(int status)
{
    switch (status) {
    case RQ_OK: return "RQ_OK";
    case RQ_EINVAL: return "RQ_EINVAL: invalid argument";
    case RQ_EALIGN: return "RQ_EALIGN: device pointer not 16-byte aligned";
    case RQ_ESIZE: return "RQ_ESIZE: size out of range";
    case RQ_EUNSUPPORTED: return "RQ_EUNSUPPORTED: unsupported combination";
    case RQ_ECUDA: return "RQ_ECUDA: CUDA runtime error";
    case RQ_EDEVICE: return "RQ_EDEVICE: a kernel gave up waiting on the tensor core; outputs are invalid";
    default: return "unknown rq_status";
    }
}

int64_t rq_code_bytes(int64_t n, int d, int bits, rq_layout layout)
{
    if ((!pow2_d(d) && !rq::bd_size(d)) || bits < 1 || bits > 8 || n < 0 || n % d) return -1;
    if (layout == RQ_CODES_INT8) return n;
    if (layout != RQ_CODES_PACKED) return -1;
    return (n / d) * ((int64_t)d * bits / 8);
}

rq_status rq_lloyd_max(int bits, float *centroids_out)
{
    if (bits < 1 || bits > 8 || !centroids_out) return RQ_EINVAL;
    const int K = 1 << bits;
    std::vector<double> c(K), t(K + 1);
    for (int i = 0; i < K; ++i) c[i] = 4.0 * (2.0 * i + 1.0 - K) / K;   // sorted start in [-4, 4]
    for (int it = 0; it < 1000000; ++it) {
        t[0] = -INFINITY;
        t[K] = INFINITY;
        for (int i = 1; i < K; ++i) t[i] = 0.5 * (c[i - 1] + c[i]);
        double worst = 0.0;
        for (int i = 0; i < K; ++i) {
            const double nc = (npdf(t[i]) - npdf(t[i + 1])) / cell_mass(t[i], t[i + 1]);
            worst = std::fmax(worst, std::fabs(nc - c[i]));
            c[i] = nc;
        }
        if (worst < 1e-13) break;
    }
    for (int i = 0; i < K / 2; ++i) {
        const double a = 0.5 * (c[K - 1 - i] - c[i]);
        c[i] = -a;
        c[K - 1 - i] = a;
    }
    for (int i = 0; i < K; ++i) centroids_out[i] = (float)c[i];
    return RQ_OK;
}

static rq_status check_common(int64_t n, int d, int bits, rq_layout layout)
{
    if (!pow2_d(d) && !rq::bd_size(d)) return d > 0 && (d & (d - 1)) == 0 ? RQ_EUNSUPPORTED : RQ_EINVAL;
    if (bits < 1 || bits > 8) return RQ_EINVAL;
    if (layout != RQ_CODES_PACKED && layout != RQ_CODES_INT8) return RQ_EINVAL;
    if (n < 0 || n % d) return RQ_EINVAL;
    if (n / 64 >= ((int64_t)1 << 31)) return RQ_ESIZE;   // TMA row coordinates are int32
    return RQ_OK;
}

static rq_status quantize_impl(const void *x, rq_dtype dtype, int64_t n, int d, int bits, rq_layout layout,
                               int use_signs, uint64_t sign_seed, const float *centroids, int m,
                               const void *proj, void *codes, uint16_t *norms, uint8_t *qjl_signs,
                               uint16_t *qjl_norms, cudaStream_t stream)
{
    rq::begin_call();
    rq_status s = check_common(n, d, bits, layout);
    if (s) return s;
    if (dtype != RQ_F16 && dtype != RQ_BF16) return RQ_EINVAL;
    const bool qjl = qjl_signs != nullptr || qjl_norms != nullptr || proj != nullptr;
    if (qjl && (!qjl_signs || !qjl_norms || !proj || m < 8 || m > 512 || m % 8)) return RQ_EINVAL;
    if (qjl && !pow2_d(d)) return RQ_EUNSUPPORTED;          // the residual sketch takes power-of-two blocks
    if (n == 0) return RQ_OK;
    if (!x || !codes || !norms) return RQ_EINVAL;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(norms)) return RQ_EALIGN;
    if (qjl && (!aligned16(proj) || !aligned16(qjl_signs) || !aligned16(qjl_norms))) return RQ_EALIGN;
    QuantTables T;
    s = tables_for(centroids, bits, d, use_signs, sign_seed, T);
    if (s) return s;
    rq::QuantArgs a{};
    a.x = x; a.nblocks = n / d; a.d = d; a.pw = layout == RQ_CODES_INT8 ? 8 : bits; a.bf16 = dtype == RQ_BF16;
    a.tables = &T; a.codes = codes; a.norms = norms;
    a.m = qjl ? m : 0; a.proj = proj; a.qsigns = qjl_signs; a.qnorms = qjl_norms;
    a.num_sms = num_sms();
    if (a.num_sms <= 0) return RQ_ECUDA;
    if (!pow2_d(d)) return cuda_status(rq::launch_quantize_bd(a, stream));
    if (!rq::make_rows64_tmap(&a.tmap_x, x, n / 64)) return RQ_ECUDA;
    a.has_tmap_v = qjl && rq::make_vectors_tmap(&a.tmap_v, x, n / d, d);
    a.has_tmap_v32 = !qjl && d == 128 && rq::make_vectors_tmap(&a.tmap_v32, x, n / d, d, 32);
    if (qjl && d >= 128) {
        const int m16 = (m + 15) / 16 * 16;
        a.has_tmap_s = (m16 <= 256 || m16 % 256 == 0) && rq::make_proj_tmap(&a.tmap_s, proj, m, d, m16 < 256 ? m16 : 256);
    }
    return cuda_status(rq::launch_quantize(a, stream));
}

rq_status rq_quantize(const void *x, rq_dtype dtype, int64_t n, int d, int bits, rq_layout layout,
                      int use_signs, uint64_t sign_seed, const float *centroids,
                      void *codes, uint16_t *norms, rq_stream_t stream)
{
    return quantize_impl(x, dtype, n, d, bits, layout, use_signs, sign_seed, centroids, 0, nullptr, codes, norms,
                         nullptr, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

rq_status rq_quantize_qjl(const void *x, rq_dtype dtype, int64_t n, int d, int bits, rq_layout layout,
                          int use_signs, uint64_t sign_seed, const float *centroids,
                          int m, const void *proj, void *codes, uint16_t *norms,
                          uint8_t *qjl_signs, uint16_t *qjl_norms, rq_stream_t stream)
{
    if (!proj || !qjl_signs || !qjl_norms) return RQ_EINVAL;
    return quantize_impl(x, dtype, n, d, bits, layout, use_signs, sign_seed, centroids, m, proj, codes, norms,
                         qjl_signs, qjl_norms, reinterpret_cast<cudaStream_t>(stream));
}

rq_status rq_dequantize(const void *codes, const uint16_t *norms, int64_t n, int d, int bits,
                        rq_layout layout, int use_signs, uint64_t sign_seed, const float *centroids,
                        void *out, rq_dtype out_dtype, rq_stream_t stream)
{
    rq::begin_call();
    rq_status s = check_common(n, d, bits, layout);
    if (s) return s;
    if (out_dtype != RQ_F16 && out_dtype != RQ_BF16) return RQ_EINVAL;
    if (n == 0) return RQ_OK;
    if (!codes || !norms || !out) return RQ_EINVAL;
    if (!aligned16(codes) || !aligned16(norms) || !aligned16(out)) return RQ_EALIGN;
    QuantTables T;
    s = tables_for(centroids, bits, d, use_signs, sign_seed, T);
    if (s) return s;
    rq::DequantArgs a{};
    a.codes = codes; a.norms = norms; a.nblocks = n / d; a.d = d; a.pw = layout == RQ_CODES_INT8 ? 8 : bits;
    a.bf16 = out_dtype == RQ_BF16; a.tables = &T; a.out = out;
    a.num_sms = num_sms();
    if (a.num_sms <= 0) return RQ_ECUDA;
    if (!pow2_d(d)) return cuda_status(rq::launch_dequantize_bd(a, reinterpret_cast<cudaStream_t>(stream)));
    if (!rq::make_rows64_tmap(&a.tmap_out, out, n / 64)) return RQ_ECUDA;
    a.has_tmap_out32 = d == 128 && rq::make_vectors_tmap(&a.tmap_out32, out, n / d, d, 32);
    return cuda_status(rq::launch_dequantize(a, reinterpret_cast<cudaStream_t>(stream)));
}

rq_status qjl_make_projection(uint64_t seed, int m, int d, rq_dtype dtype, void *proj, rq_stream_t stream)
{
    rq::begin_call();
    if (m < 8 || m > 512 || m % 8 || !pow2_d(d)) return RQ_EINVAL;
    if (dtype != RQ_F16 && dtype != RQ_BF16) return RQ_EINVAL;
    if (!proj) return RQ_EINVAL;
    if (!aligned16(proj)) return RQ_EALIGN;
    return cuda_status(rq::launch_projection(seed, m, d, dtype == RQ_BF16, proj,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

rq_status qjl_sketch(const void *x, rq_dtype dtype, int64_t n_vec, int d, int m, const void *proj,
                     uint8_t *signs, uint16_t *norms, rq_stream_t stream)
{
    rq::begin_call();
    if (!pow2_d(d)) return RQ_EINVAL;
    if (m < 8 || m > 512 || m % 8) return RQ_EINVAL;
    if (dtype != RQ_F16 && dtype != RQ_BF16) return RQ_EINVAL;
    if (n_vec < 0) return RQ_EINVAL;
    if (n_vec > ((int64_t)1 << 34)) return RQ_ESIZE;
    if (n_vec == 0) return RQ_OK;
    if (!x || !proj || !signs || !norms) return RQ_EINVAL;
    if (!aligned16(x) || !aligned16(proj) || !aligned16(signs) || !aligned16(norms)) return RQ_EALIGN;
    rq::SketchArgs a{};
    a.x = x; a.nvec = n_vec; a.d = d; a.m = m; a.bf16 = dtype == RQ_BF16; a.proj = proj; a.signs = signs;
    a.norms = norms; a.num_sms = num_sms();
    if (a.num_sms <= 0) return RQ_ECUDA;
    a.has_tmap_k = rq::make_vectors_tmap(&a.tmap_k, x, n_vec, d);
    {
        const int m16 = (m + 15) & ~15;
        a.has_tmap_s = (m16 <= 256 || m16 % 256 == 0) && rq::make_proj_tmap(&a.tmap_s, proj, m, d, m16 < 256 ? m16 : 256);
    }
    return cuda_status(rq::launch_sketch(a, reinterpret_cast<cudaStream_t>(stream)));
}

size_t qjl_attention_workspace_bytes(int64_t G, int n_q, int d, int m, int64_t T)
{
    if (G < 0 || n_q < 0 || d < 0 || m < 0 || T < 0) return 0;
    const int sms = num_sms();
    return rq::attention_workspace_bytes(G, n_q, d, m, T, sms > 0 ? sms : 1);
}

rq_status qjl_attention(const void *q, int64_t G, int n_q, int d, int m, const void *proj, rq_dtype proj_dtype,
                        const uint8_t *signs, const uint16_t *sk_norms, int64_t T_len,
                        const void *codes, const uint16_t *norms, int bits, rq_layout layout,
                        int use_signs, uint64_t sign_seed, const float *centroids,
                        const void *v_codes, const uint16_t *v_norms, int v_bits, rq_layout v_layout,
                        int v_use_signs, uint64_t v_sign_seed, const float *v_centroids,
                        float softmax_scale, float *out, void *workspace, size_t workspace_bytes,
                        rq_stream_t stream)
{
    rq::begin_call();
    if (!pow2_d(d)) return RQ_EINVAL;
    if (m < 8 || m > 512 || m % 8) return RQ_EINVAL;
    if (proj_dtype != RQ_F16 && proj_dtype != RQ_BF16) return RQ_EINVAL;
    if (G < 0 || n_q < 0 || T_len < 0) return RQ_EINVAL;
    if (!(softmax_scale == softmax_scale) || softmax_scale < 0.0f || softmax_scale > 1e30f) return RQ_EINVAL;
    if (G > 65535 || n_q > 65535 || T_len > ((int64_t)1 << 31)) return RQ_ESIZE;
    if (G == 0 || n_q == 0) return RQ_OK;
    if (T_len == 0) return RQ_EINVAL;                       // softmax over no keys
    rq_status s = check_common(0, d, v_bits, v_layout);
    if (s) return s;
    if (!q || !proj || !signs || !sk_norms || !v_codes || !v_norms || !out || !workspace) return RQ_EINVAL;
    if (!aligned16(q) || !aligned16(proj) || !aligned16(signs) || !aligned16(sk_norms) || !aligned16(v_codes) ||
        !aligned16(v_norms) || !aligned16(out) || !aligned16(workspace))
        return RQ_EALIGN;
    QuantTables T;
    std::memset(&T, 0, sizeof(T));
    int pw = 0;
    if (codes) {
        s = check_common(0, d, bits, layout);
        if (s) return s;
        if (!norms) return RQ_EINVAL;
        if (!aligned16(codes) || !aligned16(norms)) return RQ_EALIGN;
        s = tables_for(centroids, bits, d, use_signs, sign_seed, T);
        if (s) return s;
        pw = layout == RQ_CODES_INT8 ? 8 : bits;
    }
    QuantTables TV;
    s = tables_for(v_centroids, v_bits, d, v_use_signs, v_sign_seed, TV);
    if (s) return s;
    const int vpw = v_layout == RQ_CODES_INT8 ? 8 : v_bits;
    if (!rq::attention_supported(n_q, d, m, codes != nullptr, pw, vpw)) return RQ_EUNSUPPORTED;
    rq::AttnArgs a{};
    a.k.q = static_cast<const uint16_t *>(q); a.k.G = G; a.k.nq = n_q; a.k.d = d; a.k.m = m; a.k.proj = proj;
    a.k.proj_bf16 = proj_dtype == RQ_BF16; a.k.signs = signs; a.k.sk_norms = sk_norms; a.k.T = T_len;
    a.k.codes = static_cast<const uint8_t *>(codes); a.k.norms = norms; a.k.pw = pw; a.k.tables = &T;
    a.vcodes = static_cast<const uint8_t *>(v_codes); a.vnorms = v_norms; a.vpw = vpw; a.vtables = &TV;
    a.softmax_scale = softmax_scale; a.out = out; a.workspace = workspace;
    a.num_sms = num_sms();
    if (a.num_sms <= 0) return RQ_ECUDA;
    a.k.num_sms = a.num_sms;
    if (workspace_bytes < rq::attention_workspace_bytes(G, n_q, d, m, T_len, a.num_sms)) return RQ_ESIZE;
    return cuda_status(rq::launch_attention(a, reinterpret_cast<cudaStream_t>(stream)));
}

const char *rq_last_launch(void) { return rq::g_trace; }

rq_status rq_probe_bounded_wait(uint32_t polls, rq_stream_t stream)
{
    rq::begin_call();
    if (polls < 1 || polls > rq::kProbeMaxPolls) return RQ_EINVAL;
    return cuda_status(rq::launch_wait_probe(polls, reinterpret_cast<cudaStream_t>(stream)));
}

rq_status rq_device_error(int clear)
{
    unsigned int word = 0;
    if (cudaMemcpyFromSymbol(&word, rq::g_device_error, sizeof(word)) != cudaSuccess) return RQ_ECUDA;
    if (clear && word) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(rq::g_device_error, &zero, sizeof(zero)) != cudaSuccess) return RQ_ECUDA;
    }
    return word ? RQ_EDEVICE : RQ_OK;
}

size_t qjl_score_workspace_bytes(int64_t G, int n_q, int d, int m)
{
    if (G < 0 || n_q < 0 || d < 0 || m < 0) return 0;
    return rq::score_workspace_bytes(G, n_q, d, m);
}

rq_status qjl_score(const void *q, int64_t G, int n_q, int d, int m, const void *proj, rq_dtype proj_dtype,
                    const uint8_t *signs, const uint16_t *sk_norms, int64_t T_len,
                    const void *codes, const uint16_t *norms, int bits, rq_layout layout,
                    int use_signs, uint64_t sign_seed, const float *centroids,
                    float *scores, void *workspace, size_t workspace_bytes, rq_stream_t stream)
{
    rq::begin_call();
    if (!pow2_d(d)) return RQ_EINVAL;
    if (m < 8 || m > 512 || m % 8) return RQ_EINVAL;
    if (proj_dtype != RQ_F16 && proj_dtype != RQ_BF16) return RQ_EINVAL;
    if (G < 0 || n_q < 0 || T_len < 0) return RQ_EINVAL;
    if (G > 65535 || n_q > 32 * 65535 || T_len > ((int64_t)1 << 31)) return RQ_ESIZE;
    if (G == 0 || n_q == 0 || T_len == 0) return RQ_OK;
    if (!q || !proj || !signs || !sk_norms || !scores || !workspace) return RQ_EINVAL;
    if (workspace_bytes < rq::score_workspace_bytes(G, n_q, d, m)) return RQ_ESIZE;
    if (!aligned16(q) || !aligned16(proj) || !aligned16(signs) || !aligned16(sk_norms) || !aligned16(scores) ||
        !aligned16(workspace))
        return RQ_EALIGN;
    QuantTables T;
    std::memset(&T, 0, sizeof(T));
    int pw = 0;
    if (codes) {
        rq_status s = check_common(0, d, bits, layout);
        if (s) return s;
        if (!norms) return RQ_EINVAL;
        if (!aligned16(codes) || !aligned16(norms)) return RQ_EALIGN;
        s = tables_for(centroids, bits, d, use_signs, sign_seed, T);
        if (s) return s;
        pw = layout == RQ_CODES_INT8 ? 8 : bits;
    }
    rq::ScoreArgs a{};
    a.q = static_cast<const uint16_t *>(q); a.G = G; a.nq = n_q; a.d = d; a.m = m; a.proj = proj;
    a.proj_bf16 = proj_dtype == RQ_BF16; a.signs = signs; a.sk_norms = sk_norms; a.T = T_len;
    a.codes = static_cast<const uint8_t *>(codes); a.norms = norms; a.pw = pw; a.tables = &T;
    a.scores = scores; a.workspace = static_cast<float *>(workspace); a.num_sms = num_sms();
    if (a.num_sms <= 0) return RQ_ECUDA;
    a.has_tmap_scores = rq::make_scores_tmap(&a.tmap_scores, scores, T_len, n_q, G);
    return cuda_status(rq::launch_score(a, reinterpret_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------------ dense rotation

namespace {

// Gauss-Legendre nodes and weights on [-1, 1]: Newton iteration on P_n from the
// three-term recurrence (k P_k = (2k - 1) z P_{k-1} - (k - 1) P_{k-2}).
void gauss_legendre16(double *x, double *w)
{
    constexpr int n = 16;
    const double pi = 3.14159265358979323846;
    for (int i = 0; i < n / 2; ++i) {
        double z = std::cos(pi * (i + 0.75) / (n + 0.5)), dp = 1.0;
        for (int it = 0; it < 100; ++it) {
            double p0 = 1.0, p1 = z;
            for (int k = 2; k <= n; ++k) {
                const double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
                p0 = p1;
                p1 = p2;
            }
            dp = n * (z * p1 - p0) / (z * z - 1.0);
            const double dz = p1 / dp;
            z -= dz;
            if (std::fabs(dz) < 1e-16) break;
        }
        x[i] = -z;
        x[n - 1 - i] = z;
        w[i] = w[n - 1 - i] = 2.0 / ((1.0 - z * z) * dp * dp);
    }
}

// Unnormalised mass of f_d(t) ~ (1 - t^2)^((d-3)/2) over [a, b] (0 <= a < b <= 1):
// composite 16-point Gauss-Legendre, panels a quarter of the law's width 1/sqrt(d).
double beta_mass(double a, double b, int d, const double *gx, const double *gw)
{
    const double al = 0.5 * (d - 3);
    int panels = (int)std::ceil((b - a) * std::sqrt((double)d) * 4.0);
    panels = panels < 4 ? 4 : (panels > 8192 ? 8192 : panels);
    const double h = (b - a) / panels;
    double s = 0.0;
    for (int p = 0; p < panels; ++p) {
        const double m = a + (p + 0.5) * h;
        for (int k = 0; k < 16; ++k) {
            const double t = m + 0.5 * h * gx[k];
            s += gw[k] * (al == 0.0 ? 1.0 : std::exp(al * std::log1p(-t * t)));
        }
    }
    return 0.5 * h * s;
}

// Unnormalised first moment over [a, b]: d/dt (1 - t^2)^((d-1)/2) = -(d-1) t (1 - t^2)^((d-3)/2).
double beta_moment(double a, double b, int d)
{
    const double k = 0.5 * (d - 1);
    auto g = [&](double t) { return t >= 1.0 ? 0.0 : std::exp(k * std::log1p(-t * t)); };
    return (g(a) - g(b)) / (2.0 * k);
}

}  // namespace

rq_status rq_beta_lloyd_max(int d, int bits, float *centroids_out)
{
    if (d < 3 || d > 65536 || bits < 1 || bits > 8 || !centroids_out) return RQ_EINVAL;
    const int K = 1 << bits, h = K / 2;
    double gx[16], gw[16];
    gauss_legendre16(gx, gw);
    std::vector<double> c(h), t(h + 1);
    for (int k = 0; k < h; ++k) c[k] = (k + 0.5) / h * std::fmin(1.0, 3.0 / std::sqrt((double)d));
    for (int it = 0; it < 200000; ++it) {
        t[0] = 0.0;
        t[h] = 1.0;
        for (int k = 1; k < h; ++k) t[k] = 0.5 * (c[k - 1] + c[k]);
        double worst = 0.0;
        for (int k = 0; k < h; ++k) {
            const double nc = beta_moment(t[k], t[k + 1], d) / beta_mass(t[k], t[k + 1], d, gx, gw);
            worst = std::fmax(worst, std::fabs(nc - c[k]));
            c[k] = nc;
        }
        if (worst < 1e-15) break;
    }
    for (int k = 0; k < h; ++k) {
        centroids_out[h + k] = (float)c[k];
        centroids_out[h - 1 - k] = (float)-c[k];
    }
    return RQ_OK;
}

rq_status rq_make_rotation(int d, uint64_t seed, float *pi_out)
{
    if (d < 1 || d > 4096 || !pi_out) return RQ_EINVAL;
    const size_t n = (size_t)d;
    std::vector<double> A(n * n), V(n * n, 0.0), beta(n, 0.0), rdiag(n, 0.0);
    for (size_t i = 0; i < n; ++i)                  // G[i][j] = Box-Muller over SplitMix64 outputs 2k, 2k+1
        for (size_t j = 0; j < n; ++j) {
            const uint64_t k = (uint64_t)(i * n + j);
            const double u1 = (double)((splitmix64(seed, 2ull * k) >> 11) + 1ull) * 0x1p-53;
            const double u2 = (double)(splitmix64(seed, 2ull * k + 1ull) >> 11) * 0x1p-53;
            A[i * n + j] = std::sqrt(-2.0 * std::log(u1)) * std::cos(6.283185307179586476925286766559 * u2);
        }
    // Householder QR: reflection k maps column k below the diagonal onto e_k.
    for (size_t k = 0; k < n; ++k) {
        double nx = 0.0;
        for (size_t i = k; i < n; ++i) nx += A[i * n + k] * A[i * n + k];
        nx = std::sqrt(nx);
        const double x0 = A[k * n + k];
        const double alpha = x0 >= 0.0 ? -nx : nx;
        double vv = 0.0;
        for (size_t i = k; i < n; ++i) {
            V[i * n + k] = A[i * n + k] - (i == k ? alpha : 0.0);
            vv += V[i * n + k] * V[i * n + k];
        }
        rdiag[k] = nx == 0.0 ? 0.0 : alpha;
        if (vv == 0.0) continue;
        beta[k] = 2.0 / vv;
        for (size_t j = k; j < n; ++j) {
            double s = 0.0;
            for (size_t i = k; i < n; ++i) s += V[i * n + k] * A[i * n + j];
            s *= beta[k];
            for (size_t i = k; i < n; ++i) A[i * n + j] -= s * V[i * n + k];
        }
    }
    // Q = H_0 H_1 ... H_{n-1} applied to the identity, from the last reflection back.
    std::vector<double> Q(n * n, 0.0);
    for (size_t i = 0; i < n; ++i) Q[i * n + i] = 1.0;
    for (size_t kk = n; kk-- > 0;) {
        if (beta[kk] == 0.0) continue;
        for (size_t j = 0; j < n; ++j) {
            double s = 0.0;
            for (size_t i = kk; i < n; ++i) s += V[i * n + kk] * Q[i * n + j];
            s *= beta[kk];
            for (size_t i = kk; i < n; ++i) Q[i * n + j] -= s * V[i * n + kk];
        }
    }
    // sign fix: column k times sign(R_kk)
    for (size_t i = 0; i < n; ++i)
        for (size_t j = 0; j < n; ++j) pi_out[i * n + j] = (float)(rdiag[j] < 0.0 ? -Q[i * n + j] : Q[i * n + j]);
    return RQ_OK;
}

static rq_status check_dense(int64_t n, int d, int bits, rq_layout layout, rq_dtype dtype)
{
    if (d != 128) return (d > 0 && d <= 512) ? RQ_EUNSUPPORTED : RQ_EINVAL;
    if (bits < 1 || bits > 8) return RQ_EINVAL;
    if (layout != RQ_CODES_PACKED && layout != RQ_CODES_INT8) return RQ_EINVAL;
    if (dtype != RQ_F16 && dtype != RQ_BF16) return RQ_EINVAL;
    if (n < 0 || n % d) return RQ_EINVAL;
    if (n / d >= ((int64_t)1 << 31)) return RQ_ESIZE;   // TMA row coordinates are int32
    return RQ_OK;
}

rq_status rq_quantize_dense(const void *x, rq_dtype dtype, int64_t n, int d, const void *pi, int bits,
                            rq_layout layout, const float *centroids, void *codes, uint16_t *norms,
                            rq_stream_t stream)
{
    rq::begin_call();
    rq_status s = check_dense(n, d, bits, layout, dtype);
    if (s) return s;
    if (n == 0) return RQ_OK;
    if (!x || !pi || !codes || !norms) return RQ_EINVAL;
    if (!aligned16(x) || !aligned16(pi) || !aligned16(codes) || !aligned16(norms)) return RQ_EALIGN;
    QuantTables T;
    s = tables_for(centroids, bits, d, 0, 0, T);
    if (s) return s;
    rq::DenseArgs a{};
    a.nvec = n / d; a.bf16 = dtype == RQ_BF16; a.pw = layout == RQ_CODES_INT8 ? 8 : bits; a.tables = &T;
    a.codes = static_cast<uint8_t *>(codes); a.norms = norms; a.num_sms = num_sms();
    if (a.num_sms <= 0) return RQ_ECUDA;
    if (!rq::make_vectors_tmap(&a.tmap_x, x, a.nvec, d, 128) || !rq::make_proj_tmap(&a.tmap_pi, pi, d, d, 128))
        return RQ_ECUDA;
    return cuda_status(rq::launch_quantize_dense(a, reinterpret_cast<cudaStream_t>(stream)));
}

rq_status rq_dequantize_dense(const void *codes, const uint16_t *norms, int64_t n, int d, const void *pi, int bits,
                              rq_layout layout, const float *centroids, void *out, rq_dtype dtype,
                              rq_stream_t stream)
{
    rq::begin_call();
    rq_status s = check_dense(n, d, bits, layout, dtype);
    if (s) return s;
    if (n == 0) return RQ_OK;
    if (!codes || !norms || !pi || !out) return RQ_EINVAL;
    if (!aligned16(codes) || !aligned16(norms) || !aligned16(pi) || !aligned16(out)) return RQ_EALIGN;
    QuantTables T;
    s = tables_for(centroids, bits, d, 0, 0, T);
    if (s) return s;
    rq::DenseArgs a{};
    a.nvec = n / d; a.bf16 = dtype == RQ_BF16; a.pw = layout == RQ_CODES_INT8 ? 8 : bits; a.tables = &T;
    a.codes_in = static_cast<const uint8_t *>(codes); a.norms_in = norms; a.out = static_cast<uint16_t *>(out);
    a.num_sms = num_sms();
    if (a.num_sms <= 0) return RQ_ECUDA;
    if (!rq::make_proj_tmap(&a.tmap_pi, pi, d, d, 128) || !rq::make_vectors_tmap(&a.tmap_out, out, a.nvec, d, 128))
        return RQ_ECUDA;
    return cuda_status(rq::launch_dequantize_dense(a, reinterpret_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------------ outlier sketch

size_t qjl_sketch_outlier_workspace_bytes(int64_t n_vec, int d)
{
    return n_vec > 0 && d > 0 ? (size_t)n_vec * (size_t)d * 2 : 0;
}

static rq_status check_outlier(int d, int m, int m_o, int n_out)
{
    if (d != 128) return pow2_d(d) ? RQ_EUNSUPPORTED : RQ_EINVAL;
    if (m < 8 || m > 512 || m % 8) return RQ_EINVAL;
    if (n_out < 1 || n_out > 16 || m_o < 32 || m_o > m || m_o % 32) return RQ_EINVAL;
    if (m_o > 256) return RQ_EUNSUPPORTED;
    return RQ_OK;
}

rq_status qjl_sketch_outlier(const void *keys, int64_t n_vec, int d, int m, const void *proj, int m_o, int n_out,
                             uint8_t *signs, uint16_t *norms, uint8_t *out_idx, uint8_t *out_signs,
                             uint16_t *out_norms, void *workspace, size_t workspace_bytes, rq_stream_t stream)
{
    rq::begin_call();
    rq_status s = check_outlier(d, m, m_o, n_out);
    if (s) return s;
    if (n_vec < 0 || n_vec % 32) return RQ_EINVAL;
    if (n_vec > ((int64_t)1 << 34)) return RQ_ESIZE;
    if (n_vec == 0) return RQ_OK;
    if (!keys || !proj || !signs || !norms || !out_idx || !out_signs || !out_norms || !workspace) return RQ_EINVAL;
    if (workspace_bytes < qjl_sketch_outlier_workspace_bytes(n_vec, d)) return RQ_ESIZE;
    if (!aligned16(keys) || !aligned16(proj) || !aligned16(signs) || !aligned16(norms) || !aligned16(out_idx) ||
        !aligned16(out_signs) || !aligned16(out_norms) || !aligned16(workspace))
        return RQ_EALIGN;
    const int sms = num_sms();
    if (sms <= 0) return RQ_ECUDA;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = rq::launch_outlier_prep(static_cast<const uint16_t *>(keys), n_vec, n_out, m_o,
                                            static_cast<const uint16_t *>(proj), static_cast<uint16_t *>(workspace),
                                            out_idx, out_signs, out_norms, sms, st);
    if (e != cudaSuccess) return RQ_ECUDA;
    // the main sketch of the masked keys (the same checks have passed above)
    s = qjl_sketch(workspace, RQ_BF16, n_vec, d, m, proj, signs, norms, stream);
    rq::note_launch("outlier_prep_kernel");
    return s;
}

rq_status qjl_score_outlier(const void *q, int64_t G, int n_q, int d, int m, const void *proj, const uint8_t *signs,
                            const uint16_t *norms, int64_t T, int m_o, int n_out, const uint8_t *out_idx,
                            const uint8_t *out_signs, const uint16_t *out_norms, float *scores, void *workspace,
                            size_t workspace_bytes, rq_stream_t stream)
{
    rq::begin_call();
    rq_status s = check_outlier(d, m, m_o, n_out);
    if (s) return s;
    if (G < 0 || n_q < 0 || T < 0 || T % 32) return RQ_EINVAL;
    if (G > 65535 || n_q > 32 * 65535 || T > ((int64_t)1 << 31) || G * (T / 32) >= ((int64_t)1 << 31)) return RQ_ESIZE;
    if (G == 0 || n_q == 0 || T == 0) return RQ_OK;
    if (!q || !proj || !signs || !norms || !out_idx || !out_signs || !out_norms || !scores || !workspace)
        return RQ_EINVAL;
    if (workspace_bytes < rq::score_workspace_bytes(G, n_q, d, m)) return RQ_ESIZE;
    if (!aligned16(out_idx) || !aligned16(out_signs) || !aligned16(out_norms)) return RQ_EALIGN;
    s = qjl_score(q, G, n_q, d, m, proj, RQ_BF16, signs, norms, T, nullptr, nullptr, 0, RQ_CODES_PACKED, 0, 0,
                  nullptr, scores, workspace, workspace_bytes, stream);
    if (s) return s;
    cudaError_t e = rq::launch_outlier_score(static_cast<const uint16_t *>(q), G, n_q, T, m_o, n_out,
                                             static_cast<const uint16_t *>(proj), out_idx, out_signs, out_norms,
                                             scores, reinterpret_cast<cudaStream_t>(stream));
    return cuda_status(e);
}

}  // extern "C"
