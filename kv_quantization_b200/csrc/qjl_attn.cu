// qjl_attn.cu -- launcher of the attention decode over compressed keys and
// values (kernels in qjl_attention.cuh).
#define RQ_SCORE_PROLOGUE_EXTERN
#include "qjl_attention.cuh"
#include "rq_kernels.h"

namespace rq {

bool attention_supported(int nq, int d, int m, bool two, int pw, int vpw)
{
    if (!at_eligible(nq, d, m, two, pw)) return false;
    if (two && !(pw == 1 || pw == 2 || pw == 3 || pw == 4 || pw == 8)) return false;
    return vpw == 2 || vpw == 3 || vpw == 4 || vpw == 8;
}

static size_t at_prologue_bytes(int64_t G, int nq, int d, int m)
{
    return (sc2_ws_bytes(G, nq, d, m, true) + 255) & ~(size_t)255;
}

static int64_t at_grid(int64_t G, int64_t T, int num_sms)
{
    const int64_t items = G * ((T + kAtTok - 1) / kAtTok);
    return items < (int64_t)num_sms ? items : (int64_t)num_sms;
}

size_t attention_workspace_bytes(int64_t G, int nq, int d, int m, int64_t T, int num_sms)
{
    return at_prologue_bytes(G, nq, d, m) + (size_t)(at_grid(G, T, num_sms) + G) * at_part_floats(nq, d) * sizeof(float);
}

template <int PW, bool TWO, int VPW>
static cudaError_t launch_main(const AttnArgs &a, const uint16_t *wsB, const float *wsN, float *part, int grid,
                               cudaStream_t st)
{
    const ScoreArgs &k = a.k;
    struct Cfg { int kring, nrec; };
    const Cfg cfgs[] = {{3, 3}, {3, 2}, {2, 2}, {2, 1}};
    for (const Cfg &c : cfgs) {
        const size_t smem = at_smem(k.d, k.m, TWO, PW, VPW, c.kring, c.nrec);
        if (smem > kMaxSmemPerBlock) continue;
        auto kern = attention_kernel<PW, TWO, VPW>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        const float qscale = a.softmax_scale * 1.4426950408889634074f;     // log2(e)
        kern<<<(unsigned)grid, kAtThreads, smem, st>>>(wsB, wsN, k.nq, k.d, k.m, k.signs, k.sk_norms, k.T, k.G,
                                                       k.codes, k.norms, a.vcodes, a.vnorms, *k.tables, *a.vtables,
                                                       qscale, part, c.kring, c.nrec);
        note_launch("attention_kernel");
        return cudaGetLastError();
    }
    return cudaErrorNotSupported;
}

template <int PW, bool TWO>
static cudaError_t launch_v(const AttnArgs &a, const uint16_t *wsB, const float *wsN, float *part, int grid,
                            cudaStream_t st)
{
    switch (a.vpw) {
    case 2: return launch_main<PW, TWO, 2>(a, wsB, wsN, part, grid, st);
    case 3: return launch_main<PW, TWO, 3>(a, wsB, wsN, part, grid, st);
    case 4: return launch_main<PW, TWO, 4>(a, wsB, wsN, part, grid, st);
    case 8: return launch_main<PW, TWO, 8>(a, wsB, wsN, part, grid, st);
    default: return cudaErrorNotSupported;
    }
}

cudaError_t launch_attention(const AttnArgs &a, cudaStream_t st)
{
    const ScoreArgs &k = a.k;
    const bool two = k.codes != nullptr;
    if (!attention_supported(k.nq, k.d, k.m, two, k.pw, a.vpw)) return cudaErrorNotSupported;
    uint8_t *ws = static_cast<uint8_t *>(a.workspace);
    uint16_t *wsB = reinterpret_cast<uint16_t *>(ws);
    const size_t rows = (size_t)k.G * k.nq;
    float *wsN = reinterpret_cast<float *>(ws + ((rows * sc2_kb(k.d, k.m, two) * 2 + 255) & ~(size_t)255));
    float *part = reinterpret_cast<float *>(ws + at_prologue_bytes(k.G, k.nq, k.d, k.m));
    cudaError_t e = launch_score_prologue(k, two, wsB, wsN, st);
    if (e != cudaSuccess) return e;
    const int grid = (int)at_grid(k.G, k.T, a.num_sms);
    if (!two) {
        e = launch_v<1, false>(a, wsB, wsN, part, grid, st);
    } else {
        switch (k.pw) {
        case 1: e = launch_v<1, true>(a, wsB, wsN, part, grid, st); break;
        case 2: e = launch_v<2, true>(a, wsB, wsN, part, grid, st); break;
        case 3: e = launch_v<3, true>(a, wsB, wsN, part, grid, st); break;
        case 4: e = launch_v<4, true>(a, wsB, wsN, part, grid, st); break;
        case 8: e = launch_v<8, true>(a, wsB, wsN, part, grid, st); break;
        default: e = cudaErrorNotSupported; break;
        }
    }
    if (e != cudaSuccess) return e;
    attention_combine_kernel<<<dim3((unsigned)k.G, (unsigned)k.nq), kAtD, 0, st>>>(part, k.nq, k.d, k.T, k.G, grid,
                                                                                   *a.vtables, a.out);
    note_launch("attention_combine_kernel");
    return cudaGetLastError();
}

}  // namespace rq
