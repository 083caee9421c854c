// sdpa_fwd2q.cu -- host launch of the two-query-tile forward kernel
// (sdpa_fwd2q_sm100.cuh): schedule parameters, TMA tensor maps, launch.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "sdpa.h"
#include "sdpa_host.h"
#include "sdpa_fwd2q_sm100.cuh"

// Forms and K/V ring depths.  16-bit head dim 128 takes the one-warp-per-row
// softmax (two 32 KB Q tiles + 5 ring slots fill the 227 KB); 16-bit head dim
// 64 (16 KB tiles: 2 x 2 Q tiles + 8 ring slots) takes the split softmax (two
// warps per row, each over 64 of the 128 scores), which measured faster there
// and slower at 16-bit head dim 128.  e4m3 head dim 128 (16 KB tiles as well)
// takes the one-warp form with the weights computed first, about 1% faster
// than its split form.
#ifndef SDPA2_STAGES_D128
#define SDPA2_STAGES_D128 5
#endif
#ifndef SDPA2_STAGES_16K
#define SDPA2_STAGES_16K 8
#endif
#ifndef SDPA2_SPLIT_D128
#define SDPA2_SPLIT_D128 0
#endif
#ifndef SDPA2_SPLIT_16K
#define SDPA2_SPLIT_16K 1
#endif
#ifndef SDPA2_SPLIT_FP8
#define SDPA2_SPLIT_FP8 0
#endif
// the split form needs room for its halves' statistics and exchange: its
// 16-bit head dim 128 ring has 4 slots
static constexpr int kStagesD128 = SDPA2_SPLIT_D128 ? 4 : SDPA2_STAGES_D128;

namespace sdpa_host {
namespace {

using sdpa::fwd2::Cfg;
using sdpa::fwd2::Params;

template <int D, int KIND, int NS, int QB, bool SPLIT, bool STRIDED>
int launch_cfg(const Fwd2Request& r, const Params& prm, cudaStream_t stream) {
    using C = Cfg<D, KIND, NS, QB, SPLIT>;
    const CUtensorMapDataType dt = KIND == sdpa::fwd2::K2_BF16   ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                   : KIND == sdpa::fwd2::K2_FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                                 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    CUtensorMap tq, tk, tv;
    if (!encode_view(&tq, dt, C::kElem, r.q, D, r.Sq, r.Hq, r.B, r.vq, C::kElemsPerSw, !STRIDED) ||
        !encode_view(&tk, dt, C::kElem, r.k, D, r.Sk, r.Hkv, r.B, r.vk, C::kElemsPerSw, !STRIDED) ||
        !encode_view(&tv, dt, C::kElem, r.v, D, r.Sk, r.Hkv, r.B, r.vv, C::kElemsPerSw, !STRIDED))
        return SDPA_ERR_CUDA;
    auto kern = sdpa::fwd2::sdpa_fwd2q_sm100_kernel<D, KIND, NS, QB, SPLIT, STRIDED>;
    static bool attr_set[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SDPA_ERR_CUDA;
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
            return SDPA_ERR_CUDA;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    // persistent: one CTA per SM (fewer when there are fewer items)
    const unsigned grid = (unsigned)(prm.n_items < sm_count() ? prm.n_items : sm_count());
    kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, prm);
    return cudaGetLastError() == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
}

template <int D, int KIND, int NS, int QB, bool SPLIT>
int launch_form(const Fwd2Request& r, const Params& prm, cudaStream_t stream) {
    return r.contiguous ? launch_cfg<D, KIND, NS, QB, SPLIT, false>(r, prm, stream)
                        : launch_cfg<D, KIND, NS, QB, SPLIT, true>(r, prm, stream);
}

}  // namespace

int launch_fwd2q(const Fwd2Request& r, cudaStream_t stream) {
    Params prm;
    prm.o = r.o;
    prm.lse = r.lse;
    prm.B = r.B;
    prm.Hq = r.Hq;
    prm.Hkv = r.Hkv;
    prm.Sq = r.Sq;
    prm.Sk = r.Sk;
    prm.group = r.Hq / r.Hkv;
    const int nq = (r.Sq + 127) / 128;
    prm.n_pairs = (nq + 1) / 2;
    // causal items pair unit m with unit n_pairs-1-m of the same head
    prm.items_per_head = r.causal ? (prm.n_pairs + 1) / 2 : prm.n_pairs;
    const long long n_items = (long long)r.B * r.Hq * prm.items_per_head;
    if (n_items > INT32_MAX) return SDPA_ERR_INVALID_ARG;
    prm.n_items = (int)n_items;
    // about one wave of items per group of (batch, head) pairs, so that the
    // K/V of the heads in flight (2 MB per head at S = 4096, d = 128) stay
    // well inside the L2
#ifndef SDPA2_GROUP_WAVES
#define SDPA2_GROUP_WAVES 1
#endif
    int gh = (SDPA2_GROUP_WAVES * sm_count() + prm.items_per_head - 1) / prm.items_per_head;
    if (gh < 1) gh = 1;
    if (gh > r.B * r.Hq) gh = r.B * r.Hq;
    prm.group_heads = gh;
    using sdpa::fwd2::make_fastdiv;
    prm.div_items = make_fastdiv(gh * prm.items_per_head);
    prm.div_gh = make_fastdiv(gh);
    const int n_bh = r.B * r.Hq;
    prm.div_gh_last = make_fastdiv(n_bh - ((n_bh - 1) / gh) * gh);
    prm.div_hq = make_fastdiv(r.Hq);
    prm.div_group = make_fastdiv(prm.group);
    prm.causal = r.causal ? 1 : 0;
    prm.causal_off = r.causal_off;
    prm.score_log2 = r.score_log2;
    prm.out_mul = r.out_mul;
    prm.o_sb = r.vo.sb;
    prm.o_sh = r.vo.sh;
    prm.o_ss = r.vo.ss;
    using namespace sdpa::fwd2;
    constexpr bool kSplitD128 = SDPA2_SPLIT_D128 != 0, kSplit16K = SDPA2_SPLIT_16K != 0,
                   kSplitFp8 = SDPA2_SPLIT_FP8 != 0;
    switch (r.kind) {
    case K2_BF16:
        return r.d == 64 ? launch_form<64, K2_BF16, SDPA2_STAGES_16K, 2, kSplit16K>(r, prm, stream)
                         : launch_form<128, K2_BF16, kStagesD128, 1, kSplitD128>(r, prm, stream);
    case K2_FP16:
        return r.d == 64 ? launch_form<64, K2_FP16, SDPA2_STAGES_16K, 2, kSplit16K>(r, prm, stream)
                         : launch_form<128, K2_FP16, kStagesD128, 1, kSplitD128>(r, prm, stream);
    case K2_E4M3:
        if (!r.contiguous || r.d != 128) return SDPA_ERR_UNSUPPORTED;
        return launch_cfg<128, K2_E4M3, SDPA2_STAGES_16K, 2, kSplitFp8, false>(r, prm, stream);
    default:
        return SDPA_ERR_UNSUPPORTED;
    }
}

int selftest_wait(unsigned int limit_us, unsigned int* out, cudaStream_t stream) {
    sdpa::fwd2::selftest_wait_kernel<<<1, 64, 0, stream>>>((uint64_t)limit_us * 1000ull, out);
    return cudaGetLastError() == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
}

int selftest_exp2(const float* x, float* poly, float* mufu, int n, cudaStream_t stream) {
    const int pairs = (n + 1) / 2;
    sdpa::fwd2::selftest_exp2_kernel<<<(pairs + 255) / 256, 256, 0, stream>>>(x, poly, mufu, n);
    return cudaGetLastError() == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
}

int selftest_fastdiv(const int* n, const int* d, int count, int* q) {
    for (int i = 0; i < count; ++i) {
        if (n[i] < 0 || d[i] < 1) return SDPA_ERR_INVALID_ARG;
        q[i] = sdpa::fwd2::fdiv(n[i], sdpa::fwd2::make_fastdiv(d[i]));
    }
    return SDPA_OK;
}

int fwd2q_status(unsigned int out[2], int clear) {
    if (cudaMemcpyFromSymbol(out, sdpa::fwd2::g_status, 2 * sizeof(unsigned int)) != cudaSuccess)
        return SDPA_ERR_CUDA;
    if (clear) {
        const unsigned int z[2] = {0u, 0u};
        if (cudaMemcpyToSymbol(sdpa::fwd2::g_status, z, sizeof z) != cudaSuccess) return SDPA_ERR_CUDA;
    }
    return SDPA_OK;
}

}  // namespace sdpa_host
