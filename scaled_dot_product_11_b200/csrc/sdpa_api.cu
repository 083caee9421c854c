// sdpa_api.cu -- the C ABI declared in include/sdpa.h: argument checks,
// TMA tensor-map encoding, kernel selection and launch.  No allocation, no
// synchronisation, no fallback path.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>

#include "sdpa.h"
#include "sdpa_host.h"
#include "sdpa_fwd_sm100.cuh"
#include "sdpa_bwd_sm100.cuh"
#include "sdpa_bwd_pipe_sm100.cuh"

namespace {

using sdpa::FwdCfg;
using sdpa::FwdParams;

using sdpa_host::View;
using sdpa_host::bhsd;
using sdpa_host::encode_view;
using sdpa_host::same;
using sdpa_host::sm_count;

// 0 ok, else an sdpa_status.  Caches the answer per device.
int check_device() {
    static int support[64];   // 0 unknown, 1 ok, 2 unsupported
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SDPA_ERR_CUDA;
    if (dev >= 0 && dev < 64 && support[dev] != 0) return support[dev] == 1 ? SDPA_OK : SDPA_ERR_UNSUPPORTED;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return SDPA_ERR_CUDA;
    const bool ok = (major == 10 && minor == 0);
    if (dev >= 0 && dev < 64) support[dev] = ok ? 1 : 2;
    return ok ? SDPA_OK : SDPA_ERR_UNSUPPORTED;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Common argument checks of both entry points.
int check_args(const void* q, const void* k, const void* v, const void* o, const float* lse,
               int B, int Hq, int Hkv, int Sq, int Sk, int d, float scale, int causal) {
    if (!q || !k || !v || !o) return SDPA_ERR_INVALID_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Sq <= 0 || Sk <= 0 || d <= 0) return SDPA_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return SDPA_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.0f)) return SDPA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return SDPA_ERR_INVALID_ARG;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return SDPA_ERR_INVALID_ARG;
    if (causal < 0 || causal > 2) return SDPA_ERR_INVALID_ARG;
    // addressing limits: head counts and row indices fit the 32-bit TMA
    // coordinates and the grid, element offsets fit 64-bit size_t trivially
    const long long bhq = (long long)B * Hq, bhk = (long long)B * Hkv;
    const long long qblocks = (Sq + 127) / 128;
    if (bhq > INT32_MAX || bhk > INT32_MAX || bhq * qblocks > INT32_MAX) return SDPA_ERR_INVALID_ARG;
    if (d != 32 && d != 64 && d != 128) return SDPA_ERR_UNSUPPORTED;
    if (causal == SDPA_CAUSAL && Sq != Sk) return SDPA_ERR_UNSUPPORTED;
    if (causal == SDPA_CAUSAL_BOTTOM_RIGHT && Sq > Sk) return SDPA_ERR_UNSUPPORTED;
    return SDPA_OK;
}

// A view the kernel can address: positive strides whose byte sizes are
// multiples of 16 (TMA and the 16-byte output stores) and below 2^40.
bool view_ok(const long long* st, int elem_bytes) {
    if (!st) return false;
    for (int i = 0; i < 3; ++i) {
        if (st[i] <= 0 || st[i] > (1LL << 40) / elem_bytes) return false;
        if ((st[i] * elem_bytes) % 16 != 0) return false;
    }
    return true;
}

template <int D, int KIND, int NS, int QB, bool EPI, bool STRIDED, bool PACK = false>
int launch_cfg(const void* q, const void* k, const void* v, const View& vq, const View& vk,
               const View& vv, const FwdParams& prm, cudaStream_t stream) {
    using C = FwdCfg<D, KIND, NS, QB, EPI>;
    const CUtensorMapDataType dt = KIND == sdpa::KIND_BF16   ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                   : KIND == sdpa::KIND_FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                             : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    CUtensorMap tq, tk, tv;
    // PACK: Q boxes hold all Sq rows of the pk_group query heads of a K/V head
    const bool qok = PACK ? encode_view(&tq, dt, C::kElem, q, D, prm.Sq, prm.pk_hq, prm.B, vq,
                                        C::kElemsPerSw, false, prm.Sq, prm.pk_group)
                          : encode_view(&tq, dt, C::kElem, q, D, prm.Sq, prm.Hq, prm.B, vq,
                                        C::kElemsPerSw, !STRIDED);
    if (!qok ||
        !encode_view(&tk, dt, C::kElem, k, D, prm.Sk, prm.Hkv, prm.B, vk, C::kElemsPerSw, !STRIDED) ||
        !encode_view(&tv, dt, C::kElem, v, D, prm.Sk, prm.Hkv, prm.B, vv, C::kElemsPerSw, !STRIDED))
        return SDPA_ERR_CUDA;
    auto kern = sdpa::sdpa_fwd_sm100_kernel<D, KIND, NS, QB, EPI, STRIDED, PACK>;
    static bool attr_set[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
            cudaSuccess)
            return SDPA_ERR_CUDA;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    // persistent: one CTA per SM (fewer when there are fewer items)
    const unsigned grid = (unsigned)(prm.n_items < sm_count() ? prm.n_items : sm_count());
    kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, prm);
    return cudaGetLastError() == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
}

// The separate epilogue warps take the per-unit epilogue off the softmax
// warps' critical path: measured on B200 this pays when a unit (128 query
// rows of one head) averages 3 to 24 K/V tiles, and costs a few percent on
// longer units (and on units of one or two tiles).
#ifndef SDPA_EPI_MIN_AVG_TILES
#define SDPA_EPI_MIN_AVG_TILES 3
#endif
#ifndef SDPA_EPI_MAX_AVG_TILES
#define SDPA_EPI_MAX_AVG_TILES 24
#endif
bool use_epilogue_warps(const FwdParams& prm) {
    const int nk = (prm.Sk + 127) / 128;
    const double avg = prm.causal ? 0.5 * (prm.n_qtiles + 1) + prm.causal_off / 128.0 : (double)nk;
    return avg >= SDPA_EPI_MIN_AVG_TILES && avg <= SDPA_EPI_MAX_AVG_TILES;
}

// STRIDED kernels address Q/K/V through 4-D maps and O through its strides;
// contiguous [B,H,S,d] data takes the 3-D form, measured ~5% faster.
template <int D, int KIND, int NS, int QB, bool STRIDED>
int launch_form(const void* q, const void* k, const void* v, const View& vq, const View& vk,
                const View& vv, const FwdParams& prm, cudaStream_t stream) {
    return use_epilogue_warps(prm)
               ? launch_cfg<D, KIND, NS, QB, true, STRIDED>(q, k, v, vq, vk, vv, prm, stream)
               : launch_cfg<D, KIND, NS, QB, false, STRIDED>(q, k, v, vq, vk, vv, prm, stream);
}

// Decode-shaped GQA/MQA: when the Sq rows of all query heads sharing a K/V
// head fit one 128-row tile (group >= 2), one unit holds them all, so each
// K/V tile is streamed and multiplied once per K/V head instead of once per
// query head.
#ifndef SDPA_PACK_MAX_ROWS
#define SDPA_PACK_MAX_ROWS 128
#endif
bool use_packed_units(const FwdParams& prm) {
    return prm.group >= 2 && (long long)prm.group * prm.Sq <= SDPA_PACK_MAX_ROWS;
}

template <int D, int KIND, int NS, int QB>
int launch_packed(const void* q, const void* k, const void* v, const View& vq, const View& vk,
                  const View& vv, const FwdParams& prm, cudaStream_t stream) {
    using C = FwdCfg<D, KIND, NS, QB, false>;
    FwdParams pk = prm;
    pk.pk_hq = prm.Hq;
    pk.pk_group = prm.group;
    pk.pk_rows = prm.group * prm.Sq;
    pk.pk_qbytes = pk.pk_rows * C::kRowBytes;
    // units are (batch, K/V head) pairs of one tile each
    pk.Hq = prm.Hkv;
    pk.group = 1;
    pk.n_qtiles = 1;
    pk.items_per_head = 1;
    pk.n_items = prm.B * prm.Hkv;
    pk.group_heads = pk.n_items < 2 * sm_count() ? pk.n_items : 2 * sm_count();
    return launch_cfg<D, KIND, NS, QB, false, true, true>(q, k, v, vq, vk, vv, pk, stream);
}

// The two-query-tile kernel (sdpa_fwd2q.cu) serves head dims 64 and 128 in
// every layout; this file's one-tile kernel serves head dim 32 and the
// decode-shaped units with packed query heads.
#ifndef SDPA_FWD2Q
#define SDPA_FWD2Q 1
#endif

template <int D, int KIND, int NS, int QB>
int launch(const void* q, const void* k, const void* v, const View& vq, const View& vk, const View& vv,
           const FwdParams& prm, cudaStream_t stream) {
    if (use_packed_units(prm)) return launch_packed<D, KIND, NS, QB>(q, k, v, vq, vk, vv, prm, stream);
    const bool contiguous = same(vq, bhsd(prm.Hq, prm.Sq, D)) && same(vk, bhsd(prm.Hkv, prm.Sk, D)) &&
                            same(vv, bhsd(prm.Hkv, prm.Sk, D)) &&
                            prm.o_sb == (long long)prm.Hq * prm.Sq * D && prm.o_sh == (long long)prm.Sq * D &&
                            prm.o_ss == D;
    if constexpr (SDPA_FWD2Q && D != 32) {
        sdpa_host::Fwd2Request r;
        r.q = q;
        r.k = k;
        r.v = v;
        r.o = prm.o;
        r.lse = prm.lse;
        r.vq = vq;
        r.vk = vk;
        r.vv = vv;
        r.vo = View{prm.o_sb, prm.o_sh, prm.o_ss};
        r.B = prm.B;
        r.Hq = prm.Hq;
        r.Hkv = prm.Hkv;
        r.Sq = prm.Sq;
        r.Sk = prm.Sk;
        r.d = D;
        r.kind = KIND;
        r.causal = prm.causal;
        r.causal_off = prm.causal_off;
        r.contiguous = contiguous;
        r.score_log2 = prm.score_log2;
        r.out_mul = prm.out_mul;
        return sdpa_host::launch_fwd2q(r, stream);
    } else {
        return contiguous ? launch_form<D, KIND, NS, QB, false>(q, k, v, vq, vk, vv, prm, stream)
                          : launch_form<D, KIND, NS, QB, true>(q, k, v, vq, vk, vv, prm, stream);
    }
}

FwdParams make_params(void* o, const View& vo, float* lse, int B, int Hq, int Hkv, int Sq, int Sk,
                      int causal) {
    FwdParams prm;
    prm.o = o;
    prm.o_sb = vo.sb;
    prm.o_sh = vo.sh;
    prm.o_ss = vo.ss;
    prm.lse = lse;
    prm.B = B;
    prm.Hq = Hq;
    prm.Hkv = Hkv;
    prm.Sq = Sq;
    prm.Sk = Sk;
    prm.group = Hq / Hkv;
    prm.n_qtiles = (Sq + 127) / 128;
    // schedule items: causal pairs query tiles j and nq-1-j of a head
    prm.items_per_head = causal ? (prm.n_qtiles + 1) / 2 : prm.n_qtiles;
    prm.n_items = B * Hq * prm.items_per_head;
    // about two waves of items per group of (batch, head) pairs
    prm.group_heads = (2 * sm_count() + prm.items_per_head - 1) / prm.items_per_head;
    if (prm.group_heads < 1) prm.group_heads = 1;
    if (prm.group_heads > B * Hq) prm.group_heads = B * Hq;
    prm.causal = causal != 0 ? 1 : 0;
    prm.causal_off = causal == SDPA_CAUSAL_BOTTOM_RIGHT ? Sk - Sq : 0;
    prm.pk_hq = Hq;
    prm.pk_group = 1;
    prm.pk_rows = 0;
    prm.pk_qbytes = 0;
    prm.score_log2 = 0.f;
    prm.out_mul = 1.f;
    return prm;
}

int fwd_16bit(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
              int Hkv, int Sq, int Sk, int d, const View& vq, const View& vk, const View& vv,
              const View& vo, float scale, int causal, int dtype, void* stream) {
    if (dtype != SDPA_BF16 && dtype != SDPA_FP16) return SDPA_ERR_UNSUPPORTED;
    int rc = check_device();
    if (rc != SDPA_OK) return rc;
    FwdParams prm = make_params(o, vo, lse, B, Hq, Hkv, Sq, Sk, causal);
    prm.score_log2 = scale * sdpa::kLog2e;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (dtype == SDPA_BF16)
        return d == 32   ? launch<32, sdpa::KIND_BF16, SDPA_STAGES_D32, 2>(q, k, v, vq, vk, vv, prm, s)
               : d == 64 ? launch<64, sdpa::KIND_BF16, SDPA_STAGES_D64, 2>(q, k, v, vq, vk, vv, prm, s)
                         : launch<128, sdpa::KIND_BF16, SDPA_STAGES_D128, 1>(q, k, v, vq, vk, vv, prm, s);
    return d == 32   ? launch<32, sdpa::KIND_FP16, SDPA_STAGES_D32, 2>(q, k, v, vq, vk, vv, prm, s)
           : d == 64 ? launch<64, sdpa::KIND_FP16, SDPA_STAGES_D64, 2>(q, k, v, vq, vk, vv, prm, s)
                     : launch<128, sdpa::KIND_FP16, SDPA_STAGES_D128, 1>(q, k, v, vq, vk, vv, prm, s);
}

}  // namespace

extern "C" int sdpa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int Hq, int Hkv, int Sq, int Sk, int d, float scale, int causal, int dtype,
                        void* stream) {
    const int rc = check_args(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, scale, causal);
    if (rc != SDPA_OK) return rc;
    return fwd_16bit(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, bhsd(Hq, Sq, d), bhsd(Hkv, Sk, d),
                     bhsd(Hkv, Sk, d), bhsd(Hq, Sq, d), scale, causal, dtype, stream);
}

extern "C" int sdpa_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse,
                                int B, int Hq, int Hkv, int Sq, int Sk, int d,
                                const long long* q_strides, const long long* k_strides,
                                const long long* v_strides, const long long* o_strides, float scale,
                                int causal, int dtype, void* stream) {
    const int rc = check_args(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, scale, causal);
    if (rc != SDPA_OK) return rc;
    if (!view_ok(q_strides, 2) || !view_ok(k_strides, 2) || !view_ok(v_strides, 2) ||
        !view_ok(o_strides, 2))
        return SDPA_ERR_INVALID_ARG;
    auto view = [](const long long* st) { return View{st[0], st[1], st[2]}; };
    return fwd_16bit(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, view(q_strides), view(k_strides),
                     view(v_strides), view(o_strides), scale, causal, dtype, stream);
}

extern "C" int sdpa_fwd_fp8(const void* q8, const void* k8, const void* v8, float descale_q,
                            float descale_k, float descale_v, void* o, float* lse, int B, int Hq,
                            int Hkv, int Sq, int Sk, int d, float scale, int causal, void* stream) {
    int rc = check_args(q8, k8, v8, o, lse, B, Hq, Hkv, Sq, Sk, d, scale, causal);
    if (rc != SDPA_OK) return rc;
    for (float ds : {descale_q, descale_k, descale_v})
        if (!std::isfinite(ds) || !(ds > 0.0f)) return SDPA_ERR_INVALID_ARG;
    if (d != 128) return SDPA_ERR_UNSUPPORTED;
    rc = check_device();
    if (rc != SDPA_OK) return rc;
    FwdParams prm = make_params(o, bhsd(Hq, Sq, d), lse, B, Hq, Hkv, Sq, Sk, causal);
    prm.score_log2 = scale * descale_q * descale_k * sdpa::kLog2e;
    prm.out_mul = descale_v;
    return launch<128, sdpa::KIND_E4M3, SDPA_STAGES_FP8, 2>(
        q8, k8, v8, bhsd(Hq, Sq, d), bhsd(Hkv, Sk, d), bhsd(Hkv, Sk, d), prm,
        reinterpret_cast<cudaStream_t>(stream));
}

namespace {

template <int D, bool BF16>
int launch_bwd(const sdpa::BwdParams& bp, cudaStream_t stream) {
    using C = sdpa::BwdCfg<D>;
    auto kdkdv = sdpa::sdpa_bwd_dkdv_kernel<D, BF16>;
    auto kdq = sdpa::sdpa_bwd_dq_kernel<D, BF16>;
    static bool attr_set[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        if (cudaFuncSetAttribute(kdkdv, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
                cudaSuccess ||
            cudaFuncSetAttribute(kdq, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
                cudaSuccess)
            return SDPA_ERR_CUDA;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    const dim3 gkv((bp.Sk + sdpa::kBwdTile - 1) / sdpa::kBwdTile, bp.B * bp.Hkv);
    const dim3 gq((bp.Sq + sdpa::kBwdTile - 1) / sdpa::kBwdTile, bp.B * bp.Hq);
    kdkdv<<<gkv, sdpa::kBwdThreads, C::kSmemBytes, stream>>>(bp);
    if (cudaGetLastError() != cudaSuccess) return SDPA_ERR_CUDA;
    kdq<<<gq, sdpa::kBwdThreads, C::kSmemBytes, stream>>>(bp);
    return cudaGetLastError() == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
}

// Tensor-core backward (head dims 64, 128; sdpa_bwd_pipe_sm100.cuh): 3-D
// maps over (d, S, B*H) of Q, K, V, dO, then the dQ and dK/dV kernels.
template <int D, bool BF16>
int launch_bwd_pipe(const void* q, const void* k, const void* v, const sdpa::BwdParams& bp,
                    cudaStream_t stream) {
    using C = sdpa::bwdp::Cfg<D>;
    const CUtensorMapDataType dt = BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    // the dK/dV kernel streams Q, dO in 64-row boxes; everything else moves
    // in 128-row boxes
    CUtensorMap tq128, tdo128, tk128, tv128, tq64, tdo64, to128, tdq128, tdk128, tdv128;
    const View vq = bhsd(bp.Hq, bp.Sq, D), vk = bhsd(bp.Hkv, bp.Sk, D);
    const int sw = C::kElemsPerSw;
    if (!encode_view(&tq128, dt, 2, q, D, bp.Sq, bp.Hq, bp.B, vq, sw, true, 128) ||
        !encode_view(&tdo128, dt, 2, bp.dout, D, bp.Sq, bp.Hq, bp.B, vq, sw, true, 128) ||
        !encode_view(&tk128, dt, 2, k, D, bp.Sk, bp.Hkv, bp.B, vk, sw, true, 128) ||
        !encode_view(&tv128, dt, 2, v, D, bp.Sk, bp.Hkv, bp.B, vk, sw, true, 128) ||
        !encode_view(&tq64, dt, 2, q, D, bp.Sq, bp.Hq, bp.B, vq, sw, true, 64) ||
        !encode_view(&tdo64, dt, 2, bp.dout, D, bp.Sq, bp.Hq, bp.B, vq, sw, true, 64) ||
        !encode_view(&to128, dt, 2, bp.o, D, bp.Sq, bp.Hq, bp.B, vq, sw, true, 128) ||
        !encode_view(&tdq128, dt, 2, bp.dq, D, bp.Sq, bp.Hq, bp.B, vq, sw, true, 128) ||
        !encode_view(&tdk128, dt, 2, bp.dk, D, bp.Sk, bp.Hkv, bp.B, vk, sw, true, 128) ||
        !encode_view(&tdv128, dt, 2, bp.dv, D, bp.Sk, bp.Hkv, bp.B, vk, sw, true, 128))
        return SDPA_ERR_CUDA;
    sdpa::BwdTcParams tp;
    tp.o = bp.o; tp.dout = bp.dout; tp.lse = bp.lse; tp.delta = bp.delta;
    tp.dq = bp.dq; tp.dk = bp.dk; tp.dv = bp.dv;
    tp.B = bp.B; tp.Hq = bp.Hq; tp.Hkv = bp.Hkv; tp.Sq = bp.Sq; tp.Sk = bp.Sk; tp.group = bp.group;
    tp.causal = bp.causal; tp.causal_off = bp.causal_off; tp.scale = bp.scale;
    tp.dq_mul = bp.dq_mul; tp.dk_mul = bp.dk_mul; tp.dv_mul = bp.dv_mul; tp.d_mul = bp.d_mul;
    auto kdkdv = sdpa::bwdp::sdpa_bwd_dkdv_pipe_kernel<D, BF16>;
    auto kdq = sdpa::bwdp::sdpa_bwd_dq_pipe_kernel<D, BF16>;
    const int dq_smem = sdpa::bwdp::CfgQ<D>::kSmemBytes;
    static bool attr_set[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        if (cudaFuncSetAttribute(kdkdv, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
                cudaSuccess ||
            cudaFuncSetAttribute(kdq, cudaFuncAttributeMaxDynamicSharedMemorySize, dq_smem) != cudaSuccess)
            return SDPA_ERR_CUDA;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    const dim3 gkv((bp.Sk + 127) / 128, bp.B * bp.Hkv);
    const dim3 gq((bp.Sq + 127) / 128, bp.B * bp.Hq);
    // dQ first: it writes D of every row, which the dK/dV kernel reads
    kdq<<<gq, sdpa::bwdp::kThreads, dq_smem, stream>>>(tq128, tk128, tv128, tdo128, to128, tdq128, tp);
    if (cudaGetLastError() != cudaSuccess) return SDPA_ERR_CUDA;
    kdkdv<<<gkv, sdpa::bwdp::kThreads, C::kSmemBytes, stream>>>(tq64, tk128, tv128, tdo64, tdk128, tdv128, tp);
    return cudaGetLastError() == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
}

}  // namespace

extern "C" int sdpa_bwd(const void* q, const void* k, const void* v, const void* o,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv,
                        float* delta, int B, int Hq, int Hkv, int Sq, int Sk, int d, float scale,
                        int causal, int dtype, void* stream) {
    int rc = check_args(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, scale, causal);
    if (rc != SDPA_OK) return rc;
    if (!dout || !lse || !dq || !dk || !dv || !delta) return SDPA_ERR_INVALID_ARG;
    if (!aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
        reinterpret_cast<uintptr_t>(delta) % 4 != 0)
        return SDPA_ERR_INVALID_ARG;
    if ((long long)B * Hq > 65535) return SDPA_ERR_INVALID_ARG;   // grid rows
    if (dtype != SDPA_BF16 && dtype != SDPA_FP16) return SDPA_ERR_UNSUPPORTED;
    rc = check_device();
    if (rc != SDPA_OK) return rc;
    sdpa::BwdParams bp;
    bp.q = q; bp.k = k; bp.v = v; bp.o = o; bp.dout = dout; bp.lse = lse;
    bp.dq = dq; bp.dk = dk; bp.dv = dv; bp.delta = delta;
    bp.B = B; bp.Hq = Hq; bp.Hkv = Hkv; bp.Sq = Sq; bp.Sk = Sk; bp.group = Hq / Hkv;
    bp.causal = causal != 0 ? 1 : 0;
    bp.causal_off = causal == SDPA_CAUSAL_BOTTOM_RIGHT ? Sk - Sq : 0;
    bp.scale = scale;
    bp.dq_mul = scale;
    bp.dk_mul = scale;
    bp.dv_mul = 1.0f;
    bp.d_mul = 1.0f;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool bf = dtype == SDPA_BF16;
    if (d == 32) return bf ? launch_bwd<32, true>(bp, s) : launch_bwd<32, false>(bp, s);
    if (d == 64) return bf ? launch_bwd_pipe<64, true>(q, k, v, bp, s) : launch_bwd_pipe<64, false>(q, k, v, bp, s);
    return bf ? launch_bwd_pipe<128, true>(q, k, v, bp, s) : launch_bwd_pipe<128, false>(q, k, v, bp, s);
}

// ---------------------------------------------------------------------------
// sdpa_bwd_fp8: the backward of the FP8 forward under the codelab's hybrid
// recipe (section 10: E4M3 for the forward tensors, E5M2 for gradients).
// One launch widens the E4M3 Q/K/V codes and the E5M2 dO codes to bf16 --
// exactly, since both formats' values are bf16 values (3 and 2 fraction bits,
// exponents inside bf16's range) -- into the caller's workspace; the
// tensor-core backward then runs on the codes, with the per-tensor descales
// folded into the score scale and into its output and D multipliers, so that
// no value is rounded twice.  With codes q', k', v', g' (dO) and descales
// a_q, a_k, a_v, a_g:
//   scores        scale * a_q a_k (q' . k')            = scale * (q . k)
//   dP' = g' v'^T = dP / (a_g a_v);  D' = (g' . O) / a_v = D / (a_g a_v)
//   dS' = P (dP' - D') = dS / (a_g a_v)
//   dQ = (scale a_g a_v a_k) dS' k',  dK = (scale a_g a_v a_q) dS'^T q',
//   dV = a_g P^T g'.
// ---------------------------------------------------------------------------
namespace {

struct WidenSeg {
    const uint8_t* src;
    uint16_t* dst;
    long long n;      // elements
    int e5m2;         // 0: E4M3 codes, 1: E5M2 codes
};
struct WidenParams {
    WidenSeg seg[4];
    long long start[5];   // first 16-code chunk of each segment; start[4] = all chunks
};

// Two codes (low byte first) to bf16x2, exactly.
__device__ __forceinline__ uint32_t widen2(uint16_t two, int e5m2) {
    uint32_t h2;
    if (e5m2) {
        // an E5M2 code is the high byte of the binary16 with the same value
        h2 = ((uint32_t)(two & 0xffu) << 8) | ((uint32_t)(two & 0xff00u) << 16);
    } else {
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(two));
    }
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
    return sdpa::pack_bf16x2(f.x, f.y);
}

__global__ void widen_fp8_kernel(const WidenParams wp) {
    const long long total = wp.start[4];
    for (long long c = (long long)blockIdx.x * blockDim.x + threadIdx.x; c < total;
         c += (long long)gridDim.x * blockDim.x) {
        const int s = (c >= wp.start[1]) + (c >= wp.start[2]) + (c >= wp.start[3]);
        const WidenSeg sg = wp.seg[s];
        const long long i = (c - wp.start[s]) * 16;
        if (i + 16 <= sg.n) {
            const uint4 in = *reinterpret_cast<const uint4*>(sg.src + i);
            const uint32_t w[4] = {in.x, in.y, in.z, in.w};
            uint32_t o[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                o[2 * e] = widen2((uint16_t)(w[e] & 0xffffu), sg.e5m2);
                o[2 * e + 1] = widen2((uint16_t)(w[e] >> 16), sg.e5m2);
            }
            uint4* dst = reinterpret_cast<uint4*>(sg.dst + i);
            dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
            dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
        } else {
            for (long long e = i; e < sg.n; ++e) {
                const uint32_t two = widen2((uint16_t)sg.src[e], sg.e5m2);
                sg.dst[e] = (uint16_t)(two & 0xffffu);
            }
        }
    }
}

// Byte offsets of the workspace's parts, each 256-byte aligned: widened Q,
// K, V, dO (bf16), then D (fp32); returns the total.
size_t fp8_bwd_layout(int B, int Hq, int Hkv, int Sq, int Sk, int d, size_t off[5]) {
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t nq = (size_t)B * Hq * Sq * d, nk = (size_t)B * Hkv * Sk * d;
    off[0] = 0;
    off[1] = off[0] + up(nq * 2);
    off[2] = off[1] + up(nk * 2);
    off[3] = off[2] + up(nk * 2);
    off[4] = off[3] + up(nq * 2);
    return off[4] + up((size_t)B * Hq * Sq * 4);
}

}  // namespace

extern "C" size_t sdpa_bwd_fp8_workspace_bytes(int B, int Hq, int Hkv, int Sq, int Sk, int d) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Sq <= 0 || Sk <= 0 || d <= 0) return 0;
    size_t off[5];
    return fp8_bwd_layout(B, Hq, Hkv, Sq, Sk, d, off);
}

extern "C" int sdpa_bwd_fp8(const void* q8, const void* k8, const void* v8, const void* o,
                            const void* dout8, const float* lse, float descale_q, float descale_k,
                            float descale_v, float descale_do, void* dq, void* dk, void* dv,
                            void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv,
                            int Sq, int Sk, int d, float scale, int causal, void* stream) {
    int rc = check_args(q8, k8, v8, o, lse, B, Hq, Hkv, Sq, Sk, d, scale, causal);
    if (rc != SDPA_OK) return rc;
    if (!dout8 || !lse || !dq || !dk || !dv || !workspace) return SDPA_ERR_INVALID_ARG;
    if (!aligned16(dout8) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return SDPA_ERR_INVALID_ARG;
    for (float ds : {descale_q, descale_k, descale_v, descale_do})
        if (!std::isfinite(ds) || !(ds > 0.0f)) return SDPA_ERR_INVALID_ARG;
    if ((long long)B * Hq > 65535) return SDPA_ERR_INVALID_ARG;   // grid rows
    if (d != 128) return SDPA_ERR_UNSUPPORTED;
    size_t off[5];
    if (workspace_bytes < fp8_bwd_layout(B, Hq, Hkv, Sq, Sk, d, off)) return SDPA_ERR_INVALID_ARG;
    rc = check_device();
    if (rc != SDPA_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint16_t *q16 = reinterpret_cast<uint16_t*>(ws + off[0]), *k16 = reinterpret_cast<uint16_t*>(ws + off[1]);
    uint16_t *v16 = reinterpret_cast<uint16_t*>(ws + off[2]), *g16 = reinterpret_cast<uint16_t*>(ws + off[3]);
    const long long nq = (long long)B * Hq * Sq * d, nk = (long long)B * Hkv * Sk * d;
    WidenParams wp;
    wp.seg[0] = WidenSeg{static_cast<const uint8_t*>(q8), q16, nq, 0};
    wp.seg[1] = WidenSeg{static_cast<const uint8_t*>(k8), k16, nk, 0};
    wp.seg[2] = WidenSeg{static_cast<const uint8_t*>(v8), v16, nk, 0};
    wp.seg[3] = WidenSeg{static_cast<const uint8_t*>(dout8), g16, nq, 1};
    wp.start[0] = 0;
    for (int i = 0; i < 4; ++i) wp.start[i + 1] = wp.start[i] + (wp.seg[i].n + 15) / 16;
    const long long blocks = (wp.start[4] + 255) / 256;
    widen_fp8_kernel<<<(unsigned)(blocks < 4 * sm_count() ? blocks : 4 * sm_count()), 256, 0, s>>>(wp);
    if (cudaGetLastError() != cudaSuccess) return SDPA_ERR_CUDA;
    sdpa::BwdParams bp;
    bp.q = q16; bp.k = k16; bp.v = v16; bp.o = o; bp.dout = g16; bp.lse = lse;
    bp.dq = dq; bp.dk = dk; bp.dv = dv; bp.delta = reinterpret_cast<float*>(ws + off[4]);
    bp.B = B; bp.Hq = Hq; bp.Hkv = Hkv; bp.Sq = Sq; bp.Sk = Sk; bp.group = Hq / Hkv;
    bp.causal = causal != 0 ? 1 : 0;
    bp.causal_off = causal == SDPA_CAUSAL_BOTTOM_RIGHT ? Sk - Sq : 0;
    bp.scale = scale * descale_q * descale_k;
    bp.dq_mul = scale * descale_do * descale_v * descale_k;
    bp.dk_mul = scale * descale_do * descale_v * descale_q;
    bp.dv_mul = descale_do;
    bp.d_mul = 1.0f / descale_v;
    return launch_bwd_pipe<128, true>(q16, k16, v16, bp, s);
}

extern "C" const char* sdpa_strerror(int status) {
    switch (status) {
    case SDPA_OK: return "success";
    case SDPA_ERR_INVALID_ARG: return "invalid argument";
    case SDPA_ERR_UNSUPPORTED: return "unsupported configuration";
    case SDPA_ERR_CUDA: return "CUDA runtime or driver error";
    case SDPA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case SDPA_ERR_DEVICE_LAYOUT: return "shared-memory layout did not fit at the device's base address";
    case SDPA_ERR_SCRATCH_LIMIT: return "B*Hq*Sq exceeds the no-alloc backward's static workspace";
    default: return "unknown status";
    }
}

extern "C" int sdpa_device_status(int* status, int* detail, int clear) {
    unsigned int h[2] = {0u, 0u}, h2[2] = {0u, 0u};
    if (cudaDeviceSynchronize() != cudaSuccess) return SDPA_ERR_CUDA;
    if (cudaMemcpyFromSymbol(h, sdpa::g_sdpa_status, sizeof h) != cudaSuccess) return SDPA_ERR_CUDA;
    if (sdpa_host::fwd2q_status(h2, clear) != SDPA_OK) return SDPA_ERR_CUDA;
    if (h[0] == 0u) {   // the first kernel that recorded a status wins
        h[0] = h2[0];
        h[1] = h2[1];
    }
    if (status) *status = (int)h[0];
    if (detail) *detail = (int)h[1];
    if (clear) {
        const unsigned int z[2] = {0u, 0u};
        if (cudaMemcpyToSymbol(sdpa::g_sdpa_status, z, sizeof z) != cudaSuccess) return SDPA_ERR_CUDA;
    }
    return SDPA_OK;
}

extern "C" int sdpa_launches_per_call(void) { return 1; }

extern "C" int sdpa_selftest_wait(unsigned int limit_us, unsigned int* out, void* stream) {
    if (!out || limit_us == 0 || limit_us > 1000000u || (reinterpret_cast<uintptr_t>(out) & 3u))
        return SDPA_ERR_INVALID_ARG;
    const int rc = check_device();
    if (rc != SDPA_OK) return rc;
    return sdpa_host::selftest_wait(limit_us, out, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int sdpa_selftest_fastdiv(const int* n, const int* d, int count, int* q) {
    if (!n || !d || !q || count < 0) return SDPA_ERR_INVALID_ARG;
    return sdpa_host::selftest_fastdiv(n, d, count, q);
}

extern "C" int sdpa_selftest_exp2(const float* x, float* poly, float* mufu, int n, void* stream) {
    if (!x || !poly || !mufu || n <= 0) return SDPA_ERR_INVALID_ARG;
    const int rc = check_device();
    if (rc != SDPA_OK) return rc;
    return sdpa_host::selftest_exp2(x, poly, mufu, n, reinterpret_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// sdpa_bwd_noalloc: the backward for callers that cannot allocate device
// memory (a host framework that owns every allocation, or a path on which
// cudaMalloc's possible device synchronisation is not allowed).  Its
// workspace -- one float of D_i = dO_i . O_i per query row -- lives in the
// static array below instead of a caller buffer; the kernels are sdpa_bwd's.
// The article and the codelab have no counterpart: only the workspace's home
// differs.
// ---------------------------------------------------------------------------
namespace {

// 8 MiB on every GPU that loads the library, held until the process exits.
// Every call on a device shares it; no entry needs clearing, because the dQ
// kernel writes each row's D before the dK/dV kernel reads it.  Calls whose
// kernels overlap on the GPU race on it.
static __device__ __align__(256) float g_bwd_noalloc_delta[SDPA_BWD_NOALLOC_MAX_ROWS];

// Device address of the array in the current context.  In host code the
// array's name is only a host-side stand-in, so the address is looked up on
// every call, with the caller's device current: a cached address would go
// stale when the context that holds the module is destroyed and recreated
// (cudaDeviceReset) or when the caller switches to another context of the
// same device.  cudaGetSymbolAddress allocates nothing.
float* noalloc_delta(int* rc) {
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_bwd_noalloc_delta) != cudaSuccess || !addr) {
        *rc = SDPA_ERR_CUDA;
        return nullptr;
    }
    *rc = SDPA_OK;
    return static_cast<float*>(addr);
}

}  // namespace

extern "C" int sdpa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                const void* dout, const float* lse, void* dq, void* dk, void* dv,
                                int B, int Hq, int Hkv, int Sq, int Sk, int d, float scale,
                                int causal, int dtype, void* stream) {
    // the limit first: an oversized request launches nothing
    if (B > 0 && Hq > 0 && Sq > 0 && (long long)B * Hq * Sq > SDPA_BWD_NOALLOC_MAX_ROWS)
        return SDPA_ERR_SCRATCH_LIMIT;
    int rc = SDPA_OK;
    float* delta = noalloc_delta(&rc);
    if (!delta) return rc;
    return sdpa_bwd(q, k, v, o, dout, lse, dq, dk, dv, delta, B, Hq, Hkv, Sq, Sk, d, scale,
                    causal, dtype, stream);
}
