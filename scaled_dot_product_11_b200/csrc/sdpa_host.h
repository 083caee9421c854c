// sdpa_host.h -- host-side helpers shared by the library's translation
// units: the driver's tensor-map encoder (reached through the runtime's
// entry-point query, so the library links no driver library), views of
// [B, H, S, d] tensors, and per-device cached facts.  Internal; not part of
// the C ABI.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace sdpa_host {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// Streaming multiprocessors of the current device (cached; 148 on B200).
inline int sm_count() {
    static int cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

// Element strides (batch, head, row) of a [B, H, S, d] view, d contiguous.
struct View {
    long long sb, sh, ss;
};
inline View bhsd(int H, int S, int d) { return View{(long long)H * S * d, (long long)S * d, (long long)d}; }
inline bool same(const View& a, const View& b) { return a.sb == b.sb && a.sh == b.sh && a.ss == b.ss; }

// Tiled map over (d, S, H, B) with the view's strides -- 3-D (d, S, B*H) for
// contiguous [B,H,S,d] data (`rank3`); boxes of box_inner x box_rows rows of
// box_heads heads of one batch, swizzled in rows of box_inner elements (128
// bytes, or 64 for 16-bit head dim 32).
inline bool encode_view(CUtensorMap* m, CUtensorMapDataType dt, int elem_bytes, const void* base, int d,
                        int rows, int heads, int batch, const View& v, int box_inner, bool rank3,
                        int box_rows = 128, int box_heads = 1) {
    const CUtensorMapSwizzle swz =
        box_inner * elem_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint32_t rank = rank3 ? 3u : 4u;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)heads, (cuuint64_t)batch};
    cuuint64_t strides[3] = {(cuuint64_t)(v.ss * elem_bytes), (cuuint64_t)(v.sh * elem_bytes),
                             (cuuint64_t)(v.sb * elem_bytes)};
    if (rank == 3) dims[2] = (cuuint64_t)heads * (cuuint64_t)batch;
    const cuuint32_t box[4] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows, (cuuint32_t)box_heads, 1u};
    const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    return fn(m, dt, rank, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// What the two-query-tile forward kernel (its own translation unit) needs to
// launch: the problem, the views of Q, K, V, O, and the arithmetic constants.
struct Fwd2Request {
    const void* q;
    const void* k;
    const void* v;
    void* o;
    float* lse;
    View vq, vk, vv, vo;
    int B, Hq, Hkv, Sq, Sk, d;
    int kind;          // 0 bf16, 1 fp16, 2 e4m3
    int causal;        // 0 none, 1 causal (with causal_off)
    int causal_off;    // query row i sees keys 0 .. i + causal_off
    bool contiguous;   // Q, K, V, O all dense [B,H,S,d]
    float score_log2;  // scale * log2(e) (times the FP8 Q and K descales)
    float out_mul;     // the FP8 V descale, else 1
};

// Launch the two-query-tile forward (head dims 64 and 128; e4m3: 128).
// Returns an sdpa_status.
int launch_fwd2q(const Fwd2Request& r, cudaStream_t stream);
// Read (and with clear, reset) that kernel's device status word; synchronous.
int fwd2q_status(unsigned int out[2], int clear);
// Self-tests of that translation unit's device helpers (sdpa_selftest_*).
int selftest_wait(unsigned int limit_us, unsigned int* out, cudaStream_t stream);
int selftest_exp2(const float* x, float* poly, float* mufu, int n, cudaStream_t stream);
// the schedule's multiply-and-shift division, on the host
int selftest_fastdiv(const int* n, const int* d, int count, int* q);

}  // namespace sdpa_host
