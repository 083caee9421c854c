// sdpa_bwd_sm100.cuh -- backward of the fused attention forward: dQ, dK, dV
// from Q, K, V, O, dO and the forward's per-row LSE.
//
// Method (article "Self-attention, CUDA kernels and FlashAttention",
// section 3: only the per-row normalisation statistics are kept, so the
// weights are recomputed tile by tile instead of being stored): for a query
// row i and key j visible to it,
//   p_ij  = exp(s_ij - LSE_i),  s_ij = scale * q_i . k_j
//   dp_ij = dO_i . v_j,  D_i = dO_i . O_i,  ds_ij = p_ij (dp_ij - D_i)
//   dV_j += p_ij dO_i,   dK_j += scale ds_ij q_i,   dQ_i += scale ds_ij k_j
// Two kernels, each recomputing p and ds for its tiles, so that every output
// element has exactly one writer (deterministic, no atomics, no scratch):
//   sdpa_bwd_dkdv_kernel: one CTA per 64 keys of one (batch, K/V head),
//                         looping over every query head of the group and
//                         every query tile that sees those keys;
//   sdpa_bwd_dq_kernel:   one CTA per 64 query rows of one (batch, query
//                         head), looping over the key tiles they see.
// Arithmetic is fp32 on the CUDA cores (register-blocked 4x4 tiles from
// shared memory); inputs and outputs are bf16 or fp16, contiguous
// [B, H, S, d].  This form serves head dim 32; head dims 64 and 128 take the
// tensor-core kernels of sdpa_bwd_pipe_sm100.cuh.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace sdpa {

constexpr int kBwdTile = 64;         // query rows and keys per tile
constexpr int kBwdThreads = 256;

struct BwdParams {
    const void *q, *k, *v, *o, *dout;
    const float* lse;                // [B, Hq, Sq], natural log, from the forward
    float* delta;                    // [B, Hq, Sq] workspace (tensor-core kernels)
    void *dq, *dk, *dv;
    int B, Hq, Hkv, Sq, Sk, group;
    int causal, causal_off;          // key j visible to query i iff j <= i + causal_off
    float scale;
    // multipliers of the tensor-core kernels' outputs and of D (the 16-bit
    // path: scale, scale, 1, 1; the FP8 path folds the per-tensor descales
    // into them)
    float dq_mul, dk_mul, dv_mul, d_mul;
};

template <int D>
struct BwdCfg {
    static constexpr int kLd = D + 4;                 // padded fp32 row of a [64][D] tile
    static constexpr int kLdp = kBwdTile + 4;         // padded row of a [64][64] tile
    static constexpr int kTileF = kBwdTile * kLd;     // floats of one [64][D] tile
    static constexpr int kSqF = kBwdTile * kLdp;      // floats of one [64][64] tile
    // four [64][D] tiles, two [64][64] tiles, LSE and D of 64 rows
    static constexpr int kSmemBytes = (4 * kTileF + 2 * kSqF + 2 * kBwdTile) * 4;
    static constexpr int kCols = D / 16;              // output columns per thread
};

template <bool BF16>
__device__ __forceinline__ float ld16(const void* base, size_t i) {
    if constexpr (BF16)
        return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
    else
        return __half2float(reinterpret_cast<const __half*>(base)[i]);
}
template <bool BF16>
__device__ __forceinline__ void st16(void* base, size_t i, float x) {
    if constexpr (BF16)
        reinterpret_cast<__nv_bfloat16*>(base)[i] = __float2bfloat16_rn(x);
    else
        reinterpret_cast<__half*>(base)[i] = __float2half_rn(x);
}

// rows [row0, row0 + 64) of a [S, D] head at `base` (element offset `head`)
// into a padded fp32 tile; rows past S read as zero
template <int D, bool BF16>
__device__ __forceinline__ void load_tile(float* dst, const void* base, size_t head, int row0, int S) {
    using C = BwdCfg<D>;
    for (int e = threadIdx.x; e < kBwdTile * D; e += kBwdThreads) {
        const int r = e / D, c = e - r * D;
        const int row = row0 + r;
        dst[r * C::kLd + c] = row < S ? ld16<BF16>(base, head + (size_t)row * D + c) : 0.0f;
    }
}

// P and dS of one (query tile, key tile) pair into shared memory.  Qs, dOs:
// the query tile's Q and dO; Ks, Vs: the key tile's K and V; lse_s, D_s: the
// query rows' LSE and D.  Masked and out-of-range pairs get p = ds = 0.
template <int D>
__device__ __forceinline__ void tile_p_ds(const BwdParams& p, const float* Qs, const float* dOs,
                                          const float* Ks, const float* Vs, const float* lse_s,
                                          const float* D_s, float* Ps, float* dSs, int i0, int j0) {
    using C = BwdCfg<D>;
    const int r0 = (threadIdx.x / 16) * 4, c0 = (threadIdx.x % 16) * 4;
    float s[4][4] = {}, dp[4][4] = {};
    for (int c = 0; c < D; ++c) {
        float a[4], g[4], kk[4], vv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            a[i] = Qs[(r0 + i) * C::kLd + c];
            g[i] = dOs[(r0 + i) * C::kLd + c];
            kk[i] = Ks[(c0 + i) * C::kLd + c];
            vv[i] = Vs[(c0 + i) * C::kLd + c];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                s[i][j] = fmaf(a[i], kk[j], s[i][j]);
                dp[i][j] = fmaf(g[i], vv[j], dp[i][j]);
            }
    }
    const float kLog2eF = 1.44269504088896340736f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int row = i0 + r0 + i;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int key = j0 + c0 + j;
            const bool vis = row < p.Sq && key < p.Sk && (!p.causal || key <= row + p.causal_off);
            const float pij = vis ? exp2f((s[i][j] * p.scale - lse_s[r0 + i]) * kLog2eF) : 0.0f;
            Ps[(r0 + i) * C::kLdp + c0 + j] = pij;
            dSs[(r0 + i) * C::kLdp + c0 + j] = pij * (dp[i][j] - D_s[r0 + i]);
        }
    }
}

// LSE and D = dO . O of the query rows [i0, i0 + 64) of head (b, hq)
template <int D, bool BF16>
__device__ __forceinline__ void row_stats(const BwdParams& p, const float* dOs, size_t qhead, int bh,
                                          int i0, float* lse_s, float* D_s) {
    using C = BwdCfg<D>;
    // four threads per row
    const int r = threadIdx.x / 4, part = threadIdx.x % 4;
    const int row = i0 + r;
    float acc = 0.0f;
    if (row < p.Sq)
        for (int c = part; c < D; c += 4)
            acc = fmaf(dOs[r * C::kLd + c], ld16<BF16>(p.o, qhead + (size_t)row * D + c), acc);
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    if (part == 0) {
        D_s[r] = acc;
        lse_s[r] = row < p.Sq ? p.lse[(size_t)bh * p.Sq + row] : 0.0f;
    }
}

template <int D, bool BF16>
__global__ void __launch_bounds__(kBwdThreads)
sdpa_bwd_dkdv_kernel(const BwdParams p) {
    using C = BwdCfg<D>;
    extern __shared__ float sm[];
    float* Ks = sm;
    float* Vs = Ks + C::kTileF;
    float* Qs = Vs + C::kTileF;
    float* dOs = Qs + C::kTileF;
    float* Ps = dOs + C::kTileF;
    float* dSs = Ps + C::kSqF;
    float* lse_s = dSs + C::kSqF;
    float* D_s = lse_s + kBwdTile;

    const int j0 = blockIdx.x * kBwdTile;
    const int bk = blockIdx.y;                   // b * Hkv + hk
    const int b = bk / p.Hkv, hk = bk - b * p.Hkv;
    const size_t kvhead = (size_t)bk * p.Sk * D;
    load_tile<D, BF16>(Ks, p.k, kvhead, j0, p.Sk);
    load_tile<D, BF16>(Vs, p.v, kvhead, j0, p.Sk);

    // this thread's 4 keys x D/16 columns of dK and dV
    const int kb = (threadIdx.x / 16) * 4, cb = (threadIdx.x % 16) * C::kCols;
    float dk[4][C::kCols] = {}, dv[4][C::kCols] = {};
    // first query row that sees key j0
    const int i_first = p.causal ? max(0, j0 - p.causal_off) : 0;
    for (int hq = hk * p.group; hq < (hk + 1) * p.group; ++hq) {
        const int bh = b * p.Hq + hq;
        const size_t qhead = (size_t)bh * p.Sq * D;
        for (int i0 = (i_first / kBwdTile) * kBwdTile; i0 < p.Sq; i0 += kBwdTile) {
            __syncthreads();   // the previous tile's P, dS, Q, dO are consumed
            load_tile<D, BF16>(Qs, p.q, qhead, i0, p.Sq);
            load_tile<D, BF16>(dOs, p.dout, qhead, i0, p.Sq);
            __syncthreads();
            row_stats<D, BF16>(p, dOs, qhead, bh, i0, lse_s, D_s);
            __syncthreads();
            tile_p_ds<D>(p, Qs, dOs, Ks, Vs, lse_s, D_s, Ps, dSs, i0, j0);
            __syncthreads();
            for (int r = 0; r < kBwdTile; ++r) {
                float pr[4], dsr[4], g[C::kCols], a[C::kCols];
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    pr[x] = Ps[r * C::kLdp + kb + x];
                    dsr[x] = dSs[r * C::kLdp + kb + x];
                }
#pragma unroll
                for (int y = 0; y < C::kCols; ++y) {
                    g[y] = dOs[r * C::kLd + cb + y];
                    a[y] = Qs[r * C::kLd + cb + y];
                }
#pragma unroll
                for (int x = 0; x < 4; ++x)
#pragma unroll
                    for (int y = 0; y < C::kCols; ++y) {
                        dv[x][y] = fmaf(pr[x], g[y], dv[x][y]);
                        dk[x][y] = fmaf(dsr[x], a[y], dk[x][y]);
                    }
            }
        }
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) {
        const int key = j0 + kb + x;
        if (key >= p.Sk) continue;
#pragma unroll
        for (int y = 0; y < C::kCols; ++y) {
            st16<BF16>(p.dk, kvhead + (size_t)key * D + cb + y, dk[x][y] * p.scale);
            st16<BF16>(p.dv, kvhead + (size_t)key * D + cb + y, dv[x][y]);
        }
    }
}

template <int D, bool BF16>
__global__ void __launch_bounds__(kBwdThreads)
sdpa_bwd_dq_kernel(const BwdParams p) {
    using C = BwdCfg<D>;
    extern __shared__ float sm[];
    float* Qs = sm;
    float* dOs = Qs + C::kTileF;
    float* Ks = dOs + C::kTileF;
    float* Vs = Ks + C::kTileF;
    float* Ps = Vs + C::kTileF;
    float* dSs = Ps + C::kSqF;
    float* lse_s = dSs + C::kSqF;
    float* D_s = lse_s + kBwdTile;

    const int i0 = blockIdx.x * kBwdTile;
    const int bh = blockIdx.y;                   // b * Hq + hq
    const int b = bh / p.Hq, hq = bh - b * p.Hq;
    const size_t qhead = (size_t)bh * p.Sq * D;
    const size_t kvhead = ((size_t)b * p.Hkv + hq / p.group) * p.Sk * D;
    load_tile<D, BF16>(Qs, p.q, qhead, i0, p.Sq);
    load_tile<D, BF16>(dOs, p.dout, qhead, i0, p.Sq);
    __syncthreads();
    row_stats<D, BF16>(p, dOs, qhead, bh, i0, lse_s, D_s);

    // this thread's 4 rows x D/16 columns of dQ
    const int rb = (threadIdx.x / 16) * 4, cb = (threadIdx.x % 16) * C::kCols;
    float dq[4][C::kCols] = {};
    // keys up to the last one the tile's last row sees
    const int kend = p.causal ? min(p.Sk, i0 + kBwdTile + p.causal_off) : p.Sk;
    for (int j0 = 0; j0 < kend; j0 += kBwdTile) {
        __syncthreads();   // the previous key tile and dS are consumed
        load_tile<D, BF16>(Ks, p.k, kvhead, j0, p.Sk);
        load_tile<D, BF16>(Vs, p.v, kvhead, j0, p.Sk);
        __syncthreads();
        tile_p_ds<D>(p, Qs, dOs, Ks, Vs, lse_s, D_s, Ps, dSs, i0, j0);
        __syncthreads();
        for (int j = 0; j < kBwdTile; ++j) {
            float ds[4], kv[C::kCols];
#pragma unroll
            for (int x = 0; x < 4; ++x) ds[x] = dSs[(rb + x) * C::kLdp + j];
#pragma unroll
            for (int y = 0; y < C::kCols; ++y) kv[y] = Ks[j * C::kLd + cb + y];
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < C::kCols; ++y) dq[x][y] = fmaf(ds[x], kv[y], dq[x][y]);
        }
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) {
        const int row = i0 + rb + x;
        if (row >= p.Sq) continue;
#pragma unroll
        for (int y = 0; y < C::kCols; ++y)
            st16<BF16>(p.dq, qhead + (size_t)row * D + cb + y, dq[x][y] * p.scale);
    }
}

}  // namespace sdpa
