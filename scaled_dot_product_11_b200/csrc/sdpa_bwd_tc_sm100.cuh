// sdpa_bwd_tc_sm100.cuh -- tensor-core form of the attention backward for
// head dims 64 and 128 (tcgen05 MMAs, TMA tiles, TMEM accumulators).
//
// Same recomputation as sdpa_bwd_sm100.cuh (article "Self-attention, CUDA
// kernels and FlashAttention", section 3), with every product on the tensor
// cores and in the two operand forms of the forward kernel:
//   QK form  D[M=128][N=128] = A[M][d] . B[N][d]^T, A and B K-major tiles
//   PV form  D[M=128][N=d]  += A[M][128 (TMEM, bf16/fp16)] . B[128][d],
//            B an MN-major tile (d contiguous)
// dK/dV kernel, one CTA per 128 keys of one (batch, K/V head), TMEM lane =
// key:  S^T = K Q^T, dP^T = V dO^T (QK form); P^T, dS^T computed per key row
// and written over them; dV += P^T dO, dK += dS^T Q (PV form, Q and dO tiles
// used MN-major).  dQ kernel, one CTA per 128 rows of one (batch, query
// head), TMEM lane = row:  S = Q K^T, dP = dO V^T; dS; dQ += dS K.
// The dQ kernel runs first and also writes D_i = dO_i . O_i of every row to
// the caller's workspace, from which the dK/dV kernel reads it per step.
// One CTA of 256 threads per tile: thread 0 issues the TMA copies (the
// streamed tile pair one step ahead, double-buffered) and the MMAs, and
// queues the next step's S and dP products right behind the current step's
// accumulating products under one commit (the tensor pipe runs them in issue
// order, so the S/dP columns they overwrite have been read); all eight warps
// do the elementwise work, two per TMEM lane quarter splitting the columns,
// each half packing its results over columns that only it reads (no barrier
// between reading S and writing P); tiles that need no mask skip it.  Every
// wait is bounded.
#pragma once
#include <cstdint>
#include <type_traits>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include "sm100_ptx.cuh"

namespace sdpa {

// 8 warps: warps w and w+4 share TMEM lane quarter w and split the 128
// columns of every elementwise step; thread 0 issues TMA and MMAs
constexpr int kBtThreads = 256;

struct BwdTcParams {
    const void* o;                   // [B,Hq,Sq,D] (for D_i = dO_i . O_i)
    const void* dout;                // [B,Hq,Sq,D]
    const float* lse;                // [B,Hq,Sq]
    float* delta;                    // [B,Hq,Sq] D_i, written by the dQ kernel
    void *dq, *dk, *dv;
    int B, Hq, Hkv, Sq, Sk, group;
    int causal, causal_off;
    float scale;                     // score scale (P = exp(scale * s - LSE))
    // output multipliers: dQ = dq_mul * (dS K), dK = dk_mul * (dS^T Q),
    // dV = dv_mul * (P^T dO), and D = d_mul * (dO . O); 16-bit inputs use
    // scale, scale, 1, 1
    float dq_mul, dk_mul, dv_mul, d_mul;
};

template <int D>
struct BtCfg {
    static constexpr int kRowBytes = D * 2;
    static constexpr int kElemsPerSw = 64;               // 128-byte swizzle rows of 16-bit data
    static constexpr int kSwBlocks = kRowBytes / 128;
    static constexpr int kSwBlockBytes = 128 * 128;
    static constexpr int kTileBytes = 128 * kRowBytes;
    static constexpr int kQkSteps = kRowBytes / 32;
    // six tiles (the streamed pair double-buffered), per-row statistics
    // (dQ: D partial sums of two halves; dK/dV: LSE and D of the step's
    // rows), barriers, TMEM slot
    static constexpr int kStatsBytes = 4 * 128 * 4;
    static constexpr int kSmemUsed = 6 * kTileBytes + kStatsBytes + 64;
    // one CTA per SM: each allocates all 512 TMEM columns
    static constexpr int kSmemBytes = kSmemUsed + 1024 > 120 * 1024 ? kSmemUsed + 1024 : 120 * 1024;
    static_assert(D == 64 || D == 128, "tensor-core backward: head dims 64 and 128");
};

// Bounded wait (1 s) on `bar`'s phase `parity`; on expiry records a device
// timeout at `where` and returns false.
__device__ __forceinline__ bool bt_wait(uint32_t bar, uint32_t parity, uint32_t where) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > 1000000000ull) {
            if (atomicCAS(&g_sdpa_status[0], 0u, 4u) == 0u) atomicExch(&g_sdpa_status[1], where);
            return false;
        }
    }
    return true;
}

template <bool BF16>
__device__ __forceinline__ float bt_ld(const void* base, size_t i) {
    if constexpr (BF16)
        return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
    else
        return __half2float(reinterpret_cast<const __half*>(base)[i]);
}

template <bool BF16>
__device__ __forceinline__ uint32_t bt_pack(float a, float b) {
    return BF16 ? pack_bf16x2(a, b) : pack_f16x2(a, b);
}

template <bool BF16>
__device__ __forceinline__ float2 bt_unpack(uint32_t w) {
    if constexpr (BF16)
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    else
        return __half22float2(*reinterpret_cast<const __half2*>(&w));
}

// Half `half` (columns [half*D/2, (half+1)*D/2)) of D_i = dO_i . O_i of row
// `row` (0 past the end); 16-byte loads
template <int D, bool BF16>
__device__ __forceinline__ float bt_row_dot(const BwdTcParams& p, size_t head, int row, int half) {
    if (row >= p.Sq) return 0.0f;
    const size_t off = head + (size_t)row * D + (size_t)half * (D / 2);
    const uint4* g = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.dout) + off);
    const uint4* o = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.o) + off);
    uint4 gv[D / 16], ov[D / 16];
#pragma unroll
    for (int v = 0; v < D / 16; ++v) {
        gv[v] = g[v];
        ov[v] = o[v];
    }
    float acc = 0.0f;
#pragma unroll
    for (int v = 0; v < D / 16; ++v) {
        const uint32_t gw[4] = {gv[v].x, gv[v].y, gv[v].z, gv[v].w};
        const uint32_t ow[4] = {ov[v].x, ov[v].y, ov[v].z, ov[v].w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float2 a = bt_unpack<BF16>(gw[u]), b = bt_unpack<BF16>(ow[u]);
            acc = fmaf(a.x, b.x, fmaf(a.y, b.y, acc));
        }
    }
    return acc;
}

// QK form: d_tmem[128][128] = A_tile . B_tile^T over D (both K-major, SW128)
template <int D, bool BF16>
__device__ __forceinline__ void bt_mma_qk(uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem) {
    using C = BtCfg<D>;
    constexpr uint32_t idesc = make_idesc(BF16 ? 1u : 0u, false, 128, 128);
    const uint64_t da = make_smem_desc(a_smem, 16, 1024), db = make_smem_desc(b_smem, 16, 1024);
#pragma unroll
    for (int kk = 0; kk < C::kQkSteps; ++kk) {
        const uint64_t off = (uint64_t)(((kk >> 2) * C::kSwBlockBytes + (kk & 3) * 32) >> 4);
        mma_f16_ss(d_tmem, da + off, db + off, idesc, kk > 0);
    }
}

// PV form: d_tmem[128][D] (+)= A (TMEM, 128 x 128, 16-bit packed) . B_tile
// (128 x D, MN-major).  A's keys (or rows) 0-63 are packed in columns
// [0,32) and 64-127 in [64,96): each half of the threads writes its packed
// results over the first of the two 32-column chunks it read, which no other
// thread reads.
template <int D, bool BF16>
__device__ __forceinline__ void bt_mma_pv(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_smem, bool acc) {
    using C = BtCfg<D>;
    constexpr uint32_t idesc = make_idesc(BF16 ? 1u : 0u, true, 128, D);
    const uint64_t db = make_smem_desc(b_smem, C::kSwBlockBytes, 1024);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {    // 16 keys (or rows) per step
        const uint64_t off = (uint64_t)((kk * 16 * 128) >> 4);
        mma_f16_ts(d_tmem, a_tmem + kk * 8 + (kk >= 4 ? 32 : 0), db + off, idesc, (acc || kk > 0) ? 1u : 0u);
    }
}

// Shared set-up of both kernels: barriers, TMEM.  Returns the TMEM base.
struct BtSmem {
    uint32_t bar_in[2], bar_kv[2], bar_mma, bar_drain, slot;
};
__device__ __forceinline__ BtSmem bt_layout(uint32_t bars) {
    return BtSmem{{bars, bars + 8}, {bars + 16, bars + 24}, bars + 32, bars + 40, bars + 48};
}

__device__ __forceinline__ uint32_t bt_setup(const BtSmem& sm) {
    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(sm.bar_in[i], 1);
            mbar_init(sm.bar_kv[i], 1);
        }
        mbar_init(sm.bar_mma, 1);
        mbar_init(sm.bar_drain, 1);
        fence_barrier_init();
    }
    if (threadIdx.x < 32) {
        tmem_alloc(sm.slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    uint32_t t;
    asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(t) : "r"(sm.slot));
    return t;
}

// End of both kernels: after a failed wait no MMA may still write TMEM
__device__ __forceinline__ void bt_teardown(const BtSmem& sm, uint32_t tmem, bool ok) {
    if (!ok && threadIdx.x == 0) {
        mma_commit(sm.bar_drain);
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(sm.bar_drain, 0) && global_timer_ns() - t0 < 100000000ull) {
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x < 32) tmem_dealloc(tmem, 512);
}

// Whether tile (rows [i0, i0+128), keys [j0, j0+128)) needs no mask: no row
// or key past the end, and with causal every key visible to every row
__device__ __forceinline__ bool bt_tile_full(const BwdTcParams& p, int i0, int j0) {
    return i0 + 128 <= p.Sq && j0 + 128 <= p.Sk && (!p.causal || j0 + 127 <= i0 + p.causal_off);
}

// dQ: one CTA per 128 query rows of one (batch, query head); TMEM lane = row.
// Columns: S [0,128) (dS packed over [0,32) and [64,96)), dP [128,256),
// dQ [256,256+D).
template <int D, bool BF16>
__global__ void __launch_bounds__(kBtThreads, 1)
sdpa_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                      const BwdTcParams p) {
    using C = BtCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    // Q, dO once; K/V tiles double-buffered: (sK(0), sV(0)), (sK(1), sV(1))
    const uint32_t sQ = base, sdO = base + C::kTileBytes;
    auto sK = [&](int buf) { return base + (uint32_t)(2 + 2 * buf) * C::kTileBytes; };
    auto sV = [&](int buf) { return base + (uint32_t)(3 + 2 * buf) * C::kTileBytes; };
    float* const dpart = reinterpret_cast<float*>(smem_raw + (base - raw) + 6 * C::kTileBytes);
    const BtSmem sm = bt_layout(base + 6 * C::kTileBytes + C::kStatsBytes);
    const uint32_t tmem = bt_setup(sm);

    const int i0 = blockIdx.x * 128;
    const int bh = blockIdx.y;
    const int b = bh / p.Hq, hq = bh - b * p.Hq;
    const int kvrow = b * p.Hkv + hq / p.group;        // 3-D map index of the K/V head
    const int r = threadIdx.x & 127, row = i0 + r, half = threadIdx.x >> 7;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const float kL2e = 1.44269504088896340736f;
    const float sl = p.scale * kL2e;

    if (threadIdx.x == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        prefetch_tmap(&tmdO);
        mbar_arrive_expect_tx(sm.bar_in[0], 2 * C::kTileBytes);
        for (int kb = 0; kb < C::kSwBlocks; ++kb) {
            tma_load_3d(sQ + kb * C::kSwBlockBytes, &tmQ, sm.bar_in[0], kb * C::kElemsPerSw, i0, bh);
            tma_load_3d(sdO + kb * C::kSwBlockBytes, &tmdO, sm.bar_in[0], kb * C::kElemsPerSw, i0, bh);
        }
    }
    const int kend = p.causal ? min(p.Sk, i0 + 128 + p.causal_off) : p.Sk;
    const int ntiles = (kend + 127) / 128;
    // K/V tile jt goes to buffer jt & 1, one tile ahead of its use
    auto load_kv = [&](int jt) {
        const int buf = jt & 1;
        mbar_arrive_expect_tx((buf ? sm.bar_kv[1] : sm.bar_kv[0]), 2 * C::kTileBytes);
        for (int kb = 0; kb < C::kSwBlocks; ++kb) {
            tma_load_3d(sK(buf) + kb * C::kSwBlockBytes, &tmK, (buf ? sm.bar_kv[1] : sm.bar_kv[0]), kb * C::kElemsPerSw,
                        jt * 128, kvrow);
            tma_load_3d(sV(buf) + kb * C::kSwBlockBytes, &tmV, (buf ? sm.bar_kv[1] : sm.bar_kv[0]), kb * C::kElemsPerSw,
                        jt * 128, kvrow);
        }
    };
    // S = Q K^T and dP = dO V^T of tile jt, after its K/V tiles landed; warp 0
    // waits, lane 0 issues.  Returns the wait's result.
    auto issue_qk = [&](int jt) {
        const int buf = jt & 1;
        const bool got = bt_wait((buf ? sm.bar_kv[1] : sm.bar_kv[0]), (uint32_t)(jt >> 1) & 1u,
                                 0x51000u | (uint32_t)(jt & 0xfff));
        if (got && lane == 0) {
            tc_fence_after();
            bt_mma_qk<D, BF16>(tmem, sQ, sK(buf));
            bt_mma_qk<D, BF16>(tmem + 128, sdO, sV(buf));
        }
        return got;
    };
    if (threadIdx.x == 0 && ntiles > 0) load_kv(0);
    const float lse_r = row < p.Sq ? p.lse[(size_t)bh * p.Sq + row] * kL2e : 0.0f;
    dpart[threadIdx.x] = bt_row_dot<D, BF16>(p, (size_t)bh * p.Sq * D, row, half);
    bool ok = __syncthreads_and(bt_wait(sm.bar_in[0], 0, 0x50000u));
    const float d_r = (dpart[r] + dpart[r + 128]) * p.d_mul;
    if (half == 0 && row < p.Sq) p.delta[(size_t)bh * p.Sq + row] = d_r;   // for the dK/dV kernel

    // this thread's own wait results since the last block-wide check
    bool mine = true;
    if (ok && ntiles > 0 && warp == 0) {
        mine = issue_qk(0);
        if (lane == 0) mma_commit(sm.bar_mma);
        __syncwarp();
    }
    // commit jt (jt >= 1): dQ of tile jt-1, then S and dP of tile jt
    int jt = 0;
    for (; jt < ntiles && ok; ++jt) {
        const int j0 = jt * 128, buf = jt & 1;
        ok = __syncthreads_and(bt_wait(sm.bar_mma, (uint32_t)jt & 1u, 0x52000u | (uint32_t)(jt & 0xfff)) && mine);
        if (!ok) break;
        tc_fence_after();
        // the other buffer's last readers (tile jt-1's dQ MMAs) have completed
        if (threadIdx.x == 0 && jt + 1 < ntiles) load_kv(jt + 1);
        // this thread's half of the row: key chunks 2*half and 2*half+1, each
        // packed as soon as computed over the first of them (columns only
        // this thread reads)
        auto elementwise = [&](auto masked) {
            constexpr bool kMask = decltype(masked)::value;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int c = 2 * half + cc;
                float s[32], dp[32];
                uint32_t w[16];
                tmem_ld32(tmem + lane_base + 32 * c, s);
                tmem_ld32(tmem + lane_base + 128 + 32 * c, dp);
                tmem_wait_ld();
                reg_fence32(s);
                reg_fence32(dp);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float ds2[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        float pv = ex2_approx(fmaf(s[2 * e + u], sl, -lse_r));
                        if constexpr (kMask) {
                            const int key = j0 + 32 * c + 2 * e + u;
                            const bool vis = row < p.Sq && key < p.Sk && (!p.causal || key <= row + p.causal_off);
                            pv = vis ? pv : 0.0f;
                        }
                        ds2[u] = pv * (dp[2 * e + u] - d_r);
                    }
                    w[e] = bt_pack<BF16>(ds2[0], ds2[1]);
                }
                tmem_st16(tmem + lane_base + 64 * half + 16 * cc, w);    // dS
            }
        };
        if (bt_tile_full(p, i0, j0))
            elementwise(std::false_type{});
        else
            elementwise(std::true_type{});
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
        if (warp == 0) {
            if (lane == 0) {
                tc_fence_after();
                bt_mma_pv<D, BF16>(tmem + 256, tmem, sK(buf), jt > 0);   // dQ += dS K
            }
            __syncwarp();
            if (jt + 1 < ntiles) mine = issue_qk(jt + 1);
            if (lane == 0) mma_commit(sm.bar_mma);
            __syncwarp();
        }
    }
    // the last commit: dQ of the last tile
    if (ok && ntiles > 0)
        ok = __syncthreads_and(bt_wait(sm.bar_mma, (uint32_t)ntiles & 1u, 0x53000u) && mine);
    if (ok) {
        tc_fence_after();
        // dQ row: scale and round (every row sees key 0, so ntiles >= 1);
        // the TMEM loads are warp-collective, the stores per row
#pragma unroll 1
        for (int c = half * (D / 64); c < (half + 1) * (D / 64); ++c) {
            float x[32];
            tmem_ld32(tmem + lane_base + 256 + 32 * c, x);
            tmem_wait_ld();
            reg_fence32(x);
            if (row < p.Sq) {
                uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.dq) +
                                                      ((size_t)bh * p.Sq + row) * D + 32 * c);
#pragma unroll
                for (int v4 = 0; v4 < 4; ++v4)
                    dst[v4] = make_uint4(bt_pack<BF16>(x[8 * v4] * p.dq_mul, x[8 * v4 + 1] * p.dq_mul),
                                         bt_pack<BF16>(x[8 * v4 + 2] * p.dq_mul, x[8 * v4 + 3] * p.dq_mul),
                                         bt_pack<BF16>(x[8 * v4 + 4] * p.dq_mul, x[8 * v4 + 5] * p.dq_mul),
                                         bt_pack<BF16>(x[8 * v4 + 6] * p.dq_mul, x[8 * v4 + 7] * p.dq_mul));
            }
        }
    }
    bt_teardown(sm, tmem, ok);
}

// dK, dV: one CTA per 128 keys of one (batch, K/V head); TMEM lane = key.
// Columns: S^T [0,128) (P^T packed over [0,32) and [64,96)), dP^T [128,256)
// (dS^T packed over [128,160) and [192,224)), dV [256,256+D), dK [384,384+D).
template <int D, bool BF16>
__global__ void __launch_bounds__(kBtThreads, 1)
sdpa_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                        const BwdTcParams p) {
    using C = BtCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    // K, V once; Q/dO tiles double-buffered: (sQ(0), sdO(0)), (sQ(1), sdO(1))
    const uint32_t sK = base, sV = base + C::kTileBytes;
    auto sQ = [&](int buf) { return base + (uint32_t)(2 + 2 * buf) * C::kTileBytes; };
    auto sdO = [&](int buf) { return base + (uint32_t)(3 + 2 * buf) * C::kTileBytes; };
    // lse_s[128]: LSE of the step's query rows (log2 units); dl_s[128]: their D
    float* const lse_s = reinterpret_cast<float*>(smem_raw + (base - raw) + 6 * C::kTileBytes);
    float* const dl_s = lse_s + 128;
    const BtSmem sm = bt_layout(base + 6 * C::kTileBytes + C::kStatsBytes);
    const uint32_t tmem = bt_setup(sm);

    const int j0 = blockIdx.x * 128;
    const int bk = blockIdx.y;                         // b * Hkv + hk
    const int b = bk / p.Hkv, hk = bk - b * p.Hkv;
    const int r = threadIdx.x & 127, key = j0 + r, half = threadIdx.x >> 7;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const float kL2e = 1.44269504088896340736f;
    const float sl = p.scale * kL2e;

    if (threadIdx.x == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        prefetch_tmap(&tmdO);
        mbar_arrive_expect_tx(sm.bar_kv[0], 2 * C::kTileBytes);
        for (int kb = 0; kb < C::kSwBlocks; ++kb) {
            tma_load_3d(sK + kb * C::kSwBlockBytes, &tmK, sm.bar_kv[0], kb * C::kElemsPerSw, j0, bk);
            tma_load_3d(sV + kb * C::kSwBlockBytes, &tmV, sm.bar_kv[0], kb * C::kElemsPerSw, j0, bk);
        }
    }
    // steps: the (query head of the group, query tile) pairs that see these
    // keys, query tiles from the first row that sees key j0
    const int i_start = ((p.causal ? max(0, j0 - p.causal_off) : 0) / 128) * 128;
    const int tiles_per_head = i_start < p.Sq ? (p.Sq - i_start + 127) / 128 : 0;
    const int nsteps = tiles_per_head * p.group;
    auto step_bh = [&](int st) { return b * p.Hq + hk * p.group + st / tiles_per_head; };
    auto step_i0 = [&](int st) { return i_start + (st % tiles_per_head) * 128; };
    // step st's Q/dO go to buffer st & 1, one step ahead of their use
    auto load_q = [&](int st) {
        const int buf = st & 1, bh = step_bh(st), i0 = step_i0(st);
        mbar_arrive_expect_tx((buf ? sm.bar_in[1] : sm.bar_in[0]), 2 * C::kTileBytes);
        for (int kb = 0; kb < C::kSwBlocks; ++kb) {
            tma_load_3d(sQ(buf) + kb * C::kSwBlockBytes, &tmQ, (buf ? sm.bar_in[1] : sm.bar_in[0]), kb * C::kElemsPerSw, i0, bh);
            tma_load_3d(sdO(buf) + kb * C::kSwBlockBytes, &tmdO, (buf ? sm.bar_in[1] : sm.bar_in[0]), kb * C::kElemsPerSw, i0, bh);
        }
    };
    // LSE (log2 units) and D of step st's 128 query rows, loaded by warps
    // 1-7: warp 0 issues the MMAs meanwhile, and its loads would land after
    // them
    auto load_stats = [&](int st) {
        if (warp == 0) return;
        const int si0 = step_i0(st);
        const size_t rows = (size_t)step_bh(st) * p.Sq;
        for (int i = (int)threadIdx.x - 32; i < 256; i += kBtThreads - 32) {
            const int qr = si0 + (i & 127);
            if (i < 128)
                lse_s[i] = qr < p.Sq ? p.lse[rows + qr] * kL2e : 0.0f;
            else
                dl_s[i - 128] = qr < p.Sq ? p.delta[rows + qr] : 0.0f;
        }
    };
    // S^T = K Q^T and dP^T = V dO^T of step st, after its Q/dO tiles landed;
    // warp 0 waits, lane 0 issues.  Returns the wait's result.
    auto issue_qk = [&](int st) {
        const int buf = st & 1;
        const bool got = bt_wait((buf ? sm.bar_in[1] : sm.bar_in[0]), (uint32_t)(st >> 1) & 1u,
                                 0x59000u | (uint32_t)(st & 0xfff));
        if (got && lane == 0) {
            tc_fence_after();
            bt_mma_qk<D, BF16>(tmem, sK, sQ(buf));
            bt_mma_qk<D, BF16>(tmem + 128, sV, sdO(buf));
        }
        return got;
    };
    if (threadIdx.x == 0 && nsteps > 0) load_q(0);
    bool ok = __syncthreads_and(bt_wait(sm.bar_kv[0], 0, 0x58000u));
    // this thread's own wait results since the last block-wide check
    bool mine = true;
    if (ok && nsteps > 0) {
        load_stats(0);
        if (warp == 0) {
            mine = issue_qk(0);
            if (lane == 0) mma_commit(sm.bar_mma);
            __syncwarp();
        }
    }

    // commit it (it >= 1): dV, dK of step it-1, then S^T and dP^T of step it
    int it = 0;
    for (; it < nsteps && ok; ++it) {
        const int i0 = step_i0(it), buf = it & 1;
        ok = __syncthreads_and(bt_wait(sm.bar_mma, (uint32_t)it & 1u, 0x5a000u | (uint32_t)(it & 0xfff)) && mine);
        if (!ok) break;
        tc_fence_after();
        // the other buffer's last readers (step it-1's MMAs) have completed
        if (threadIdx.x == 0 && it + 1 < nsteps) load_q(it + 1);
        // this thread's half of the key row: query chunks 2*half and
        // 2*half+1, each packed as soon as computed over the first of them
        // in S^T and dP^T (columns only this thread reads)
        auto elementwise = [&](auto masked) {
            constexpr bool kMask = decltype(masked)::value;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int c = 2 * half + cc;
                float s[32], dp[32];
                uint32_t wp[16], wd[16];
                tmem_ld32(tmem + lane_base + 32 * c, s);
                tmem_ld32(tmem + lane_base + 128 + 32 * c, dp);
                tmem_wait_ld();
                reg_fence32(s);
                reg_fence32(dp);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float pv2[2], ds2[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int col = 32 * c + 2 * e + u;
                        float pv = ex2_approx(fmaf(s[2 * e + u], sl, -lse_s[col]));
                        if constexpr (kMask) {
                            const int qi = i0 + col;
                            const bool vis = key < p.Sk && qi < p.Sq && (!p.causal || key <= qi + p.causal_off);
                            pv = vis ? pv : 0.0f;
                        }
                        pv2[u] = pv;
                        ds2[u] = pv * (dp[2 * e + u] - dl_s[col]);
                    }
                    wp[e] = bt_pack<BF16>(pv2[0], pv2[1]);
                    wd[e] = bt_pack<BF16>(ds2[0], ds2[1]);
                }
                tmem_st16(tmem + lane_base + 64 * half + 16 * cc, wp);          // P^T
                tmem_st16(tmem + lane_base + 128 + 64 * half + 16 * cc, wd);    // dS^T
            }
        };
        if (bt_tile_full(p, i0, j0))
            elementwise(std::false_type{});
        else
            elementwise(std::true_type{});
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
        if (warp == 0) {
            if (lane == 0) {
                tc_fence_after();
                bt_mma_pv<D, BF16>(tmem + 256, tmem, sdO(buf), it > 0);         // dV += P^T dO
                bt_mma_pv<D, BF16>(tmem + 384, tmem + 128, sQ(buf), it > 0);    // dK += dS^T Q
            }
            __syncwarp();
            if (it + 1 < nsteps) mine = issue_qk(it + 1);
            if (lane == 0) mma_commit(sm.bar_mma);
            __syncwarp();
        }
        // this step's reads of the statistics finished before the barrier above
        if (it + 1 < nsteps) load_stats(it + 1);
    }
    // the last commit: dV, dK of the last step
    if (ok && nsteps > 0)
        ok = __syncthreads_and(bt_wait(sm.bar_mma, (uint32_t)nsteps & 1u, 0x5b000u) && mine);
    if (ok) {
        tc_fence_after();
        // dV and dK rows (zero when no query sees these keys); the TMEM loads
        // are warp-collective, the stores per key.  Warps 0-3 write dV, 4-7 dK.
        const size_t orow = ((size_t)bk * p.Sk + (size_t)key) * D;
        void* out = half ? p.dk : p.dv;
        const float mul = half ? p.dk_mul : p.dv_mul;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
            float x[32];
            tmem_ld32(tmem + lane_base + (half ? 384 : 256) + 32 * c, x);
            tmem_wait_ld();
            reg_fence32(x);
            if (key < p.Sk) {
                // with no step the accumulators were never written: zeros
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] = it > 0 ? x[e] * mul : 0.0f;
                uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(out) + orow + 32 * c);
#pragma unroll
                for (int v4 = 0; v4 < 4; ++v4)
                    dst[v4] = make_uint4(bt_pack<BF16>(x[8 * v4], x[8 * v4 + 1]),
                                         bt_pack<BF16>(x[8 * v4 + 2], x[8 * v4 + 3]),
                                         bt_pack<BF16>(x[8 * v4 + 4], x[8 * v4 + 5]),
                                         bt_pack<BF16>(x[8 * v4 + 6], x[8 * v4 + 7]));
            }
        }
    }
    bt_teardown(sm, tmem, ok);
}

}  // namespace sdpa
