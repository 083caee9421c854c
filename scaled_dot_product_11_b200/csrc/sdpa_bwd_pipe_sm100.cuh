// sdpa_bwd_pipe_sm100.cuh -- pipelined tensor-core backward of attention for
// head dims 64 and 128 (tcgen05 MMAs, TMA tiles, TMEM accumulators).
//
// Method (article "Self-attention, CUDA kernels and FlashAttention", section
// 3): the weights are recomputed from the kept row statistics,
//   P = exp(scale * S - LSE),  dP = dO V^T,  D_i = dO_i . O_i,
//   dS = P * (dP - D),  dQ = scale * dS K,  dK = scale * dS^T Q,  dV = P^T dO,
// arranged so that the tensor pipe and the elementwise warps overlap.
//
// The dK/dV kernel walks its streamed operand in steps of 64 rows, so that the
// two products the elementwise step reads (S and dP, 64 fp32 columns each)
// fit twice in tensor memory next to the two accumulators: while the sixteen
// elementwise warps turn step t's S, dP into P, dS (written back over them,
// 16-bit), the tensor pipe runs step t-1's accumulating products and step
// t+1's S and dP (committed separately, so that step t+1's exponentials can
// start before its dP lands).  A TMA producer warp streams the 64-row tiles
// through a ring; an MMA warp issues every product from one elected lane (in
// issue order, so a product that overwrites a buffer cannot overtake the one
// that reads it, which is issued just before it).
//
// dK/dV kernel, one CTA per 128 keys of one (batch, K/V head); TMEM lane =
// key; steps = 64 query rows of one query head of the group:
//   S^T = K Q^T, dP^T = V dO^T            (M 128 keys, N 64 rows, K d)
//   dV += P^T dO, dK += dS^T Q            (A = P^T / dS^T from TMEM, K 64)
// dQ kernel, one CTA per 128 query rows of one (batch, query head); TMEM lane
// = row; steps = 128 keys (its one accumulator leaves room for two 128-column
// S buffers and one dP, see CfgQ):
//   S = Q K^T, dP = dO V^T                (M 128 rows, N 128 keys, K d)
//   dQ += dS K                            (A = dS from TMEM, K 128)
// The dQ kernel runs first and writes D_i of every row to the caller's
// workspace, which the dK/dV kernel's producer reads per step with the LSE.
// dK/dV tensor memory (512 columns): S_b at [64 b, 64 b + 64), dP_b at
// [128 + 64 b, ...) for buffers b = 0, 1; dV, dK from column 256.  The 16-bit
// P / dS of a buffer's 16-column chunk c (owned by warps 4c..4c+3) are packed
// over the chunk's first 8 columns, which is where the accumulating product's
// k-th 16-row slice reads them (k = c).
// Warps: 0-15 elementwise (four per TMEM lane quarter, warp w on quarter
// w & 3 and chunk w >> 2: four warps per SM sub-partition to hide the
// latencies of one step's short chain), 16 TMA producer, 17 MMA issuer and
// TMEM owner.  Every wait is bounded; a warp that gives up raises the CTA's
// abort flag and the others leave their waits.
#pragma once
#include <cstdint>
#include <type_traits>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include "sm100_ptx.cuh"

namespace sdpa {

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

// Half of D_i = dO_i . O_i for row r of a 128-row tile, from the dO and O
// tiles in shared memory (128-byte swizzle: 16-byte unit u of a row's
// 128-byte segment sits at unit u ^ (row & 7)); half h covers columns
// [h D/2, (h + 1) D/2), summed in column order.
template <int D, bool BF16>
__device__ __forceinline__ float bt_row_dot_smem(uint32_t sdo, uint32_t so, int r, int half) {
    constexpr int kUnits = D / 16;   // 16-byte units per half row
    uint4 gv[kUnits], ov[kUnits];
#pragma unroll
    for (int v = 0; v < kUnits; ++v) {
        const int gu = half * kUnits + v;
        const uint32_t off = (uint32_t)((gu >> 3) * 128 * 128 + r * 128 + (((gu & 7) ^ (r & 7)) << 4));
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(gv[v].x), "=r"(gv[v].y), "=r"(gv[v].z), "=r"(gv[v].w) : "r"(sdo + off));
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(ov[v].x), "=r"(ov[v].y), "=r"(ov[v].z), "=r"(ov[v].w) : "r"(so + off));
    }
    float acc = 0.0f;
#pragma unroll
    for (int v = 0; v < kUnits; ++v) {
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

namespace bwdp {

constexpr int kEwWarps = 16;      // elementwise warps 0-15
constexpr int kEwThreads = 32 * kEwWarps;
constexpr int kLoadWarp = kEwWarps;
constexpr int kMmaWarp = kEwWarps + 1;
constexpr int kThreads = kEwThreads + 64;
constexpr int kStep = 64;         // query rows per dK/dV step
constexpr int kChunk = 16;        // columns of a dK/dV step per elementwise warp

// dK/dV kernel layout (the dQ kernel's is CfgQ below)
template <int D>
struct Cfg {
    static constexpr int kRowBytes = D * 2;
    static constexpr int kElemsPerSw = 64;                  // 128-byte swizzle rows of 16-bit data
    static constexpr int kSwBlocks = kRowBytes / 128;
    static constexpr int kBlock128 = 128 * 128;             // one swizzle block of a 128-row tile
    static constexpr int kBlock64 = 64 * 128;               // ... of a 64-row tile
    static constexpr int kTile128 = 128 * kRowBytes;
    static constexpr int kTile64 = 64 * kRowBytes;
    static constexpr int kQkSteps = kRowBytes / 32;         // K steps of 16 elements
    // ring of streamed 64-row (Q, dO) tile pairs: 4 slots at d = 128, 8 at
    // d = 64 (32 KB / 16 KB a slot)
    static constexpr int kRing = D == 128 ? 4 : 8;
    // shared memory: resident pair (2 x 128-row tiles), ring, per-slot
    // statistics (64 -LSE + 64 D floats), barriers, TMEM slot, abort flag
    static constexpr int kSmemRes = 0;
    static constexpr int kSmemRing = 2 * kTile128;
    static constexpr int kSmemStats = kSmemRing + kRing * 2 * kTile64;
    static constexpr int kSmemBar = kSmemStats + kRing * 2 * kStep * 4;
    // barriers: res_full, ring_full[R], ring_empty[R], s_full[2] (S or S^T
    // of a buffer landed), dp_full[2] (dP or dP^T landed), p_full[2] (the
    // elementwise step's results written), done, drain
    static constexpr int kBarResFull = 0;
    static constexpr int kBarRingFull = 1;
    static constexpr int kBarRingEmpty = 1 + kRing;
    static constexpr int kBarSFull = 1 + 2 * kRing;
    static constexpr int kBarDPFull = 3 + 2 * kRing;
    static constexpr int kBarPFull = 5 + 2 * kRing;
    static constexpr int kBarDone = 7 + 2 * kRing;
    static constexpr int kBarDrain = 8 + 2 * kRing;
    static constexpr int kNumBars = 9 + 2 * kRing;
    static constexpr int kSmemSlot = kSmemBar + 8 * kNumBars;
    static constexpr int kSmemAbort = kSmemSlot + 4;
    static constexpr int kSmemUsed = kSmemAbort + 4;
    static constexpr int kSmemBytes = kSmemUsed + 1024;
    // TMEM columns
    static constexpr uint32_t kColS = 0, kColDP = 128, kColAcc = 256;
    static_assert(D == 64 || D == 128, "pipelined backward: head dims 64 and 128");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static_assert(kSmemBytes > 116 * 1024, "one CTA per SM (each allocates all of TMEM)");
};

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ void sts_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.volatile.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Bounded wait on `bar`'s phase `parity`: gives up after 1 s (records a
// device timeout at `where` and raises the CTA's abort flag) or when another
// warp has raised the flag.
__device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity, uint32_t abort_addr, uint32_t where) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t k = 1;; ++k) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((k & 15u) == 0) {
            if (lds_u32(abort_addr) != 0u) return false;
            if (global_timer_ns() - t0 > 1000000000ull) {
                sts_u32(abort_addr, 1u);
                if (atomicCAS(&g_sdpa_status[0], 0u, 4u) == 0u) atomicExch(&g_sdpa_status[1], where);
                return false;
            }
        }
    }
}

// QK form: d[128][64] = A[128 rows][D] . B[64 rows][D]^T, both K-major SW128
// tiles (A a 128-row tile, B a 64-row tile)
template <int D, bool BF16>
__device__ __forceinline__ void mma_qk(uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem) {
    using C = Cfg<D>;
    constexpr uint32_t idesc = make_idesc(BF16 ? 1u : 0u, false, 128, kStep);
    const uint64_t da = make_smem_desc(a_smem, 16, 1024), db = make_smem_desc(b_smem, 16, 1024);
#pragma unroll
    for (int kk = 0; kk < C::kQkSteps; ++kk) {
        const uint64_t oa = (uint64_t)(((kk >> 2) * C::kBlock128 + (kk & 3) * 32) >> 4);
        const uint64_t ob = (uint64_t)(((kk >> 2) * C::kBlock64 + (kk & 3) * 32) >> 4);
        mma_f16_ss(d_tmem, da + oa, db + ob, idesc, kk > 0);
    }
}

// PV form: d[128][D] (+)= A (TMEM, 128 x 64, 16-bit, 16-column chunk k packed
// over its first 8 columns) . B[64 rows][D] (MN-major 64-row tile)
template <int D, bool BF16>
__device__ __forceinline__ void mma_pv(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_smem, bool acc) {
    using C = Cfg<D>;
    constexpr uint32_t idesc = make_idesc(BF16 ? 1u : 0u, true, 128, D);
    const uint64_t db = make_smem_desc(b_smem, C::kBlock64, 1024);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {    // 16 rows (or keys) per product
        const uint64_t off = (uint64_t)((kk * 16 * 128) >> 4);
        mma_f16_ts(d_tmem, a_tmem + kChunk * kk, db + off, idesc, (acc || kk > 0) ? 1u : 0u);
    }
}

// Set-up shared by both kernels: barriers (thread 0), TMEM (the MMA warp).
// Returns the TMEM base.
template <int D>
__device__ __forceinline__ uint32_t setup(uint32_t base) {
    using C = Cfg<D>;
    auto bar = [&](int i) -> uint32_t { return base + C::kSmemBar + 8u * (uint32_t)i; };
    if (threadIdx.x == 0) {
        mbar_init(bar(C::kBarResFull), 1);
        for (int i = 0; i < C::kRing; ++i) {
            mbar_init(bar(C::kBarRingFull + i), 1);
            mbar_init(bar(C::kBarRingEmpty + i), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(C::kBarSFull + b), 1);
            mbar_init(bar(C::kBarDPFull + b), 1);
            mbar_init(bar(C::kBarPFull + b), kEwWarps);   // one arrival per warp
        }
        mbar_init(bar(C::kBarDone), 1);
        mbar_init(bar(C::kBarDrain), 1);
        sts_u32(base + C::kSmemAbort, 0u);
        fence_barrier_init();
    }
    if ((threadIdx.x >> 5) == kMmaWarp) {
        tmem_alloc(base + C::kSmemSlot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return lds_u32(base + C::kSmemSlot);
}

// End of both kernels: after a failed wait no MMA may still write TMEM when
// it is freed.
template <int D>
__device__ __forceinline__ void teardown(uint32_t base, uint32_t tmem, bool mma_ok) {
    using C = Cfg<D>;
    const int warp = threadIdx.x >> 5;
    if (warp == kMmaWarp && !mma_ok) {
        const uint32_t drain = base + C::kSmemBar + 8u * C::kBarDrain;
        if (elect_one()) mma_commit(drain);
        __syncwarp();
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < 100000000ull) {
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

// The producer's exit: wait (bounded, 100 ms) until its own copies have
// landed -- the resident pair and the last `issued` ring loads -- so that
// none is in flight when the CTA ends (on the normal path the MMA warp has
// already waited for every one of them).
template <int D>
__device__ __forceinline__ void drain_loads(uint32_t base, int issued) {
    using C = Cfg<D>;
    auto bar = [&](int i) -> uint32_t { return base + C::kSmemBar + 8u * (uint32_t)i; };
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar(C::kBarResFull), 0) && global_timer_ns() - t0 < 100000000ull) {
    }
    for (int st = issued > C::kRing ? issued - C::kRing : 0; st < issued; ++st)
        while (!mbar_try_wait(bar(C::kBarRingFull + st % C::kRing), (uint32_t)(st / C::kRing) & 1u) &&
               global_timer_ns() - t0 < 100000000ull) {
        }
}

// One row's 16-column accumulator chunk (TMEM address t): times `mul` (or
// zeros), rounded, into the row's 32 bytes at 16-bit column `col` of a
// 128-row tile in shared memory, in the 128-byte swizzled layout its TMA
// store reads (64-column blocks of 128 rows x 128 bytes; 16-byte unit u of a
// row segment at u ^ (row & 7)).
template <bool BF16>
__device__ __forceinline__ void stage_chunk16(uint32_t t, uint32_t tile, int r, int col, float mul, bool zero) {
    float x[16];
    tmem_ld16(t, x);
    tmem_wait_ld();
    reg_fence16(x);
    if (zero) {
#pragma unroll
        for (int e = 0; e < 16; ++e) x[e] = 0.0f;
    }
#pragma unroll
    for (int v4 = 0; v4 < 2; ++v4) {
        const int gu = col / 8 + v4;
        const uint32_t addr = tile + (uint32_t)((gu >> 3) * 128 * 128 + r * 128 + (((gu & 7) ^ (r & 7)) << 4));
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                     "r"(bt_pack<BF16>(x[8 * v4] * mul, x[8 * v4 + 1] * mul)),
                     "r"(bt_pack<BF16>(x[8 * v4 + 2] * mul, x[8 * v4 + 3] * mul)),
                     "r"(bt_pack<BF16>(x[8 * v4 + 4] * mul, x[8 * v4 + 5] * mul)),
                     "r"(bt_pack<BF16>(x[8 * v4 + 6] * mul, x[8 * v4 + 7] * mul))
                     : "memory");
    }
}

// dK, dV: one CTA per 128 keys of one (batch, K/V head).
template <int D, bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
sdpa_bwd_dkdv_pipe_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                          const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                          const BwdTcParams p) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const uint32_t sK = base + C::kSmemRes, sV = sK + C::kTile128;
    auto sQ = [&](int slot) -> uint32_t { return base + C::kSmemRing + (uint32_t)slot * 2u * C::kTile64; };
    auto sdO = [&](int slot) -> uint32_t { return sQ(slot) + C::kTile64; };
    // per ring slot: -LSE (log2 units) and D of the step's 64 query rows
    float* const stats = reinterpret_cast<float*>(smem_raw + (base - raw) + C::kSmemStats);
    auto bar = [&](int i) -> uint32_t { return base + C::kSmemBar + 8u * (uint32_t)i; };
    const uint32_t abort_addr = base + C::kSmemAbort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float kL2e = 1.44269504088896340736f;

    const int j0 = blockIdx.x * 128;
    const int bk = blockIdx.y;                         // b * Hkv + hk
    const int b = bk / p.Hkv, hk = bk - b * p.Hkv;
    // steps: 64 query rows of one query head of the group, from the first
    // row that sees key j0
    const int i_start = ((p.causal ? max(0, j0 - p.causal_off) : 0) / kStep) * kStep;
    const int tiles_per_head = i_start < p.Sq ? (p.Sq - i_start + kStep - 1) / kStep : 0;
    const int nsteps = tiles_per_head * p.group;
    auto step_bh = [&](int st) { return b * p.Hq + hk * p.group + st / tiles_per_head; };
    auto step_i0 = [&](int st) { return i_start + (st % tiles_per_head) * kStep; };

    const uint32_t tmem = setup<D>(base);
    bool mma_ok = true;

    if (warp == kLoadWarp) {
        // ================= TMA producer (lane 0) and statistics ===========
        bool ok = true;
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            prefetch_tmap(&tmdO);
            mbar_arrive_expect_tx(bar(C::kBarResFull), 2 * C::kTile128);
            for (int kb = 0; kb < C::kSwBlocks; ++kb) {
                tma_load_3d(sK + kb * C::kBlock128, &tmK, bar(C::kBarResFull), kb * C::kElemsPerSw, j0, bk);
                tma_load_3d(sV + kb * C::kBlock128, &tmV, bar(C::kBarResFull), kb * C::kElemsPerSw, j0, bk);
            }
        }
        int issued = 0;
        for (int st = 0; st < nsteps && ok; ++st) {
            const int slot = st % C::kRing;
            if (st >= C::kRing)
                ok = wait(bar(C::kBarRingEmpty + slot), (uint32_t)(st / C::kRing - 1) & 1u, abort_addr,
                          0x61000u | (uint32_t)(st & 0xfff));
            if (!ok) break;
            const int bh = step_bh(st), i0 = step_i0(st);
            // the tiles first (their bytes are expected before the copies
            // start), then the statistics, whose load latency overlaps the
            // copies; lane 0's arrival after them completes the slot
            const uint32_t fb = bar(C::kBarRingFull + slot);
            if (lane == 0) {
                mbar_expect_tx(fb, 2 * C::kTile64);
                for (int kb = 0; kb < C::kSwBlocks; ++kb) {
                    tma_load_3d(sQ(slot) + kb * C::kBlock64, &tmQ, fb, kb * C::kElemsPerSw, i0, bh);
                    tma_load_3d(sdO(slot) + kb * C::kBlock64, &tmdO, fb, kb * C::kElemsPerSw, i0, bh);
                }
            }
            float* const st_lse = stats + slot * 2 * kStep;
            const size_t rows = (size_t)bh * p.Sq;
            for (int i = lane; i < kStep; i += 32) {
                const int qr = i0 + i;
                st_lse[i] = qr < p.Sq ? -(p.lse[rows + qr] * kL2e) : 0.0f;
                st_lse[kStep + i] = qr < p.Sq ? p.delta[rows + qr] : 0.0f;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(fb);
            __syncwarp();
            issued = st + 1;
        }
        if (lane == 0) drain_loads<D>(base, issued);
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ================= MMA issuer =====================================
        const bool leader = elect_one();
        auto wait_all = [&](uint32_t b_, uint32_t par, uint32_t where) {
            return __all_sync(0xffffffffu, wait(b_, par, abort_addr, where));
        };
        auto commit = [&](uint32_t b_) {
            if (leader) mma_commit(b_);
            __syncwarp();
        };
        // Step st's Q / dO landed (its ring slot)
        auto wait_in = [&](int st) -> bool {
            return wait_all(bar(C::kBarRingFull + st % C::kRing), (uint32_t)(st / C::kRing) & 1u,
                            0x62000u | (uint32_t)(st & 0xfff));
        };
        // S^T (or dP^T) of step st into buffer st & 1, with its own commit
        auto issue_s = [&](int st) {
            if (leader) mma_qk<D, BF16>(tmem + C::kColS + 64 * (st & 1), sK, sQ(st % C::kRing));
            __syncwarp();
            commit(bar(C::kBarSFull + (st & 1)));
        };
        auto issue_dp = [&](int st) {
            if (leader) mma_qk<D, BF16>(tmem + C::kColDP + 64 * (st & 1), sV, sdO(st % C::kRing));
            __syncwarp();
            commit(bar(C::kBarDPFull + (st & 1)));
        };
        bool ok = wait_all(bar(C::kBarResFull), 0, 0x60000u);
        for (int st = 0; st < 2 && st < nsteps && ok; ++st) {
            ok = wait_in(st);
            if (!ok) break;
            tc_fence_after();
            issue_s(st);
            issue_dp(st);
        }
        // Per step, in issue order: dV(st) (reads P^T over S^T_b), S^T(st+2)
        // (overwrites it), dK(st) (reads dS^T over dP^T_b), dP^T(st+2): the
        // elementwise step st+2 starts on S^T while dK and dP^T still run.
        for (int st = 0; st < nsteps && ok; ++st) {
            const int slot = st % C::kRing, bf = st & 1;
            const bool next = st + 2 < nsteps;
            ok = wait_all(bar(C::kBarPFull + bf), (uint32_t)(st >> 1) & 1u, 0x63000u | (uint32_t)(st & 0xfff));
            if (ok && next) ok = wait_in(st + 2);
            if (!ok) break;
            tc_fence_after();
            if (leader) mma_pv<D, BF16>(tmem + C::kColAcc, tmem + C::kColS + 64 * bf, sdO(slot), st > 0);  // dV += P^T dO
            __syncwarp();
            if (next) issue_s(st + 2);
            if (leader) mma_pv<D, BF16>(tmem + C::kColAcc + D, tmem + C::kColDP + 64 * bf, sQ(slot), st > 0);  // dK += dS^T Q
            __syncwarp();
            commit(bar(C::kBarRingEmpty + slot));
            if (next) issue_dp(st + 2);
        }
        if (ok) commit(bar(C::kBarDone));
        mma_ok = ok;
    } else {
        // ================= elementwise (warps 0-15) =======================
        const int quarter = warp & 3, c = warp >> 2;   // lane quarter, column chunk
        const int r = quarter * 32 + lane, key = j0 + r;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const float sl = p.scale * kL2e;
        const uint64_t sl2 = f2_pack(sl, sl);
        bool ok = true;
        for (int st = 0; st < nsteps && ok; ++st) {
            const int slot = st % C::kRing, bf = st & 1, i0 = step_i0(st);
            // -LSE and D of this chunk's 16 query rows (broadcast loads),
            // landed long before the step's products
            ok = wait(bar(C::kBarRingFull + slot), (uint32_t)(st / C::kRing) & 1u, abort_addr,
                      0x65000u | (uint32_t)(st & 0xfff));
            const float4* const st4 = reinterpret_cast<const float4*>(stats + slot * 2 * kStep + kChunk * c);
            float nl[16], dl[16];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const float4 a4 = st4[v], d4 = st4[kStep / 4 + v];
                nl[4 * v] = a4.x; nl[4 * v + 1] = a4.y; nl[4 * v + 2] = a4.z; nl[4 * v + 3] = a4.w;
                dl[4 * v] = d4.x; dl[4 * v + 1] = d4.y; dl[4 * v + 2] = d4.z; dl[4 * v + 3] = d4.w;
            }
            ok = ok && wait(bar(C::kBarSFull + bf), (uint32_t)(st >> 1) & 1u, abort_addr,
                            0x64000u | (uint32_t)(st & 0xfff));
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            const uint32_t tS = tmem + lane_base + C::kColS + 64 * bf + kChunk * c;
            const uint32_t tP = tmem + lane_base + C::kColDP + 64 * bf + kChunk * c;
            float s[16];
            tmem_ld16(tS, s);
            tmem_wait_ld();
            reg_fence16(s);
            // P^T = 2^(s sl - LSE) (0 where masked), while dP^T is computed
            float pv[16];
            uint32_t wp[8];
            auto weights = [&](auto masked) {
                constexpr bool kMask = decltype(masked)::value;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    float x0, x1;
                    f2_unpack(f2_fma(f2_pack(s[2 * e], s[2 * e + 1]), sl2, f2_pack(nl[2 * e], nl[2 * e + 1])), x0, x1);
                    float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                    if constexpr (kMask) {
                        const int qi = i0 + kChunk * c + 2 * e;
                        const bool kin = key < p.Sk;
                        p0 = (kin && qi < p.Sq && (!p.causal || key <= qi + p.causal_off)) ? p0 : 0.0f;
                        p1 = (kin && qi + 1 < p.Sq && (!p.causal || key <= qi + 1 + p.causal_off)) ? p1 : 0.0f;
                    }
                    pv[2 * e] = p0;
                    pv[2 * e + 1] = p1;
                    wp[e] = bt_pack<BF16>(p0, p1);
                }
            };
            if (i0 + kStep <= p.Sq && j0 + 128 <= p.Sk && (!p.causal || j0 + 127 <= i0 + p.causal_off))
                weights(std::false_type{});
            else
                weights(std::true_type{});
            tmem_st8(tS, wp);    // P^T
            // dS^T = P^T (dP^T - D)
            ok = __all_sync(0xffffffffu, wait(bar(C::kBarDPFull + bf), (uint32_t)(st >> 1) & 1u, abort_addr,
                                              0x67000u | (uint32_t)(st & 0xfff)));
            if (!ok) break;
            tc_fence_after();
            float dp[16];
            tmem_ld16(tP, dp);
            tmem_wait_ld();
            reg_fence16(dp);
            uint32_t wd[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float d0, d1;
                f2_unpack(f2_mul(f2_pack(pv[2 * e], pv[2 * e + 1]),
                                 f2_sub(f2_pack(dp[2 * e], dp[2 * e + 1]), f2_pack(dl[2 * e], dl[2 * e + 1]))),
                          d0, d1);
                wd[e] = bt_pack<BF16>(d0, d1);
            }
            tmem_st8(tP, wd);    // dS^T
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::kBarPFull + bf));
        }
        // dV (chunks 0, 1: columns [0, D/2), [D/2, D)) and dK (chunks 2, 3)
        // rows, zero when no query row sees these keys, staged in the ring's
        // first 64 KB (every product that read the ring has completed) and
        // written by two TMA stores (rows past Sk are not written)
        if (ok && nsteps > 0) ok = __all_sync(0xffffffffu, wait(bar(C::kBarDone), 0, abort_addr, 0x66000u));
        const uint32_t tile_v = base + C::kSmemRing, tile_k = tile_v + C::kTile128;
        if (ok) {
            tc_fence_after();
            const bool is_k = c >= 2;
            const float mul = is_k ? p.dk_mul : p.dv_mul;
            const int col0 = (c & 1) * (D / 2);
            const uint32_t tacc = tmem + lane_base + C::kColAcc + (is_k ? D : 0) + col0;
#pragma unroll 1
            for (int cc = 0; cc < D / 2; cc += 16)
                stage_chunk16<BF16>(tacc + cc, is_k ? tile_k : tile_v, r, col0 + cc, mul, nsteps == 0);
            fence_proxy_async_smem();
        }
        named_bar_sync(1, kEwThreads);
        if (ok && threadIdx.x == 0) {
            for (int kb = 0; kb < C::kSwBlocks; ++kb) {
                tma_store_3d(&tmdV, tile_v + kb * C::kBlock128, kb * C::kElemsPerSw, j0, bk);
                tma_store_3d(&tmdK, tile_k + kb * C::kBlock128, kb * C::kElemsPerSw, j0, bk);
            }
            bulk_commit_group();
            bulk_wait_group_read0();   // the stores have read the tiles before the CTA ends
        }
    }
    teardown<D>(base, tmem, mma_ok);
}

// ---------------------------------------------------------------------------
// The dQ kernel takes 128-key steps.  It needs only S double-buffered:
// its dS goes over S, and dP is free as soon as the elementwise step has read
// it, so S_b [128 b, 128 b + 128) (b = 0, 1), one dP [256, 384) and dQ
// [384, 384 + d) fit 512 TMEM columns at N = 128: per 128 keys 24 products at
// the full rate (an N = 128 Q K^T-form product takes 64 cycles, two N = 64
// ones 96) and one step's turnaround instead of two.  K and V stream through
// separate rings (V is free after dP, K only after dQ), sized to the 227 KB:
// 3 K and 2 V slots at d = 128, 4 and 4 at d = 64.
// ---------------------------------------------------------------------------
template <int D>
struct CfgQ {
    static constexpr int kRowBytes = D * 2;
    static constexpr int kElemsPerSw = 64;
    static constexpr int kSwBlocks = kRowBytes / 128;
    static constexpr int kBlock = 128 * 128;                 // swizzle block of a 128-row tile
    static constexpr int kTile = 128 * kRowBytes;
    static constexpr int kQkSteps = kRowBytes / 32;
    static constexpr int kRingK = D == 128 ? 3 : 4;
    static constexpr int kRingV = D == 128 ? 2 : 4;
    static constexpr int kSmemQ = 0, kSmemDO = kTile, kSmemK = 2 * kTile;
    static constexpr int kSmemV = kSmemK + kRingK * kTile;
    static constexpr int kSmemPart = kSmemV + kRingV * kTile;   // D_i partial sums [2][128]
    static constexpr int kSmemBar = kSmemPart + 2 * 128 * 4;
    static constexpr int kBarResFull = 0;
    static constexpr int kBarKFull = 1;
    static constexpr int kBarKEmpty = 1 + kRingK;
    static constexpr int kBarVFull = 1 + 2 * kRingK;
    static constexpr int kBarVEmpty = 1 + 2 * kRingK + kRingV;
    static constexpr int kBarSFull = 1 + 2 * kRingK + 2 * kRingV;   // [2]
    static constexpr int kBarDPFull = kBarSFull + 2;
    static constexpr int kBarPFull = kBarDPFull + 1;               // [2]
    static constexpr int kBarDone = kBarPFull + 2;
    static constexpr int kBarDrain = kBarDone + 1;
    static constexpr int kBarOFull = kBarDrain + 1;   // the O tile landed (in V slot kOSlot)
    static constexpr int kBarOFree = kBarOFull + 1;   // D_i computed: V slot kOSlot is free
    static constexpr int kNumBars = kBarOFree + 1;
    static constexpr int kSmemSlot = kSmemBar + 8 * kNumBars;
    static constexpr int kSmemAbort = kSmemSlot + 4;
    static constexpr int kSmemUsed = kSmemAbort + 4;
    static constexpr int kSmemBytes = kSmemUsed + 1024;
    static constexpr uint32_t kColS = 0, kColDP = 256, kColAcc = 384;
    // the rows' O tile borrows the last V slot until D_i is computed (its
    // first V tile, kOSlot, is loaded after that)
    static constexpr int kOSlot = kRingV - 1;
    static_assert(D == 64 || D == 128, "pipelined backward: head dims 64 and 128");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// d[128][128] = A[128 rows][D] . B[128 rows][D]^T, both K-major 128-row tiles
template <int D, bool BF16>
__device__ __forceinline__ void mma_qk128(uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem) {
    using C = CfgQ<D>;
    constexpr uint32_t idesc = make_idesc(BF16 ? 1u : 0u, false, 128, 128);
    const uint64_t da = make_smem_desc(a_smem, 16, 1024), db = make_smem_desc(b_smem, 16, 1024);
#pragma unroll
    for (int kk = 0; kk < C::kQkSteps; ++kk) {
        const uint64_t off = (uint64_t)(((kk >> 2) * C::kBlock + (kk & 3) * 32) >> 4);
        mma_f16_ss(d_tmem, da + off, db + off, idesc, kk > 0);
    }
}

// d[128][D] (+)= A (TMEM, 128 x 128, 16-bit; 32-column chunk c packed over
// its first 16 columns) . B[128 rows][D] (MN-major 128-row tile)
template <int D, bool BF16>
__device__ __forceinline__ void mma_pv128(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_smem, bool acc) {
    using C = CfgQ<D>;
    constexpr uint32_t idesc = make_idesc(BF16 ? 1u : 0u, true, 128, D);
    const uint64_t db = make_smem_desc(b_smem, C::kBlock, 1024);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {    // 16 keys per product
        const uint64_t off = (uint64_t)((kk * 16 * 128) >> 4);
        mma_f16_ts(d_tmem, a_tmem + 32 * (kk >> 1) + 8 * (kk & 1), db + off, idesc, (acc || kk > 0) ? 1u : 0u);
    }
}

// dQ: one CTA per 128 query rows of one (batch, query head), 128-key steps;
// also writes D_i = dO_i . O_i of its rows for the dK/dV kernel (from a TMA-loaded
// O tile that borrows the last V slot, and the resident dO).
template <int D, bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
sdpa_bwd_dq_pipe_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                        const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmdQ,
                        const BwdTcParams p) {
    using C = CfgQ<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const uint32_t sQ = base + C::kSmemQ, sdO = base + C::kSmemDO;
    auto sK = [&](int slot) -> uint32_t { return base + C::kSmemK + (uint32_t)slot * C::kTile; };
    auto sV = [&](int slot) -> uint32_t { return base + C::kSmemV + (uint32_t)slot * C::kTile; };
    float* const dpart = reinterpret_cast<float*>(smem_raw + (base - raw) + C::kSmemPart);
    auto bar = [&](int i) -> uint32_t { return base + C::kSmemBar + 8u * (uint32_t)i; };
    const uint32_t abort_addr = base + C::kSmemAbort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float kL2e = 1.44269504088896340736f;

    // causal: a head's last query tiles (the most keys) first, so that the
    // light ones end the launch
    const int i0 = (p.causal ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x) * 128;
    const int bh = blockIdx.y;
    const int b = bh / p.Hq, hq = bh - b * p.Hq;
    const int kvrow = b * p.Hkv + hq / p.group;        // 3-D map index of the K/V head
    const int kend = p.causal ? min(p.Sk, i0 + 128 + p.causal_off) : p.Sk;
    const int nsteps = kend > 0 ? (kend + 127) / 128 : 0;

    if (threadIdx.x == 0) {
        mbar_init(bar(C::kBarResFull), 1);
        for (int i = 0; i < C::kRingK; ++i) {
            mbar_init(bar(C::kBarKFull + i), 1);
            mbar_init(bar(C::kBarKEmpty + i), 1);
        }
        for (int i = 0; i < C::kRingV; ++i) {
            mbar_init(bar(C::kBarVFull + i), 1);
            mbar_init(bar(C::kBarVEmpty + i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(C::kBarSFull + i), 1);
            mbar_init(bar(C::kBarPFull + i), kEwWarps);   // one arrival per warp
        }
        mbar_init(bar(C::kBarDPFull), 1);
        mbar_init(bar(C::kBarDone), 1);
        mbar_init(bar(C::kBarDrain), 1);
        mbar_init(bar(C::kBarOFull), 1);
        mbar_init(bar(C::kBarOFree), 1);
        sts_u32(abort_addr, 0u);
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(base + C::kSmemSlot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = lds_u32(base + C::kSmemSlot);
    bool mma_ok = true;

    if (warp == kLoadWarp) {
        // ================= TMA producer (lane 0) ==========================
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            prefetch_tmap(&tmdO);
            prefetch_tmap(&tmO);
            mbar_arrive_expect_tx(bar(C::kBarResFull), 2 * C::kTile);
            for (int kb = 0; kb < C::kSwBlocks; ++kb) {
                tma_load_3d(sQ + kb * C::kBlock, &tmQ, bar(C::kBarResFull), kb * C::kElemsPerSw, i0, bh);
                tma_load_3d(sdO + kb * C::kBlock, &tmdO, bar(C::kBarResFull), kb * C::kElemsPerSw, i0, bh);
            }
            mbar_arrive_expect_tx(bar(C::kBarOFull), C::kTile);
            for (int kb = 0; kb < C::kSwBlocks; ++kb)
                tma_load_3d(sV(C::kOSlot) + kb * C::kBlock, &tmO, bar(C::kBarOFull), kb * C::kElemsPerSw, i0, bh);
            bool ok = true;
            int kiss = 0, viss = 0;   // K / V tiles issued
            for (int jt = 0; jt < nsteps && ok; ++jt) {
                const int ks = jt % C::kRingK, vs = jt % C::kRingV;
                if (jt >= C::kRingK)
                    ok = wait(bar(C::kBarKEmpty + ks), (uint32_t)(jt / C::kRingK - 1) & 1u, abort_addr,
                              0x71000u | (uint32_t)(jt & 0xfff));
                if (!ok) break;
                mbar_arrive_expect_tx(bar(C::kBarKFull + ks), C::kTile);
                for (int kb = 0; kb < C::kSwBlocks; ++kb)
                    tma_load_3d(sK(ks) + kb * C::kBlock, &tmK, bar(C::kBarKFull + ks), kb * C::kElemsPerSw,
                                jt * 128, kvrow);
                kiss = jt + 1;
                if (jt >= C::kRingV)
                    ok = wait(bar(C::kBarVEmpty + vs), (uint32_t)(jt / C::kRingV - 1) & 1u, abort_addr,
                              0x72000u | (uint32_t)(jt & 0xfff));
                else if (jt == C::kOSlot)   // the O tile there has been read
                    ok = wait(bar(C::kBarOFree), 0, abort_addr, 0x7a000u);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(C::kBarVFull + vs), C::kTile);
                for (int kb = 0; kb < C::kSwBlocks; ++kb)
                    tma_load_3d(sV(vs) + kb * C::kBlock, &tmV, bar(C::kBarVFull + vs), kb * C::kElemsPerSw,
                                jt * 128, kvrow);
                viss = jt + 1;
            }
            // let the copies already issued land before the CTA ends
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(bar(C::kBarResFull), 0) && global_timer_ns() - t0 < 100000000ull) {
            }
            while (!mbar_try_wait(bar(C::kBarOFull), 0) && global_timer_ns() - t0 < 100000000ull) {
            }
            for (int jt = kiss > C::kRingK ? kiss - C::kRingK : 0; jt < kiss; ++jt)
                while (!mbar_try_wait(bar(C::kBarKFull + jt % C::kRingK), (uint32_t)(jt / C::kRingK) & 1u) &&
                       global_timer_ns() - t0 < 100000000ull) {
                }
            for (int jt = viss > C::kRingV ? viss - C::kRingV : 0; jt < viss; ++jt)
                while (!mbar_try_wait(bar(C::kBarVFull + jt % C::kRingV), (uint32_t)(jt / C::kRingV) & 1u) &&
                       global_timer_ns() - t0 < 100000000ull) {
                }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ================= MMA issuer =====================================
        const bool leader = elect_one();
        auto wait_all = [&](uint32_t b_, uint32_t par, uint32_t where) {
            return __all_sync(0xffffffffu, wait(b_, par, abort_addr, where));
        };
        auto commit = [&](uint32_t b_) {
            if (leader) mma_commit(b_);
            __syncwarp();
        };
        // S of step jt into buffer jt & 1 (its K landed)
        auto issue_s = [&](int jt) -> bool {
            const int ks = jt % C::kRingK;
            if (!wait_all(bar(C::kBarKFull + ks), (uint32_t)(jt / C::kRingK) & 1u, 0x73000u | (uint32_t)(jt & 0xfff)))
                return false;
            tc_fence_after();
            if (leader) mma_qk128<D, BF16>(tmem + C::kColS + 128 * (jt & 1), sQ, sK(ks));
            __syncwarp();
            commit(bar(C::kBarSFull + (jt & 1)));
            return true;
        };
        // dP of step jt (its V landed); V's slot is free once it has run
        auto issue_dp = [&](int jt) -> bool {
            const int vs = jt % C::kRingV;
            if (!wait_all(bar(C::kBarVFull + vs), (uint32_t)(jt / C::kRingV) & 1u, 0x74000u | (uint32_t)(jt & 0xfff)))
                return false;
            tc_fence_after();
            if (leader) mma_qk128<D, BF16>(tmem + C::kColDP, sdO, sV(vs));
            __syncwarp();
            commit(bar(C::kBarDPFull));
            commit(bar(C::kBarVEmpty + vs));
            return true;
        };
        bool ok = wait_all(bar(C::kBarResFull), 0, 0x70000u);
        if (ok && nsteps > 0) ok = issue_s(0);
        if (ok && nsteps > 0) ok = issue_dp(0);
        if (ok && nsteps > 1) ok = issue_s(1);
        // Per step, in issue order: dP(jt+1) (the single dP buffer was read
        // by the elementwise step jt), dQ(jt) (reads dS over S_b; K's slot is
        // then free), S(jt+2) (overwrites S_b)
        for (int jt = 0; jt < nsteps && ok; ++jt) {
            const int bf = jt & 1, ks = jt % C::kRingK;
            ok = wait_all(bar(C::kBarPFull + bf), (uint32_t)(jt >> 1) & 1u, 0x75000u | (uint32_t)(jt & 0xfff));
            if (!ok) break;
            tc_fence_after();
            if (jt + 1 < nsteps) {
                ok = issue_dp(jt + 1);
                if (!ok) break;
            }
            if (leader) mma_pv128<D, BF16>(tmem + C::kColAcc, tmem + C::kColS + 128 * bf, sK(ks), jt > 0);  // dQ += dS K
            __syncwarp();
            commit(bar(C::kBarKEmpty + ks));
            if (jt + 2 < nsteps) ok = issue_s(jt + 2);
        }
        if (ok) commit(bar(C::kBarDone));
        mma_ok = ok;
    } else {
        // ================= elementwise (warps 0-15) =======================
        const int quarter = warp & 3, c = warp >> 2;   // lane quarter, 32-column chunk
        const int r = quarter * 32 + lane, row = i0 + r;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const float sl = p.scale * kL2e;
        const uint64_t sl2 = f2_pack(sl, sl);
        const float nlse_r = row < p.Sq ? -(p.lse[(size_t)bh * p.Sq + row] * kL2e) : 0.0f;
        const uint64_t nl2 = f2_pack(nlse_r, nlse_r);
        // D_i: chunks 0 and 1 compute the two halves of the row's dot
        // product from the dO and O tiles (rows past Sq were filled with
        // zeros), summed through shared memory; then O's slot is released
        bool ok = true;
        if (c < 2) {
            ok = wait(bar(C::kBarResFull), 0, abort_addr, 0x79000u) &&
                 wait(bar(C::kBarOFull), 0, abort_addr, 0x7b000u);
            dpart[c * 128 + r] = ok ? bt_row_dot_smem<D, BF16>(sdO, sV(C::kOSlot), r, c) : 0.0f;
        }
        named_bar_sync(1, kEwThreads);
        if (threadIdx.x == 0) mbar_arrive(bar(C::kBarOFree));
        const float d_r = (dpart[r] + dpart[128 + r]) * p.d_mul;
        const uint64_t d2 = f2_pack(d_r, d_r);
        if (c == 0 && row < p.Sq) p.delta[(size_t)bh * p.Sq + row] = d_r;
        for (int jt = 0; jt < nsteps && ok; ++jt) {
            const int bf = jt & 1, j0 = jt * 128;
            ok = __all_sync(0xffffffffu, wait(bar(C::kBarSFull + bf), (uint32_t)(jt >> 1) & 1u, abort_addr,
                                              0x76000u | (uint32_t)(jt & 0xfff)));
            if (!ok) break;
            tc_fence_after();
            const uint32_t tS = tmem + lane_base + C::kColS + 128 * bf + 32 * c;
            const uint32_t tP = tmem + lane_base + C::kColDP + 32 * c;
            float s[32];
            tmem_ld32(tS, s);
            tmem_wait_ld();
            reg_fence32(s);
            // P = 2^(s sl - LSE) (0 where masked), while dP is computed
            float pv[32];
            auto weights = [&](auto masked) {
                constexpr bool kMask = decltype(masked)::value;
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float x0, x1;
                    f2_unpack(f2_fma(f2_pack(s[2 * e], s[2 * e + 1]), sl2, nl2), x0, x1);
                    float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                    if constexpr (kMask) {
                        const int key = j0 + 32 * c + 2 * e;
                        const bool rin = row < p.Sq;
                        p0 = (rin && key < p.Sk && (!p.causal || key <= row + p.causal_off)) ? p0 : 0.0f;
                        p1 = (rin && key + 1 < p.Sk && (!p.causal || key + 1 <= row + p.causal_off)) ? p1 : 0.0f;
                    }
                    pv[2 * e] = p0;
                    pv[2 * e + 1] = p1;
                }
            };
            if (i0 + 128 <= p.Sq && j0 + 128 <= p.Sk && (!p.causal || j0 + 127 <= i0 + p.causal_off))
                weights(std::false_type{});
            else
                weights(std::true_type{});
            // dS = P (dP - D)
            ok = __all_sync(0xffffffffu, wait(bar(C::kBarDPFull), (uint32_t)jt & 1u, abort_addr,
                                              0x77000u | (uint32_t)(jt & 0xfff)));
            if (!ok) break;
            tc_fence_after();
            float dp[32];
            tmem_ld32(tP, dp);
            tmem_wait_ld();
            reg_fence32(dp);
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                float d0, d1;
                f2_unpack(f2_mul(f2_pack(pv[2 * e], pv[2 * e + 1]), f2_sub(f2_pack(dp[2 * e], dp[2 * e + 1]), d2)), d0, d1);
                w[e] = bt_pack<BF16>(d0, d1);
            }
            tmem_st16(tS, w);    // dS
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::kBarPFull + bf));
        }
        // dQ row, this warp's quarter of the columns, zero when the row sees
        // no key, staged in K slot 0 (every product that read K has
        // completed) and written by one TMA store (rows past Sq are not
        // written)
        if (ok && nsteps > 0) ok = __all_sync(0xffffffffu, wait(bar(C::kBarDone), 0, abort_addr, 0x78000u));
        const uint32_t tile = sK(0);
        if (ok) {
            tc_fence_after();
            const int col0 = c * (D / 4);
#pragma unroll 1
            for (int cc = 0; cc < D / 4; cc += 16)
                stage_chunk16<BF16>(tmem + lane_base + C::kColAcc + col0 + cc, tile, r, col0 + cc, p.dq_mul,
                                    nsteps == 0);
            fence_proxy_async_smem();
        }
        named_bar_sync(1, kEwThreads);
        if (ok && threadIdx.x == 0) {
            for (int kb = 0; kb < C::kSwBlocks; ++kb)
                tma_store_3d(&tmdQ, tile + kb * C::kBlock, kb * C::kElemsPerSw, i0, bh);
            bulk_commit_group();
            bulk_wait_group_read0();   // the store has read the tile before the CTA ends
        }
    }
    // end: after a failed wait no MMA may still write TMEM when it is freed
    if (warp == kMmaWarp && !mma_ok) {
        if (elect_one()) mma_commit(bar(C::kBarDrain));
        __syncwarp();
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(bar(C::kBarDrain), 0) && global_timer_ns() - t0 < 100000000ull) {
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

}  // namespace bwdp
}  // namespace sdpa
