// sdpa_fwd_sm100.cuh -- fused scaled-dot-product attention forward for
// sm_100a (B200): TMA-fed K/V ring, tcgen05 MMAs with accumulators in tensor
// memory, warp-specialised roles, exp2 online softmax, causal tile skipping,
// GQA/MQA K/V heads shared by index.
//
// Method (article "Self-attention, CUDA kernels and FlashAttention", section
// 3): Q, K, V are cut into on-chip tiles, scores of a tile are turned into
// weights with a softmax that keeps a running row maximum and row sum, the
// partial output is rescaled when the maximum moves, and only the output and
// the per-row normaliser (LSE) are written to global memory; the Sq x Sk
// score matrix never leaves the SM.  Formula and steps: codelab "JAX on GPU,
// Lab 5: attention on GPU", section 1; causal mask section 7; MHA/GQA/MQA
// section 9; FP8 E4M3 forward section 10.
//
// One CTA owns 2 x 128 query rows of one (batch, query head) and walks the
// K/V tiles of that head's KV head.  Warp roles (384 threads):
//   warps 0-3  softmax group 0: query tile 0, thread = row = TMEM lane
//   warps 4-7  softmax group 1: query tile 1
//   warp  8    TMA producer: Q tiles once, then K_0, V_0, K_1, V_1, ...
//   warp  9    MMA issuer (one elected lane) and TMEM owner
//   warps 10-11 idle (they complete warpgroup 2 for the register split)
// Registers are moved with setmaxnreg from warpgroup 2 to the softmax groups.
// Tensor memory (512 columns x 128 lanes, fp32):
//   [0,128) S0   [128,256) S1   [256,256+d) O0   [384,384+d) O1
//   P_w (the weights, packed 2 x 16-bit or 4 x e4m3 per column) overwrites
//   the upper half of S_w once the softmax group has read S_w.
// MMA issue order per K/V tile i: S0=Q0 K_i^T, O1+=P1(i-1) V_(i-1),
// S1=Q1 K_i^T, O0+=P0(i) V_i -- while one softmax group works, the tensor
// pipe always has the other group's products queued.  tcgen05 MMAs from one
// thread execute in issue order, so an S_w write queued after the P_w read
// of the previous tile cannot overtake it, and the commit that signals S_w(i)
// also covers O_w += P_w(i-1) V_(i-1): when a softmax group sees S_w(i) its
// O_w is quiescent and may be rescaled in place.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include "sm100_ptx.cuh"

// Tuning knobs (compile-time; the defaults are the measured best on B200).
// Pairs e (0..15) of a 32-column chunk whose exponentials go to the FMA pipe:
// bit (e & 7) of this mask.
#ifndef SDPA_POLY_MASK
#define SDPA_POLY_MASK 0x88
#endif
// 1: the softmax signals each P tile once; 2: once per half of the keys.
#ifndef SDPA_P_SPLIT
#define SDPA_P_SPLIT 2
#endif
// K/V ring depth for d = 128 (16-bit) and d = 64.
#ifndef SDPA_STAGES_D128
#define SDPA_STAGES_D128 4
#endif
#ifndef SDPA_STAGES_D64
#define SDPA_STAGES_D64 8
#endif

namespace sdpa {

enum Kind { KIND_BF16 = 0, KIND_FP16 = 1, KIND_E4M3 = 2 };

constexpr int kBlockM = 128;        // query rows per tile (= TMEM lanes)
constexpr int kBlockN = 128;        // keys per K/V tile
constexpr int kQTiles = 2;          // query tiles per CTA
constexpr int kThreads = 384;       // 3 warpgroups
constexpr int kSoftmaxRegs = 208;   // per thread after setmaxnreg, warpgroups 0-1
constexpr int kOtherRegs = 88;      // warpgroup 2 (TMA, MMA, two idle warps)
constexpr int kLaunchRegs = 168;    // registers per thread at launch (384 threads, 1 CTA/SM)
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kTmemCols = 512;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // bounded waits: 1 s

// Device status word: [0] status (0 ok, 4 = device timeout), [1] location.
__device__ unsigned int g_sdpa_status[2];

struct FwdParams {
    void* o;            // [B,Hq,Sq,D] 16-bit
    float* lse;         // [B,Hq,Sq] or null
    int B, Hq, Hkv, Sq, Sk;
    int group;          // Hq / Hkv
    int n_qblocks;      // ceil(Sq / 256)
    int causal;
    float score_log2;   // multiplier from raw MMA score to log2 units
    float out_mul;      // multiplier on (sum_j p_j v_j) / l: the V descale for FP8, else 1
};

template <int D, int KIND, int NS>
struct FwdCfg {
    static constexpr int kElem = (KIND == KIND_E4M3) ? 1 : 2;
    static constexpr int kRowBytes = D * kElem;
    static constexpr int kElemsPerSw = 128 / kElem;      // elements in one 128-byte swizzle row
    static constexpr int kSwBlocks = kRowBytes / 128;    // 128-byte column blocks per row
    static constexpr int kSwBlockBytes = 128 * 128;      // one column block of a 128-row tile
    static constexpr int kTileBytes = 128 * kRowBytes;
    static constexpr int kQkSteps = kRowBytes / 32;      // every MMA consumes 32 bytes of K
    static constexpr int kPvKeysPerStep = 32 / kElem;
    static constexpr int kPvSteps = kBlockN / kPvKeysPerStep;
    static constexpr int kPCols = kBlockN * kElem / 4;   // TMEM columns of one P row
    static constexpr float kRescaleThreshold = (KIND == KIND_E4M3) ? 0.0f : 8.0f;
    // log2 of the factor applied to p before it is rounded for the PV MMA:
    // 448 (the e4m3 maximum) for FP8, so that p in (0, 1] fills the format
    static constexpr float kPLog2 = (KIND == KIND_E4M3) ? 8.807354922057604f : 0.0f;
    // shared memory map (offsets from a 1024-byte aligned base)
    static constexpr int kSmemQ = 0;
    static constexpr int kSmemKV = kQTiles * kTileBytes;
    static constexpr int kSmemBar = kSmemKV + NS * kTileBytes;
    // barriers: q_full[2] kv_full[NS] kv_empty[NS] s_full[2] p_full[2 tiles][2 halves]
    //           o_full[2] drain[1]
    static constexpr int kBarQFull = 0;
    static constexpr int kBarKVFull = 2;
    static constexpr int kBarKVEmpty = 2 + NS;
    static constexpr int kBarSFull = 2 + 2 * NS;
    static constexpr int kBarPFull = 4 + 2 * NS;
    static constexpr int kBarOFull = 8 + 2 * NS;
    static constexpr int kBarDrain = 10 + 2 * NS;
    static constexpr int kNumBars = 11 + 2 * NS;
    static constexpr int kSmemTmemSlot = kSmemBar + 8 * kNumBars;
    static constexpr int kSmemAbort = kSmemTmemSlot + 4;
    static constexpr int kSmemUsed = kSmemAbort + 4;
    static constexpr int kSmemBytes = kSmemUsed + 1024;  // slack for the 1024-byte alignment
    // TMEM columns
    static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 384;
    static constexpr uint32_t kPOffset = 64;
    static_assert(kRowBytes % 128 == 0, "rows must fill whole 128-byte swizzle rows");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static_assert(D <= 128, "O tile must fit its 128 TMEM columns");
};

// ---------------------------------------------------------------------------
// bounded waiting
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.volatile.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Wait for the phase of `bar` with parity `parity`.  Gives up (returning
// false) when another role of the CTA has aborted, or after kWaitLimitNs, in
// which case it records the timeout and `where` in the device status word and
// raises the CTA's abort flag.
__device__ __forceinline__ bool wait_bar_slow(uint32_t bar, uint32_t parity, uint32_t abort_addr,
                                           uint32_t where) {
    const uint64_t t0 = global_timer_ns();
    for (uint32_t k = 1;; ++k) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((k & 63u) == 0) {
            if (ld_shared_u32(abort_addr) != 0u) return false;
            if (global_timer_ns() - t0 > kWaitLimitNs) {
                st_shared_u32(abort_addr, 1u);
                if (atomicCAS(&g_sdpa_status[0], 0u, 4u) == 0u)
                    atomicExch(&g_sdpa_status[1], where);
                return false;
            }
        }
    }
}
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, uint32_t abort_addr,
                                         uint32_t where) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_bar_slow(bar, parity, abort_addr, where);
}

// Pairs of one 32-column chunk (e = 0..15) whose exponentials are evaluated
// on the FMA pipe instead of the MUFU (SDPA_POLY_MASK).
__device__ __forceinline__ constexpr bool poly_pair(int e) {
    return ((SDPA_POLY_MASK >> (e & 7)) & 1) != 0;
}

// Row-tile key counts of one CTA: number of K/V tiles query tile w needs.
__device__ __forceinline__ int tiles_for(int row0, int Sq, int Sk, int causal) {
    if (row0 >= Sq) return 0;
    const int kend = causal ? min(Sk, row0 + kBlockM) : Sk;
    return (kend + kBlockN - 1) / kBlockN;
}

template <int D, int KIND, int NS>
__global__ void __launch_bounds__(kThreads, 1)
sdpa_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV,
                      const FwdParams p) {
    using C = FwdCfg<D, KIND, NS>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- work unit: longest (last) query blocks first --------------------
    const int n_bh = p.B * p.Hq;
    const int qblk = p.n_qblocks - 1 - (int)(blockIdx.x / (unsigned)n_bh);
    const int bh = (int)(blockIdx.x % (unsigned)n_bh);
    const int b = bh / p.Hq;
    const int hq = bh - b * p.Hq;
    const int kvh = b * p.Hkv + hq / p.group;
    const int m0 = qblk * (kQTiles * kBlockM);
    const int nt0 = tiles_for(m0, p.Sq, p.Sk, p.causal);
    const int nt1 = tiles_for(m0 + kBlockM, p.Sq, p.Sk, p.causal);
    const int n = max(nt0, nt1);

    auto bar = [&](int i) -> uint32_t { return sbase + C::kSmemBar + 8u * (uint32_t)i; };
    const uint32_t abort_addr = sbase + C::kSmemAbort;
    const uint32_t slot_addr = sbase + C::kSmemTmemSlot;

    if (threadIdx.x == 0) {
        for (int w = 0; w < kQTiles; ++w) {
            mbar_init(bar(C::kBarQFull + w), 1);
            mbar_init(bar(C::kBarSFull + w), 1);
            mbar_init(bar(C::kBarPFull + 2 * w), kBlockM);
            mbar_init(bar(C::kBarPFull + 2 * w + 1), kBlockM);
            mbar_init(bar(C::kBarOFull + w), 1);
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(bar(C::kBarKVFull + s), 1);
            mbar_init(bar(C::kBarKVEmpty + s), 1);
        }
        mbar_init(bar(C::kBarDrain), 1);
        st_shared_u32(abort_addr, 0u);
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(slot_addr, kTmemCols);
        tmem_relinquish();
    }
    if (warp == kLoadWarp && lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ld_shared_u32(slot_addr);
    // launch: 384 x 168 registers; split: 256 x 208 + 128 x 88 = 64512 <= 64512 (the host
    // checks the compiled register count before the first launch)
    static_assert(2 * 128 * kSoftmaxRegs + 128 * kOtherRegs <= kThreads * kLaunchRegs, "register split");

    const uint32_t sQ = sbase + C::kSmemQ;
    const uint32_t sKV = sbase + C::kSmemKV;

    if (warp >= 8) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kOtherRegs));
    if (warp == kLoadWarp) {
        // ================= TMA producer =================================
        if (lane == 0) {
            bool ok = true;
            for (int w = 0; w < kQTiles; ++w) {
                if ((w ? nt1 : nt0) == 0) continue;
                const uint32_t qb = bar(C::kBarQFull + w);
                mbar_arrive_expect_tx(qb, C::kTileBytes);
                for (int kb = 0; kb < C::kSwBlocks; ++kb)
                    tma_load_3d(sQ + w * C::kTileBytes + kb * C::kSwBlockBytes, &tmQ, qb,
                                kb * C::kElemsPerSw, m0 + w * kBlockM, bh);
            }
            int t = 0;
            for (; t < 2 * n && ok; ++t) {
                const int slot = t % NS;
                const uint32_t par = ((uint32_t)(t / NS) & 1u) ^ 1u;
                ok = wait_bar(bar(C::kBarKVEmpty + slot), par, abort_addr, 0x10000u | (uint32_t)t);
                if (!ok) break;
                const uint32_t fb = bar(C::kBarKVFull + slot);
                mbar_arrive_expect_tx(fb, C::kTileBytes);
                const CUtensorMap* m = (t & 1) ? &tmV : &tmK;
                for (int kb = 0; kb < C::kSwBlocks; ++kb)
                    tma_load_3d(sKV + slot * C::kTileBytes + kb * C::kSwBlockBytes, m, fb,
                                kb * C::kElemsPerSw, (t >> 1) * kBlockN, kvh);
            }
            if (!ok) {
                // let the copies already issued land before the CTA exits
                for (int u = max(0, t - NS); u < t; ++u) {
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(bar(C::kBarKVFull + u % NS), (uint32_t)(u / NS) & 1u) &&
                           global_timer_ns() - t0 < 100000000ull) {
                    }
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ================= MMA issuer ===================================
        // The whole warp runs the loop (so descriptors and addresses stay
        // warp-uniform); one elected lane issues the MMAs and commits.
        const bool leader = elect_one();
        constexpr uint32_t fmt = (KIND == KIND_BF16) ? 1u : 0u;
        constexpr uint32_t idesc_qk = make_idesc(fmt, false, kBlockM, kBlockN);
        constexpr uint32_t idesc_pv = make_idesc(fmt, true, kBlockM, D);
        const uint64_t desc_q0 = make_smem_desc(sQ, 16, 1024);
        const uint64_t desc_q1 = make_smem_desc(sQ + C::kTileBytes, 16, 1024);
        const uint64_t desc_k = make_smem_desc(sKV, 16, 1024);
        const uint64_t desc_v = make_smem_desc(sKV, C::kSwBlockBytes, 1024);
        bool ok = true;

        auto wait_all = [&](uint32_t b_, uint32_t par, uint32_t where) {
            const bool r_ = wait_bar(b_, par, abort_addr, where);
            return __all_sync(0xffffffffu, r_);
        };
        auto commit = [&](uint32_t b_) {
            if (leader) mma_commit(b_);
            __syncwarp();
        };
        auto issue_qk = [&](int w, int slot) {
            const uint32_t d_tmem = tmem + (w ? C::kColS1 : C::kColS0);
            const uint64_t dq = w ? desc_q1 : desc_q0;
            const uint64_t dk = desc_k + (uint64_t)((slot * C::kTileBytes) >> 4);
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < C::kQkSteps; ++kk) {
                    const uint64_t off = (uint64_t)(((kk >> 2) * C::kSwBlockBytes + (kk & 3) * 32) >> 4);
                    if constexpr (KIND == KIND_E4M3)
                        mma_f8_ss(d_tmem, dq + off, dk + off, idesc_qk, kk > 0);
                    else
                        mma_f16_ss(d_tmem, dq + off, dk + off, idesc_qk, kk > 0);
                }
            }
            __syncwarp();
        };
        // O_w (+)= P_w V over the keys of one half of the tile (K steps
        // [h * kPvSteps / 2, (h + 1) * kPvSteps / 2)); P is read from TMEM.
        auto issue_pv_half = [&](int w, int slot, bool acc, int h) {
            const uint32_t d_tmem = tmem + (w ? C::kColO1 : C::kColO0);
            const uint32_t a_tmem = tmem + (w ? C::kColS1 : C::kColS0) + C::kPOffset;
            const uint64_t dv = desc_v + (uint64_t)((slot * C::kTileBytes) >> 4);
            if (leader) {
#pragma unroll
                for (int kk = h * C::kPvSteps / 2; kk < (h + 1) * C::kPvSteps / 2; ++kk) {
                    const uint64_t off = (uint64_t)((kk * C::kPvKeysPerStep * 128) >> 4);
                    const uint32_t accum = (acc || kk > 0) ? 1u : 0u;
                    if constexpr (KIND == KIND_E4M3)
                        mma_f8_ts(d_tmem, a_tmem + kk * 8, dv + off, idesc_pv, accum);
                    else
                        mma_f16_ts(d_tmem, a_tmem + kk * 8, dv + off, idesc_pv, accum);
                }
            }
            __syncwarp();
        };
        // wait for each half of P_w(j) and issue its MMAs
        auto pv = [&](int w, int slot, int j) -> bool {
            for (int h = 0; h < SDPA_P_SPLIT; ++h) {
                if (!wait_all(bar(C::kBarPFull + 2 * w + h), (uint32_t)j & 1u,
                              0x22000u | (w << 11) | (h << 10) | (uint32_t)j))
                    return false;
                tc_fence_after();
                if (SDPA_P_SPLIT == 1) {
                    issue_pv_half(w, slot, j > 0, 0);
                    issue_pv_half(w, slot, j > 0, 1);
                } else {
                    issue_pv_half(w, slot, j > 0, h);
                }
            }
            return true;
        };

        if (nt0 > 0) ok = wait_all(bar(C::kBarQFull + 0), 0, 0x20000u);
        if (ok && nt1 > 0) ok = wait_all(bar(C::kBarQFull + 1), 0, 0x20001u);

        for (int i = 0; i <= n && ok; ++i) {
            const int tK = 2 * i, tV = 2 * i + 1;
            const int slotK = tK % NS, slotV = tV % NS;
            if (i < n) {
                ok = wait_all(bar(C::kBarKVFull + slotK), (uint32_t)(tK / NS) & 1u, 0x21000u | (uint32_t)i);
                if (!ok) break;
                if (i < nt0) {
                    issue_qk(0, slotK);
                    commit(bar(C::kBarSFull + 0));
                }
            }
            if (i >= 1) {
                const int j = i - 1;
                if (j < nt1) {
                    ok = pv(1, (2 * j + 1) % NS, j);
                    if (!ok) break;
                    if (j == nt1 - 1) commit(bar(C::kBarOFull + 1));
                }
                commit(bar(C::kBarKVEmpty + (2 * j + 1) % NS));   // V_(i-1) free
            }
            if (i < n) {
                if (i < nt1) {
                    issue_qk(1, slotK);
                    commit(bar(C::kBarSFull + 1));
                }
                commit(bar(C::kBarKVEmpty + slotK));               // K_i free
                ok = wait_all(bar(C::kBarKVFull + slotV), (uint32_t)(tV / NS) & 1u, 0x23000u | (uint32_t)i);
                if (!ok) break;
                if (i < nt0) {
                    ok = pv(0, slotV, i);
                    if (!ok) break;
                    if (i == nt0 - 1) commit(bar(C::kBarOFull + 0));
                }
            }
        }
        if (!ok) {
            // make sure no MMA is still writing tensor memory at exit
            commit(bar(C::kBarDrain));
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(bar(C::kBarDrain), 0) && global_timer_ns() - t0 < 100000000ull) {
            }
        }
        // teardown: the softmax groups have read O for the last time
        named_bar_sync(1, 256 + 32);
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    } else if (warp < 8) {
        // ================= softmax groups (warps 0-7) ====================
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
        const int w = warp >> 2;                 // query tile
        const int quarter = warp & 3;            // TMEM lane quarter of this warp
        const int r = (int)(threadIdx.x & 127);  // row within the tile
        const int row = m0 + w * kBlockM + r;
        const int nw = w ? nt1 : nt0;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint32_t tS = tmem + lane_base + (w ? C::kColS1 : C::kColS0);
        const uint32_t tP = tS + C::kPOffset;
        const uint32_t tO = tmem + lane_base + (w ? C::kColO1 : C::kColO0);
        const float sl = p.score_log2;
        const uint64_t sl2 = f2_pack(sl, sl);
        float m_run = -INFINITY;   // running max of the scaled scores (log2 units)
        float l_run = 0.0f;        // running sum of 2^(s*sl - m_run + kPLog2)
        bool ok = true;

        for (int i = 0; i < nw; ++i) {
            ok = wait_bar(bar(C::kBarSFull + w), (uint32_t)i & 1u, abort_addr, 0x30000u | (w << 12) | i);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();

            // S row in two halves: the second half's load overlaps the first
            // half's masking and max
            float s[kBlockN];
            tmem_ld32(tS + 0, *reinterpret_cast<float(*)[32]>(&s[0]));
            tmem_ld32(tS + 32, *reinterpret_cast<float(*)[32]>(&s[32]));
            tmem_wait_ld();
            reg_fence32(&s[0]);
            reg_fence32(&s[32]);
            tmem_ld32(tS + 64, *reinterpret_cast<float(*)[32]>(&s[64]));
            tmem_ld32(tS + 96, *reinterpret_cast<float(*)[32]>(&s[96]));

            // mask: keys past Sk, and (causal) keys after the row
            const int key0 = i * kBlockN;
            const bool edge = (key0 + kBlockN > p.Sk) ||
                              (p.causal && key0 + kBlockN - 1 > m0 + w * kBlockM);
            int lim = p.Sk - key0;
            if (p.causal) lim = min(lim, row - key0 + 1);
            if (edge) {
#pragma unroll
                for (int c = 0; c < kBlockN / 2; ++c)
                    if (c >= lim) s[c] = -INFINITY;
            }
            // first half only: columns 0..63 (64..127 are still in flight)
            float mx0 = s[0], mx1 = s[1];
#pragma unroll
            for (int c = 2; c + 4 <= kBlockN / 2 - 2; c += 4) {
                mx0 = fmax3(mx0, s[c], s[c + 1]);
                mx1 = fmax3(mx1, s[c + 2], s[c + 3]);
            }
            mx0 = fmax3(mx0, s[kBlockN / 2 - 2], s[kBlockN / 2 - 1]);
            tmem_wait_ld();
            reg_fence32(&s[64]);
            reg_fence32(&s[96]);
            if (edge) {
#pragma unroll
                for (int c = kBlockN / 2; c < kBlockN; ++c)
                    if (c >= lim) s[c] = -INFINITY;
            }
#pragma unroll
            for (int c = kBlockN / 2; c < kBlockN; c += 4) {
                mx0 = fmax3(mx0, s[c], s[c + 1]);
                mx1 = fmax3(mx1, s[c + 2], s[c + 3]);
            }
            const float tile_max = fmaxf(mx0, mx1) * sl;

            // The running max only moves when the new one exceeds it by more
            // than the threshold; weights computed against a stale max are
            // bounded by 2^threshold and the final O / l and LSE are exact
            // for any reference value as long as O and l share it.
            float alpha = 1.0f;
            if (tile_max > m_run + C::kRescaleThreshold) {
                alpha = ex2_approx(m_run - tile_max);   // 0 on the first tile
                m_run = tile_max;
            }
            l_run *= alpha;
            // O_w (quiescent: its last update is covered by the S_w(i) commit)
            // takes the same factor as l before any of P_w(i) V_i is added.
            if (i > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    float o[32];
                    tmem_ld32(tO + 32 * c, o);
                    tmem_wait_ld();
                    reg_fence32(o);
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] *= alpha;
                    tmem_st32(tO + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(o));
                }
            }

            // weights p = 2^(s*sl - m [+ log2 of the P scale]): most pairs on
            // the MUFU, kPolyPairs in every 8 on the FMA pipe
            // (exp2_poly_x2); row sums from the fp32 values, P rounded for the
            // PV product and stored to TMEM one half of the keys at a time so
            // the MMA warp can start on the first half.
            const float neg_m = C::kPLog2 - m_run;
            const uint64_t nm2 = f2_pack(neg_m, neg_m);
            uint64_t sum2[2] = {0ull, 0ull};
#pragma unroll
            for (int c = 0; c < kBlockN / 32; ++c) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const uint64_t x2 = f2_fma(f2_pack(s[32 * c + 2 * e], s[32 * c + 2 * e + 1]), sl2, nm2);
                    float x0, x1;
                    f2_unpack(x2, x0, x1);
                    uint64_t p2;
                    if (poly_pair(e)) {
                        p2 = exp2_poly_x2(f2_pack(fmaxf(x0, -126.0f), fmaxf(x1, -126.0f)));
                    } else {
                        p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
                    }
                    sum2[e & 1] = f2_add(sum2[e & 1], p2);
                    float q0, q1;
                    f2_unpack(p2, q0, q1);
                    if constexpr (KIND == KIND_E4M3) {
                        if (e & 1) pk[e >> 1] |= pack_e4m3x4(0.f, 0.f, q0, q1) & 0xFFFF0000u;
                        else pk[e >> 1] = pack_e4m3x4(q0, q1, 0.f, 0.f) & 0x0000FFFFu;
                    } else {
                        pk[e] = (KIND == KIND_BF16) ? pack_bf16x2(q0, q1) : pack_f16x2(q0, q1);
                    }
                }
                // first half of the keys: its stores were issued one chunk ago,
                // so this wait finds them done
                if (SDPA_P_SPLIT == 2 && c == 2) {
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(bar(C::kBarPFull + 2 * w));
                }
                if constexpr (KIND == KIND_E4M3)
                    tmem_st8(tP + 8 * c, pk);
                else
                    tmem_st16(tP + 16 * c, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(C::kBarPFull + 2 * w + (SDPA_P_SPLIT - 1)));
            {
                float a0, a1, b0, b1;
                f2_unpack(sum2[0], a0, a1);
                f2_unpack(sum2[1], b0, b1);
                l_run += (a0 + a1) + (b0 + b1);
            }
        }

        // ---- epilogue: O / l -> 16-bit, LSE ---------------------------------
        if (ok && nw > 0) {
            ok = wait_bar(bar(C::kBarOFull + w), 0, abort_addr, 0x40000u | w);
            ok = __all_sync(0xffffffffu, ok);
        }
        if (ok && nw > 0) {
            tc_fence_after();
            const float inv_l = p.out_mul / l_run;
            const bool live = row < p.Sq;
            const size_t orow = ((size_t)bh * p.Sq + (size_t)(live ? row : 0)) * D;
            uint16_t* obase = reinterpret_cast<uint16_t*>(p.o) + orow;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                float o[32];
                tmem_ld32(tO + 32 * c, o);
                tmem_wait_ld();
                reg_fence32(o);
                uint32_t u[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    u[e] = (KIND == KIND_FP16) ? pack_f16x2(o[2 * e] * inv_l, o[2 * e + 1] * inv_l)
                                               : pack_bf16x2(o[2 * e] * inv_l, o[2 * e + 1] * inv_l);
                if (live) {
                    uint4* dst = reinterpret_cast<uint4*>(obase + 32 * c);
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4)
                        dst[v4] = make_uint4(u[4 * v4], u[4 * v4 + 1], u[4 * v4 + 2], u[4 * v4 + 3]);
                }
            }
            if (p.lse != nullptr && live)
                p.lse[(size_t)bh * p.Sq + row] = (m_run + __log2f(l_run) - C::kPLog2) * kLn2;
        }
        tc_fence_before();
        named_bar_sync(1, 256 + 32);
    }

}

}  // namespace sdpa
