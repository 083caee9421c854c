// sdpa_fwd_sm100.cuh -- fused scaled-dot-product attention forward for
// sm_100a (B200): TMA-fed K/V ring, tcgen05 MMAs with accumulators in tensor
// memory, warp-specialised roles, exp2 online softmax, causal tile skipping,
// GQA/MQA K/V heads shared by index, persistent CTAs.
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
// Work units are 128 query rows of one (batch, query head).  One CTA runs
// per SM and walks a static list of schedule items: for causal attention an
// item pairs query tile j with tile nq-1-j of the same head (together always
// nq+1 K/V tiles), so a round-robin assignment of items balances the SMs;
// items come in groups of heads so their K/V stay in L2.  The CTA treats the
// K/V tiles of all its units as one stream, so the scores of the next unit
// are computed while the current one finishes.  Warp roles (320 threads):
//   warps 0-3    softmax group 0: keys 0-63 of every tile, thread = row = lane
//   warps 4-7    softmax group 1: keys 64-127 of every tile
//   warps 8-11   (EPI) epilogue: merge the halves of a finished unit,
//                O -> 16-bit, LSE, while the softmax groups go on with the
//                next unit; without EPI the softmax groups do it themselves
//   next warp    TMA producer: Q per unit, K/V tiles in MMA consumption
//                order K_0, K_1, V_0, K_2, V_1, ... over the stream
//   last warp    MMA issuer (one elected lane) and TMEM owner
// With EPI the roles follow warp groups, so that the softmax warp groups can
// take registers from the epilogue one (setmaxnreg).  EPI pays when units
// are short (the epilogue leaves the softmax critical path once per unit)
// and costs a few percent on long ones.
// Tensor memory (512 columns x 128 lanes, fp32):
//   [0,128) S_a  [128,256) S_b  [256,256+d) O_0  [384,384+d) O_1
// S is double-buffered: S(g) of stream tile g lives in S_(g&1), and
// Q K_(g+2)^T is issued as soon as O += P(g) V_g has been issued, so the
// next scores are ready when the softmax finishes a tile and the tensor pipe
// works while the softmax does.  Each softmax group keeps its own running max
// m_h, sum l_h and output O_h over its half of the keys; the halves never
// exchange data inside the loop and are merged once per unit, by the
// epilogue warps:
//   O = (2^(m_0-m) O_0 + 2^(m_1-m) O_1) / (2^(m_0-m) l_0 + 2^(m_1-m) l_1),
//   m = max(m_0, m_1),  LSE = (m + log2(2^(m_0-m) l_0 + 2^(m_1-m) l_1)) ln 2.
// P_h(g) (the weights, packed 2 x 16-bit or 4 x e4m3 per column) overwrites
// group h's own columns of S_(g&1) once the group has read them.
// tcgen05 MMAs from one thread execute in issue order, so the S write of
// Q K_(g+2)^T queued after the P(g) reads cannot overtake them.
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
#define SDPA_POLY_MASK 0x00
#endif
// K/V ring depth for 16-bit d = 128 (with one Q buffer: the next unit's Q is
// loaded once the current unit's last QK has completed, one tile ahead),
// 16-bit d = 64 and e4m3 d = 128 (two Q buffers each).
#ifndef SDPA_STAGES_D128
#define SDPA_STAGES_D128 6
#endif
#ifndef SDPA_STAGES_D64
#define SDPA_STAGES_D64 8
#endif
#ifndef SDPA_STAGES_D32
#define SDPA_STAGES_D32 16
#endif
#ifndef SDPA_STAGES_FP8
#define SDPA_STAGES_FP8 10
#endif

namespace sdpa {

enum Kind { KIND_BF16 = 0, KIND_FP16 = 1, KIND_E4M3 = 2 };

constexpr int kBlockM = 128;        // query rows per unit (= TMEM lanes)
constexpr int kBlockN = 128;        // keys per K/V tile
constexpr int kHalfN = 64;          // keys per softmax group
constexpr int kEpiWarp0 = 8;        // EPI: warps 8-11, TMEM lane quarters 0-3
constexpr uint32_t kTmemCols = 512;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // bounded waits: 1 s

// Device status word: [0] status (0 ok, 4 = device timeout, 5 = shared
// memory layout does not fit the allocation), [1] location.
__device__ unsigned int g_sdpa_status[2];

struct FwdParams {
    void* o;            // [B,Hq,Sq,D] view, 16-bit, D contiguous (strides below)
    float* lse;         // [B,Hq,Sq] contiguous, or null
    int B, Hq, Hkv, Sq, Sk;
    int group;          // Hq / Hkv
    int n_qtiles;       // ceil(Sq / 128)
    int items_per_head; // schedule items per (batch, head): causal ceil(nq/2), else nq
    int n_items;        // B * Hq * items_per_head
    int group_heads;    // (batch, head) pairs per schedule group
    int causal;
    float score_log2;   // multiplier from raw MMA score to log2 units
    float out_mul;      // multiplier on (sum_j p_j v_j) / l: the V descale for FP8, else 1
    long long o_sb, o_sh, o_ss;   // O's batch, head, row strides in elements (STRIDED)
    int causal_off;     // causal: query row i sees keys 0 .. i + causal_off (0, or Sk - Sq
                        // when the queries are aligned to the end of the keys)
    // PACK form: a unit holds the Sq rows of all pk_group query heads of one
    // K/V head (pk_rows = pk_group * Sq <= 128 TMEM lanes, row r = head
    // r / Sq, position r % Sq); Hq and group above then describe units
    // (Hq = Hkv, group = 1) and these the query heads.
    int pk_hq, pk_group, pk_rows, pk_qbytes;
};

template <int D, int KIND, int NS, int QB, bool EPI>
struct FwdCfg {
    static constexpr int kThreads = EPI ? 448 : 320;     // 14 or 10 warps
    static constexpr int kLoadWarp = EPI ? 12 : 8;
    static constexpr int kMmaWarp = EPI ? 13 : 9;
    static constexpr int kTmemUsers = 256 + 32 + (EPI ? 128 : 0);   // softmax, MMA, epilogue threads
    static constexpr int kElem = (KIND == KIND_E4M3) ? 1 : 2;
    static constexpr int kRowBytes = D * kElem;
    // swizzle rows of 128 bytes (64 when a whole row is 64 bytes: d = 32)
    static constexpr int kSwBytes = kRowBytes >= 128 ? 128 : kRowBytes;
    static constexpr uint32_t kSwLayout = kSwBytes == 128 ? 2u : 4u;   // descriptor swizzle field
    static constexpr int kSbo = 8 * kSwBytes;            // 8-row core-matrix group stride
    static constexpr int kElemsPerSw = kSwBytes / kElem; // elements in one swizzle row
    static constexpr int kSwBlocks = kRowBytes / kSwBytes;   // swizzle column blocks per row
    static constexpr int kSwBlockBytes = 128 * kSwBytes; // one column block of a 128-row tile
    static constexpr int kStepsPerBlock = kSwBytes / 32; // MMA K steps (32 bytes) per block
    static constexpr int kTileBytes = 128 * kRowBytes;
    static constexpr int kQkSteps = kRowBytes / 32;      // every MMA consumes 32 bytes of K
    static constexpr int kPvKeysPerStep = 32 / kElem;
    static constexpr int kPvStepsHalf = kHalfN / kPvKeysPerStep;
    static constexpr int kPWordsPer32 = 32 * kElem / 4;  // TMEM columns of P per 32 keys
    static constexpr float kRescaleThreshold = (KIND == KIND_E4M3) ? 0.0f : 8.0f;
    // log2 of the factor applied to p before it is rounded for the PV MMA:
    // 448 (the e4m3 maximum) for FP8, so that p in (0, 1] fills the format
    static constexpr float kPLog2 = (KIND == KIND_E4M3) ? 8.807354922057604f : 0.0f;
    // shared memory map (offsets from a 1024-byte aligned base)
    static constexpr int kSmemQ = 0;                      // QB Q tiles
    static constexpr int kSmemKV = QB * kTileBytes;
    static constexpr int kSmemStats = kSmemKV + NS * kTileBytes;   // [2 groups][128 rows][m, l] fp32
    static constexpr int kSmemBar = kSmemStats + 2 * 128 * 2 * 4;
    // barriers (Q ones: [QB buffers], QB <= 2)
    static constexpr int kBarQFull = 0;
    static constexpr int kBarQEmpty = 2;
    static constexpr int kBarKVFull = 4;                  // [NS]
    static constexpr int kBarKVEmpty = 4 + NS;            // [NS]
    static constexpr int kBarSFull = 4 + 2 * NS;          // [2 S buffers]
    static constexpr int kBarPFull = 6 + 2 * NS;          // [2 S buffers][2 groups]
    static constexpr int kBarODone = 10 + 2 * NS;         // [2 groups], once per tile
    static constexpr int kBarOFull = 12 + 2 * NS;         // once per unit
    static constexpr int kBarOEmpty = 13 + 2 * NS;        // once per unit
    static constexpr int kBarStatsFull = 14 + 2 * NS;     // softmax -> epilogue, once per unit
    static constexpr int kBarStatsEmpty = 15 + 2 * NS;    // epilogue -> softmax, once per unit
    static constexpr int kBarXchg1 = 16 + 2 * NS;         // no EPI: group 1 -> group 0, once per unit
    static constexpr int kBarXchg2 = 17 + 2 * NS;         // no EPI: group 0 -> group 1, once per unit
    static constexpr int kBarDrain = 18 + 2 * NS;
    static constexpr int kNumBars = 19 + 2 * NS;
    static constexpr int kSmemTmemSlot = kSmemBar + 8 * kNumBars;
    static constexpr int kSmemAbort = kSmemTmemSlot + 4;
    static constexpr int kSmemUsed = kSmemAbort + 4;
    // slack for the 1024-byte alignment of the tiles, as far as the budget
    // allows; the kernel checks at entry that its layout fits
    static constexpr int kSmemBytes = (kSmemUsed + 1024 <= 232448) ? kSmemUsed + 1024 : 232448;
    // TMEM columns
    static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 384;
    static_assert(kSwBytes == 128 || kSwBytes == 64, "rows of 64 bytes or whole 128-byte swizzle rows");
    static_assert(kRowBytes % kSwBytes == 0, "rows must fill whole swizzle rows");
    static_assert(kSmemUsed <= 232448, "shared memory budget");
    static_assert(kSmemBytes > 116 * 1024, "one CTA per SM (each allocates all of TMEM)");
    static_assert(D <= 128, "O tile must fit its 128 TMEM columns");
    static_assert(QB == 1 || QB == 2, "one or two Q buffers");
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

// Registers per thread of the softmax and epilogue warp groups (0: leave
// the launch budget of 65536 / 448 -> 128 each).  The producer and MMA warps
// keep the launch budget; the sum must stay within the launch allocation.
#ifndef SDPA_REGS_SOFTMAX
#define SDPA_REGS_SOFTMAX 152
#endif
#ifndef SDPA_REGS_EPILOGUE
#define SDPA_REGS_EPILOGUE 80
#endif
static_assert(SDPA_REGS_SOFTMAX == 0 || 8 * SDPA_REGS_SOFTMAX + 4 * SDPA_REGS_EPILOGUE + 2 * 128 <= 14 * 128,
              "register split exceeds the launch allocation");

#ifndef SDPA_EPI_SLEEP_NS
#define SDPA_EPI_SLEEP_NS 256
#endif
// As wait_bar, for warps off the critical path: sleeps between polls so that
// the waiting warp takes no issue slots from the softmax warps.
__device__ __forceinline__ bool wait_bar_sleep(uint32_t bar, uint32_t parity, uint32_t abort_addr,
                                               uint32_t where) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t k = 1;; ++k) {
        __nanosleep(SDPA_EPI_SLEEP_NS);
        if (mbar_try_wait(bar, parity)) return true;
        if ((k & 15u) == 0) {
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

// Pairs of one 32-column chunk (e = 0..15) whose exponentials are evaluated
// on the FMA pipe instead of the MUFU (SDPA_POLY_MASK).
__device__ __forceinline__ constexpr bool poly_pair(int e) {
    return ((SDPA_POLY_MASK >> (e & 7)) & 1) != 0;
}

// Maximum of 32 consecutive registers (3-input max, two chains).
__device__ __forceinline__ float chunk_max32(const float* s) {
    float a = s[0], b = s[1];
#pragma unroll
    for (int c = 2; c + 4 <= 30; c += 4) {
        a = fmax3(a, s[c], s[c + 1]);
        b = fmax3(b, s[c + 2], s[c + 3]);
    }
    a = fmax3(a, s[30], s[31]);
    return fmaxf(a, b);
}

// Element offset of row `row` of (batch, head) pair bh in O: contiguous
// [B,Hq,Sq,D], or the strided view.
template <int D, bool STRIDED>
__device__ __forceinline__ long long o_offset(const FwdParams& p, int bh, int row, int heads = 0) {
    if constexpr (STRIDED) {
        const int h_n = heads > 0 ? heads : p.Hq;
        const int b = bh / h_n;
        return (long long)b * p.o_sb + (long long)(bh - b * h_n) * p.o_sh + (long long)row * p.o_ss;
    } else {
        return ((long long)bh * p.Sq + row) * D;
    }
}

// PACK form: (batch, query head) index b * pk_hq + hq of lane r of the unit
// of (batch, K/V head) pair ubh.
__device__ __forceinline__ int packed_qhead(const FwdParams& p, int ubh, int r) {
    const int b = ubh / p.Hq;                       // p.Hq = K/V heads here
    return b * p.pk_hq + (ubh - b * p.Hq) * p.pk_group + r / p.Sq;
}

// Number of K/V tiles the query rows [row0, row0 + 128) need.
__device__ __forceinline__ int tiles_for(int row0, int Sq, int Sk, int causal, int off) {
    if (row0 >= Sq) return 0;
    const int kend = causal ? min(Sk, row0 + kBlockM + off) : Sk;
    return (kend + kBlockN - 1) / kBlockN;
}


// ---------------------------------------------------------------------------
// schedule: the units (128 query rows of one (batch, head)) a CTA processes
// ---------------------------------------------------------------------------
// Unit `sub` (0 or 1) of this CTA's k-th schedule item.  Item index
// blockIdx.x + k * gridDim.x; items come in groups of p.group_heads heads;
// within a group, item j of a head holds query tile nq-1-j (and, for causal
// attention, also tile j: long and short tiles of the same head paired).
__device__ __forceinline__ bool sched_unit(const FwdParams& p, int k, int sub, int& bh,
                                           int& qtile) {
    const long long item = (long long)blockIdx.x + (long long)k * gridDim.x;
    if (item >= p.n_items) return false;
    const int n_bh = p.B * p.Hq;
    const int per_group = p.group_heads * p.items_per_head;
    const int grp = (int)(item / per_group);
    const int within = (int)(item - (long long)grp * per_group);
    const int gsize = min(p.group_heads, n_bh - grp * p.group_heads);
    const int j = within / gsize;
    bh = grp * p.group_heads + within % gsize;
    const int hi = p.n_qtiles - 1 - j;
    if (sub == 0) {
        qtile = hi;
        return true;
    }
    if (!p.causal || j == hi) return false;
    qtile = j;
    return true;
}

struct UnitCursor {
    int k, sub;      // schedule position
    int bh, qtile;   // the unit
    int n;           // its K/V tiles
    int ku;          // units of this CTA before it
    bool valid;
};

__device__ __forceinline__ void unit_load(const FwdParams& p, UnitCursor& u) {
    u.valid = sched_unit(p, u.k, u.sub, u.bh, u.qtile);
    u.n = u.valid ? tiles_for(u.qtile * kBlockM, p.Sq, p.Sk, p.causal, p.causal_off) : 0;
}
__device__ __forceinline__ void unit_first(const FwdParams& p, UnitCursor& u) {
    u.k = 0;
    u.sub = 0;
    u.ku = 0;
    unit_load(p, u);
}
__device__ __forceinline__ void unit_next(const FwdParams& p, UnitCursor& u) {
    ++u.ku;
    if (u.sub == 0) {
        u.sub = 1;
        unit_load(p, u);
        if (u.valid) return;
    }
    ++u.k;
    u.sub = 0;
    unit_load(p, u);
}

// One position in the CTA's stream of K/V tiles.
struct TileCursor {
    UnitCursor u;
    int i;           // tile within the unit
    int g;           // tile within the stream
};
__device__ __forceinline__ void tile_first(const FwdParams& p, TileCursor& c) {
    unit_first(p, c.u);
    c.i = 0;
    c.g = 0;
}
__device__ __forceinline__ void tile_next(const FwdParams& p, TileCursor& c) {
    ++c.g;
    if (++c.i == c.u.n) {
        unit_next(p, c.u);
        c.i = 0;
    }
}

template <int D, int KIND, int NS, int QB, bool EPI, bool STRIDED, bool PACK>
__global__ void __launch_bounds__(FwdCfg<D, KIND, NS, QB, EPI>::kThreads, 1)
sdpa_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV,
                      const FwdParams p) {
    using C = FwdCfg<D, KIND, NS, QB, EPI>;
    static_assert(!PACK || (STRIDED && !EPI), "packed units use the strided form without epilogue warps");
    constexpr int kLoadWarp = C::kLoadWarp;
    constexpr int kMmaWarp = C::kMmaWarp;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    float* const stats = reinterpret_cast<float*>(smem_raw + (sbase - raw) + C::kSmemStats);
    // the aligned layout must end inside the allocation (uniform exit)
    if (sbase - raw + (uint32_t)C::kSmemUsed > (uint32_t)C::kSmemBytes) {
        if (threadIdx.x == 0 && atomicCAS(&g_sdpa_status[0], 0u, 5u) == 0u)
            atomicExch(&g_sdpa_status[1], sbase - raw);
        return;
    }

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    auto bar = [&](int i) -> uint32_t { return sbase + C::kSmemBar + 8u * (uint32_t)i; };
    const uint32_t abort_addr = sbase + C::kSmemAbort;
    const uint32_t slot_addr = sbase + C::kSmemTmemSlot;

    if (threadIdx.x == 0) {
        for (int j = 0; j < 2; ++j) {
            mbar_init(bar(C::kBarQFull + j), 1);
            mbar_init(bar(C::kBarQEmpty + j), 1);
            mbar_init(bar(C::kBarSFull + j), 1);
            mbar_init(bar(C::kBarODone + j), 1);
            mbar_init(bar(C::kBarPFull + 2 * j), kBlockM);
            mbar_init(bar(C::kBarPFull + 2 * j + 1), kBlockM);
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(bar(C::kBarKVFull + s), 1);
            mbar_init(bar(C::kBarKVEmpty + s), 1);
        }
        mbar_init(bar(C::kBarOFull), 1);
        mbar_init(bar(C::kBarOEmpty), EPI ? kBlockM : 2 * kBlockM);
        mbar_init(bar(C::kBarXchg1), kBlockM);
        mbar_init(bar(C::kBarXchg2), kBlockM);
        mbar_init(bar(C::kBarStatsFull), 2 * kBlockM);
        mbar_init(bar(C::kBarStatsEmpty), kBlockM);
        mbar_init(bar(C::kBarDrain), 1);
        st_shared_u32(abort_addr, 0u);
        fence_barrier_init();
    }
    if constexpr (PACK) {
        // rows pk_rows..127 of every Q buffer stay zero: the packed Q box
        // never writes them, and their scores are then finite
        const int dead = (kBlockM - p.pk_rows) * C::kSwBytes;   // bytes per column block
        for (int qb = 0; qb < QB; ++qb)
            for (int kb = 0; kb < C::kSwBlocks; ++kb) {
                uint8_t* blk = smem_raw + (sbase - raw) + C::kSmemQ + qb * C::kTileBytes +
                               kb * C::kSwBlockBytes + p.pk_rows * C::kSwBytes;
                for (int i = threadIdx.x * 16; i < dead; i += C::kThreads * 16)
                    *reinterpret_cast<uint4*>(blk + i) = make_uint4(0u, 0u, 0u, 0u);
            }
        fence_proxy_async_smem();
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
    const uint32_t sQ = sbase + C::kSmemQ;
    const uint32_t sKV = sbase + C::kSmemKV;

    if (warp == kLoadWarp) {
        // ================= TMA producer =================================
        if (lane == 0) {
            bool ok = true;
            int t = 0;        // K/V tiles issued
            int q_last = -1;  // last unit whose Q was issued
            TileCursor kc, vc;
            tile_first(p, kc);
            tile_first(p, vc);
            // Issue the K (or V) tile of stream position c into the ring; a
            // unit's Q goes in right before its first K tile.
            auto emit = [&](const TileCursor& c, bool is_v) -> bool {
                if (!is_v && c.i == 0) {
                    const int qb = c.u.ku % QB, qm = c.u.ku / QB;
                    if (qm >= 1 &&
                        !wait_bar(bar(C::kBarQEmpty + qb), (uint32_t)(qm - 1) & 1u,
                                  abort_addr, 0x11000u | (uint32_t)c.u.ku))
                        return false;
                    mbar_arrive_expect_tx(bar(C::kBarQFull + qb), PACK ? p.pk_qbytes : C::kTileBytes);
                    for (int kb = 0; kb < C::kSwBlocks; ++kb) {
                        const uint32_t dst = sQ + qb * C::kTileBytes + kb * C::kSwBlockBytes;
                        if constexpr (PACK) {
                            // box: all Sq rows of the group's pk_group query heads
                            const int qbat = c.u.bh / p.Hq;
                            tma_load_4d(dst, &tmQ, bar(C::kBarQFull + qb), kb * C::kElemsPerSw, 0,
                                        (c.u.bh - qbat * p.Hq) * p.pk_group, qbat);
                        } else if constexpr (STRIDED) {
                            const int qbat = c.u.bh / p.Hq;
                            tma_load_4d(dst, &tmQ, bar(C::kBarQFull + qb), kb * C::kElemsPerSw,
                                        c.u.qtile * kBlockM, c.u.bh - qbat * p.Hq, qbat);
                        } else {
                            tma_load_3d(dst, &tmQ, bar(C::kBarQFull + qb), kb * C::kElemsPerSw,
                                        c.u.qtile * kBlockM, c.u.bh);
                        }
                    }
                    q_last = c.u.ku;
                }
                const int slot = t % NS;
                if (!wait_bar(bar(C::kBarKVEmpty + slot), ((uint32_t)(t / NS) & 1u) ^ 1u, abort_addr,
                              0x10000u | (uint32_t)t))
                    return false;
                const int b = c.u.bh / p.Hq;
                const int kvh = (c.u.bh - b * p.Hq) / p.group;   // K/V head of the group
                const uint32_t fb = bar(C::kBarKVFull + slot);
                mbar_arrive_expect_tx(fb, C::kTileBytes);
                for (int kb = 0; kb < C::kSwBlocks; ++kb) {
                    if constexpr (STRIDED)
                        tma_load_4d(sKV + slot * C::kTileBytes + kb * C::kSwBlockBytes,
                                    is_v ? &tmV : &tmK, fb, kb * C::kElemsPerSw, c.i * kBlockN, kvh, b);
                    else
                        tma_load_3d(sKV + slot * C::kTileBytes + kb * C::kSwBlockBytes,
                                    is_v ? &tmV : &tmK, fb, kb * C::kElemsPerSw, c.i * kBlockN,
                                    b * p.Hkv + kvh);
                }
                ++t;
                return true;
            };
            // MMA consumption order: K(0), K(1), then V(g), K(g+2), ..., then
            // the last V tiles
            for (int j = 0; j < 2 && ok && kc.u.valid; ++j) {
                ok = emit(kc, false);
                tile_next(p, kc);
            }
            while (ok && vc.u.valid) {
                ok = emit(vc, true);
                tile_next(p, vc);
                if (ok && kc.u.valid) {
                    ok = emit(kc, false);
                    tile_next(p, kc);
                }
            }
            if (!ok) {
                // let the copies already issued land before the CTA exits
                for (int u = max(0, t - NS); u < t; ++u) {
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(bar(C::kBarKVFull + u % NS), (uint32_t)(u / NS) & 1u) &&
                           global_timer_ns() - t0 < 100000000ull) {
                    }
                }
                for (int u = max(0, q_last - QB + 1); u <= q_last; ++u) {
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(bar(C::kBarQFull + u % QB), (uint32_t)(u / QB) & 1u) &&
                           global_timer_ns() - t0 < 100000000ull) {
                    }
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ================= MMA issuer ===================================
        // The whole warp runs the loop (descriptors stay warp-uniform); one
        // elected lane issues the MMAs and commits.
        const bool leader = elect_one();
        constexpr uint32_t fmt = (KIND == KIND_BF16) ? 1u : 0u;
        constexpr uint32_t idesc_qk = make_idesc(fmt, false, kBlockM, kBlockN);
        constexpr uint32_t idesc_pv = make_idesc(fmt, true, kBlockM, D);
        const uint64_t desc_q = make_smem_desc(sQ, 16, C::kSbo, C::kSwLayout);
        const uint64_t desc_k = make_smem_desc(sKV, 16, C::kSbo, C::kSwLayout);
        const uint64_t desc_v = make_smem_desc(sKV, C::kSwBlockBytes, C::kSbo, C::kSwLayout);
        bool ok = true;
        int t = 0;   // K/V tiles consumed

        auto wait_all = [&](uint32_t b_, uint32_t par, uint32_t where) {
            const bool r_ = wait_bar(b_, par, abort_addr, where);
            return __all_sync(0xffffffffu, r_);
        };
        auto commit = [&](uint32_t b_) {
            if (leader) mma_commit(b_);
            __syncwarp();
        };
        auto next_kv = [&](uint32_t where) -> int {
            const int slot = t % NS;
            ok = wait_all(bar(C::kBarKVFull + slot), (uint32_t)(t / NS) & 1u, where | (uint32_t)(t & 0xfff));
            return slot;
        };
        // S_buf = Q_qb K^T for the K tile in `slot`
        auto issue_qk = [&](int buf, int qb, int slot) {
            const uint32_t d_tmem = tmem + (buf ? C::kColS1 : C::kColS0);
            const uint64_t dq = desc_q + (uint64_t)((qb * C::kTileBytes) >> 4);
            const uint64_t dk = desc_k + (uint64_t)((slot * C::kTileBytes) >> 4);
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < C::kQkSteps; ++kk) {
                    const uint64_t off = (uint64_t)(((kk / C::kStepsPerBlock) * C::kSwBlockBytes +
                                                     (kk % C::kStepsPerBlock) * 32) >> 4);
                    if constexpr (KIND == KIND_E4M3)
                        mma_f8_ss(d_tmem, dq + off, dk + off, idesc_qk, kk > 0);
                    else
                        mma_f16_ss(d_tmem, dq + off, dk + off, idesc_qk, kk > 0);
                }
            }
            __syncwarp();
        };
        // O_h (+)= P_h V[keys of half h]; P_h is in TMEM over group h's
        // columns of S_buf
        auto issue_pv = [&](int h, int buf, int slot, bool acc) {
            const uint32_t d_tmem = tmem + (h ? C::kColO1 : C::kColO0);
            const uint32_t a_tmem = tmem + (buf ? C::kColS1 : C::kColS0) + h * kHalfN;
            const uint64_t dv = desc_v + (uint64_t)((slot * C::kTileBytes + h * kHalfN * C::kSwBytes) >> 4);
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < C::kPvStepsHalf; ++kk) {
                    const uint64_t off = (uint64_t)((kk * C::kPvKeysPerStep * C::kSwBytes) >> 4);
                    const uint32_t accum = (acc || kk > 0) ? 1u : 0u;
                    if constexpr (KIND == KIND_E4M3)
                        mma_f8_ts(d_tmem, a_tmem + kk * 8, dv + off, idesc_pv, accum);
                    else
                        mma_f16_ts(d_tmem, a_tmem + kk * 8, dv + off, idesc_pv, accum);
                }
            }
            __syncwarp();
        };

        TileCursor kc, vc;
        tile_first(p, kc);
        tile_first(p, vc);
        // S_(g&1) = Q K^T for stream tile kc (g = kc.g)
        auto qk_tile = [&]() -> bool {
            const int qb = kc.u.ku % QB;
            if (kc.i == 0 &&
                !wait_all(bar(C::kBarQFull + qb), (uint32_t)(kc.u.ku / QB) & 1u, 0x20000u | (uint32_t)kc.u.ku))
                return false;
            const int slot = next_kv(0x21000u);
            if (!ok) return false;
            issue_qk(kc.g & 1, qb, slot);
            commit(bar(C::kBarSFull + (kc.g & 1)));
            commit(bar(C::kBarKVEmpty + slot));
            if (kc.i == kc.u.n - 1) commit(bar(C::kBarQEmpty + qb));   // Q_qb free
            ++t;
            tile_next(p, kc);
            return true;
        };

        for (int j = 0; j < 2 && ok && kc.u.valid; ++j) ok = qk_tile();
        while (ok && vc.u.valid) {
            const int buf = vc.g & 1;
            const int slotV = next_kv(0x22000u);
            if (!ok) break;
            // the first product of a unit overwrites O: the previous unit's
            // epilogue must have read it
            if (vc.i == 0 && vc.u.ku > 0) {
                ok = wait_all(bar(C::kBarOEmpty), (uint32_t)(vc.u.ku - 1) & 1u, 0x25000u | (uint32_t)vc.u.ku);
                if (!ok) break;
            }
            for (int h = 0; h < 2 && ok; ++h) {
                ok = wait_all(bar(C::kBarPFull + 2 * buf + h), (uint32_t)(vc.g >> 1) & 1u,
                              0x23000u | (h << 11) | (uint32_t)(vc.g & 0x7ff));
                if (!ok) break;
                tc_fence_after();
                issue_pv(h, buf, slotV, vc.i > 0);
                commit(bar(C::kBarODone + h));
            }
            if (!ok) break;
            if (vc.i == vc.u.n - 1) commit(bar(C::kBarOFull));
            commit(bar(C::kBarKVEmpty + slotV));
            ++t;
            tile_next(p, vc);
            if (kc.u.valid) ok = qk_tile();
        }
        if (!ok) {
            // make sure no MMA is still writing tensor memory at exit
            commit(bar(C::kBarDrain));
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(bar(C::kBarDrain), 0) && global_timer_ns() - t0 < 100000000ull) {
            }
        }
        // teardown: the softmax and epilogue warps are done with TMEM
        named_bar_sync(1, C::kTmemUsers);
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    } else if (warp < 8) {
        // ================= softmax groups (warps 0-7) ====================
        if constexpr (EPI && SDPA_REGS_SOFTMAX > 0) regs_inc<(SDPA_REGS_SOFTMAX > 0 ? SDPA_REGS_SOFTMAX : 128)>();
        const int h = warp >> 2;                 // key half of every tile
        const int quarter = warp & 3;            // TMEM lane quarter of this warp
        const int r = (int)(threadIdx.x & 127);  // row within the unit
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint32_t tO = tmem + lane_base + (h ? C::kColO1 : C::kColO0);
        const float sl = p.score_log2;
        const uint64_t sl2 = f2_pack(sl, sl);
        bool ok = true;

        // -m [+ log2 of the P scale] as a pair; a row whose keys of this half
        // have all been masked so far keeps m = -inf and gets p = 0
        auto neg_m_of = [&](float m) -> uint64_t {
            const float nm = (m == -INFINITY) ? 0.0f : C::kPLog2 - m;
            return f2_pack(nm, nm);
        };
        // Weights p = 2^(s*sl + nm) of 32 scores: pairs on the MUFU, or on the
        // FMA pipe for the pairs SDPA_POLY_MASK selects; P rounded for the PV
        // product and stored into chunk c of this group's columns of S.
        // Returns the fp32 sum of the weights as a pair.
        auto exp_chunk = [&](const float* sc, uint64_t sl2_, uint64_t nm2, uint32_t tS_,
                             int c) -> uint64_t {
            uint64_t sum2[2] = {0ull, 0ull};
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const uint64_t x2 = f2_fma(f2_pack(sc[2 * e], sc[2 * e + 1]), sl2_, nm2);
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
            if constexpr (KIND == KIND_E4M3)
                tmem_st8(tS_ + C::kPWordsPer32 * c, pk);
            else
                tmem_st16(tS_ + C::kPWordsPer32 * c, pk);
            return f2_add(sum2[0], sum2[1]);
        };

        UnitCursor u;
        unit_first(p, u);
        int g = 0;   // stream tile
        while (ok && u.valid) {
            const int m0 = u.qtile * kBlockM;
            // a packed unit's lane r is position r % Sq of query head r / Sq
            const int row = PACK ? r % p.Sq : m0 + r;
            const int n = u.n;
            float m_run = -INFINITY;   // running max of this half's scaled scores (log2 units)
            float l_run = 0.0f;        // running sum of 2^(s*sl - m_run + kPLog2)

            for (int i = 0; i < n && ok; ++i, ++g) {
                const int buf = g & 1;
                ok = wait_bar(bar(C::kBarSFull + buf), (uint32_t)(g >> 1) & 1u, abort_addr,
                              0x30000u | (h << 12) | (uint32_t)(g & 0xfff));
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();
                const uint32_t tS = tmem + lane_base + (buf ? C::kColS1 : C::kColS0) + h * kHalfN;

                float s[kHalfN];
                // chunk 0 (keys 0-31 of this half); chunk 1 is loaded while the
                // exponentials of chunk 0 run
                tmem_ld32(tS + 0, *reinterpret_cast<float(*)[32]>(&s[0]));
                tmem_wait_ld();
                reg_fence32(&s[0]);
                tmem_ld32(tS + 32, *reinterpret_cast<float(*)[32]>(&s[32]));

                // mask: keys past Sk, and (causal) keys after the row's last
                // visible key row + causal_off
                const int key0 = i * kBlockN + h * kHalfN;
                const bool edge = (key0 + kHalfN > p.Sk) ||
                                  (p.causal && key0 + kHalfN - 1 > m0 + p.causal_off);
                int lim = kHalfN;
                if (edge) {
                    lim = p.Sk - key0;
                    if (p.causal) lim = min(lim, row + p.causal_off - key0 + 1);
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        if (c >= lim) s[c] = -INFINITY;
                }
                const float cmax0 = chunk_max32(&s[0]) * sl;

                // Fast path: while a chunk's maximum stays within the rescale
                // threshold of the running max m_run, its weights are computed
                // against m_run at once.  Otherwise (always on the first tile)
                // the tile takes the full path: maximum of both chunks, new
                // m_run, l and O rescaled, chunk 0 recomputed.
                const bool fast0 = !__any_sync(0xffffffffu, cmax0 > m_run + C::kRescaleThreshold);
                uint64_t sum0 = 0ull, sum1 = 0ull;
                if (fast0) sum0 = exp_chunk(&s[0], sl2, neg_m_of(m_run), tS, 0);

                tmem_wait_ld();
                reg_fence32(&s[32]);
                if (edge) {
#pragma unroll
                    for (int c = 32; c < kHalfN; ++c)
                        if (c >= lim) s[c] = -INFINITY;
                }
                const float cmax1 = chunk_max32(&s[32]) * sl;
                if (!fast0 || __any_sync(0xffffffffu, cmax1 > m_run + C::kRescaleThreshold)) {
                    const float tile_max = fmaxf(cmax0, cmax1);
                    float alpha = 1.0f;
                    if (tile_max > m_run + C::kRescaleThreshold) {
                        alpha = ex2_approx(m_run - tile_max);   // 0 on the first live tile
                        m_run = tile_max;
                    }
                    l_run *= alpha;
                    // O_h takes the same factor before P_h V is added; its last
                    // update (stream tile g-1, same unit since i > 0) must have
                    // completed.  o_done[h] completes once per tile; this
                    // parity wait is exact because the barrier is within one
                    // phase of tile g-1: the S(g) commit covered tile g-2's
                    // product and tile g's cannot exist yet.
                    if (i > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
                        ok = wait_bar(bar(C::kBarODone + h), (uint32_t)(g - 1) & 1u, abort_addr,
                                      0x31000u | (h << 12) | (uint32_t)(g & 0xfff));
                        ok = __all_sync(0xffffffffu, ok);
                        if (!ok) break;
                        tc_fence_after();
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
                    sum0 = exp_chunk(&s[0], sl2, neg_m_of(m_run), tS, 0);
                }
                sum1 = exp_chunk(&s[32], sl2, neg_m_of(m_run), tS, 1);
                {
                    float a0, a1, b0, b1;
                    f2_unpack(sum0, a0, a1);
                    f2_unpack(sum1, b0, b1);
                    l_run += (a0 + a1) + (b0 + b1);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(C::kBarPFull + 2 * buf + h));
            }
            if (!ok) break;

            if constexpr (EPI) {
                // ---- end of the unit: hand (m_h, l_h) of every row to the
                // epilogue warps and go on with the next unit ----
                if (u.ku > 0) {
                    ok = wait_bar(bar(C::kBarStatsEmpty), (uint32_t)(u.ku - 1) & 1u, abort_addr,
                                  0x40000u | (h << 12) | (uint32_t)(u.ku & 0xfff));
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                }
                stats[(h * kBlockM + r) * 2] = m_run;
                stats[(h * kBlockM + r) * 2 + 1] = l_run;
                mbar_arrive(bar(C::kBarStatsFull));
            } else {
                // ---- epilogue of the unit: merge the halves, O -> 16-bit,
                // LSE.  Group 1 hands (m_1, l_1) to group 0 through `stats`;
                // group 0 computes the merge factors c_0, c_1 and hands them
                // back; each group writes half of O's columns. ----
                const uint32_t xpar = (uint32_t)u.ku & 1u;
                float c0 = 0.f, c1 = 0.f;
                if (h == 1) {
                    stats[2 * r] = m_run;
                    stats[2 * r + 1] = l_run;
                    mbar_arrive(bar(C::kBarXchg1));
                    ok = wait_bar(bar(C::kBarXchg2), xpar, abort_addr, 0x43000u | (uint32_t)(u.ku & 0xfff));
                    ok = __all_sync(0xffffffffu, ok);
                    c0 = stats[2 * r];
                    c1 = stats[2 * r + 1];
                } else {
                    ok = wait_bar(bar(C::kBarXchg1), xpar, abort_addr, 0x44000u | (uint32_t)(u.ku & 0xfff));
                    ok = __all_sync(0xffffffffu, ok);
                    const float m_1 = stats[2 * r], l_1 = stats[2 * r + 1];
                    const float m = fmaxf(m_run, m_1);
                    const float a0 = (m_run == -INFINITY) ? 0.0f : ex2_approx(m_run - m);
                    const float a1 = (m_1 == -INFINITY) ? 0.0f : ex2_approx(m_1 - m);
                    const float l = l_run * a0 + l_1 * a1;
                    c0 = a0 * (p.out_mul / l);
                    c1 = a1 * (p.out_mul / l);
                    stats[2 * r] = c0;
                    stats[2 * r + 1] = c1;
                    mbar_arrive(bar(C::kBarXchg2));
                    if constexpr (PACK) {
                        if (ok && p.lse != nullptr && r < p.pk_rows)
                            p.lse[(size_t)packed_qhead(p, u.bh, r) * p.Sq + row] =
                                (m + __log2f(l) - C::kPLog2) * kLn2;
                    } else {
                        if (ok && p.lse != nullptr && row < p.Sq)
                            p.lse[(size_t)u.bh * p.Sq + row] = (m + __log2f(l) - C::kPLog2) * kLn2;
                    }
                }
                if (ok) {
                    ok = wait_bar(bar(C::kBarOFull), xpar, abort_addr, 0x45000u | (uint32_t)(u.ku & 0xfff));
                    ok = __all_sync(0xffffffffu, ok);
                }
                if (!ok) break;
                tc_fence_after();
                const bool live = PACK ? r < p.pk_rows : row < p.Sq;
                uint16_t* obase = reinterpret_cast<uint16_t*>(p.o);
                if constexpr (PACK)
                    obase += o_offset<D, true>(p, live ? packed_qhead(p, u.bh, r) : 0, live ? row : 0,
                                               p.pk_hq);
                else
                    obase += o_offset<D, STRIDED>(p, u.bh, live ? row : 0);
                const uint32_t tO0 = tmem + lane_base + C::kColO0, tO1 = tmem + lane_base + C::kColO1;
                // group h writes output columns [h * D / 2, (h + 1) * D / 2)
                if constexpr (D == 32) {
                    float x[16], y[16];
                    tmem_ld16(tO0 + 16 * h, x);
                    tmem_ld16(tO1 + 16 * h, y);
                    tmem_wait_ld();
                    reg_fence16(x);
                    reg_fence16(y);
                    uint32_t w4[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float v0 = x[2 * e] * c0 + y[2 * e] * c1;
                        const float v1 = x[2 * e + 1] * c0 + y[2 * e + 1] * c1;
                        w4[e] = (KIND == KIND_FP16) ? pack_f16x2(v0, v1) : pack_bf16x2(v0, v1);
                    }
                    if (live) {
                        uint4* dst = reinterpret_cast<uint4*>(obase + 16 * h);
                        dst[0] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                        dst[1] = make_uint4(w4[4], w4[5], w4[6], w4[7]);
                    }
                }
#pragma unroll 1
                for (int c = h * (D / 64); c < (h + 1) * (D / 64); ++c) {
                    float x[32], y[32];
                    tmem_ld32(tO0 + 32 * c, x);
                    tmem_ld32(tO1 + 32 * c, y);
                    tmem_wait_ld();
                    reg_fence32(x);
                    reg_fence32(y);
                    uint32_t w4[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float v0 = x[2 * e] * c0 + y[2 * e] * c1;
                        const float v1 = x[2 * e + 1] * c0 + y[2 * e + 1] * c1;
                        w4[e] = (KIND == KIND_FP16) ? pack_f16x2(v0, v1) : pack_bf16x2(v0, v1);
                    }
                    if (live) {
                        uint4* dst = reinterpret_cast<uint4*>(obase + 32 * c);
#pragma unroll
                        for (int v4 = 0; v4 < 4; ++v4)
                            dst[v4] = make_uint4(w4[4 * v4], w4[4 * v4 + 1], w4[4 * v4 + 2], w4[4 * v4 + 3]);
                    }
                }
                // O may now be overwritten by the next unit's first product
                tc_fence_before();
                mbar_arrive(bar(C::kBarOEmpty));
            }
            unit_next(p, u);
        }
        tc_fence_before();
        named_bar_sync(1, C::kTmemUsers);
    } else if (EPI && warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
        // ================= epilogue (warps 8-11) =========================
        if constexpr (EPI && SDPA_REGS_SOFTMAX > 0) regs_dec<(SDPA_REGS_SOFTMAX > 0 ? SDPA_REGS_EPILOGUE : 128)>();
        // Per unit: O = (2^(m_0-m) O_0 + 2^(m_1-m) O_1) / l with l the
        // halves' sums on the common max m; O is read from this warp's TMEM
        // lane quarter, rounded to 16 bits and stored, then LSE.
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;       // row within the unit = TMEM lane
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint32_t tO0 = tmem + lane_base + C::kColO0, tO1 = tmem + lane_base + C::kColO1;
        bool ok = true;
        UnitCursor u;
        unit_first(p, u);
        while (ok && u.valid) {
            const uint32_t par = (uint32_t)u.ku & 1u;
            ok = wait_bar_sleep(bar(C::kBarStatsFull), par, abort_addr, 0x41000u | (uint32_t)(u.ku & 0xfff));
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            const float m_0 = stats[r * 2], l_0 = stats[r * 2 + 1];
            const float m_1 = stats[(kBlockM + r) * 2], l_1 = stats[(kBlockM + r) * 2 + 1];
            mbar_arrive(bar(C::kBarStatsEmpty));
            const float m = fmaxf(m_0, m_1);
            const float a0 = (m_0 == -INFINITY) ? 0.0f : ex2_approx(m_0 - m);
            const float a1 = (m_1 == -INFINITY) ? 0.0f : ex2_approx(m_1 - m);
            const float l = l_0 * a0 + l_1 * a1;
            const float c0 = a0 * (p.out_mul / l);
            const float c1 = a1 * (p.out_mul / l);
            const int row = u.qtile * kBlockM + r;
            const bool live = row < p.Sq;
            if (live && p.lse != nullptr)
                p.lse[(size_t)u.bh * p.Sq + row] = (m + __log2f(l) - C::kPLog2) * kLn2;
            ok = wait_bar_sleep(bar(C::kBarOFull), par, abort_addr, 0x42000u | (uint32_t)(u.ku & 0xfff));
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            uint16_t* obase = reinterpret_cast<uint16_t*>(p.o) + o_offset<D, STRIDED>(p, u.bh, live ? row : 0);
#pragma unroll 1
            for (int c = 0; c < D / 16; ++c) {
                float x[16], y[16];
                tmem_ld16(tO0 + 16 * c, x);
                tmem_ld16(tO1 + 16 * c, y);
                tmem_wait_ld();
                reg_fence16(x);
                reg_fence16(y);
                if (c == D / 16 - 1) {
                    // O is read: the next unit's first product may overwrite it
                    tc_fence_before();
                    mbar_arrive(bar(C::kBarOEmpty));
                }
                uint32_t w4[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float v0 = x[2 * e] * c0 + y[2 * e] * c1;
                    const float v1 = x[2 * e + 1] * c0 + y[2 * e + 1] * c1;
                    w4[e] = (KIND == KIND_FP16) ? pack_f16x2(v0, v1) : pack_bf16x2(v0, v1);
                }
                if (live) {
                    uint4* dst = reinterpret_cast<uint4*>(obase + 16 * c);
                    dst[0] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    dst[1] = make_uint4(w4[4], w4[5], w4[6], w4[7]);
                }
            }
            unit_next(p, u);
        }
        tc_fence_before();
        named_bar_sync(1, C::kTmemUsers);
    }
}


}  // namespace sdpa
