// sdpa_fwd2q_sm100.cuh -- fused scaled-dot-product attention forward for
// sm_100a (B200) with two 128-row query tiles per CTA sharing every K/V tile.
//
// Method (article "Self-attention, CUDA kernels and FlashAttention", section
// 3): Q, K, V are cut into on-chip tiles, the scores of a tile become weights
// through a softmax that keeps a running row maximum and row sum, the partial
// output is rescaled when the maximum moves, and only O and the per-row
// normaliser (LSE) reach global memory.  Formula and steps: codelab "JAX on
// GPU, Lab 5: attention on GPU", section 1; causal mask section 7; MHA / GQA
// / MQA section 9; FP8 E4M3 forward section 10.
//
// A work unit is 256 query rows of one (batch, query head): query tiles 2m
// ("stage 0") and 2m+1 ("stage 1").  Both stages read the same K/V tiles, so
// each K/V byte brought into shared memory feeds 256 rows of products, half
// the L2->SMEM traffic per flop of a one-tile CTA.  Each stage has its own
// score tile S_s and output accumulator O_s in tensor memory and its own
// softmax warp group, so the two softmax groups run out of phase: while one
// computes exponentials, the tensor pipe works on the other stage's products.
//
// Warp roles (512 threads):
//   warps 0-3    softmax, stage 0: thread = query row = TMEM lane
//   warps 4-7    softmax, stage 1
//   warps 8-11   epilogue: O_s / l -> 16-bit rows, LSE, once per unit and
//                stage, off the softmax groups' path
//   warp 12      TMA producer: Q tiles per unit, K/V tiles in stream order
//                K_0 V_0 K_1 V_1 ... (the ring spans unit boundaries)
//   warp 13      MMA issuer (one elected lane) and TMEM owner; a single
//                in-order issuer keeps each stage's PV + QK block contiguous
//                in the tensor pipe (two issuers, one per stage, interleave
//                the blocks and lengthen both stages' chains)
//   warps 14-15  idle (they complete the fourth warp group's register split)
// The split form (768 threads) doubles the softmax warps: warps 0-7 stage 0,
// 8-15 stage 1, two warps per TMEM lane quarter, each over 64 of a row's 128
// scores (the halves exchange tile maxima through shared memory and keep
// their own row sums); the epilogue, producer and MMA warps follow (16-19,
// 20, 21).  It halves each softmax warp's serial work, at the price of a
// 32-score register budget (80 registers a thread at launch), so its scores
// are read from TMEM twice (max, then weights).
// Tensor memory (128 lanes x 512 columns, fp32):
//   [0,128) S_0   [128,256) S_1   [256,256+d) O_0   [256+d,256+2d) O_1
// The weights P_s (16-bit pairs, or e4m3 quads, per column) overwrite the
// first columns of S_s once the softmax has read the scores; they are the
// TMEM A operand of O_s += P_s V.  Per stage the chain is
//   S_s = Q_s K_j^T -> softmax_s(j) -> O_s += P_s V_j -> S_s = Q_s K_(j+1)^T
// and the MMA warp interleaves the stages: PV_0(j-1) QK_0(j) PV_1(j-1)
// QK_1(j).  tcgen05 MMAs of one thread complete in issue order, so the QK
// that overwrites S_s cannot overtake the PV that reads P_s, and S_s(j)
// complete implies O_s += P_s(j-1) V complete (the softmax may then rescale
// O_s in place before it releases P_s(j)).
// Causal units: query tile 2m needs one K/V tile fewer than tile 2m+1; stage
// 0 simply has no product on that tile.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include "sm100_ptx.cuh"

// Pairs e (0..15) of a 32-column chunk whose exponentials are evaluated on
// the FMA pipe (exp2_poly_x2) instead of the MUFU: bit (e & 7) of the mask,
// for 16-bit inputs and for e4m3.  None measured fastest in the forms that
// are launched (the split e4m3 form was fastest with 0x11 or 0x01).
#ifndef SDPA2_POLY_MASK
#define SDPA2_POLY_MASK 0x00
#endif
#ifndef SDPA2_POLY_MASK_FP8
#define SDPA2_POLY_MASK_FP8 0x00
#endif
// Register budgets (setmaxnreg) of the softmax, epilogue and producer/MMA
// warp groups: 8 * S + 4 * E + 4 * W <= 16 * 128 (the launch allocation; per
// SM sub-partition 2 * S + E + W <= 512).
#ifndef SDPA2_REGS_SOFTMAX
#define SDPA2_REGS_SOFTMAX 184
#endif
#ifndef SDPA2_REGS_EPILOGUE
#define SDPA2_REGS_EPILOGUE 56
#endif
#ifndef SDPA2_REGS_OTHER
#define SDPA2_REGS_OTHER 88
#endif
static_assert(8 * SDPA2_REGS_SOFTMAX + 4 * SDPA2_REGS_EPILOGUE + 4 * SDPA2_REGS_OTHER <= 16 * 128,
              "register split exceeds the launch allocation");
// e4m3 inputs (one-warp form): the softmax holds packed e4m3 words besides
// the fp32 scores and takes more, the other groups less
#ifndef SDPA2_REGS_SOFTMAX_FP8
#define SDPA2_REGS_SOFTMAX_FP8 200
#endif
#ifndef SDPA2_REGS_EPILOGUE_FP8
#define SDPA2_REGS_EPILOGUE_FP8 40
#endif
#ifndef SDPA2_REGS_OTHER_FP8
#define SDPA2_REGS_OTHER_FP8 72
#endif
static_assert(8 * SDPA2_REGS_SOFTMAX_FP8 + 4 * SDPA2_REGS_EPILOGUE_FP8 + 4 * SDPA2_REGS_OTHER_FP8 <= 16 * 128,
              "register split exceeds the launch allocation");
// The split form (two softmax warps per lane quarter and stage, 768 threads)
// is launched with 80 registers a thread (65536 / 768, rounded down to a
// multiple of 8); setmaxnreg moves registers only within that allocation, so
// per SM sub-partition (4 softmax, 1 epilogue, 1 other warp) 4 S + E + W <= 6 * 80.
#ifndef SDPA2S_REGS_SOFTMAX
#define SDPA2S_REGS_SOFTMAX 88
#endif
#ifndef SDPA2S_REGS_EPILOGUE
#define SDPA2S_REGS_EPILOGUE 48
#endif
#ifndef SDPA2S_REGS_OTHER
#define SDPA2S_REGS_OTHER 80
#endif
static_assert(4 * SDPA2S_REGS_SOFTMAX + SDPA2S_REGS_EPILOGUE + SDPA2S_REGS_OTHER <= 6 * 80,
              "split register budget exceeds the launch allocation");
// 1: the MMA warp commits a step's K/V slot releases at the next step's top
#ifndef SDPA2_DEFER_RELEASE
#define SDPA2_DEFER_RELEASE 1
#endif
// 1: split form, edge tiles: a 32-key chunk that every row of a warp has
// masked gets zero weights without exponentials
#ifndef SDPA2_SKIP_MASKED
#define SDPA2_SKIP_MASKED 1
#endif
// 1: the one-warp form computes the weights before the tile max (see the softmax)
#ifndef SDPA2_WEIGHTS_FIRST
#define SDPA2_WEIGHTS_FIRST 1
#endif
#ifndef SDPA2_EPI_SLEEP_NS
#define SDPA2_EPI_SLEEP_NS 128
#endif

namespace sdpa {
namespace fwd2 {

enum Kind2 { K2_BF16 = 0, K2_FP16 = 1, K2_E4M3 = 2 };

constexpr int kRows = 128;            // query rows per stage (= TMEM lanes)
constexpr int kKeys = 128;            // keys per K/V tile
constexpr uint32_t kTmemCols = 512;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // bounded waits: 1 s

// Device status word of this kernel's module: [0] status (0 ok, 4 = a wait
// timed out, 5 = the shared-memory layout does not fit), [1] location code.
__device__ unsigned int g_status[2];

// n / d for 0 <= n < 2^31 by one multiply and a shift: m = ceil(2^(31+l) / d)
// with l = ceil(log2 d) satisfies 2^(31+l) <= m d <= 2^(31+l) + 2^l, which
// makes floor(m n / 2^(31+l)) = floor(n / d) for every 31-bit n (Granlund and
// Montgomery, "Division by invariant integers using multiplication", 1994,
// Theorem 4.2).  The schedule decodes every unit with a few of these in the
// MMA issuer's thread, where a 64-bit division cost over a thousand cycles.
struct FastDiv {
    unsigned int m;
    int s;   // 31 + l
};
inline FastDiv make_fastdiv(int d) {
    int l = 0;
    while ((1ull << l) < (unsigned long long)d) ++l;
    FastDiv f;
    f.m = (unsigned int)(((1ull << (31 + l)) + (unsigned long long)d - 1) / (unsigned long long)d);
    f.s = 31 + l;
    return f;
}
__host__ __device__ __forceinline__ int fdiv(int n, FastDiv f) {
    return (int)(((unsigned long long)(unsigned int)n * f.m) >> f.s);
}

struct Params {
    void* o;                // [B,Hq,Sq,D] view, 16-bit, D contiguous (strides below)
    float* lse;             // [B,Hq,Sq] contiguous, or null
    int B, Hq, Hkv, Sq, Sk;
    int group;              // Hq / Hkv
    int n_pairs;            // ceil(ceil(Sq / 128) / 2): units per (batch, head)
    int items_per_head;     // schedule items per (batch, head): causal ceil(n_pairs/2), else n_pairs
    int n_items;            // B * Hq * items_per_head
    int group_heads;        // (batch, head) pairs per schedule group
    FastDiv div_items;      // by group_heads * items_per_head (items per group)
    FastDiv div_gh;         // by group_heads
    FastDiv div_gh_last;    // by the size of the last group (B * Hq - its first pair)
    FastDiv div_hq;         // by Hq
    FastDiv div_group;      // by Hq / Hkv
    int causal;             // 0 / 1
    int causal_off;         // query row i sees keys 0 .. i + causal_off
    float score_log2;       // raw MMA score -> log2 units
    float out_mul;          // multiplier on (sum_j p_j v_j) / l: V descale for FP8, else 1
    long long o_sb, o_sh, o_ss;   // O's batch, head, row strides in elements
};

template <int D, int KIND, int NS, int QB, bool SPLIT = false>
struct Cfg {
    // SPLIT: two softmax warps per TMEM lane quarter and stage, each over 64
    // of a row's 128 scores (16 softmax warps); else one (8 softmax warps)
    static constexpr int kSmWarpsPerStage = SPLIT ? 8 : 4;
    static constexpr int kSoftmaxWarps = 2 * kSmWarpsPerStage;
    static constexpr int kSmThreadsPerStage = 32 * kSmWarpsPerStage;
    static constexpr int kThreads = SPLIT ? 768 : 512;
    static constexpr int kEpiWarp0 = kSoftmaxWarps;
    static constexpr int kLoadWarp = kSoftmaxWarps + 4;
    static constexpr int kMmaWarp = kLoadWarp + 1;
    static constexpr int kTmemUsers = 2 * kSmThreadsPerStage + 128 + 32;   // softmax, epilogue, MMA
    static constexpr int kThreadKeys = SPLIT ? 64 : 128;   // scores per softmax thread and tile
    static constexpr int kElem = (KIND == K2_E4M3) ? 1 : 2;
    static constexpr int kRowBytes = D * kElem;
    static constexpr int kSwBytes = 128;                   // 128-byte swizzle rows
    static constexpr uint32_t kSwLayout = 2u;
    static constexpr int kSbo = 8 * kSwBytes;
    static constexpr int kElemsPerSw = kSwBytes / kElem;
    static constexpr int kSwBlocks = kRowBytes / kSwBytes;
    static constexpr int kSwBlockBytes = 128 * kSwBytes;
    static constexpr int kStepsPerBlock = kSwBytes / 32;
    static constexpr int kTileBytes = 128 * kRowBytes;
    static constexpr int kQkSteps = kRowBytes / 32;        // MMA K steps of 32 bytes
    static constexpr int kPvKeysPerStep = 32 / kElem;
    static constexpr int kPvSteps = kKeys / kPvKeysPerStep;
    static constexpr int kPWordsPer32 = 32 * kElem / 4;    // TMEM columns of P per 32 keys
    // PV products per 64-key half: a half's weights sit in its own score
    // columns (S_s + 64 h) in the split form, so the A operand address jumps
    // by 64 columns between the halves
    static constexpr int kPvStepsPerHalf = kThreadKeys / kPvKeysPerStep;
    // lazy rescale: the running max only moves when a tile's max exceeds it
    // by more than this (log2 units), so a weight 2^(s - m_run) can reach
    // 2^threshold
    static constexpr float kRescaleThreshold = (KIND == K2_E4M3) ? 4.0f : 8.0f;
    // log2 of the factor applied to the weights before they are rounded for
    // the PV product: for e4m3, 448 * 2^-threshold, so that the largest
    // weight (2^threshold) maps to the format's largest value, 448
    static constexpr float kPLog2 = (KIND == K2_E4M3) ? 8.807354922057604f - 4.0f : 0.0f;
    // one-warp form: weights against the running max before the tile max
    // (recomputed in the rare tile whose max moves it)
    static constexpr bool kWeightsFirst = SDPA2_WEIGHTS_FIRST != 0;
    // shared memory (offsets from a 1024-byte aligned base)
    static constexpr int kSmemQ = 0;                                 // [2 stages][QB] tiles
    static constexpr int kSmemKV = 2 * QB * kTileBytes;              // [NS] tiles
    // [2 stages][halves][128 rows][m, l], then (split) the halves' tile-max
    // exchange [2 stages][2 tile parities][2 halves][128 rows]
    static constexpr int kSmemStats = kSmemKV + NS * kTileBytes;
    static constexpr int kStatsBytes = (SPLIT ? 2 : 1) * 2 * 128 * 2 * 4;
    static constexpr int kSmemXchg = kSmemStats + kStatsBytes;
    static constexpr int kSmemBar = kSmemXchg + (SPLIT ? 2 * 2 * 2 * 128 * 4 : 0);
    // barriers
    static constexpr int kBarQFull = 0;            // [2 stages][2 buffers]
    static constexpr int kBarQEmpty = 4;           // [2][2]
    static constexpr int kBarKVFull = 8;           // [NS]
    static constexpr int kBarKVEmpty = 8 + NS;     // [NS]
    static constexpr int kBarSFull = 8 + 2 * NS;   // [2 stages]
    static constexpr int kBarPFull = 10 + 2 * NS;  // [2]
    static constexpr int kBarOFull = 12 + 2 * NS;  // [2], once per unit
    static constexpr int kBarOEmpty = 14 + 2 * NS; // [2], once per unit
    static constexpr int kBarStFull = 16 + 2 * NS; // [2], softmax -> epilogue
    static constexpr int kBarStEmpty = 18 + 2 * NS;// [2], epilogue -> softmax
    static constexpr int kBarDrain = 20 + 2 * NS;
    static constexpr int kBarXchg = 21 + 2 * NS;   // split: [2 stages][4 lane quarters], both halves arrive
    static constexpr int kNumBars = 29 + 2 * NS;
    static constexpr int kSmemTmemSlot = kSmemBar + 8 * kNumBars;
    static constexpr int kSmemAbort = kSmemTmemSlot + 4;
    static constexpr int kSmemUsed = kSmemAbort + 4;
    static constexpr int kSmemBytes = (kSmemUsed + 1024 <= 232448) ? kSmemUsed + 1024 : 232448;
    // TMEM columns
    static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 256 + D;
    static_assert(kRowBytes % 128 == 0, "rows of whole 128-byte swizzle rows");
    static_assert(kSmemUsed <= 232448, "shared memory budget");
    static_assert(kSmemBytes > 116 * 1024, "one CTA per SM (each allocates all of TMEM)");
    static_assert(D <= 128, "O_s must fit 128 TMEM columns");
    static_assert(QB == 1 || QB == 2, "one or two Q buffers per stage");
};

// ---------------------------------------------------------------------------
// bounded waiting (every wait gives up after kWaitLimitNs, records where in
// the status word and raises the CTA's abort flag; no trap)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ void sts_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.volatile.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ bool wait_slow(uint32_t bar, uint32_t parity, uint32_t abort_addr,
                                          unsigned int* status, uint32_t where, uint32_t sleep_ns,
                                          uint64_t limit_ns = kWaitLimitNs) {
    const uint64_t t0 = global_timer_ns();
    for (uint32_t k = 1;; ++k) {
        if (sleep_ns) __nanosleep(sleep_ns);
        if (mbar_try_wait(bar, parity)) return true;
        if ((k & 15u) == 0) {
            if (lds_u32(abort_addr) != 0u) return false;
            if (global_timer_ns() - t0 > limit_ns) {
                sts_u32(abort_addr, 1u);
                if (atomicCAS(&status[0], 0u, 4u) == 0u) atomicExch(&status[1], where);
                return false;
            }
        }
    }
}
__device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity, uint32_t abort_addr,
                                     unsigned int* status, uint32_t where) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_slow(bar, parity, abort_addr, status, where, 0u);
}
__device__ __forceinline__ bool wait_sleep(uint32_t bar, uint32_t parity, uint32_t abort_addr,
                                           unsigned int* status, uint32_t where) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_slow(bar, parity, abort_addr, status, where, SDPA2_EPI_SLEEP_NS);
}

// Zero weights into chunk c (32 keys) of a P tile starting at TMEM address tP.
template <int KIND, int WORDS_PER_32>
__device__ __forceinline__ void zero_p_chunk(uint32_t tP, int c) {
    uint32_t z[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) z[i] = 0u;
    if constexpr (KIND == K2_E4M3)
        tmem_st8(tP + WORDS_PER_32 * c, z);
    else
        tmem_st16(tP + WORDS_PER_32 * c, z);
}
template <int KIND>
__device__ __forceinline__ constexpr bool poly_pair(int e) {
    return (((KIND == K2_E4M3 ? SDPA2_POLY_MASK_FP8 : SDPA2_POLY_MASK) >> (e & 7)) & 1) != 0;
}

// Maximum of 128 registers (3-input max, four chains).
__device__ __forceinline__ float max128(const float* s) {
    float a = s[0], b = s[1], c = s[2], d = s[3];
#pragma unroll
    for (int i = 4; i + 8 <= 128; i += 8) {
        a = fmax3(a, s[i], s[i + 1]);
        b = fmax3(b, s[i + 2], s[i + 3]);
        c = fmax3(c, s[i + 4], s[i + 5]);
        d = fmax3(d, s[i + 6], s[i + 7]);
    }
    a = fmax3(a, s[124], s[125]);
    b = fmax3(b, s[126], s[127]);
    return fmax3(fmaxf(a, b), c, d);
}

// Maximum of 32 registers.
__device__ __forceinline__ float max32(const float* s) {
    float a = s[0], b = s[1];
#pragma unroll
    for (int i = 2; i + 4 <= 32; i += 4) {
        a = fmax3(a, s[i], s[i + 1]);
        b = fmax3(b, s[i + 2], s[i + 3]);
    }
    return fmax3(fmaxf(a, b), s[30], s[31]);
}

// K/V tiles the query rows [row0, row0 + 128) need (0 when the tile starts
// past Sq).
__device__ __forceinline__ int tiles_for(int row0, int Sq, int Sk, int causal, int off) {
    if (row0 >= Sq) return 0;
    const int kend = causal ? min(Sk, row0 + kRows + off) : Sk;
    return (kend + kKeys - 1) / kKeys;
}

// ---------------------------------------------------------------------------
// schedule: items are dealt round-robin to the persistent CTAs; items come in
// groups of `group_heads` (batch, head) pairs (their K/V stay in L2); within
// a group, item j of a head is unit n_pairs-1-j (the longest first) and, for
// causal attention, also unit j, so every causal item costs the same.
// ---------------------------------------------------------------------------
struct Unit {
    int k, sub;     // schedule position
    int bh, m;      // (batch, head) and pair index: stage s holds query tile 2m+s
    int n0, n1, n;  // K/V tiles of stage 0, stage 1, and of the unit (max)
    bool valid;
};

__device__ __forceinline__ bool sched(const Params& p, int k, int sub, int& bh, int& m) {
    // item < n_items < 2^31 once the bound holds; the sum cannot wrap 32 bits
    const unsigned int item = blockIdx.x + (unsigned int)k * gridDim.x;
    if (item >= (unsigned int)p.n_items) return false;
    const int per_group = p.group_heads * p.items_per_head;
    const int grp = fdiv((int)item, p.div_items);
    const int within = (int)item - grp * per_group;
    const int rest = p.B * p.Hq - grp * p.group_heads;   // pairs from this group's first on
    const bool last = rest < p.group_heads;
    const int gsize = last ? rest : p.group_heads;
    const int j = fdiv(within, last ? p.div_gh_last : p.div_gh);
    bh = grp * p.group_heads + (within - j * gsize);
    const int hi = p.n_pairs - 1 - j;
    if (sub == 0) {
        m = hi;
        return true;
    }
    if (!p.causal || j == hi) return false;
    m = j;
    return true;
}
__device__ __forceinline__ void unit_load(const Params& p, Unit& u) {
    u.valid = sched(p, u.k, u.sub, u.bh, u.m);
    if (u.valid) {
        u.n0 = tiles_for(2 * u.m * kRows, p.Sq, p.Sk, p.causal, p.causal_off);
        u.n1 = tiles_for((2 * u.m + 1) * kRows, p.Sq, p.Sk, p.causal, p.causal_off);
        u.n = max(u.n0, u.n1);
    } else {
        u.n0 = u.n1 = u.n = 0;
    }
}
__device__ __forceinline__ void unit_first(const Params& p, Unit& u) {
    u.k = 0;
    u.sub = 0;
    unit_load(p, u);
}
__device__ __forceinline__ void unit_next(const Params& p, Unit& u) {
    if (u.sub == 0 && p.causal) {   // only causal items hold a second unit
        u.sub = 1;
        unit_load(p, u);
        if (u.valid) return;
    }
    ++u.k;
    u.sub = 0;
    unit_load(p, u);
}
__device__ __forceinline__ int stage_tiles(const Unit& u, int s) { return s ? u.n1 : u.n0; }

// One position in the CTA's stream of K/V tiles.
struct Cursor {
    Unit u;
    int j;   // tile within the unit
};
__device__ __forceinline__ void cur_first(const Params& p, Cursor& c) {
    unit_first(p, c.u);
    c.j = 0;
}
__device__ __forceinline__ void cur_next(const Params& p, Cursor& c) {
    if (++c.j == c.u.n) {
        unit_next(p, c.u);
        c.j = 0;
    }
}

template <int D, bool STRIDED>
__device__ __forceinline__ long long o_offset(const Params& p, int bh, int row) {
    if constexpr (STRIDED) {
        const int b = fdiv(bh, p.div_hq);
        return (long long)b * p.o_sb + (long long)(bh - b * p.Hq) * p.o_sh + (long long)row * p.o_ss;
    } else {
        return ((long long)bh * p.Sq + row) * D;
    }
}

template <int D, int KIND, int NS, int QB, bool SPLIT, bool STRIDED>
__global__ void __launch_bounds__(SPLIT ? 768 : 512, 1)
sdpa_fwd2q_sm100_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV,
                        const Params p) {
    using C = Cfg<D, KIND, NS, QB, SPLIT>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    float* const stats = reinterpret_cast<float*>(smem_raw + (sbase - raw) + C::kSmemStats);
    unsigned int* const status = g_status;
    // the aligned layout must end inside the allocation (uniform exit)
    if (sbase - raw + (uint32_t)C::kSmemUsed > (uint32_t)C::kSmemBytes) {
        if (threadIdx.x == 0 && atomicCAS(&status[0], 0u, 5u) == 0u) atomicExch(&status[1], sbase - raw);
        return;
    }
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    auto bar = [&](int i) -> uint32_t { return sbase + C::kSmemBar + 8u * (uint32_t)i; };
    const uint32_t abort_addr = sbase + C::kSmemAbort;
    const uint32_t slot_addr = sbase + C::kSmemTmemSlot;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 4; ++i) {
            mbar_init(bar(C::kBarQFull + i), 1);
            mbar_init(bar(C::kBarQEmpty + i), 1);
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(bar(C::kBarKVFull + s), 1);
            mbar_init(bar(C::kBarKVEmpty + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(C::kBarSFull + s), 1);
            mbar_init(bar(C::kBarPFull + s), C::kSmThreadsPerStage);
            mbar_init(bar(C::kBarOFull + s), 1);
            mbar_init(bar(C::kBarOEmpty + s), kRows);
            mbar_init(bar(C::kBarStFull + s), C::kSmThreadsPerStage);
            mbar_init(bar(C::kBarStEmpty + s), kRows);
        }
        mbar_init(bar(C::kBarDrain), 1);
        for (int i = 0; i < 8; ++i) mbar_init(bar(C::kBarXchg + i), 64);
        sts_u32(abort_addr, 0u);
        fence_barrier_init();
    }
    if (warp == C::kMmaWarp) {
        tmem_alloc(slot_addr, kTmemCols);
        tmem_relinquish();
    }
    if (warp == C::kLoadWarp && lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = lds_u32(slot_addr);
    const uint32_t sQ = sbase + C::kSmemQ;
    const uint32_t sKV = sbase + C::kSmemKV;

    if (warp >= C::kLoadWarp) {
        if constexpr (SPLIT) regs_dec<SDPA2S_REGS_OTHER>();
        else regs_dec<KIND == K2_E4M3 ? SDPA2_REGS_OTHER_FP8 : SDPA2_REGS_OTHER>();
        if (warp == C::kLoadWarp && lane == 0) {
            // ================= TMA producer ==============================
            bool ok = true;
            int kq[2] = {0, 0};   // units loaded per stage (Q buffer uses)
            int t = 0;            // ring positions issued
            auto load_q = [&](const Unit& u, int s, uint32_t fb, uint32_t dst) {
                const int row0 = (2 * u.m + s) * kRows;
                for (int kb = 0; kb < C::kSwBlocks; ++kb) {
                    if constexpr (STRIDED) {
                        const int b = fdiv(u.bh, p.div_hq);
                        tma_load_4d(dst + kb * C::kSwBlockBytes, &tmQ, fb, kb * C::kElemsPerSw, row0,
                                    u.bh - b * p.Hq, b);
                    } else {
                        tma_load_3d(dst + kb * C::kSwBlockBytes, &tmQ, fb, kb * C::kElemsPerSw, row0, u.bh);
                    }
                }
            };
            auto prefetch_q = [&](const Unit& u) {
                for (int s = 0; s < 2; ++s) {
                    if (stage_tiles(u, s) == 0) continue;
                    const int row0 = (2 * u.m + s) * kRows;
                    for (int kb = 0; kb < C::kSwBlocks; ++kb) {
                        if constexpr (STRIDED) {
                            const int b = fdiv(u.bh, p.div_hq);
                            tma_prefetch_l2_4d(&tmQ, kb * C::kElemsPerSw, row0, u.bh - b * p.Hq, b);
                        } else {
                            tma_prefetch_l2_3d(&tmQ, kb * C::kElemsPerSw, row0, u.bh);
                        }
                    }
                }
            };
            auto load_kv = [&](const Unit& u, int j, bool is_v) -> bool {
                const int slot = t % NS;
                if (!wait(bar(C::kBarKVEmpty + slot), ((uint32_t)(t / NS) & 1u) ^ 1u, abort_addr, status,
                          0x10000u | (uint32_t)(t & 0xffff)))
                    return false;
                const int b = fdiv(u.bh, p.div_hq);
                const int kvh = fdiv(u.bh - b * p.Hq, p.div_group);
                const uint32_t fb = bar(C::kBarKVFull + slot);
                mbar_arrive_expect_tx(fb, C::kTileBytes);
                for (int kb = 0; kb < C::kSwBlocks; ++kb) {
                    const uint32_t dst = sKV + slot * C::kTileBytes + kb * C::kSwBlockBytes;
                    if constexpr (STRIDED)
                        tma_load_4d(dst, is_v ? &tmV : &tmK, fb, kb * C::kElemsPerSw, j * kKeys, kvh, b);
                    else
                        tma_load_3d(dst, is_v ? &tmV : &tmK, fb, kb * C::kElemsPerSw, j * kKeys,
                                    b * p.Hkv + kvh);
                }
                ++t;
                return true;
            };
            Unit u, un;
            unit_first(p, u);
            while (ok && u.valid) {
                // Q tiles of the unit (each stage's buffer is free once the
                // previous unit's last Q K^T of that stage has completed)
                for (int s = 0; s < 2 && ok; ++s) {
                    if (stage_tiles(u, s) == 0) continue;
                    const int qb = kq[s] % QB, use = kq[s] / QB;
                    if (use >= 1 && !wait(bar(C::kBarQEmpty + 2 * s + qb), (uint32_t)(use - 1) & 1u, abort_addr,
                                          status, 0x11000u | (s << 11) | (uint32_t)(kq[s] & 0x7ff))) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = bar(C::kBarQFull + 2 * s + qb);
                    mbar_arrive_expect_tx(fb, C::kTileBytes);
                    load_q(u, s, fb, sQ + (s * QB + qb) * C::kTileBytes);
                    ++kq[s];
                }
                if (!ok) break;
                // warm L2 with the next unit's Q tiles
                un = u;
                unit_next(p, un);
                if (un.valid) prefetch_q(un);
                for (int j = 0; j < u.n && ok; ++j) {
                    ok = load_kv(u, j, false);
                    if (ok) ok = load_kv(u, j, true);
                }
                u = un;
            }
            if (!ok) {
                // let the copies already issued land before the CTA exits
                for (int v = max(0, t - NS); v < t; ++v) {
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(bar(C::kBarKVFull + v % NS), (uint32_t)(v / NS) & 1u) &&
                           global_timer_ns() - t0 < 100000000ull) {
                    }
                }
                for (int s = 0; s < 2; ++s)
                    for (int v = max(0, kq[s] - QB); v < kq[s]; ++v) {
                        const uint64_t t0 = global_timer_ns();
                        while (!mbar_try_wait(bar(C::kBarQFull + 2 * s + v % QB), (uint32_t)(v / QB) & 1u) &&
                               global_timer_ns() - t0 < 100000000ull) {
                        }
                    }
            }
        } else if (warp == C::kMmaWarp) {
            // ================= MMA issuer ================================
            const bool leader = elect_one();
            constexpr uint32_t fmt = (KIND == K2_BF16) ? 1u : 0u;
            constexpr uint32_t idesc_qk = make_idesc(fmt, false, kRows, kKeys);
            constexpr uint32_t idesc_pv = make_idesc(fmt, true, kRows, D);
            // Shared-memory descriptors: the high word (stride offset, fixed
            // bits, swizzle) is the same for every operand; the low word is
            // start address >> 4 plus the leading offset, and stepping
            // through a tile only adds to the start address (no carry: the
            // addresses stay below 2^18).
            const uint64_t dq0 = make_smem_desc(sQ, 16, C::kSbo, C::kSwLayout);
            const uint64_t dk0 = make_smem_desc(sKV, 16, C::kSbo, C::kSwLayout);
            const uint64_t dv0 = make_smem_desc(sKV, C::kSwBlockBytes, C::kSbo, C::kSwLayout);
            const uint32_t desc_hi = (uint32_t)(dq0 >> 32);
            const uint32_t dq_lo = (uint32_t)dq0, dk_lo = (uint32_t)dk0, dv_lo = (uint32_t)dv0;
            auto desc = [&](uint32_t lo) -> uint64_t { return ((uint64_t)desc_hi << 32) | lo; };
            bool ok = true;
            int cp[2] = {0, 0};    // P_s tiles consumed (P_full phase)
            int kqk[2] = {0, 0};   // units started, QK side (Q_full phase)
            int kpv[2] = {0, 0};   // units started, PV side (O_empty phase)

            auto wait_all = [&](uint32_t b_, uint32_t par, uint32_t where) {
                const bool r_ = wait(b_, par, abort_addr, status, where);
                return __all_sync(0xffffffffu, r_);
            };
            auto commit = [&](uint32_t b_) {
                if (leader) mma_commit(b_);
                __syncwarp();
            };
            // The issue loops are unrolled: every MMA's descriptors are one
            // add of an immediate to a 32-bit base, so the single issuing
            // thread keeps up with the tensor pipe.
            auto issue_qk = [&](int s, int qb, int slot) {
                const uint32_t d_tmem = tmem + (s ? C::kColS1 : C::kColS0);
                const uint32_t aq = dq_lo + (uint32_t)(((s * QB + qb) * C::kTileBytes) >> 4);
                const uint32_t bk = dk_lo + (uint32_t)((slot * C::kTileBytes) >> 4);
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < C::kQkSteps; ++kk) {
                        constexpr int kBlk = C::kSwBlockBytes, kSpb = C::kStepsPerBlock;
                        const uint32_t off = (uint32_t)(((kk / kSpb) * kBlk + (kk % kSpb) * 32) >> 4);
                        if constexpr (KIND == K2_E4M3)
                            mma_f8_ss(d_tmem, desc(aq + off), desc(bk + off), idesc_qk, kk > 0);
                        else
                            mma_f16_ss(d_tmem, desc(aq + off), desc(bk + off), idesc_qk, kk > 0);
                    }
                }
                __syncwarp();
            };
            auto issue_pv = [&](int s, int slot, bool acc) {
                const uint32_t d_tmem = tmem + (s ? C::kColO1 : C::kColO0);
                const uint32_t a_tmem = tmem + (s ? C::kColS1 : C::kColS0);
                const uint32_t bv = dv_lo + (uint32_t)((slot * C::kTileBytes) >> 4);
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < C::kPvSteps; ++kk) {
                        const uint32_t off = (uint32_t)((kk * C::kPvKeysPerStep * C::kSwBytes) >> 4);
                        const uint32_t accum = (acc || kk > 0) ? 1u : 0u;
                        constexpr int kPh = C::kPvStepsPerHalf;
                        const uint32_t a_col = (uint32_t)((kk / kPh) * 64 + (kk % kPh) * 8);
                        if constexpr (KIND == K2_E4M3)
                            mma_f8_ts(d_tmem, a_tmem + a_col, desc(bv + off), idesc_pv, accum);
                        else
                            mma_f16_ts(d_tmem, a_tmem + a_col, desc(bv + off), idesc_pv, accum);
                    }
                }
                __syncwarp();
            };
            // Q K^T of stream tile kc for stage s (K already landed in slotK)
            auto qk_stage = [&](const Cursor& kc, int s, int slotK) -> bool {
                const int qb = kqk[s] % QB;
                if (kc.j == 0 &&
                    !wait_all(bar(C::kBarQFull + 2 * s + qb), (uint32_t)(kqk[s] / QB) & 1u,
                              0x20000u | (s << 11) | (uint32_t)(kqk[s] & 0x7ff)))
                    return false;
                issue_qk(s, qb, slotK);
                commit(bar(C::kBarSFull + s));
                if (kc.j == stage_tiles(kc.u, s) - 1) {
                    commit(bar(C::kBarQEmpty + 2 * s + qb));   // Q_s buffer free
                    ++kqk[s];
                }
                return true;
            };
            // O_s (+)= P_s V for stream tile vc (V landed in slotV)
            auto pv_stage = [&](const Cursor& vc, int s, int slotV) -> bool {
                if (!wait_all(bar(C::kBarPFull + s), (uint32_t)cp[s] & 1u,
                              0x23000u | (s << 11) | (uint32_t)(cp[s] & 0x7ff)))
                    return false;
                // the unit's first product overwrites O_s: the epilogue must
                // have read the previous unit's
                if (vc.j == 0 && kpv[s] > 0 &&
                    !wait_all(bar(C::kBarOEmpty + s), (uint32_t)(kpv[s] - 1) & 1u,
                              0x25000u | (s << 11) | (uint32_t)(kpv[s] & 0x7ff)))
                    return false;
                tc_fence_after();
                issue_pv(s, slotV, vc.j > 0);
                if (vc.j == stage_tiles(vc.u, s) - 1) {
                    commit(bar(C::kBarOFull + s));
                    ++kpv[s];
                }
                ++cp[s];
                return true;
            };

            Cursor kc, vc;
            cur_first(p, kc);
            cur_first(p, vc);
            int t = 0;   // ring positions consumed: K(g) at 2g, V(g) at 2g + 1
            if (kc.u.valid) {
                const int slotK = t % NS;
                ok = wait_all(bar(C::kBarKVFull + slotK), (uint32_t)(t / NS) & 1u, 0x21000u);
                for (int s = 0; s < 2 && ok; ++s)
                    if (stage_tiles(kc.u, s) > 0) ok = qk_stage(kc, s, slotK);
                if (ok) commit(bar(C::kBarKVEmpty + slotK));
                ++t;
                cur_next(p, kc);
            }
            // Release commits of the previous step's K/V slots, deferred to
            // the top of the next step, where the thread is about to wait for
            // weights anyway (measured faster on long units than committing
            // them at the end of the step or right after the PV products).
            int pend_v = -1, pend_k = -1;
            auto release = [&]() {
                if (pend_v >= 0) commit(bar(C::kBarKVEmpty + pend_v));
                if (pend_k >= 0) commit(bar(C::kBarKVEmpty + pend_k));
                pend_v = pend_k = -1;
            };
            while (ok && vc.u.valid) {
                const int slotV = t % NS;
                ok = wait_all(bar(C::kBarKVFull + slotV), (uint32_t)(t / NS) & 1u,
                              0x22000u | (uint32_t)(t & 0xfff));
                if (!ok) break;
                if (SDPA2_DEFER_RELEASE) release();
                const int slotK = (t + 1) % NS;
                bool k_ready = false;
                for (int s = 0; s < 2 && ok; ++s) {
                    if (vc.j < stage_tiles(vc.u, s)) ok = pv_stage(vc, s, slotV);
                    if (ok && kc.u.valid && kc.j < stage_tiles(kc.u, s)) {
                        if (!k_ready) {
                            ok = wait_all(bar(C::kBarKVFull + slotK), (uint32_t)((t + 1) / NS) & 1u,
                                          0x21000u | (uint32_t)((t + 1) & 0xfff));
                            k_ready = true;
                        }
                        if (ok) ok = qk_stage(kc, s, slotK);
                    }
                }
                if (!ok) break;
                pend_v = slotV;
                ++t;
                if (kc.u.valid) {
                    // a unit whose stage tiles are all inactive on this K
                    // tile does not exist (stage 1's count is the unit's)
                    pend_k = slotK;
                    ++t;
                    cur_next(p, kc);
                }
                if (!SDPA2_DEFER_RELEASE) release();
                cur_next(p, vc);
            }
            if (ok) release();
            if (!ok) {
                // make sure no MMA is still writing tensor memory at exit
                commit(bar(C::kBarDrain));
                const uint64_t t0 = global_timer_ns();
                while (!mbar_try_wait(bar(C::kBarDrain), 0) && global_timer_ns() - t0 < 100000000ull) {
                }
            }
            named_bar_sync(1, C::kTmemUsers);
            __syncwarp();
            tc_fence_after();
            tmem_dealloc(tmem, kTmemCols);
        }
    } else if (warp < C::kSoftmaxWarps && !SPLIT) {
        // ================= softmax, one stage per warp group ==============
        regs_inc<KIND == K2_E4M3 ? SDPA2_REGS_SOFTMAX_FP8 : SDPA2_REGS_SOFTMAX>();
        const int s = warp >> 2;                 // stage
        const int quarter = warp & 3;            // TMEM lane quarter
        const int r = (int)(threadIdx.x & 127);  // row within the stage tile
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint32_t tS = tmem + lane_base + (s ? C::kColS1 : C::kColS0);
        const uint32_t tO = tmem + lane_base + (s ? C::kColO1 : C::kColO0);
        const float sl = p.score_log2;
        const uint64_t sl2 = f2_pack(sl, sl);
        bool ok = true;
        int cs = 0;   // tiles of this stage so far (S_full / P_full phase)
        int ks = 0;   // units of this stage so far (stats phase)

        // weights of 32 scores against nm2 = (-m + log2 of the P scale) x 2,
        // rounded for the PV product into chunk c of P; returns the fp32 sum
        // and, in cmax, the largest of the 32 raw scores
        auto exp_chunk = [&](const float* sc, uint64_t nm2, int c, float& cmax) -> uint64_t {
            uint64_t sum2[2] = {0ull, 0ull};
            uint32_t pk[16];
            float mx0 = sc[0], mx1 = sc[1];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                if (e > 0) {
                    if (e & 1) mx1 = fmax3(mx1, sc[2 * e], sc[2 * e + 1]);
                    else mx0 = fmax3(mx0, sc[2 * e], sc[2 * e + 1]);
                }
                const uint64_t x2 = f2_fma(f2_pack(sc[2 * e], sc[2 * e + 1]), sl2, nm2);
                float x0, x1;
                f2_unpack(x2, x0, x1);
                uint64_t p2;
                if (poly_pair<KIND>(e))
                    p2 = exp2_poly_x2(f2_pack(fmaxf(x0, -126.0f), fmaxf(x1, -126.0f)));
                else
                    p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
                sum2[e & 1] = f2_add(sum2[e & 1], p2);
                float q0, q1;
                f2_unpack(p2, q0, q1);
                if constexpr (KIND == K2_E4M3) {
                    // one conversion per pair; pairs 2i and 2i+1 share a word
                    if (e & 1) pk[e >> 1] |= pack_e4m3x2(q0, q1) << 16;
                    else pk[e >> 1] = pack_e4m3x2(q0, q1);
                } else {
                    pk[e] = (KIND == K2_BF16) ? pack_bf16x2(q0, q1) : pack_f16x2(q0, q1);
                }
            }
            cmax = fmaxf(mx0, mx1);
            if constexpr (KIND == K2_E4M3)
                tmem_st8(tS + C::kPWordsPer32 * c, pk);
            else
                tmem_st16(tS + C::kPWordsPer32 * c, pk);
            return f2_add(sum2[0], sum2[1]);
        };

        Unit u;
        unit_first(p, u);
        while (ok && u.valid) {
            const int ns = stage_tiles(u, s);
            if (ns == 0) {   // stage 1 of a unit past the last query tile
                unit_next(p, u);
                continue;
            }
            const int row0 = (2 * u.m + s) * kRows;
            const int row = row0 + r;
            float m_run = -INFINITY;   // running max of scaled scores (log2 units)
            float l_run = 0.0f;        // running sum of 2^(s*sl - m_run + kPLog2)
            for (int j = 0; j < ns && ok; ++j, ++cs) {
                ok = wait(bar(C::kBarSFull + s), (uint32_t)cs & 1u, abort_addr, status,
                          0x30000u | (s << 12) | (uint32_t)(cs & 0xfff));
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();
                float sc[kKeys];
                tmem_ld32(tS + 0, *reinterpret_cast<float(*)[32]>(&sc[0]));
                tmem_ld32(tS + 32, *reinterpret_cast<float(*)[32]>(&sc[32]));
                tmem_ld32(tS + 64, *reinterpret_cast<float(*)[32]>(&sc[64]));
                tmem_ld32(tS + 96, *reinterpret_cast<float(*)[32]>(&sc[96]));
                tmem_wait_ld();
                reg_fence32(&sc[0]);
                reg_fence32(&sc[32]);
                reg_fence32(&sc[64]);
                reg_fence32(&sc[96]);
                // mask keys past Sk and (causal) keys after row + causal_off
                const int key0 = j * kKeys;
                const bool edge = (key0 + kKeys > p.Sk) || (p.causal && key0 + kKeys - 1 > row0 + p.causal_off);
                if (edge) {
                    int lim = p.Sk - key0;
                    if (p.causal) lim = min(lim, row + p.causal_off - key0 + 1);
#pragma unroll
                    for (int c = 0; c < kKeys; ++c)
                        if (c >= lim) sc[c] = -INFINITY;
                }
                // Lazy rescale: the reference max m_run moves only when a
                // tile's max exceeds it by more than the threshold; O_s and l
                // share the reference max at all times.  With kWeightsFirst,
                // past the unit's first tile the weights are computed against
                // m_run at once and the tile's max is found alongside them,
                // off the MUFU; in the rare case that it exceeds m_run by more
                // than the threshold, m_run moves, l and O_s are rescaled and
                // the weights are computed again (the PV product has not been
                // released yet).  Otherwise the max comes first.
                // all weights against m_run; tmax receives the tile's max
                // raw score
                auto all_weights = [&](float& tmax) -> uint64_t {
                    const float nm = C::kPLog2 - m_run;
                    const uint64_t nm2 = f2_pack(nm, nm);
                    float c0, c1, c2, c3;
                    uint64_t a = exp_chunk(&sc[0], nm2, 0, c0);
                    a = f2_add(a, exp_chunk(&sc[32], nm2, 1, c1));
                    a = f2_add(a, exp_chunk(&sc[64], nm2, 2, c2));
                    a = f2_add(a, exp_chunk(&sc[96], nm2, 3, c3));
                    tmax = fmaxf(fmaxf(c0, c1), fmaxf(c2, c3));
                    return a;
                };
                uint64_t acc;
                float traw;
                // O_s *= alpha row by row; O_s += P_s V of the previous tile
                // has completed (it was issued before the Q K^T that produced
                // this S)
                auto rescale_o = [&](float alpha) {
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
                };
                if (j == 0) {
                    // every row of the unit's first tile has a visible key
                    m_run = max128(sc) * sl;
                    acc = all_weights(traw);
                } else if constexpr (!C::kWeightsFirst) {
                    const float tmax = max128(sc) * sl;
                    const bool need = tmax > m_run + C::kRescaleThreshold;
                    if (__any_sync(0xffffffffu, need)) {
                        float alpha = 1.0f;
                        if (need) {
                            alpha = ex2_approx(m_run - tmax);
                            m_run = tmax;
                        }
                        l_run *= alpha;
                        rescale_o(alpha);
                    }
                    acc = all_weights(traw);
                } else {
                    acc = all_weights(traw);
                    const float tmax = traw * sl;
                    const bool need = tmax > m_run + C::kRescaleThreshold;
                    if (__any_sync(0xffffffffu, need)) {
                        float alpha = 1.0f;
                        if (need) {
                            alpha = ex2_approx(m_run - tmax);
                            m_run = tmax;
                        }
                        l_run *= alpha;
                        rescale_o(alpha);
                        acc = all_weights(traw);   // P_s overwritten in place
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(C::kBarPFull + s));
                float a0, a1;
                f2_unpack(acc, a0, a1);
                l_run += a0 + a1;
            }
            if (!ok) break;
            // hand (m, l) of every row to the epilogue warps
            if (ks > 0) {
                ok = wait(bar(C::kBarStEmpty + s), (uint32_t)(ks - 1) & 1u, abort_addr, status,
                          0x40000u | (s << 12) | (uint32_t)(ks & 0xfff));
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
            }
            stats[(s * kRows + r) * 2] = m_run;
            stats[(s * kRows + r) * 2 + 1] = l_run;
            mbar_arrive(bar(C::kBarStFull + s));
            ++ks;
            unit_next(p, u);
        }
        tc_fence_before();
        named_bar_sync(1, C::kTmemUsers);
    } else if (warp < C::kSoftmaxWarps) {
        // ================= softmax, split form: two warps per lane quarter
        // and stage, each over 64 of a row's 128 scores ====================
        // The two halves of a row share its reference max m_run (moved on
        // both sides by the same decision) and keep their own row sums; once
        // per tile they exchange their tile maxima (shared memory and a
        // two-warp mbarrier), which is all a rescale decision needs.  A
        // half's weights go into its own score columns, S_s + 64 h.
        if constexpr (SPLIT) regs_inc<SDPA2S_REGS_SOFTMAX>();
        const int s = warp / C::kSmWarpsPerStage;               // stage
        const int quarter = warp & 3;                            // TMEM lane quarter
        const int h = (warp % C::kSmWarpsPerStage) >> 2;         // key half
        const int r = quarter * 32 + lane;                       // row within the stage tile
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint32_t tS = tmem + lane_base + (s ? C::kColS1 : C::kColS0) + 64 * h;
        const uint32_t tO = tmem + lane_base + (s ? C::kColO1 : C::kColO0) + h * (D / 2);
        float* const xchg = reinterpret_cast<float*>(smem_raw + (sbase - raw) + C::kSmemXchg);
        const uint32_t xbar = bar(C::kBarXchg + 4 * s + quarter);
        const float sl = p.score_log2;
        const uint64_t sl2 = f2_pack(sl, sl);
        bool ok = true;
        int cs = 0;   // tiles of this stage so far (S_full / P_full / exchange phase)
        int ks = 0;   // units of this stage so far (stats phase)

        // weights of 32 scores against nm2 = (-m + log2 of the P scale) x 2,
        // rounded into chunk c of this half's P; returns the fp32 sum
        auto exp_chunk = [&](const float* sc, uint64_t nm2, int c) -> uint64_t {
            uint64_t sum2[2] = {0ull, 0ull};
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const uint64_t x2 = f2_fma(f2_pack(sc[2 * e], sc[2 * e + 1]), sl2, nm2);
                float x0, x1;
                f2_unpack(x2, x0, x1);
                uint64_t p2;
                if (poly_pair<KIND>(e))
                    p2 = exp2_poly_x2(f2_pack(fmaxf(x0, -126.0f), fmaxf(x1, -126.0f)));
                else
                    p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
                sum2[e & 1] = f2_add(sum2[e & 1], p2);
                float q0, q1;
                f2_unpack(p2, q0, q1);
                if constexpr (KIND == K2_E4M3) {
                    if (e & 1) pk[e >> 1] |= pack_e4m3x2(q0, q1) << 16;
                    else pk[e >> 1] = pack_e4m3x2(q0, q1);
                } else {
                    pk[e] = (KIND == K2_BF16) ? pack_bf16x2(q0, q1) : pack_f16x2(q0, q1);
                }
            }
            if constexpr (KIND == K2_E4M3)
                tmem_st8(tS + C::kPWordsPer32 * c, pk);
            else
                tmem_st16(tS + C::kPWordsPer32 * c, pk);
            return f2_add(sum2[0], sum2[1]);
        };

        Unit u;
        unit_first(p, u);
        while (ok && u.valid) {
            const int ns = stage_tiles(u, s);
            if (ns == 0) {
                unit_next(p, u);
                continue;
            }
            const int row0 = (2 * u.m + s) * kRows;
            const int row = row0 + r;
            float m_run = -INFINITY;   // the row's reference max (log2 units), shared by the halves
            float l_run = 0.0f;        // this half's sum of 2^(s*sl - m_run + kPLog2)
            for (int j = 0; j < ns && ok; ++j, ++cs) {
                ok = wait(bar(C::kBarSFull + s), (uint32_t)cs & 1u, abort_addr, status,
                          0x30000u | (s << 12) | (uint32_t)(cs & 0xfff));
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();
                const int key0 = j * kKeys + 64 * h;
                const bool edge = (key0 + 64 > p.Sk) || (p.causal && key0 + 63 > row0 + p.causal_off);
                int lim = 64;
                int nch = 2;   // leading 32-key chunks of the half not masked for the whole warp
                if (edge) {
                    lim = p.Sk - key0;
                    if (p.causal) lim = min(lim, row + p.causal_off - key0 + 1);
                    if (SDPA2_SKIP_MASKED)
                        nch = min(2, max(0, (__reduce_max_sync(0xffffffffu, lim) + 31) >> 5));
                }
                // 32 scores of the half (chunk c), masked past Sk and after
                // row + causal_off
                auto load32 = [&](int c, float (&sc)[32]) {
                    tmem_ld32(tS + 32 * c, sc);
                    tmem_wait_ld();
                    reg_fence32(sc);
                    if (edge) {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (32 * c + e >= lim) sc[e] = -INFINITY;
                    }
                };
                // The max comes first, one chunk at a time; the scores are
                // read again for the weights (the chunk-0 weights overwrite
                // only chunk-0 columns), so 32 of them are live at a time.
                float hm = -INFINITY;
                if (nch > 0) {
                    float sc[32];
                    load32(0, sc);
                    hm = max32(sc);
                    if (nch > 1) {
                        load32(1, sc);
                        hm = fmaxf(hm, max32(sc));
                    }
                }
                // the row's tile max: this half's and the partner's, through
                // shared memory (slots alternate with the tile parity)
                const int par = cs & 1;
                xchg[((s * 2 + par) * 2 + h) * kRows + r] = hm * sl;
                mbar_arrive(xbar);
                ok = wait(xbar, (uint32_t)par, abort_addr, status, 0x33000u | (s << 11) | (uint32_t)(cs & 0x7ff));
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                const float tmax = fmaxf(hm * sl, xchg[((s * 2 + par) * 2 + (1 - h)) * kRows + r]);
                // lazy rescale, as in the one-warp form; both halves take the
                // same decision on the same m_run
                const bool need = tmax > m_run + C::kRescaleThreshold;
                if (__any_sync(0xffffffffu, need)) {
                    float alpha = 1.0f;
                    if (need) {
                        alpha = ex2_approx(m_run - tmax);   // 0 on the first live tile
                        m_run = tmax;
                    }
                    l_run *= alpha;
                    if (j > 0) {
                        // this half's columns of O_s; O_s += P_s V of the
                        // previous tile has completed
#pragma unroll 1
                        for (int c = 0; c < D / 64; ++c) {
                            float o[32];
                            tmem_ld32(tO + 32 * c, o);
                            tmem_wait_ld();
                            reg_fence32(o);
#pragma unroll
                            for (int e = 0; e < 32; ++e) o[e] *= alpha;
                            tmem_st32(tO + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(o));
                        }
                    }
                }
                const float nm = C::kPLog2 - m_run;
                const uint64_t nm2 = f2_pack(nm, nm);
                uint64_t acc = 0ull;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    if (c < nch) {
                        float sc[32];
                        load32(c, sc);
                        acc = f2_add(acc, exp_chunk(sc, nm2, c));
                    } else {
                        zero_p_chunk<KIND, C::kPWordsPer32>(tS, c);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(C::kBarPFull + s));
                float a0, a1;
                f2_unpack(acc, a0, a1);
                l_run += a0 + a1;
            }
            if (!ok) break;
            if (ks > 0) {
                ok = wait(bar(C::kBarStEmpty + s), (uint32_t)(ks - 1) & 1u, abort_addr, status,
                          0x40000u | (s << 12) | (uint32_t)(ks & 0xfff));
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
            }
            stats[((s * 2 + h) * kRows + r) * 2] = m_run;
            stats[((s * 2 + h) * kRows + r) * 2 + 1] = l_run;
            mbar_arrive(bar(C::kBarStFull + s));
            ++ks;
            unit_next(p, u);
        }
        tc_fence_before();
        named_bar_sync(1, C::kTmemUsers);
    } else {
        // ================= epilogue (4 warps after the softmax warps) =====
        if constexpr (SPLIT) regs_dec<SDPA2S_REGS_EPILOGUE>();
        else regs_dec<KIND == K2_E4M3 ? SDPA2_REGS_EPILOGUE_FP8 : SDPA2_REGS_EPILOGUE>();
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;       // row within the stage tile = TMEM lane
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        bool ok = true;
        int ks[2] = {0, 0};
        Unit u;
        unit_first(p, u);
        while (ok && u.valid) {
            for (int s = 0; s < 2 && ok; ++s) {
                if (stage_tiles(u, s) == 0) continue;
                const uint32_t par = (uint32_t)ks[s] & 1u;
                ok = wait_sleep(bar(C::kBarStFull + s), par, abort_addr, status,
                                0x41000u | (s << 11) | (uint32_t)(ks[s] & 0x7ff));
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                float m, l;
                if constexpr (SPLIT) {
                    // the halves share m; their sums add
                    m = stats[((s * 2) * kRows + r) * 2];
                    l = stats[((s * 2) * kRows + r) * 2 + 1] + stats[((s * 2 + 1) * kRows + r) * 2 + 1];
                } else {
                    m = stats[(s * kRows + r) * 2];
                    l = stats[(s * kRows + r) * 2 + 1];
                }
                mbar_arrive(bar(C::kBarStEmpty + s));
                const float cmul = p.out_mul / l;
                const int row = (2 * u.m + s) * kRows + r;
                const bool live = row < p.Sq;
                if (live && p.lse != nullptr)
                    p.lse[(size_t)u.bh * p.Sq + row] = (m + __log2f(l) - C::kPLog2) * kLn2;
                ok = wait_sleep(bar(C::kBarOFull + s), par, abort_addr, status,
                                0x42000u | (s << 11) | (uint32_t)(ks[s] & 0x7ff));
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();
                const uint32_t tO = tmem + lane_base + (s ? C::kColO1 : C::kColO0);
                // Stores in whole 32-byte sectors: lanes 2i and 2i+1 swap
                // halves of each 16-column chunk, so that one store
                // instruction writes 16 bytes of each of the pair's rows
                // next to each other (16 full sectors per instruction).
                const bool odd = (lane & 1) != 0;
                const int prow = (2 * u.m + s) * kRows + (r ^ 1);   // the partner's row
                const bool plive = prow < p.Sq;
                uint16_t* const rowA = reinterpret_cast<uint16_t*>(p.o) +
                                       o_offset<D, STRIDED>(p, u.bh, odd ? (plive ? prow : 0) : (live ? row : 0));
                uint16_t* const rowB = reinterpret_cast<uint16_t*>(p.o) +
                                       o_offset<D, STRIDED>(p, u.bh, odd ? (live ? row : 0) : (plive ? prow : 0));
                const bool liveA = odd ? plive : live, liveB = odd ? live : plive;
#pragma unroll 1
                for (int c = 0; c < D / 16; ++c) {
                    float x[16];
                    tmem_ld16(tO + 16 * c, x);
                    tmem_wait_ld();
                    reg_fence16(x);
                    if (c == D / 16 - 1) {
                        // O_s is read: the next unit's first product may overwrite it
                        tc_fence_before();
                        mbar_arrive(bar(C::kBarOEmpty + s));
                    }
                    uint32_t w[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float v0 = x[2 * e] * cmul, v1 = x[2 * e + 1] * cmul;
                        w[e] = (KIND == K2_FP16) ? pack_f16x2(v0, v1) : pack_bf16x2(v0, v1);
                    }
                    // even lanes keep columns 0-7 of the chunk and receive the
                    // partner's; odd lanes keep columns 8-15 and receive the
                    // partner's
                    uint32_t y[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) y[e] = __shfl_xor_sync(0xffffffffu, odd ? w[e] : w[4 + e], 1);
                    // first store: the even row of the pair; second: the odd row
                    const uint4 first = odd ? make_uint4(y[0], y[1], y[2], y[3]) : make_uint4(w[0], w[1], w[2], w[3]);
                    const uint4 second = odd ? make_uint4(w[4], w[5], w[6], w[7]) : make_uint4(y[0], y[1], y[2], y[3]);
                    const int colA = 16 * c + (odd ? 8 : 0);
                    if (liveA) *reinterpret_cast<uint4*>(rowA + colA) = first;
                    if (liveB) *reinterpret_cast<uint4*>(rowB + colA) = second;
                }
                ++ks[s];
            }
            unit_next(p, u);
        }
        tc_fence_before();
        named_bar_sync(1, C::kTmemUsers);
    }
}

// ---------------------------------------------------------------------------
// self-test kernels (not part of the attention path)
// ---------------------------------------------------------------------------
// The kernels' bounded-wait path on a barrier that nothing completes: warp 0
// waits with a limit of limit_ns, gives up, raises the CTA's abort flag and
// records SDPA_ERR_DEVICE_TIMEOUT with location kSelftestWhere in the status
// word; warp 1 waits on the same barrier with the full limit and must give up
// as soon as it sees the abort flag.  out[0..3]: warp 0's wait result, the
// abort flag after it, warp 1's wait result, the abort flag warp 1 saw.
constexpr uint32_t kSelftestWhere = 0x7e000u;
__global__ void __launch_bounds__(64, 1) selftest_wait_kernel(uint64_t limit_ns, unsigned int* out) {
    __shared__ __align__(8) uint64_t bar_word;
    __shared__ uint32_t abort_word;
    const uint32_t bar = smem_u32(&bar_word), abort_addr = smem_u32(&abort_word);
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        sts_u32(abort_addr, 0u);
        fence_barrier_init();
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5;
    bool ok;
    if (warp == 0)
        ok = wait_slow(bar, 0u, abort_addr, g_status, kSelftestWhere, 0u, limit_ns);
    else
        ok = wait_slow(bar, 0u, abort_addr, g_status, kSelftestWhere + 1u, 0u, kWaitLimitNs);
    ok = __all_sync(0xffffffffu, ok);
    if ((threadIdx.x & 31) == 0) {
        out[2 * warp] = ok ? 1u : 0u;
        out[2 * warp + 1] = lds_u32(abort_addr);
    }
}

// 2^x by the FMA-pipe polynomial (exp2_poly_x2) and by ex2.approx, for n
// inputs (pairs of consecutive elements through the packed form; an odd last
// element is paired with itself).
__global__ void selftest_exp2_kernel(const float* x, float* poly, float* mufu, int n) {
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const float a = x[i], b = (i + 1 < n) ? x[i + 1] : a;
    float p0, p1;
    f2_unpack(exp2_poly_x2(f2_pack(a, b)), p0, p1);
    poly[i] = p0;
    mufu[i] = ex2_approx(a);
    if (i + 1 < n) {
        poly[i + 1] = p1;
        mufu[i + 1] = ex2_approx(b);
    }
}

}  // namespace fwd2
}  // namespace sdpa
