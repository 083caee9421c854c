/*
 * sdpa.h -- C ABI of the B200 (sm_100a) fused scaled-dot-product attention
 * forward library (libsdpa_b200.so).
 *
 * The operation (codelab "JAX on GPU, Lab 5: attention on GPU", section 1 "How
 * attention works": Attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V in four
 * steps -- score, scale + softmax, attend, output of Q's shape; section 7: the
 * causal (lower-triangular) mask applied inside the fused kernel; section 9:
 * K/V heads shared by groups of query heads, MHA / GQA / MQA; article
 * "Self-attention, CUDA kernels and FlashAttention", section 3: tiles kept on
 * chip, online softmax with running max and sum, only the per-row
 * normalisation statistic written to memory):
 *
 *   for b < B, hq < Hq, i < Sq:
 *     hk = hq / (Hq / Hkv)                         contiguous head groups
 *     s_j = scale * <Q[b,hq,i,:], K[b,hk,j,:]>     j < Sk  (j <= i if causal)
 *     O[b,hq,i,:] = sum_j softmax_j(s) * V[b,hk,j,:]
 *     LSE[b,hq,i] = ln sum_j exp(s_j)              natural log, fp32
 *
 * The Sq x Sk score matrix never reaches global memory.
 *
 * Layout (all entry points): Q [B,Hq,Sq,d], K and V [B,Hkv,Sk,d],
 * O [B,Hq,Sq,d], LSE [B,Hq,Sq]; every tensor dense row-major ("BHSD"), device
 * pointers, 16-byte aligned.  (The codelab's JAX arrays are (B,T,N,H); this
 * library takes the head-major order.)
 *
 * Ownership: the caller owns every buffer.  The entry points allocate no
 * memory, keep no state between calls other than cached per-device set-up
 * (driver entry points, kernel attributes) and a device status word, and
 * never synchronise: work is queued on `stream` (a cudaStream_t; NULL = the
 * legacy default stream) and errors raised while it runs surface at the
 * caller's next synchronisation.
 *
 * CUDA graphs: the compute entry points may be called while `stream` is being
 * captured.  The host work (argument checks, tensor-map encoding) runs at
 * capture time and the captured graph holds only the kernel launches, whose
 * arguments -- including every device pointer -- are fixed then; a replay
 * reads the inputs found at those addresses at replay time.  Make one call of
 * each entry point on the device before the capture: the first call sets the
 * kernels' shared-memory attribute and (with lazy module loading) loads the
 * module.
 *
 * Errors: every entry point returns an sdpa_status.  There is no fallback
 * path: a request the kernels cannot serve is refused with a status (the
 * codelab's cuDNN back-end likewise raises instead of silently falling back,
 * section 6).  Q/K/V/O/LSE must not overlap; O and LSE may be any device
 * memory of the right size.
 */
#ifndef SDPA_B200_H
#define SDPA_B200_H

#include <stddef.h>

#if defined(__GNUC__)
#define SDPA_API __attribute__((visibility("default")))
#else
#define SDPA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SDPA_BF16 = 0,   /* bfloat16 Q/K/V/O */
    SDPA_FP16 = 1    /* float16  Q/K/V/O */
} sdpa_dtype;

/* Values of the `causal` argument. */
typedef enum {
    SDPA_NO_MASK = 0,              /* every query sees every key */
    SDPA_CAUSAL = 1,               /* query i sees keys 0..i (codelab section 7);
                                      needs Sq == Sk */
    SDPA_CAUSAL_BOTTOM_RIGHT = 2   /* the queries are the last Sq positions of the
                                      Sk-long sequence (a KV cache): query i
                                      sees keys 0..i+Sk-Sq; needs Sq <= Sk and
                                      equals SDPA_CAUSAL when Sq == Sk */
} sdpa_causal;

typedef enum {
    SDPA_OK = 0,
    SDPA_ERR_INVALID_ARG = 1,    /* null pointer, a size <= 0, Hq % Hkv != 0,
                                    causal not an sdpa_causal value,
                                    non-finite or non-positive scale, a pointer
                                    not 16-byte aligned, sizes whose element
                                    counts overflow the addressing limits */
    SDPA_ERR_UNSUPPORTED = 2,    /* d not 32, 64 or 128 (FP8: not 128),
                                    SDPA_CAUSAL with Sq != Sk,
                                    SDPA_CAUSAL_BOTTOM_RIGHT with Sq > Sk,
                                    unknown dtype, device not sm_100 */
    SDPA_ERR_CUDA = 3,           /* the CUDA runtime or driver reported an
                                    error while preparing or launching */
    SDPA_ERR_DEVICE_TIMEOUT = 4, /* a kernel's bounded wait expired (reported
                                    by sdpa_device_status only) */
    SDPA_ERR_DEVICE_LAYOUT = 5,  /* the kernel's shared-memory layout did not
                                    fit its allocation at the base address the
                                    device gave it; nothing was computed
                                    (reported by sdpa_device_status only) */
    SDPA_ERR_SCRATCH_LIMIT = 6   /* sdpa_bwd_noalloc: B*Hq*Sq is above
                                    SDPA_BWD_NOALLOC_MAX_ROWS; nothing was
                                    launched */
} sdpa_status;

/*
 * sdpa_fwd -- fused attention forward, bf16 or fp16.
 *
 *   d                head dim: 32, 64 or 128
 *   q    [B,Hq,Sq,d]  in,  dtype
 *   k, v [B,Hkv,Sk,d] in,  dtype
 *   o    [B,Hq,Sq,d]  out, dtype (rounded to nearest even from fp32)
 *   lse  [B,Hq,Sq]    out, float32, natural-log logsumexp of the scaled
 *                     scores of each row (may be NULL to skip it)
 *   scale            applied to Q K^T as given; pass 1/sqrt(d) for the
 *                    codelab's default (section 4, scale = 1/sqrt(H))
 *   causal           an sdpa_causal: 0 every key; 1 key j only for query
 *                    i >= j (needs Sq == Sk); 2 key j only for query
 *                    i >= j - (Sk - Sq) (needs Sq <= Sk)
 *   dtype            an sdpa_dtype
 *   stream           cudaStream_t to enqueue on
 *
 * Accumulation is fp32 in tensor memory; the softmax weights are rounded to
 * the input dtype before the P*V product while the row sums use fp32.
 */
SDPA_API int sdpa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
             int B, int Hq, int Hkv, int Sq, int Sk, int d,
             float scale, int causal, int dtype, void* stream);

/*
 * sdpa_fwd_strided -- sdpa_fwd on strided views, so that the codelab's
 * [batch, time, heads, head_dim] layout (the layout JAX expects; codelab
 * "JAX on GPU, Lab 5: attention on GPU", section 3, the table of array
 * dimensions) or any other layout whose head_dim elements are contiguous is
 * read and written in place, with no transpose copy.
 *
 *   q_strides, k_strides, v_strides, o_strides
 *       host arrays of three element strides each: {batch, head, row} of
 *       the [B,H,S,d] view (d contiguous).  For BTNH data [B,T,N,d] they
 *       are {T*N*d, d, N*d}.  Every stride is positive and its byte size a
 *       multiple of 16, else SDPA_ERR_INVALID_ARG.  The library reads the
 *       arrays during the call only.
 *   lse  stays contiguous [B,Hq,Sq] float32 (or NULL).
 *
 * The other arguments, results and errors are those of sdpa_fwd.  O must
 * not overlap Q, K or V.
 */
SDPA_API int sdpa_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse,
                              int B, int Hq, int Hkv, int Sq, int Sk, int d,
                              const long long* q_strides, const long long* k_strides,
                              const long long* v_strides, const long long* o_strides,
                              float scale, int causal, int dtype, void* stream);

/*
 * sdpa_fwd_fp8 -- the same forward with FP8 E4M3 ("fn", max 448) Q/K/V.
 *
 * The codelab runs attention in E4M3 for the forward pass with per-tensor
 * scaling factors (section 10, "Check the FP8 path").  Here the scaling is
 * per tensor and current: the caller quantises x8 = e4m3(x / descale_x) with
 * descale_x = amax(|x|) / 448 and passes descale_x, so the value a code
 * stands for is code * descale_x.
 *
 *   q8, k8, v8       e4m3 codes, layouts as above
 *   descale_q/k/v    host floats, > 0 and finite
 *   o                bf16 [B,Hq,Sq,d]
 *   lse              float32 [B,Hq,Sq] or NULL
 *
 * The softmax weights are themselves quantised to e4m3 for the P*V product,
 * by the amax rule: against a reference max m_ref that is moved only when a
 * tile's scores exceed it by more than 4 (log2 units), a weight is
 * 2^(s - m_ref) <= 2^4 and is stored as e4m3(448 * 2^-4 * 2^(s - m_ref)), so
 * that the largest possible weight maps to 448; the product is multiplied
 * back by descale_v and divided by the fp32 row sum of the same scaled
 * weights.
 * Errors as sdpa_fwd; d must be 128 (SDPA_ERR_UNSUPPORTED otherwise).
 */
SDPA_API int sdpa_fwd_fp8(const void* q8, const void* k8, const void* v8,
                 float descale_q, float descale_k, float descale_v,
                 void* o, float* lse,
                 int B, int Hq, int Hkv, int Sq, int Sk, int d,
                 float scale, int causal, void* stream);

/*
 * sdpa_bwd -- gradients of sdpa_fwd: dQ, dK, dV for the loss whose gradient
 * with respect to O is dout (article "Self-attention, CUDA kernels and
 * FlashAttention", section 3: the weights are recomputed from the kept
 * per-row statistics instead of being stored).
 *
 *   q, o, dout, dq  [B,Hq,Sq,d]  dtype, contiguous (dq written)
 *   k, v, dk, dv    [B,Hkv,Sk,d] dtype, contiguous (dk, dv written; for GQA
 *                   summed over the query heads sharing each K/V head)
 *   lse             [B,Hq,Sq] float32 as written by sdpa_fwd for the same
 *                   q, k, v, scale and causal (required)
 *   delta           [B,Hq,Sq] float32 workspace, device memory owned by the
 *                   caller, 4-byte aligned; the call overwrites it (for head
 *                   dims 64 and 128 it holds D_i = dO_i . O_i on return, for
 *                   32 its contents are unspecified)
 *   other arguments as sdpa_fwd.
 *
 * Two kernel launches (rows-major for dQ, which also writes D to delta, then
 * keys-major for dK/dV, which reads it), each output element written once:
 * deterministic.  The library allocates nothing.  Arithmetic is fp32.
 * Errors as sdpa_fwd, plus SDPA_ERR_INVALID_ARG for a null dout, lse, dq,
 * dk, dv or delta, a misaligned delta, and B*Hq above 65535.
 */
SDPA_API int sdpa_bwd(const void* q, const void* k, const void* v, const void* o,
                      const void* dout, const float* lse, void* dq, void* dk, void* dv,
                      float* delta, int B, int Hq, int Hkv, int Sq, int Sk, int d,
                      float scale, int causal, int dtype, void* stream);

/*
 * sdpa_bwd_fp8 -- gradients of sdpa_fwd_fp8 under the codelab's FP8 hybrid
 * recipe ("JAX on GPU, Lab 5: attention on GPU", section 10: E4M3 for the
 * forward tensors, E5M2 for the gradients): E4M3 Q/K/V codes with their
 * per-tensor descales (as passed to sdpa_fwd_fp8), the forward's bf16 O and
 * fp32 LSE, and the output gradient as E5M2 codes with its own per-tensor
 * descale (current scaling: descale_do = amax(|dO|) / 57344).  The weights are
 * recomputed from LSE (article "Self-attention, CUDA kernels and
 * FlashAttention", section 3).
 *
 *   q8               E4M3 [B,Hq,Sq,d];  k8, v8  E4M3 [B,Hkv,Sk,d]
 *   o                bf16 [B,Hq,Sq,d], lse float32 [B,Hq,Sq] (sdpa_fwd_fp8's)
 *   dout8            E5M2 [B,Hq,Sq,d]
 *   descale_q/k/v/do host floats, > 0 and finite
 *   dq               bf16 [B,Hq,Sq,d];  dk, dv  bf16 [B,Hkv,Sk,d] (out; for GQA
 *                    summed over the query heads sharing each K/V head)
 *   workspace        device memory owned by the caller, 256-byte aligned, at
 *                    least sdpa_bwd_fp8_workspace_bytes(B, Hq, Hkv, Sq, Sk, d)
 *                    bytes; overwritten
 *   d                128
 *
 * Three launches: the codes are widened exactly to bf16 into the workspace
 * (both formats' values are bf16 values), then the two tensor-core backward
 * kernels of sdpa_bwd run on them with the descales folded into the score
 * scale and into their output multipliers, so no value is rounded twice; P
 * and dS are rounded to bf16 for their products, accumulation is fp32.
 * Deterministic.  Errors as sdpa_bwd, plus SDPA_ERR_INVALID_ARG for a
 * non-positive or non-finite descale, a null or misaligned workspace or one
 * smaller than required, and SDPA_ERR_UNSUPPORTED for d != 128.
 */
SDPA_API size_t sdpa_bwd_fp8_workspace_bytes(int B, int Hq, int Hkv, int Sq, int Sk, int d);
SDPA_API int sdpa_bwd_fp8(const void* q8, const void* k8, const void* v8, const void* o,
                          const void* dout8, const float* lse, float descale_q, float descale_k,
                          float descale_v, float descale_do, void* dq, void* dk, void* dv,
                          void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv,
                          int Sq, int Sk, int d, float scale, int causal, void* stream);

/*
 * sdpa_bwd_noalloc -- sdpa_bwd without the delta argument, for callers that
 * cannot allocate device memory: code running inside a host framework that
 * owns every device allocation and lends none to its extensions, or code on
 * a path that must not call cudaMalloc / cudaFree because those calls can
 * synchronise the device.  The article and the codelab have no counterpart
 * to it: it changes where the backward's workspace lives, not what it
 * computes.
 *
 * The workspace (D_i = dO_i . O_i, one float per query row) is a static
 * device array of SDPA_BWD_NOALLOC_MAX_ROWS floats (8 MiB), which every GPU
 * that loads the library holds until the process exits.  Arguments, outputs
 * and errors as sdpa_bwd, plus SDPA_ERR_SCRATCH_LIMIT, with nothing launched,
 * when B*Hq*Sq is above SDPA_BWD_NOALLOC_MAX_ROWS.  The call allocates
 * nothing.
 *
 * The array belongs to the library's device code, which the CUDA runtime
 * loads into a device's context on the first call of any library entry point
 * on that device (lazy module loading, the default since CUDA 12): that load
 * places the array in device memory and may synchronise the device.  Make one
 * call on each device before entering a region that must not allocate or
 * synchronise (a stream capture included).  Every call looks the array's
 * address up in the current context, so a context recreated in between
 * (cudaDeviceReset) is followed correctly.
 * All calls on a device share the one array, which keeps the D values of the
 * last call: nothing in it has to start at zero, since every call writes each
 * row's D before reading it.  Calls whose kernels overlap on the GPU (on
 * streams with no order between them) race on the array and give wrong
 * gradients: order them on one stream, or with events.
 */
#define SDPA_BWD_NOALLOC_MAX_ROWS (1 << 21)
SDPA_API int sdpa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                              const void* dout, const float* lse, void* dq, void* dk,
                              void* dv, int B, int Hq, int Hkv, int Sq, int Sk, int d,
                              float scale, int causal, int dtype, void* stream);

/* Static, NUL-terminated description of a status code. */
SDPA_API const char* sdpa_strerror(int status);

/*
 * sdpa_device_status -- read (and with clear != 0, reset) the device status
 * word of the current device.  The kernels never trap: a wait that does not
 * complete within about one second stops the kernel and records
 * SDPA_ERR_DEVICE_TIMEOUT here; a kernel whose shared-memory layout does not
 * fit at the base address it was given computes nothing and records
 * SDPA_ERR_DEVICE_LAYOUT.  *status receives SDPA_OK or one of those codes and
 * *detail a kernel-specific location code (0 when none).  This call
 * synchronises the current device.  Returns SDPA_OK or SDPA_ERR_CUDA.
 */
SDPA_API int sdpa_device_status(int* status, int* detail, int clear);

/* Number of kernel launches sdpa_fwd / sdpa_fwd_strided / sdpa_fwd_fp8 issue
 * per call (1); sdpa_bwd and sdpa_bwd_noalloc issue 2, sdpa_bwd_fp8 3. */
SDPA_API int sdpa_launches_per_call(void);

/*
 * Self-tests of the kernels' device-side machinery.  They are not part of the
 * attention path; the library's test suite calls them to check, on the GPU,
 * behaviour that the attention kernels only show when something goes wrong
 * or that sits deep inside them.
 *
 * sdpa_selftest_wait -- runs the attention kernels' bounded-wait path (the
 * forward kernel's) on an mbarrier that nothing ever completes: one CTA, two
 * warps.  Warp 0 waits with a limit of limit_us microseconds, gives up,
 * raises the CTA's abort flag and records SDPA_ERR_DEVICE_TIMEOUT with
 * location code 0x7e000 in the device status word (read it with
 * sdpa_device_status); warp 1 waits on the same barrier with the kernels'
 * full one-second limit and must give up as soon as it sees the abort flag.
 * No trap, no fault: the kernel returns and the context stays usable.
 *   limit_us  1 .. 1000000
 *   out       device memory, 4 x uint32, 4-byte aligned: warp 0's wait result
 *             (0 = gave up), the abort flag after it (1), warp 1's wait result
 *             (0), the abort flag warp 1 saw (1)
 * Returns SDPA_OK after the launch, SDPA_ERR_INVALID_ARG for a null or
 * misaligned out or a limit outside the range, SDPA_ERR_UNSUPPORTED off
 * sm_100, SDPA_ERR_CUDA for a launch error.
 *
 * sdpa_selftest_exp2 -- evaluates 2^x for n floats x (device memory, x in
 * [-126, 64]) both with the FMA-pipe polynomial the softmax can use for part
 * of its exponentials (range reduction to [-1/2, 1/2] by rounding, a cubic
 * fitted to the relative error of 2^f, the exponent added to the result's
 * bits) and with the MUFU instruction ex2.approx; results to poly and mufu
 * (device memory, n floats each).  Errors as sdpa_selftest_wait.
 */
/*
 * sdpa_selftest_fastdiv -- host only, needs no GPU: q[i] = floor(n[i] / d[i])
 * for count pairs (host memory, n[i] >= 0, d[i] >= 1) by the multiply-and-
 * shift division the forward's schedule decodes its units with (a magic
 * number m = ceil(2^(31+l) / d), l = ceil(log2 d), computed on the host;
 * q = (n m) >> (31 + l); Granlund and Montgomery 1994, Theorem 4.2).
 * SDPA_ERR_INVALID_ARG for a null pointer, count < 0 or a pair out of range
 * (q is then filled up to that pair).
 */
SDPA_API int sdpa_selftest_wait(unsigned int limit_us, unsigned int* out, void* stream);
SDPA_API int sdpa_selftest_exp2(const float* x, float* poly, float* mufu, int n, void* stream);
SDPA_API int sdpa_selftest_fastdiv(const int* n, const int* d, int count, int* q);

#ifdef __cplusplus
}
#endif

#endif /* SDPA_B200_H */
