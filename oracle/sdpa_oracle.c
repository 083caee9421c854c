/*
 * sdpa_oracle.c -- fp64 CPU oracle for the fused scaled-dot-product attention
 * forward.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline leg may call it; the product path never does, and
 * this file shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (codelab "JAX on GPU, Lab 5: attention on GPU", section 1
 * "How attention works", the formula Attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V
 * and its four steps score -> scale+softmax -> attend -> output of Q's shape;
 * article "Self-attention, CUDA kernels and FlashAttention", section 1, the
 * same formula for one head and "run per head in parallel"):
 *
 *   for every batch b, query head hq, query row i:
 *     hk  = hq / (Hq / Hkv)                         (codelab section 9: KV heads
 *                                                    are shared by groups of
 *                                                    query heads; contiguous groups)
 *     J_i = {0 .. Sk-1}, or {0 .. i} when causal     (codelab section 7: each
 *                                                    position sees earlier ones)
 *           or {0 .. i + Sk - Sq} when causal is 2   (the Sq queries are the last
 *                                                    Sq positions of a sequence of
 *                                                    Sk, as with a KV cache: codelab
 *                                                    section 9 and its closing
 *                                                    suggestions; Sq <= Sk)
 *     s_j = scale * sum_c Q[b,hq,i,c] * K[b,hk,j,c]  for j in J_i
 *     m   = max_j s_j ;  l = sum_j exp(s_j - m)
 *     O[b,hq,i,:] = sum_j exp(s_j - m) / l * V[b,hk,j,:]
 *     LSE[b,hq,i] = m + ln(l)                        (article section 3: only the
 *                                                    small per-row normalisation
 *                                                    statistic is kept; natural log
 *                                                    of the scaled scores)
 *
 * Two passes over the row (max, then exp/sum/accumulate) in fp64; no tiling, no
 * online rescaling.  A second routine materialises the whole score matrix of a
 * head, applies a row softmax and multiplies by V, the structure of the
 * codelab's from-scratch attention (section 4); it serves tiny inputs only.
 *
 * Layouts: Q [B,Hq,Sq,d], K and V [B,Hkv,Sk,d], O [B,Hq,Sq,d], LSE [B,Hq,Sq],
 * all contiguous row-major.  Inputs are read in their storage type and widened
 * exactly to double: bf16, fp16, e4m3 (OCP "fn" variant, times a per-tensor
 * descale) or fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F64 = 0, ORC_BF16 = 1, ORC_F16 = 2, ORC_E4M3 = 3, ORC_E5M2 = 4 };

/* ---- exact widening of the storage formats to double ------------------- */

/* bf16 is the upper half of an IEEE binary32 pattern. */
double oracle_decode_bf16(uint16_t h) {
    uint32_t bits = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
double oracle_decode_f16(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double mag;
    if (e == 0) {
        mag = ldexp((double)f, -24);            /* subnormal: f * 2^-10 * 2^-14 */
    } else if (e == 31) {
        mag = f ? NAN : INFINITY;
    } else {
        mag = ldexp((double)(1024 + f), e - 25); /* (1 + f/1024) * 2^(e-15) */
    }
    return sign ? -mag : mag;
}

/* OCP FP8 E4M3 ("fn": finite, no infinities): 1 sign, 4 exponent (bias 7),
 * 3 fraction bits; S.1111.111 is NaN, the largest finite is 448. */
double oracle_decode_e4m3(uint8_t c) {
    int sign = (c >> 7) & 1;
    int e = (c >> 3) & 0xf;
    int f = c & 0x7;
    double mag;
    if (e == 15 && f == 7) {
        mag = NAN;
    } else if (e == 0) {
        mag = ldexp((double)f, -9);             /* subnormal: f/8 * 2^-6 */
    } else {
        mag = ldexp((double)(8 + f), e - 10);   /* (1 + f/8) * 2^(e-7) */
    }
    return sign ? -mag : mag;
}

/* OCP FP8 E5M2: 1 sign, 5 exponent (bias 15), 2 fraction bits; IEEE-like,
 * exponent 31 holds the infinities and NaNs; the largest finite is 57344. */
double oracle_decode_e5m2(uint8_t c) {
    int sign = (c >> 7) & 1;
    int e = (c >> 2) & 0x1f;
    int f = c & 0x3;
    double mag;
    if (e == 31) {
        mag = f ? NAN : INFINITY;
    } else if (e == 0) {
        mag = ldexp((double)f, -16);            /* subnormal: f/4 * 2^-14 */
    } else {
        mag = ldexp((double)(4 + f), e - 17);   /* (1 + f/4) * 2^(e-15) */
    }
    return sign ? -mag : mag;
}

static double load_elem(const void* base, int dtype, size_t idx, double descale) {
    switch (dtype) {
    case ORC_BF16: return oracle_decode_bf16(((const uint16_t*)base)[idx]);
    case ORC_F16:  return oracle_decode_f16(((const uint16_t*)base)[idx]);
    case ORC_E4M3: return oracle_decode_e4m3(((const uint8_t*)base)[idx]) * descale;
    case ORC_E5M2: return oracle_decode_e5m2(((const uint8_t*)base)[idx]) * descale;
    default:       return ((const double*)base)[idx];
    }
}

typedef struct {
    const void *q, *k, *v;
    int dtype;
    double dq, dk, dv;
    int B, Hq, Hkv, Sq, Sk, d;
    double scale;
    int causal;
} problem_t;

static int check_problem(const problem_t* p) {
    if (!p->q || !p->k || !p->v) return 1;
    if (p->B <= 0 || p->Hq <= 0 || p->Hkv <= 0 || p->Sq <= 0 || p->Sk <= 0 || p->d <= 0) return 1;
    if (p->Hq % p->Hkv != 0) return 1;
    if (p->causal < 0 || p->causal > 2) return 1;
    if (p->causal == 1 && p->Sq != p->Sk) return 2;
    if (p->causal == 2 && p->Sq > p->Sk) return 2;
    if (p->dtype < ORC_F64 || p->dtype > ORC_E4M3) return 1;
    return 0;
}

/* One output row (b, hq, i).  `work` holds Sk doubles. */
static void one_row(const problem_t* p, int b, int hq, int i, double* work,
                    double* o_row, double* lse_out) {
    const int group = p->Hq / p->Hkv;
    const int hk = hq / group;
    const size_t qoff = (((size_t)b * p->Hq + hq) * p->Sq + i) * p->d;
    const size_t kvhead = ((size_t)b * p->Hkv + hk) * p->Sk;
    /* keys 0 .. last visible: all, the diagonal, or the diagonal shifted by
       Sk - Sq (queries aligned to the end of the key sequence) */
    const int nkeys = p->causal == 1 ? i + 1 : p->causal == 2 ? i + 1 + (p->Sk - p->Sq) : p->Sk;

    /* score step: s_j = scale * q_i . k_j */
    double m = -INFINITY;
    for (int j = 0; j < nkeys; ++j) {
        const size_t koff = (kvhead + j) * p->d;
        double acc = 0.0;
        for (int c = 0; c < p->d; ++c)
            acc += load_elem(p->q, p->dtype, qoff + c, p->dq) *
                   load_elem(p->k, p->dtype, koff + c, p->dk);
        work[j] = p->scale * acc;
        if (work[j] > m) m = work[j];
    }
    /* softmax step (second pass) and attend step */
    double l = 0.0;
    for (int c = 0; c < p->d; ++c) o_row[c] = 0.0;
    for (int j = 0; j < nkeys; ++j) {
        const double w = exp(work[j] - m);
        l += w;
        const size_t voff = (kvhead + j) * p->d;
        for (int c = 0; c < p->d; ++c)
            o_row[c] += w * load_elem(p->v, p->dtype, voff + c, p->dv);
    }
    for (int c = 0; c < p->d; ++c) o_row[c] /= l;
    *lse_out = m + log(l);
}

/*
 * Full forward.  o: [B,Hq,Sq,d] doubles, lse: [B,Hq,Sq] doubles.
 * Returns 0 on success, 1 for invalid arguments, 2 for causal 1 with Sq != Sk
 * or causal 2 with Sq > Sk.
 */
int oracle_sdpa_fwd(const void* q, const void* k, const void* v, int dtype,
                    double dq, double dk, double dv, double* o, double* lse,
                    int B, int Hq, int Hkv, int Sq, int Sk, int d,
                    double scale, int causal, int nthreads) {
    problem_t p = {q, k, v, dtype, dq, dk, dv, B, Hq, Hkv, Sq, Sk, d, scale, causal};
    int rc = check_problem(&p);
    if (rc) return rc;
    if (!o || !lse) return 1;
    const long long nrows = (long long)B * Hq * Sq;
    if (nthreads <= 0) nthreads = 1;
    int failed = 0;
#pragma omp parallel num_threads(nthreads)
    {
        double* work = (double*)malloc(sizeof(double) * (size_t)Sk);
        if (!work) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (long long r = 0; r < nrows; ++r) {
                const int i = (int)(r % Sq);
                const int hq = (int)((r / Sq) % Hq);
                const int b = (int)(r / ((long long)Sq * Hq));
                one_row(&p, b, hq, i, work, o + (size_t)r * d, lse + r);
            }
            free(work);
        }
    }
    return failed ? 3 : 0;
}

/*
 * Selected rows only: rows[t] is the flat row index (b*Hq + hq)*Sq + i.
 * o_rows: [nrows, d], lse_rows: [nrows].  Used where the full problem is too
 * large for the CPU (the output of every row depends on its own row only).
 */
int oracle_sdpa_rows(const void* q, const void* k, const void* v, int dtype,
                     double dq, double dk, double dv,
                     const int64_t* rows, int64_t nrows, double* o_rows, double* lse_rows,
                     int B, int Hq, int Hkv, int Sq, int Sk, int d,
                     double scale, int causal, int nthreads) {
    problem_t p = {q, k, v, dtype, dq, dk, dv, B, Hq, Hkv, Sq, Sk, d, scale, causal};
    int rc = check_problem(&p);
    if (rc) return rc;
    if (!rows || !o_rows || !lse_rows || nrows < 0) return 1;
    const long long total = (long long)B * Hq * Sq;
    for (int64_t t = 0; t < nrows; ++t)
        if (rows[t] < 0 || rows[t] >= total) return 1;
    if (nthreads <= 0) nthreads = 1;
    int failed = 0;
#pragma omp parallel num_threads(nthreads)
    {
        double* work = (double*)malloc(sizeof(double) * (size_t)Sk);
        if (!work) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t t = 0; t < nrows; ++t) {
                const long long r = rows[t];
                const int i = (int)(r % Sq);
                const int hq = (int)((r / Sq) % Hq);
                const int b = (int)(r / ((long long)Sq * Hq));
                one_row(&p, b, hq, i, work, o_rows + (size_t)t * d, lse_rows + t);
            }
            free(work);
        }
    }
    return failed ? 3 : 0;
}

/*
 * Brute force, the explicit-matrix structure of the codelab's from-scratch
 * attention (section 4): per head, build the whole Sq x Sk score matrix
 * (masked entries = -inf), scale it, apply a row softmax in place (weights),
 * then multiply the weight matrix by V.  The weights are also returned when
 * `weights` is non-null ([B,Hq,Sq,Sk]).  Meant for tiny inputs.
 */
int oracle_sdpa_bruteforce(const void* q, const void* k, const void* v, int dtype,
                           double dq, double dk, double dv, double* o, double* lse,
                           double* weights,
                           int B, int Hq, int Hkv, int Sq, int Sk, int d,
                           double scale, int causal) {
    problem_t p = {q, k, v, dtype, dq, dk, dv, B, Hq, Hkv, Sq, Sk, d, scale, causal};
    int rc = check_problem(&p);
    if (rc) return rc;
    if (!o || !lse) return 1;
    double* S = (double*)malloc(sizeof(double) * (size_t)Sq * Sk);
    if (!S) return 3;
    const int group = Hq / Hkv;
    for (int b = 0; b < B; ++b) {
        for (int hq = 0; hq < Hq; ++hq) {
            const int hk = hq / group;
            const size_t qh = ((size_t)b * Hq + hq) * Sq;
            const size_t kh = ((size_t)b * Hkv + hk) * Sk;
            /* scores = (Q K^T) * scale; masked entries (above the diagonal,
               shifted by Sk - Sq when causal is 2) -inf */
            for (int i = 0; i < Sq; ++i)
                for (int j = 0; j < Sk; ++j) {
                    double acc = 0.0;
                    for (int c = 0; c < d; ++c)
                        acc += load_elem(q, dtype, (qh + i) * d + c, dq) *
                               load_elem(k, dtype, (kh + j) * d + c, dk);
                    const int last = causal == 2 ? i + Sk - Sq : i;
                    S[(size_t)i * Sk + j] = (causal && j > last) ? -INFINITY : acc * scale;
                }
            /* row softmax in place; keep each row's log normaliser */
            for (int i = 0; i < Sq; ++i) {
                double* row = S + (size_t)i * Sk;
                double m = -INFINITY;
                for (int j = 0; j < Sk; ++j) m = row[j] > m ? row[j] : m;
                double l = 0.0;
                for (int j = 0; j < Sk; ++j) { row[j] = exp(row[j] - m); l += row[j]; }
                for (int j = 0; j < Sk; ++j) row[j] /= l;
                lse[qh + i] = m + log(l);
            }
            if (weights)
                memcpy(weights + qh * (size_t)Sk, S, sizeof(double) * (size_t)Sq * Sk);
            /* weights @ V */
            for (int i = 0; i < Sq; ++i)
                for (int c = 0; c < d; ++c) {
                    double acc = 0.0;
                    for (int j = 0; j < Sk; ++j)
                        acc += S[(size_t)i * Sk + j] * load_elem(v, dtype, (kh + j) * d + c, dv);
                    o[(qh + i) * d + c] = acc;
                }
        }
    }
    free(S);
    return 0;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Backward of the same forward: given dO = dL/dO for a loss L, the gradients
 * dL/dQ, dL/dK, dL/dV (codelab section 12 suggests training with these
 * kernels; the article's section 3 keeps the per-row statistics so that the
 * backward can recompute the weights).  For every (b, hq, i), with the
 * weights p_j of the forward (recomputed here in fp64, two-pass):
 *
 *   dp_j = dO_i . V_j                      (gradient of the weights)
 *   D_i  = sum_j p_j dp_j                  (= dO_i . O_i)
 *   ds_j = p_j (dp_j - D_i)                (softmax Jacobian applied to dp)
 *   dQ_i   = scale * sum_j ds_j K_j
 *   dK_j  += scale * ds_j Q_i              (summed over the rows and over the
 *   dV_j  += p_j dO_i                       query heads sharing K/V head hk)
 *
 * dout has Q's shape and storage type.  dq: [B,Hq,Sq,d], dk, dv: [B,Hkv,Sk,d]
 * doubles.  Work is split by (b, hk), so every dK/dV row has one writer.
 */
static int bwd_impl(const void* q, const void* k, const void* v, const void* dout, int dtype,
                    int dout_dtype, double dsq, double dsk, double dsv, double dsdo,
                    double* dq_out, double* dk_out, double* dv_out,
                    int B, int Hq, int Hkv, int Sq, int Sk, int d,
                    double scale, int causal, int nthreads) {
    problem_t p = {q, k, v, dtype, dsq, dsk, dsv, B, Hq, Hkv, Sq, Sk, d, scale, causal};
    int rc = check_problem(&p);
    if (rc) return rc;
    if (!dout || !dq_out || !dk_out || !dv_out) return 1;
    memset(dk_out, 0, sizeof(double) * (size_t)B * Hkv * Sk * d);
    memset(dv_out, 0, sizeof(double) * (size_t)B * Hkv * Sk * d);
    const int group = Hq / Hkv;
    if (nthreads <= 0) nthreads = 1;
    int failed = 0;
#pragma omp parallel num_threads(nthreads)
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)Sk * 2);
        if (!s) {
#pragma omp atomic write
            failed = 1;
        } else {
            double* dp = s + Sk;
#pragma omp for schedule(dynamic, 1)
            for (long long bk = 0; bk < (long long)B * Hkv; ++bk) {
                const int b = (int)(bk / Hkv), hk = (int)(bk % Hkv);
                const size_t kvhead = ((size_t)b * Hkv + hk) * Sk;
                for (int hq = hk * group; hq < (hk + 1) * group; ++hq) {
                    for (int i = 0; i < Sq; ++i) {
                        const size_t qoff = (((size_t)b * Hq + hq) * Sq + i) * d;
                        const int nkeys = causal == 1 ? i + 1 : causal == 2 ? i + 1 + (Sk - Sq) : Sk;
                        double m = -INFINITY;
                        for (int j = 0; j < nkeys; ++j) {
                            double acc = 0.0, accd = 0.0;
                            for (int c = 0; c < d; ++c) {
                                acc += load_elem(q, dtype, qoff + c, dsq) *
                                       load_elem(k, dtype, (kvhead + j) * d + c, dsk);
                                accd += load_elem(dout, dout_dtype, qoff + c, dsdo) *
                                        load_elem(v, dtype, (kvhead + j) * d + c, dsv);
                            }
                            s[j] = scale * acc;
                            dp[j] = accd;
                            if (s[j] > m) m = s[j];
                        }
                        double l = 0.0;
                        for (int j = 0; j < nkeys; ++j) {
                            s[j] = exp(s[j] - m);
                            l += s[j];
                        }
                        double Di = 0.0;
                        for (int j = 0; j < nkeys; ++j) {
                            s[j] /= l;                 /* p_j */
                            Di += s[j] * dp[j];
                        }
                        double* dqi = dq_out + qoff;
                        for (int c = 0; c < d; ++c) dqi[c] = 0.0;
                        for (int j = 0; j < nkeys; ++j) {
                            const double ds = s[j] * (dp[j] - Di);
                            double* dkj = dk_out + (kvhead + j) * d;
                            double* dvj = dv_out + (kvhead + j) * d;
                            for (int c = 0; c < d; ++c) {
                                dqi[c] += scale * ds * load_elem(k, dtype, (kvhead + j) * d + c, dsk);
                                dkj[c] += scale * ds * load_elem(q, dtype, qoff + c, dsq);
                                dvj[c] += s[j] * load_elem(dout, dout_dtype, qoff + c, dsdo);
                            }
                        }
                    }
                }
            }
            free(s);
        }
    }
    return failed ? 3 : 0;
}

/* 16-bit inputs: dout has Q's storage type. */
int oracle_sdpa_bwd(const void* q, const void* k, const void* v, const void* dout, int dtype,
                    double* dq_out, double* dk_out, double* dv_out,
                    int B, int Hq, int Hkv, int Sq, int Sk, int d,
                    double scale, int causal, int nthreads) {
    if (dtype == ORC_E4M3 || dtype == ORC_E5M2) return 1;
    return bwd_impl(q, k, v, dout, dtype, dtype, 1.0, 1.0, 1.0, 1.0, dq_out, dk_out, dv_out,
                    B, Hq, Hkv, Sq, Sk, d, scale, causal, nthreads);
}

/* The FP8 hybrid recipe (codelab section 10: E4M3 for the forward tensors,
 * E5M2 for gradients): Q, K, V as E4M3 codes times their per-tensor
 * descales, dO as E5M2 codes times its descale; the same exact gradients. */
int oracle_sdpa_bwd_fp8(const void* q8, const void* k8, const void* v8, const void* dout8,
                        double descale_q, double descale_k, double descale_v, double descale_do,
                        double* dq_out, double* dk_out, double* dv_out,
                        int B, int Hq, int Hkv, int Sq, int Sk, int d,
                        double scale, int causal, int nthreads) {
    return bwd_impl(q8, k8, v8, dout8, ORC_E4M3, ORC_E5M2, descale_q, descale_k, descale_v,
                    descale_do, dq_out, dk_out, dv_out, B, Hq, Hkv, Sq, Sk, d, scale, causal,
                    nthreads);
}
