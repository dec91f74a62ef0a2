/*
 * swa_oracle.c -- plain fp64 CPU oracle for causal sliding-window attention.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this library. The CUDA product path never calls
 * it, and it shares no code, header or constant with the CUDA path.
 *
 * What it computes (the definition, written out with no blocking, fusion or
 * reordering):
 *
 *   The nanochat GPT calls attention as flash_attn_func(q, k, v, causal=True,
 *   window_size=...) (apidog guide "Train your own ChatGPT", section 5 "Flash
 *   Attention unification"), alternating short and long windows per layer
 *   ("SSSL", same guide, section 1 "GPT model", architecture features).  The
 *   window convention used here: query i attends to key j iff i-W < j <= i,
 *   and W >= T is full causal attention.  So row i has n_i = min(i+1, W) keys.
 *
 *   Forward, per (b, h, i):
 *     S_ij  = s * <q_i, k_j>            for j in band(i)
 *     m_i   = max_j S_ij
 *     l_i   = sum_j exp(S_ij - m_i)
 *     P_ij  = exp(S_ij - m_i) / l_i
 *     O_i   = sum_j P_ij v_j
 *     lse_i = m_i + ln(l_i)             (natural log)
 *
 *   Backward (gradient of sum(dO * O)), per (b, h):
 *     Delta_i = sum_d dO_id O_id
 *     dP_ij   = <dO_i, v_j>
 *     dS_ij   = P_ij (dP_ij - Delta_i)
 *     dQ_i    = s * sum_j dS_ij k_j
 *     dK_j    = s * sum_i dS_ij q_i
 *     dV_j    = sum_i P_ij dO_i
 *
 *   Decode over a KV cache (the inference engine's KV cache, same guide,
 *   section 6 "Inference engine"): sequence b holds L = cache_len[b] tokens;
 *   its query sits at position L-1 and attends to cache slots
 *   max(0, L-W) .. L-1.  The result is row L-1 of the forward above.
 *
 * Grouped K/V heads (the GPT config's n_kv_head, same guide, section 1): K and V
 * have Hk heads, Hk dividing H, and query head h reads K/V head h / (H / Hk), so
 * H / Hk consecutive query heads share one K/V head; dK and dV of a K/V head sum
 * over its query heads.  Hk = H is plain multi-head attention.
 *
 * Layouts: q, dO, o, dq are [B, T, H, D] row-major; k, v, dk, dv are
 * [B, T, Hk, D]; lse is [B, H, T].  Decode: q, o are [B, H, D]; caches
 * [B, cap, Hk, D]; lse [B, H].
 * Inputs are either bf16 bit patterns (uint16, widened exactly to double) or
 * doubles, selected by `in_bf16`.  Outputs are always double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_f64(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double ld(const void *p, int in_bf16, size_t i) {
    return in_bf16 ? bf16_to_f64(((const uint16_t *)p)[i]) : ((const double *)p)[i];
}

/* Element (b, t, h, d) of a [B, T, H, D] tensor. */
static size_t at4(long T, long H, long D, long b, long t, long h, long d) {
    return (((size_t)b * T + t) * H + h) * D + d;
}

/* First key of the band of query i: max(0, i - W + 1). */
static long band_lo(long i, long W) {
    long lo = i - W + 1;
    return lo < 0 ? 0 : lo;
}

/*
 * One query row: scores, softmax and output.  Fills p[j - lo] = P_ij for
 * j in [lo, i] and returns o_i (length D) and lse_i.
 */
static void row_forward(const void *q, const void *k, const void *v, int in_bf16,
                        long T, long H, long Hk, long D, long W, double scale,
                        long b, long h, long i, double *p, double *o_i, double *lse_i) {
    long hk = h / (H / Hk);
    long lo = band_lo(i, W);
    long n = i - lo + 1;
    double m = -INFINITY;
    for (long j = lo; j <= i; ++j) {
        double s = 0.0;
        for (long d = 0; d < D; ++d)
            s += ld(q, in_bf16, at4(T, H, D, b, i, h, d)) * ld(k, in_bf16, at4(T, Hk, D, b, j, hk, d));
        s *= scale;
        p[j - lo] = s;
        if (s > m) m = s;
    }
    double l = 0.0;
    for (long c = 0; c < n; ++c) {
        p[c] = exp(p[c] - m);
        l += p[c];
    }
    for (long c = 0; c < n; ++c) p[c] /= l;
    for (long d = 0; d < D; ++d) {
        double acc = 0.0;
        for (long j = lo; j <= i; ++j) acc += p[j - lo] * ld(v, in_bf16, at4(T, Hk, D, b, j, hk, d));
        o_i[d] = acc;
    }
    *lse_i = m + log(l);
}

/* Full forward: o [B,T,H,D], lse [B,H,T]. */
void swa_oracle_fwd(const void *q, const void *k, const void *v, int in_bf16,
                    long B, long T, long H, long Hk, long D, long W, double scale,
                    double *o, double *lse) {
    #pragma omp parallel for collapse(2) schedule(dynamic)
    for (long b = 0; b < B; ++b) {
        for (long h = 0; h < H; ++h) {
            double *p = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
            for (long i = 0; i < T; ++i)
                row_forward(q, k, v, in_bf16, T, H, Hk, D, W, scale, b, h, i, p,
                            &o[at4(T, H, D, b, i, h, 0)], &lse[((size_t)b * H + h) * T + i]);
            free(p);
        }
    }
}

/* Forward for n selected rows; idx holds (b, h, i) triplets.  o [n, D], lse [n]. */
void swa_oracle_fwd_rows(const void *q, const void *k, const void *v, int in_bf16,
                         long B, long T, long H, long Hk, long D, long W, double scale,
                         long n, const long *idx, double *o, double *lse) {
    (void)B;
    #pragma omp parallel for schedule(dynamic)
    for (long r = 0; r < n; ++r) {
        double *p = (double *)malloc(sizeof(double) * (size_t)T);
        row_forward(q, k, v, in_bf16, T, H, Hk, D, W, scale, idx[3 * r], idx[3 * r + 1], idx[3 * r + 2],
                    p, &o[(size_t)r * D], &lse[r]);
        free(p);
    }
}

/*
 * Full backward: dq [B,T,H,D], dk, dv [B,T,Hk,D].  O and Delta are the
 * oracle's own (recomputed here in fp64 from q, k, v).  One task per
 * (b, K/V head) walks that head's query heads, so dk and dv accumulate in one
 * thread.
 */
void swa_oracle_bwd(const void *q, const void *k, const void *v, const void *dout, int in_bf16,
                    long B, long T, long H, long Hk, long D, long W, double scale,
                    double *dq, double *dk, double *dv) {
    memset(dq, 0, (size_t)B * T * H * D * sizeof(double));
    memset(dk, 0, (size_t)B * T * Hk * D * sizeof(double));
    memset(dv, 0, (size_t)B * T * Hk * D * sizeof(double));
    long G = H / Hk;
    #pragma omp parallel for collapse(2) schedule(dynamic)
    for (long b = 0; b < B; ++b) {
        for (long hk = 0; hk < Hk; ++hk) {
            double *p = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
            double *o_i = (double *)malloc(sizeof(double) * (size_t)D);
            for (long h = hk * G; h < (hk + 1) * G; ++h) {
                for (long i = 0; i < T; ++i) {
                    double lse_i;
                    row_forward(q, k, v, in_bf16, T, H, Hk, D, W, scale, b, h, i, p, o_i, &lse_i);
                    double delta = 0.0;
                    for (long d = 0; d < D; ++d) delta += ld(dout, in_bf16, at4(T, H, D, b, i, h, d)) * o_i[d];
                    long lo = band_lo(i, W);
                    for (long j = lo; j <= i; ++j) {
                        double dp = 0.0;
                        for (long d = 0; d < D; ++d)
                            dp += ld(dout, in_bf16, at4(T, H, D, b, i, h, d)) *
                                  ld(v, in_bf16, at4(T, Hk, D, b, j, hk, d));
                        double pij = p[j - lo];
                        double ds = pij * (dp - delta);
                        for (long d = 0; d < D; ++d) {
                            dq[at4(T, H, D, b, i, h, d)] += scale * ds * ld(k, in_bf16, at4(T, Hk, D, b, j, hk, d));
                            dk[at4(T, Hk, D, b, j, hk, d)] += scale * ds * ld(q, in_bf16, at4(T, H, D, b, i, h, d));
                            dv[at4(T, Hk, D, b, j, hk, d)] += pij * ld(dout, in_bf16, at4(T, H, D, b, i, h, d));
                        }
                    }
                }
            }
            free(o_i);
            free(p);
        }
    }
}

/* dQ for n selected query rows (b, h, i): dq [n, D]. */
void swa_oracle_dq_rows(const void *q, const void *k, const void *v, const void *dout, int in_bf16,
                        long B, long T, long H, long Hk, long D, long W, double scale,
                        long n, const long *idx, double *dq) {
    (void)B;
    #pragma omp parallel for schedule(dynamic)
    for (long r = 0; r < n; ++r) {
        long b = idx[3 * r], h = idx[3 * r + 1], i = idx[3 * r + 2];
        double *p = (double *)malloc(sizeof(double) * (size_t)T);
        double *o_i = (double *)malloc(sizeof(double) * (size_t)D);
        double lse_i;
        row_forward(q, k, v, in_bf16, T, H, Hk, D, W, scale, b, h, i, p, o_i, &lse_i);
        long hk = h / (H / Hk);
        double delta = 0.0;
        for (long d = 0; d < D; ++d) delta += ld(dout, in_bf16, at4(T, H, D, b, i, h, d)) * o_i[d];
        double *out = &dq[(size_t)r * D];
        for (long d = 0; d < D; ++d) out[d] = 0.0;
        long lo = band_lo(i, W);
        for (long j = lo; j <= i; ++j) {
            double dp = 0.0;
            for (long d = 0; d < D; ++d)
                dp += ld(dout, in_bf16, at4(T, H, D, b, i, h, d)) * ld(v, in_bf16, at4(T, Hk, D, b, j, hk, d));
            double ds = p[j - lo] * (dp - delta);
            for (long d = 0; d < D; ++d) out[d] += scale * ds * ld(k, in_bf16, at4(T, Hk, D, b, j, hk, d));
        }
        free(o_i);
        free(p);
    }
}

/*
 * dK and dV for n selected key rows (b, hk, j) of K/V head hk: dk, dv [n, D].
 * Key j is in the band of queries i = j .. min(T-1, j+W-1) of every query head
 * of the group; each such row's softmax is recomputed in full.
 */
void swa_oracle_dkv_rows(const void *q, const void *k, const void *v, const void *dout, int in_bf16,
                         long B, long T, long H, long Hk, long D, long W, double scale,
                         long n, const long *idx, double *dk, double *dv) {
    (void)B;
    long G = H / Hk;
    #pragma omp parallel for schedule(dynamic)
    for (long r = 0; r < n; ++r) {
        long b = idx[3 * r], hk = idx[3 * r + 1], j = idx[3 * r + 2];
        double *p = (double *)malloc(sizeof(double) * (size_t)T);
        double *o_i = (double *)malloc(sizeof(double) * (size_t)D);
        double *dk_r = &dk[(size_t)r * D], *dv_r = &dv[(size_t)r * D];
        for (long d = 0; d < D; ++d) dk_r[d] = dv_r[d] = 0.0;
        long last = j + W - 1;
        if (last > T - 1) last = T - 1;
        for (long h = hk * G; h < (hk + 1) * G; ++h) {
            for (long i = j; i <= last; ++i) {
                double lse_i;
                row_forward(q, k, v, in_bf16, T, H, Hk, D, W, scale, b, h, i, p, o_i, &lse_i);
                double delta = 0.0, dp = 0.0;
                for (long d = 0; d < D; ++d) {
                    delta += ld(dout, in_bf16, at4(T, H, D, b, i, h, d)) * o_i[d];
                    dp += ld(dout, in_bf16, at4(T, H, D, b, i, h, d)) * ld(v, in_bf16, at4(T, Hk, D, b, j, hk, d));
                }
                double pij = p[j - band_lo(i, W)];
                double ds = pij * (dp - delta);
                for (long d = 0; d < D; ++d) {
                    dk_r[d] += scale * ds * ld(q, in_bf16, at4(T, H, D, b, i, h, d));
                    dv_r[d] += pij * ld(dout, in_bf16, at4(T, H, D, b, i, h, d));
                }
            }
        }
        free(o_i);
        free(p);
    }
}

/*
 * Single-token decode over a KV cache.  q [B,H,D]; k_cache, v_cache
 * [B,cap,Hk,D]; cache_len [B] with values in [1, cap].  o [B,H,D], lse [B,H].
 */
void swa_oracle_decode(const void *q, const void *k_cache, const void *v_cache, int in_bf16,
                       const int *cache_len, long B, long cap, long H, long Hk, long D, long W, double scale,
                       double *o, double *lse) {
    #pragma omp parallel for collapse(2) schedule(dynamic)
    for (long b = 0; b < B; ++b) {
        for (long h = 0; h < H; ++h) {
            long hk = h / (H / Hk);
            long L = cache_len[b];
            long lo = L - W;
            if (lo < 0) lo = 0;
            long n = L - lo;
            double *s = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
            double m = -INFINITY;
            for (long j = lo; j < L; ++j) {
                double acc = 0.0;
                for (long d = 0; d < D; ++d)
                    acc += ld(q, in_bf16, ((size_t)b * H + h) * D + d) *
                           ld(k_cache, in_bf16, at4(cap, Hk, D, b, j, hk, d));
                s[j - lo] = acc * scale;
                if (s[j - lo] > m) m = s[j - lo];
            }
            double l = 0.0;
            for (long c = 0; c < n; ++c) {
                s[c] = exp(s[c] - m);
                l += s[c];
            }
            for (long d = 0; d < D; ++d) {
                double acc = 0.0;
                for (long j = lo; j < L; ++j) acc += s[j - lo] / l * ld(v_cache, in_bf16, at4(cap, Hk, D, b, j, hk, d));
                o[((size_t)b * H + h) * D + d] = acc;
            }
            lse[(size_t)b * H + h] = m + log(l);
            free(s);
        }
    }
}
