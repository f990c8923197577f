/*
 * attn_oracle.c -- plain, slow, fp64 CPU oracle for prefix-masked attention forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this
 * file: only the tests, the package's smoke check and the benchmark's CPU-baseline leg
 * use it.  It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (the plain definition, no blocking, no fusion, no reordering):
 *
 *   For batch element b, head h, query row i, with n = kv_len[b] valid keys:
 *     s_j   = scale * sum_d q[b,h,i,d] * k[b,h,j,d]        for j < n
 *     m     = max_j s_j
 *     l     = sum_{j<n} exp(s_j - m)
 *     out_i = sum_{j<n} exp(s_j - m) * v[b,h,j,:] / l
 *     lse_i = m + ln(l)
 *   and n = 0 gives out_i = 0, lse_i = -inf.
 *
 * Sources (the pages this method is described on):
 *   - "Rewrite prefix key-padding masks as k/v truncation to keep SDPA on the flash path",
 *     sections "Problem" and "Fix": scaled-dot-product attention with a [B,1,1,S] boolean
 *     key-prefix mask, and the statement that masking all keys but the first n is the
 *     same computation as truncating k/v to n rows with no mask.  A ragged n per batch
 *     element is the same computation per element (section "Tests").
 *   - "Add sequence-parallel multi-GPU inference ... and a cuDNN flash attention option",
 *     section "Sequence-parallel inference": partial results over disjoint key shards
 *     combine exactly through their log-sum-exp values (oracle_lse_combine below), and
 *     padded key slots are masked; section "cuDNN flash attention": the boolean prefix
 *     mask is a per-batch count of valid keys (key_value_seq_lengths).
 *   - "Broadcast SDPA attn_mask instead of materializing a per-head copy", section
 *     "What": one mask per batch element serves every head.
 *
 * Readings where the pages are silent (each one applied the same way by every mode):
 *   - lse is the natural logarithm of sum_j exp(scale * q.k_j), scale included;
 *   - n = 0 gives out = 0 and lse = -inf (the pages leave an empty prefix undefined);
 *   - key selection is exact: keys j >= n are never read in truncation mode.
 *
 * Inputs are bf16 bit patterns (uint16); each is widened exactly to double.  All
 * arithmetic is double precision.  Build: gcc -O2 -fopenmp -shared -fPIC (no fast-math).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 is the top 16 bits of an IEEE binary32; widening is a shift, then an exact
 * float -> double conversion. */
static double widen_bf16(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* One query row against keys [j0, j1) of one (b, h) slice.
 * qrow: D values; kbase/vbase: the slice's [Tk, D] key and value rows.
 * s: scratch of at least (j1 - j0) doubles.  Writes out[D] and *lse. */
static void attend_row(const uint16_t* qrow, const uint16_t* kbase, const uint16_t* vbase,
                       long j0, long j1, int D, double scale, double* s,
                       double* out, double* lse) {
    if (j1 <= j0) {
        for (int d = 0; d < D; ++d) out[d] = 0.0;
        *lse = -INFINITY;
        return;
    }
    /* scores */
    double m = -INFINITY;
    for (long j = j0; j < j1; ++j) {
        const uint16_t* krow = kbase + (size_t)j * D;
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += widen_bf16(qrow[d]) * widen_bf16(krow[d]);
        double sj = scale * dot;
        s[j - j0] = sj;
        if (sj > m) m = sj;
    }
    /* softmax weights (unnormalised) and their sum */
    double l = 0.0;
    for (long j = j0; j < j1; ++j) {
        double w = exp(s[j - j0] - m);
        s[j - j0] = w;
        l += w;
    }
    /* weighted sum of value rows, then normalise */
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    for (long j = j0; j < j1; ++j) {
        const uint16_t* vrow = vbase + (size_t)j * D;
        double w = s[j - j0];
        for (int d = 0; d < D; ++d) out[d] += w * widen_bf16(vrow[d]);
    }
    for (int d = 0; d < D; ++d) out[d] /= l;
    *lse = m + log(l);
}

/* Core loop shared by the truncation and chunk entry points: for every (b, h) and every
 * selected query row, attend over keys [max(key_begin,0), min(key_end, kv_len[b])).
 * rows == NULL selects all Tq rows (n_rows must then equal Tq).
 * Returns 0, or -1 on bad arguments / allocation failure. */
static int attend_range(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                        const int32_t* kv_len, int B, int H, int Tq, int Tk, int D,
                        double scale, const int64_t* rows, int n_rows,
                        long key_begin, long key_end, double* out, double* lse) {
    if (!q || !k || !v || !kv_len || !out || !lse) return -1;
    if (B <= 0 || H <= 0 || Tq <= 0 || Tk <= 0 || D <= 0 || n_rows <= 0) return -1;
    if (!rows && n_rows != Tq) return -1;
    for (int b = 0; b < B; ++b)
        if (kv_len[b] < 0 || kv_len[b] > Tk) return -1;
    if (rows)
        for (int r = 0; r < n_rows; ++r)
            if (rows[r] < 0 || rows[r] >= Tq) return -1;

    int failed = 0;
    long total = (long)B * H * n_rows;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)(Tk > 0 ? Tk : 1));
        if (!s) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 4)
        for (long idx = 0; idx < total; ++idx) {
            if (!s) continue;
            int r = (int)(idx % n_rows);
            long bh = idx / n_rows;
            int b = (int)(bh / H);
            long i = rows ? rows[r] : r;
            long n = kv_len[b];
            long j0 = key_begin > 0 ? key_begin : 0;
            long j1 = key_end < n ? key_end : n;
            const uint16_t* qrow = q + ((size_t)bh * Tq + (size_t)i) * D;
            const uint16_t* kbase = k + (size_t)bh * Tk * D;
            const uint16_t* vbase = v + (size_t)bh * Tk * D;
            attend_row(qrow, kbase, vbase, j0, j1, D, scale, s,
                       out + (size_t)idx * D, lse + idx);
        }
        free(s);
    }
    return failed ? -1 : 0;
}

/* Truncation mode (the primary oracle): keys j < kv_len[b] only.
 * q: [B,H,Tq,D], k/v: [B,H,Tk,D] bf16 bits; out: [B,H,n_rows,D]; lse: [B,H,n_rows]. */
int oracle_attn_prefix(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                       const int32_t* kv_len, int B, int H, int Tq, int Tk, int D,
                       double scale, const int64_t* rows, int n_rows,
                       double* out, double* lse) {
    return attend_range(q, k, v, kv_len, B, H, Tq, Tk, D, scale, rows, n_rows,
                        0, (long)Tk, out, lse);
}

/* One key chunk [key_begin, key_end) intersected with the valid prefix: the normalised
 * partial output O_c and its log-sum-exp lse_c, as one shard of the exact combination. */
int oracle_attn_chunk(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                      const int32_t* kv_len, int B, int H, int Tq, int Tk, int D,
                      double scale, const int64_t* rows, int n_rows,
                      long key_begin, long key_end, double* out, double* lse) {
    if (key_begin < 0 || key_end < key_begin) return -1;
    return attend_range(q, k, v, kv_len, B, H, Tq, Tk, D, scale, rows, n_rows,
                        key_begin, key_end, out, lse);
}

/* Dense boolean mask mode: the scaled-dot-product attention of the pages with a
 * [B,1,1,Tk] key mask broadcast over heads and queries.  Every key is scored; masked
 * keys get score -inf, the softmax runs over the whole row, and the weighted sum runs
 * over all Tk value rows.  Meant for finite key/value padding (a non-finite padded
 * value would reach the sum through 0 * value).  An all-false mask row gives NaN, as
 * the definition does.  mask: [B, Tk] bytes, nonzero = key takes part. */
int oracle_attn_masked(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                       const uint8_t* mask, int B, int H, int Tq, int Tk, int D,
                       double scale, double* out, double* lse) {
    if (!q || !k || !v || !mask || !out || !lse) return -1;
    if (B <= 0 || H <= 0 || Tq <= 0 || Tk <= 0 || D <= 0) return -1;
    long total = (long)B * H * Tq;
    int failed = 0;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)Tk);
        if (!s) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 4)
        for (long idx = 0; idx < total; ++idx) {
            if (!s) continue;
            long bh = idx / Tq;
            long i = idx % Tq;
            int b = (int)(bh / H);
            const uint16_t* qrow = q + ((size_t)bh * Tq + (size_t)i) * D;
            const uint16_t* kbase = k + (size_t)bh * Tk * D;
            const uint16_t* vbase = v + (size_t)bh * Tk * D;
            const uint8_t* mrow = mask + (size_t)b * Tk;
            double m = -INFINITY;
            for (long j = 0; j < Tk; ++j) {
                double dot = 0.0;
                for (int d = 0; d < D; ++d)
                    dot += widen_bf16(qrow[d]) * widen_bf16(kbase[(size_t)j * D + d]);
                double sj = mrow[j] ? scale * dot : -INFINITY;
                s[j] = sj;
                if (sj > m) m = sj;
            }
            double l = 0.0;
            for (long j = 0; j < Tk; ++j) {
                s[j] = exp(s[j] - m);
                l += s[j];
            }
            double* o = out + (size_t)idx * D;
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            for (long j = 0; j < Tk; ++j)
                for (int d = 0; d < D; ++d)
                    o[d] += s[j] * widen_bf16(vbase[(size_t)j * D + d]);
            for (int d = 0; d < D; ++d) o[d] /= l;
            lse[idx] = m + log(l);
        }
        free(s);
    }
    return failed ? -1 : 0;
}

/* Exact combination of C partial results over disjoint key ranges:
 *   M = max_c lse_c;  lse = M + ln sum_c exp(lse_c - M);  out = sum_c exp(lse_c - lse) O_c.
 * All partials empty (every lse_c = -inf) gives out = 0, lse = -inf.
 * part_out: [C, rows, D]; part_lse: [C, rows]; out: [rows, D]; lse: [rows]. */
int oracle_lse_combine(const double* part_out, const double* part_lse, int C, long rows,
                       int D, double* out, double* lse) {
    if (!part_out || !part_lse || !out || !lse || C <= 0 || rows <= 0 || D <= 0) return -1;
#pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r) {
        double M = -INFINITY;
        for (int c = 0; c < C; ++c) {
            double x = part_lse[(size_t)c * rows + r];
            if (x > M) M = x;
        }
        double* o = out + (size_t)r * D;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        if (M == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double sum = 0.0;
        for (int c = 0; c < C; ++c) sum += exp(part_lse[(size_t)c * rows + r] - M);
        double L = M + log(sum);
        for (int c = 0; c < C; ++c) {
            double w = exp(part_lse[(size_t)c * rows + r] - L);
            const double* oc = part_out + ((size_t)c * rows + r) * D;
            for (int d = 0; d < D; ++d) o[d] += w * oc[d];
        }
        lse[r] = L;
    }
    return 0;
}

/* Multi-range key mask: batch element b attends to the keys of its S segments,
 *   [seg_start[b*S + s], seg_start[b*S + s] + seg_len[b*S + s]),   s = 0 .. S-1,
 * taken in segment order (the softmax does not depend on the order).  This is the
 * gathered-shards case of "Add sequence-parallel multi-GPU inference ...", section
 * "Sequence-parallel inference": each device's context K/V is gathered with padded key
 * slots, so the valid keys are one range per shard rather than one prefix.
 * Readings where the pages are silent:
 *   - a segment is intersected with [0, Tk); a negative length counts as 0;
 *   - a key that lies in two segments takes part twice (the segments are concatenated);
 *   - the concatenation is cut after Tk keys;
 *   - no valid key gives out = 0 and lse = -inf, as for an empty prefix.
 * Keys outside every segment are never read.  out: [B,H,n_rows,D]; lse: [B,H,n_rows]. */
int oracle_attn_segments(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                         const int32_t* seg_start, const int32_t* seg_len, int S,
                         int B, int H, int Tq, int Tk, int D, double scale,
                         const int64_t* rows, int n_rows, double* out, double* lse) {
    if (!q || !k || !v || !seg_start || !seg_len || !out || !lse) return -1;
    if (S <= 0 || B <= 0 || H <= 0 || Tq <= 0 || Tk <= 0 || D <= 0 || n_rows <= 0) return -1;
    if (!rows && n_rows != Tq) return -1;
    if (rows)
        for (int r = 0; r < n_rows; ++r)
            if (rows[r] < 0 || rows[r] >= Tq) return -1;

    /* the key index list of every batch element */
    long* keys = (long*)malloc(sizeof(long) * (size_t)B * (size_t)Tk);
    long* n_keys = (long*)malloc(sizeof(long) * (size_t)B);
    if (!keys || !n_keys) {
        free(keys);
        free(n_keys);
        return -1;
    }
    for (int b = 0; b < B; ++b) {
        long n = 0;
        for (int s = 0; s < S && n < Tk; ++s) {
            long lo = seg_start[(size_t)b * S + s];
            long len = seg_len[(size_t)b * S + s];
            long hi = len > 0 ? lo + len : lo;
            if (lo < 0) lo = 0;
            if (hi > Tk) hi = Tk;
            for (long j = lo; j < hi && n < Tk; ++j) keys[(size_t)b * Tk + n++] = j;
        }
        n_keys[b] = n;
    }

    int failed = 0;
    long total = (long)B * H * n_rows;
#pragma omp parallel
    {
        double* w = (double*)malloc(sizeof(double) * (size_t)Tk);
        if (!w) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 4)
        for (long idx = 0; idx < total; ++idx) {
            if (!w) continue;
            int r = (int)(idx % n_rows);
            long bh = idx / n_rows;
            int b = (int)(bh / H);
            long i = rows ? rows[r] : r;
            const long* kl = keys + (size_t)b * Tk;
            long n = n_keys[b];
            const uint16_t* qrow = q + ((size_t)bh * Tq + (size_t)i) * D;
            const uint16_t* kbase = k + (size_t)bh * Tk * D;
            const uint16_t* vbase = v + (size_t)bh * Tk * D;
            double* o = out + (size_t)idx * D;
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            if (n == 0) {
                lse[idx] = -INFINITY;
                continue;
            }
            double m = -INFINITY;
            for (long t = 0; t < n; ++t) {
                double dot = 0.0;
                for (int d = 0; d < D; ++d)
                    dot += widen_bf16(qrow[d]) * widen_bf16(kbase[(size_t)kl[t] * D + d]);
                w[t] = scale * dot;
                if (w[t] > m) m = w[t];
            }
            double l = 0.0;
            for (long t = 0; t < n; ++t) {
                w[t] = exp(w[t] - m);
                l += w[t];
            }
            for (long t = 0; t < n; ++t)
                for (int d = 0; d < D; ++d) o[d] += w[t] * widen_bf16(vbase[(size_t)kl[t] * D + d]);
            for (int d = 0; d < D; ++d) o[d] /= l;
            lse[idx] = m + log(l);
        }
        free(w);
    }
    free(keys);
    free(n_keys);
    return failed ? -1 : 0;
}
