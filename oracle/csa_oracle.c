/*
 * csa_oracle.c -- plain fp64 CPU oracle for the DeepSeek-V4 hybrid compressed attention
 * layer (KV Compressor -> Lightning Indexer + top-k -> shared K=V MQA with sink, partial
 * interleaved RoPE and output de-rotation).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this
 * file; only the CPU tests, the smoke check and the benchmark's CPU-baseline leg use it.
 * It shares no code, header, table or constant with the CUDA library.
 *
 * Every quantity is computed in double precision from the caller's double inputs, with
 * plain loops in the order the definitions state them.  No blocking, fusion or
 * reordering beyond the definitions.  OpenMP only splits independent query rows.
 *
 * Sources (the web pages this layer is described on):
 *  [HF-PR]   HF transformers PR #45616 "add DeepSeek-V4": compressor/indexer state,
 *            empty pool before the first closed window, interleaved RoPE, GPT-OSS
 *            eager sink attention, output rope-slice un-rotation.
 *  [HF-DOC]  HF docs model_doc/deepseek_v4: section "Hybrid attention (2.3)" (CSA m=4
 *            overlapping, HCA m'=128 non-overlapping, shared K=V MQA, partial RoPE with
 *            the -i output rotation of eq. 26, per-head sink of eq. 27) and section
 *            "Attention mask layout" (sliding window, -1 top-k marker, HCA visibility
 *            w < (t+1)//m with the m=8 worked example).
 *  [OV-1748] optimum-intel issue #1748: V4-Flash window 128, ratios 4 / 128.
 *  Formulas the pages leave open are fixed here as: indexer score
 *  sum_h w[t,h] ReLU(q_I[t,h].k_I[j]); CSA window of entry j is tokens
 *  [max(0,(j-1)m), (j+1)m); HCA window [jm,(j+1)m); entry j visible to t iff
 *  (j+1)m-1 <= t.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - RoPE position of compressed entry j is j*m (parity unpinned by the pages).
 *  - Pooling acts on un-rotated kv; the entry is rotated at its own position.
 *  - One RoPE base per call, used for q, window keys, entries and de-rotation.
 *  - Softmax scale is a caller argument (the layer uses 1/sqrt(head_dim)).
 *  - A key in the window that is also covered by a selected entry counts twice.
 *  - Top-k order: score descending, ties by lower entry index.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_BAD_ARG (-1)
#define ORC_NO_MEM (-2)

/* ---------------------------------------------------------------------------------
 * RoPE, [HF-DOC] "Partial rotary positional embedding (2.3.3)", [HF-PR] "RoPE apply:
 * interleaved-pair rotation via complex mul".  The last R channels of a D-vector form
 * R/2 pairs (a, a+1), a = D-R+2i; pair i turns by angle pos * base^(-2i/R).
 * ------------------------------------------------------------------------------- */
static void rope_rotate(double *x, double pos, int64_t D, int64_t R, double base)
{
    for (int64_t i = 0; i < R / 2; ++i) {
        double theta = pow(base, -2.0 * (double)i / (double)R);
        double phi = pos * theta;
        double c = cos(phi), s = sin(phi);
        int64_t a = D - R + 2 * i;
        double xa = x[a], xb = x[a + 1];
        x[a] = xa * c - xb * s;
        x[a + 1] = xa * s + xb * c;
    }
}

/* Rotate n rows of D doubles in place, row r at position pos[r]. */
int orc_rope_rows(double *x, const double *pos, int64_t n, int64_t D, int64_t R, double base)
{
    if (R < 0 || R > D || (R % 2) != 0) return ORC_BAD_ARG;
    for (int64_t r = 0; r < n; ++r) rope_rotate(x + r * D, pos[r], D, R, base);
    return ORC_OK;
}

/* ---------------------------------------------------------------------------------
 * KV Compressor, [HF-DOC] 2.3.1 / 2.3.2 and [HF-PR] "Compressor.forward always returns
 * a tensor (empty when no window has closed yet)".  Entry j of sequence b, channel d:
 *   pool[b,j,d] = sum_{s in Win_j} exp(g[b,s,d]) kv[b,s,d] / sum_{s in Win_j} exp(g[b,s,d])
 * (a per-channel softmax of the gate logits over the window, subtracting the window
 * max first), Win_j = [max(0,(j-1)m), (j+1)m) with overlap, [jm,(j+1)m) without.
 * P = floor(S/m) entries; a trailing partial window is not emitted.
 * ------------------------------------------------------------------------------- */
int orc_compress(const double *kv, const double *gate, double *pool,
                 int64_t B, int64_t S, int64_t D, int64_t m, int overlap)
{
    if (B < 0 || S < 0 || D <= 0 || m <= 0) return ORC_BAD_ARG;
    int64_t P = S / m;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t j = 0; j < P; ++j) {
            int64_t lo = overlap ? (j - 1) * m : j * m;
            if (lo < 0) lo = 0;
            int64_t hi = (j + 1) * m;
            for (int64_t d = 0; d < D; ++d) {
                double mx = -INFINITY;
                for (int64_t s = lo; s < hi; ++s) {
                    double g = gate[(b * S + s) * D + d];
                    if (g > mx) mx = g;
                }
                double num = 0.0, den = 0.0;
                for (int64_t s = lo; s < hi; ++s) {
                    double e = exp(gate[(b * S + s) * D + d] - mx);
                    num += e * kv[(b * S + s) * D + d];
                    den += e;
                }
                pool[(b * P + j) * D + d] = num / den;
            }
        }
    }
    return ORC_OK;
}

/* ---------------------------------------------------------------------------------
 * Stateful compressor for decode, [HF-PR] note on compressor and indexer state: the state
 * lives in the model's cache, one compressor state and one indexer state per layer, each
 * a buffer of raw kv and gate rows plus the pooled cache, and one call accumulates the
 * new rows and updates the pool once; [HF-DOC] section "Cache layers": the HCA cache
 * keeps a compressor buffer, pool and counter, the CSA cache the same plus its overlap
 * state.
 *
 * State of sequence b (the layout is this oracle's own):
 *   buf_kv, buf_gate [B, m, D]  tokens of the window that has not closed yet; the first
 *                               counter[b] mod m rows are live
 *   ovl_kv, ovl_gate [B, m, D]  the last closed block of m tokens (overlap=1 only);
 *                               n_ovl[b] rows are live (0 before the first close)
 *   counter [B]                 tokens seen so far
 * Each new token goes into the buffer.  When the buffer holds m tokens the window
 * closes: its entry pools the overlap block followed by the buffer (overlap=1), or the
 * buffer alone (overlap=0), by the per-channel gate softmax of orc_compress; then, with
 * overlap, the buffer becomes the overlap block; the buffer starts empty again.
 * Entries are written in closing order to out[b, 0 .. n_out[b]).
 * ------------------------------------------------------------------------------- */
static void pool_window(const double *kv, const double *gate, int64_t n, int64_t D,
                        double *entry)
{
    for (int64_t d = 0; d < D; ++d) {
        double gmax = -INFINITY;
        for (int64_t s = 0; s < n; ++s)
            if (gate[s * D + d] > gmax) gmax = gate[s * D + d];
        double acc = 0.0, z = 0.0;
        for (int64_t s = 0; s < n; ++s) {
            double wgt = exp(gate[s * D + d] - gmax);
            acc += wgt * kv[s * D + d];
            z += wgt;
        }
        entry[d] = acc / z;
    }
}

int orc_compress_step(double *buf_kv, double *buf_gate, double *ovl_kv, double *ovl_gate,
                      int64_t *counter, int64_t *n_ovl, const double *kv_new,
                      const double *gate_new, int64_t n_new, int64_t B, int64_t D, int64_t m,
                      int overlap, double *out, int64_t max_out, int64_t *n_out)
{
    if (B < 0 || n_new < 0 || D <= 0 || m <= 0 || max_out < 0) return ORC_BAD_ARG;
    double *win_kv = (double *)malloc(sizeof(double) * (size_t)(2 * m * D));
    double *win_gate = (double *)malloc(sizeof(double) * (size_t)(2 * m * D));
    if (!win_kv || !win_gate) {
        free(win_kv);
        free(win_gate);
        return ORC_NO_MEM;
    }
    int rc = ORC_OK;
    for (int64_t b = 0; b < B && rc == ORC_OK; ++b) {
        n_out[b] = 0;
        for (int64_t i = 0; i < n_new; ++i) {
            int64_t fill = counter[b] % m;   /* live rows in the buffer */
            memcpy(buf_kv + (b * m + fill) * D, kv_new + (b * n_new + i) * D, sizeof(double) * (size_t)D);
            memcpy(buf_gate + (b * m + fill) * D, gate_new + (b * n_new + i) * D, sizeof(double) * (size_t)D);
            counter[b] += 1;
            if (fill + 1 < m) continue;      /* the window is still open */
            int64_t n = 0;
            if (overlap) {
                memcpy(win_kv, ovl_kv + b * m * D, sizeof(double) * (size_t)(n_ovl[b] * D));
                memcpy(win_gate, ovl_gate + b * m * D, sizeof(double) * (size_t)(n_ovl[b] * D));
                n = n_ovl[b];
            }
            memcpy(win_kv + n * D, buf_kv + b * m * D, sizeof(double) * (size_t)(m * D));
            memcpy(win_gate + n * D, buf_gate + b * m * D, sizeof(double) * (size_t)(m * D));
            n += m;
            if (n_out[b] >= max_out) {
                rc = ORC_BAD_ARG;
                break;
            }
            pool_window(win_kv, win_gate, n, D, out + (b * max_out + n_out[b]) * D);
            n_out[b] += 1;
            if (overlap) {
                memcpy(ovl_kv + b * m * D, buf_kv + b * m * D, sizeof(double) * (size_t)(m * D));
                memcpy(ovl_gate + b * m * D, buf_gate + b * m * D, sizeof(double) * (size_t)(m * D));
                n_ovl[b] = m;
            }
        }
    }
    free(win_kv);
    free(win_gate);
    return rc;
}

/* Entry j is visible to the query at absolute position t iff (j+1)m-1 <= t, so the
 * visible entries are j < min(P, floor((t+1)/m)).  [HF-DOC] "Attention mask layout":
 * with m=8, entry 0 opens at t >= 7 and entry 1 at t >= 15. */
int64_t orc_n_visible(int64_t t, int64_t m, int64_t P)
{
    if (t < 0 || m <= 0) return 0;
    int64_t n = (t + 1) / m;
    return n < P ? n : P;
}

/* ---------------------------------------------------------------------------------
 * Lightning Indexer score, [HF-DOC] 2.3.1 (eq. 13-17 are named there but not printed;
 * the form is fixed here as):
 *   score[t,j] = sum_h w[t,h] * max(0, sum_d q_I[t,h,d] k_I[j,d])   for visible j.
 * Rows are the caller's query rows with absolute positions tpos[i]; invisible entries
 * get NaN.  qI [B,n,HI,dI], w [B,n,HI], kI [B,P,dI], scores [B,n,P].
 * ------------------------------------------------------------------------------- */
int orc_index_scores(const double *qI, const double *w, const double *kI,
                     const int64_t *tpos, int64_t B, int64_t n, int64_t P,
                     int64_t HI, int64_t dI, int64_t m, double *scores)
{
    if (B < 0 || n < 0 || P < 0 || HI <= 0 || dI <= 0 || m <= 0) return ORC_BAD_ARG;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t i = 0; i < n; ++i) {
            int64_t nv = orc_n_visible(tpos[i], m, P);
            double *srow = scores + (b * n + i) * P;
            for (int64_t j = 0; j < P; ++j) {
                if (j >= nv) { srow[j] = NAN; continue; }
                double acc = 0.0;
                for (int64_t h = 0; h < HI; ++h) {
                    const double *q = qI + ((b * n + i) * HI + h) * dI;
                    const double *k = kI + (b * P + j) * dI;
                    double dot = 0.0;
                    for (int64_t d = 0; d < dI; ++d) dot += q[d] * k[d];
                    double relu = dot > 0.0 ? dot : 0.0;
                    acc += w[(b * n + i) * HI + h] * relu;
                }
                srow[j] = acc;
            }
        }
    }
    return ORC_OK;
}

/* ---------------------------------------------------------------------------------
 * Top-k with the -1 marker, [HF-DOC] "Attention mask layout" (CSA): a query keeps the
 * k best visible entries; before the first closed window it gets only -1.  Visible
 * entries are sorted by (score descending, index ascending); the first min(k, n_vis)
 * are kept in that order and the rest of the k slots hold -1 (score slot NaN).
 * ------------------------------------------------------------------------------- */
typedef struct { double s; int64_t j; } orc_pair;

static int pair_cmp(const void *pa, const void *pb)
{
    const orc_pair *a = (const orc_pair *)pa, *b = (const orc_pair *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->j < b->j) ? -1 : (a->j > b->j);
}

int orc_topk(const double *scores, const int64_t *tpos, int64_t B, int64_t n, int64_t P,
             int64_t m, int64_t k, int32_t *idx, double *sel_scores)
{
    if (B < 0 || n < 0 || P < 0 || m <= 0 || k <= 0) return ORC_BAD_ARG;
    int fail = 0;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t i = 0; i < n; ++i) {
            int64_t nv = orc_n_visible(tpos[i], m, P);
            orc_pair *v = (orc_pair *)malloc((size_t)(nv > 0 ? nv : 1) * sizeof(orc_pair));
            if (!v) { fail = 1; continue; }
            const double *srow = scores + (b * n + i) * P;
            for (int64_t j = 0; j < nv; ++j) { v[j].s = srow[j]; v[j].j = j; }
            qsort(v, (size_t)nv, sizeof(orc_pair), pair_cmp);
            for (int64_t r = 0; r < k; ++r) {
                int64_t o = (b * n + i) * k + r;
                if (r < nv) {
                    idx[o] = (int32_t)v[r].j;
                    if (sel_scores) sel_scores[o] = v[r].s;
                } else {
                    idx[o] = -1;
                    if (sel_scores) sel_scores[o] = NAN;
                }
            }
            free(v);
        }
    }
    return fail ? ORC_NO_MEM : ORC_OK;
}

/* ---------------------------------------------------------------------------------
 * Sink attention over an explicit key list for one query, [HF-DOC] 2.3 "shared K=V
 * MQA", eq. 26 and eq. 27; [HF-PR] "port eager_attention_forward from GPT-OSS" and the
 * un-rotation note.  For each head h:
 *   q_r = Rot(q[h], tq);  k_x = v_x = Rot(key_x, pos_x)
 *   l_x = scale * <q_r, k_x>;  M = max(max_x l_x, sink_h)
 *   Z = exp(sink_h - M) + sum_x exp(l_x - M)
 *   o = sum_x exp(l_x - M) / Z * v_x;   o[D-R:] <- Rot(o[D-R:], -tq)
 * q [H,D]; keys: n_keys pointers to un-rotated D-rows; kpos positions; out [H,D].
 * work must hold n_keys*D + n_keys + D doubles.
 * ------------------------------------------------------------------------------- */
static void attend_query(const double *q, double tq, const double *const *keys,
                         const double *kpos, int64_t n_keys, const double *sink,
                         int64_t H, int64_t D, int64_t R, double base, double scale,
                         double *out, double *work)
{
    double *krot = work;                 /* n_keys * D */
    double *logit = krot + n_keys * D;   /* n_keys     */
    double *qr = logit + n_keys;         /* D          */
    for (int64_t x = 0; x < n_keys; ++x) {
        memcpy(krot + x * D, keys[x], (size_t)D * sizeof(double));
        rope_rotate(krot + x * D, kpos[x], D, R, base);
    }
    for (int64_t h = 0; h < H; ++h) {
        memcpy(qr, q + h * D, (size_t)D * sizeof(double));
        rope_rotate(qr, tq, D, R, base);
        double M = sink[h];
        for (int64_t x = 0; x < n_keys; ++x) {
            double dot = 0.0;
            for (int64_t d = 0; d < D; ++d) dot += qr[d] * krot[x * D + d];
            logit[x] = scale * dot;
            if (logit[x] > M) M = logit[x];
        }
        double Z = (sink[h] == -INFINITY) ? 0.0 : exp(sink[h] - M);
        for (int64_t x = 0; x < n_keys; ++x) Z += exp(logit[x] - M);
        double *o = out + h * D;
        for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
        for (int64_t x = 0; x < n_keys; ++x) {
            double p = exp(logit[x] - M) / Z;
            for (int64_t d = 0; d < D; ++d) o[d] += p * krot[x * D + d];
        }
        rope_rotate(o, -tq, D, R, base);
    }
}

/* One query against explicit keys (used by the invariance and closed-form checks). */
int orc_attend_keys(const double *q, double tq, const double *keys, const double *kpos,
                    int64_t n_keys, const double *sink, int64_t H, int64_t D, int64_t R,
                    double base, double scale, double *out)
{
    if (n_keys < 0 || H <= 0 || D <= 0 || R < 0 || R > D || (R % 2)) return ORC_BAD_ARG;
    const double **kp = (const double **)malloc((size_t)(n_keys > 0 ? n_keys : 1) * sizeof(double *));
    double *work = (double *)malloc((size_t)(n_keys * D + n_keys + D) * sizeof(double));
    if (!kp || !work) { free(kp); free(work); return ORC_NO_MEM; }
    for (int64_t x = 0; x < n_keys; ++x) kp[x] = keys + x * D;
    attend_query(q, tq, kp, kpos, n_keys, sink, H, D, R, base, scale, out, work);
    free(kp);
    free(work);
    return ORC_OK;
}

/* ---------------------------------------------------------------------------------
 * The layer's attention for a set of query rows.
 *   Keys of query t (absolute position tpos[i]):
 *     window: raw rows at positions s with t-W < s <= t that the caller supplied
 *             (kv row r sits at kv_pos0 + r), [HF-DOC] sliding branch, window of W
 *             rows including the query's own;
 *     entries: mode 0 (CSA) the entries idx[b,i,:] other than -1;
 *              mode 1 (HCA) every visible entry j < min(P, floor((t+1)/m));
 *              P = 0 gives the sliding-only layer.
 *   Entry j is rotated at position j*m.
 * q [B,n,H,D]; kv [B,S_kv,D]; pool [B,P,D]; idx [B,n,k] int32; sink [H]; out [B,n,H,D].
 * Returns ORC_BAD_ARG for an idx entry that is out of range or not visible to its row.
 * ------------------------------------------------------------------------------- */
int orc_attend(const double *q, const int64_t *tpos, int64_t n,
               const double *kv, int64_t S_kv, int64_t kv_pos0,
               const double *pool, int64_t P, int64_t m,
               const int32_t *idx, int64_t k, int mode,
               const double *sink, int64_t B, int64_t H, int64_t D, int64_t R,
               double base, int64_t W, double scale, double *out)
{
    if (B < 0 || n < 0 || H <= 0 || D <= 0 || R < 0 || R > D || (R % 2) || W < 0 || m <= 0)
        return ORC_BAD_ARG;
    if (mode == 0 && P > 0 && (k <= 0 || !idx)) return ORC_BAD_ARG;
    int64_t max_keys = W + (mode == 0 ? k : P) + 1;
    int fail = 0;
#pragma omp parallel
    {
        const double **kp = (const double **)malloc((size_t)max_keys * sizeof(double *));
        double *kpos = (double *)malloc((size_t)max_keys * sizeof(double));
        double *work = (double *)malloc((size_t)(max_keys * D + max_keys + D) * sizeof(double));
        if (!kp || !kpos || !work) {
#pragma omp atomic write
            fail = ORC_NO_MEM;
        }
#pragma omp for collapse(2) schedule(dynamic)
        for (int64_t b = 0; b < B; ++b) {
            for (int64_t i = 0; i < n; ++i) {
                if (!kp || !kpos || !work) continue;
                int64_t t = tpos[i];
                int64_t nk = 0;
                for (int64_t r = 0; r < S_kv; ++r) {
                    int64_t s = kv_pos0 + r;
                    if (s > t - W && s <= t) {
                        kp[nk] = kv + (b * S_kv + r) * D;
                        kpos[nk] = (double)s;
                        ++nk;
                    }
                }
                int64_t nv = orc_n_visible(t, m, P);
                if (mode == 0) {
                    for (int64_t r = 0; r < k && P > 0; ++r) {
                        int32_t j = idx[(b * n + i) * k + r];
                        if (j == -1) continue;
                        if (j < 0 || j >= nv) {
#pragma omp atomic write
                            fail = ORC_BAD_ARG;
                            break;
                        }
                        kp[nk] = pool + (b * P + j) * D;
                        kpos[nk] = (double)j * (double)m;
                        ++nk;
                    }
                } else {
                    for (int64_t j = 0; j < nv; ++j) {
                        kp[nk] = pool + (b * P + j) * D;
                        kpos[nk] = (double)j * (double)m;
                        ++nk;
                    }
                }
                attend_query(q + (b * n + i) * H * D, (double)t, kp, kpos, nk, sink, H, D, R,
                             base, scale, out + (b * n + i) * H * D, work);
            }
        }
        free(kp);
        free(kpos);
        free(work);
    }
    return fail;
}
