/*
 * ratp_oracle.c -- plain fp64 CPU oracle for the RAT+ sequence mixer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the test-suite, the package's smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, table or
 * constant with the CUDA library.
 *
 * Sources (web pages on RAT+, arXiv 2602.18196):
 *   [abs]  "RAT+: Train Dense, Infer Sparse -- Recurrence Augmented Attention
 *          for Dilated Inference", abstract (paperdance.org/p/2602.18196):
 *          dilated attention of dilation D cuts attention FLOPs and the KV
 *          cache by D; optional local windows; hybrid layer/head compositions.
 *   [zc]   "RAT+ 深度拆解：Dense 预训练 + Dilated 推理的 KV Cache 压缩新范式"
 *          (zhichai.net): section 1 (dilated attention skips tokens at a fixed
 *          interval), section 2.1 (full-sequence forget-gate recurrence,
 *          associative scan at prefill), section 6 (head-wise hybrid: first
 *          heads dense, the rest dilated).
 *
 * Readings taken where the pages are silent or garbled (the recurrence
 * formula itself is missing from the extracted section 2.1):
 *   - recurrence  h_t = g_t * h_{t-1} + (1 - g_t) * x_t  per channel, h_{-1} = 0,
 *     over the whole sequence, one gate tensor shared by the key and value
 *     streams;
 *   - dilated key set of query t: { j < t : j mod D == D-1 } U { t };
 *   - local window of W >= 1 positions { j : t-W < j <= t, j >= 0 }, united
 *     with the dilated set (each key once); W == 0 means no window;
 *   - scores q_t . hk_j / sqrt(Dh), softmax over the key set, output
 *     sum_j p_j hv_j; queries are not recurrent, keys/values are;
 *   - a dense head (dense_mask[h] != 0) uses D = 1;
 *   - chunk-local variant (the original RAT that [zc] section 2.1 contrasts
 *     with RAT+: each token recurs only inside its own block of L tokens):
 *     the state is zeroed before position t whenever t mod L == 0, at
 *     prefill and at decode alike; the key and value streams restart
 *     together;
 *   - fixed look-back variant (the window L* = 64 that the same section
 *     attributes to RAT+ before it moved to the full sequence): h_t is the
 *     recurrence over the L positions max(0, t-L+1) .. t, started from zero.
 *
 * Parity pins for every function live in the CPU test-suite (closed forms,
 * brute-force masks, dense causal attention from a library routine,
 * hand-worked fixtures).
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC ratp_oracle.c -lm
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Recurrence ([zc] section 2.1): a sequential loop, the plain definition.   */
/* x, g, h: [B][T][C] row-major, C = H*Dh channels per token.                */
/* ------------------------------------------------------------------------ */
void orc_scan(const double* x, const double* g, double* h,
              long B, long T, long C)
{
    long b;
#pragma omp parallel for schedule(static)
    for (b = 0; b < B; ++b) {
        for (long c = 0; c < C; ++c) {
            double state = 0.0;                      /* h_{-1} = 0 */
            for (long t = 0; t < T; ++t) {
                long i = (b * T + t) * C + c;
                state = g[i] * state + (1.0 - g[i]) * x[i];
                h[i] = state;
            }
        }
    }
}

/* Chunk-local recurrence of the original RAT ([zc] section 2.1: the state
 * restarts at every chunk of L tokens, L = D there): the same recurrence with
 * h_{t-1} taken as 0 whenever t mod L == 0.  L <= 0 means no restart (the
 * full-sequence recurrence of orc_scan). */
void orc_scan_reset(const double* x, const double* g, double* h,
                    long B, long T, long C, long L)
{
    long b;
#pragma omp parallel for schedule(static)
    for (b = 0; b < B; ++b) {
        for (long c = 0; c < C; ++c) {
            double state = 0.0;
            for (long t = 0; t < T; ++t) {
                long i = (b * T + t) * C + c;
                if (L > 0 && t % L == 0) state = 0.0;    /* a chunk starts at t */
                state = g[i] * state + (1.0 - g[i]) * x[i];
                h[i] = state;
            }
        }
    }
}

/* Fixed look-back recurrence ([zc] section 2.1: an earlier RAT+ design whose
 * recurrence window is the L tokens up to and including t, L* = 64): h_t is
 * the recurrence started from zero at position max(0, t-L+1) and run to t.
 * A plain O(T * L) loop per channel; L >= T gives the full sequence. */
void orc_scan_window(const double* x, const double* g, double* h,
                     long B, long T, long C, long L)
{
    long b;
#pragma omp parallel for schedule(static)
    for (b = 0; b < B; ++b) {
        for (long c = 0; c < C; ++c) {
            for (long t = 0; t < T; ++t) {
                long j0 = t - L + 1;
                if (j0 < 0) j0 = 0;
                double state = 0.0;
                for (long j = j0; j <= t; ++j) {
                    long i = (b * T + j) * C + c;
                    state = g[i] * state + (1.0 - g[i]) * x[i];
                }
                h[(b * T + t) * C + c] = state;
            }
        }
    }
}

/* One recurrence step for decode: state <- g*state + (1-g)*x, n channels. */
void orc_scan_step(const double* x, const double* g, double* state, long n)
{
    for (long i = 0; i < n; ++i)
        state[i] = g[i] * state[i] + (1.0 - g[i]) * x[i];
}

/* ------------------------------------------------------------------------ */
/* Key set K(t) by enumeration ([abs]; [zc] section 1).                      */
/* Writes the sorted, duplicate-free positions to out; returns the count.    */
/* out must hold at least t/D + W + 1 entries.                               */
/* ------------------------------------------------------------------------ */
static void insert_sorted(long* out, long* n, long j)
{
    long k = *n;
    for (long i = 0; i < k; ++i) {
        if (out[i] == j) return;                     /* already present */
    }
    long pos = k;
    while (pos > 0 && out[pos - 1] > j) {
        out[pos] = out[pos - 1];
        --pos;
    }
    out[pos] = j;
    *n = k + 1;
}

long orc_key_set(long t, long D, long W, long* out)
{
    long n = 0;
    for (long j = D - 1; j < t; j += D)              /* dilated positions */
        insert_sorted(out, &n, j);
    insert_sorted(out, &n, t);                       /* the query itself */
    if (W > 0) {                                     /* local window */
        long lo = t - W + 1;
        if (lo < 0) lo = 0;
        for (long j = lo; j <= t; ++j)
            insert_sorted(out, &n, j);
    }
    return n;
}

/* Softmax attention of one query row over an explicit key list.            */
/* q, hk, hv point at [T][H][Dh] slices of one batch item.                   */
static void attend_row(const double* q, const double* hk, const double* hv,
                       double* o, long t, long h, long H, long Dh,
                       const long* keys, long nk, double* scores)
{
    const double scale = 1.0 / sqrt((double)Dh);
    const double* qt = q + (t * H + h) * Dh;
    double m = -INFINITY;
    for (long i = 0; i < nk; ++i) {
        const double* kj = hk + (keys[i] * H + h) * Dh;
        double s = 0.0;
        for (long d = 0; d < Dh; ++d) s += qt[d] * kj[d];
        scores[i] = s * scale;
        if (scores[i] > m) m = scores[i];
    }
    double denom = 0.0;
    for (long i = 0; i < nk; ++i) {
        scores[i] = exp(scores[i] - m);
        denom += scores[i];
    }
    for (long d = 0; d < Dh; ++d) o[d] = 0.0;
    for (long i = 0; i < nk; ++i) {
        const double* vj = hv + (keys[i] * H + h) * Dh;
        double p = scores[i] / denom;
        for (long d = 0; d < Dh; ++d) o[d] += p * vj[d];
    }
}

/* ------------------------------------------------------------------------ */
/* Dilated (+ windowed) attention by key-set enumeration.                    */
/* q, hk, hv: [B][T][H][Dh].  dense_mask: [H] (NULL = no dense heads).       */
/* rows == NULL: o is [B][T][H][Dh], every query is computed.                */
/* rows != NULL: n_rows triples (b, t, h); o is [n_rows][Dh].                */
/* ------------------------------------------------------------------------ */
void orc_attention(const double* q, const double* hk, const double* hv,
                   double* o, long B, long T, long H, long Dh, long D, long W,
                   const unsigned char* dense_mask,
                   const long* rows, long n_rows)
{
    long total = rows ? n_rows : B * T * H;
    long r;
#pragma omp parallel
    {
        long* keys = (long*)malloc(sizeof(long) * (size_t)(T + W + 2));
        double* scores = (double*)malloc(sizeof(double) * (size_t)(T + W + 2));
#pragma omp for schedule(dynamic, 16)
        for (r = 0; r < total; ++r) {
            long b, t, h;
            double* out;
            if (rows) {
                b = rows[3 * r]; t = rows[3 * r + 1]; h = rows[3 * r + 2];
                out = o + r * Dh;
            } else {
                b = r / (T * H); t = (r / H) % T; h = r % H;
                out = o + r * Dh;
            }
            long Dh_eff = (dense_mask && dense_mask[h]) ? 1 : D;
            long nk = orc_key_set(t, Dh_eff, W, keys);
            const long off = b * T * H * Dh;
            attend_row(q + off, hk + off, hv + off, out, t, h, H, Dh,
                       keys, nk, scores);
        }
        free(keys);
        free(scores);
    }
}

/* ------------------------------------------------------------------------ */
/* Brute force: explicit T x T mask with -inf entries and a full softmax.    */
/* A separate path from the enumeration above (tiny T only).                 */
/* ------------------------------------------------------------------------ */
void orc_attention_mask(const double* q, const double* hk, const double* hv,
                        double* o, long B, long T, long H, long Dh, long D,
                        long W, const unsigned char* dense_mask)
{
    const double scale = 1.0 / sqrt((double)Dh);
    double* S = (double*)malloc(sizeof(double) * (size_t)(T * T));
    for (long b = 0; b < B; ++b) {
        for (long h = 0; h < H; ++h) {
            long Dd = (dense_mask && dense_mask[h]) ? 1 : D;
            for (long t = 0; t < T; ++t) {
                for (long j = 0; j < T; ++j) {
                    int allowed = (j <= t) &&
                                  ((j % Dd == Dd - 1) || (j == t) ||
                                   (W > 0 && t - j < W));
                    double s = 0.0;
                    for (long d = 0; d < Dh; ++d)
                        s += q[((b * T + t) * H + h) * Dh + d] *
                             hk[((b * T + j) * H + h) * Dh + d];
                    S[t * T + j] = allowed ? s * scale : -INFINITY;
                }
                double m = -INFINITY;
                for (long j = 0; j < T; ++j) if (S[t * T + j] > m) m = S[t * T + j];
                double z = 0.0;
                for (long j = 0; j < T; ++j) {
                    S[t * T + j] = exp(S[t * T + j] - m);   /* exp(-inf) = 0 */
                    z += S[t * T + j];
                }
                for (long d = 0; d < Dh; ++d) {
                    double acc = 0.0;
                    for (long j = 0; j < T; ++j)
                        acc += S[t * T + j] / z * hv[((b * T + j) * H + h) * Dh + d];
                    o[((b * T + t) * H + h) * Dh + d] = acc;
                }
            }
        }
    }
    free(S);
}

/* ------------------------------------------------------------------------ */
/* D-compressed KV cache layout ([abs]: the cache shrinks by D).             */
/*                                                                            */
/* Dilated rows: head h with dilation D_h keeps the recurrent key/value of   */
/* position p = s*D_h + D_h - 1 in slot s.  Per-head capacity                */
/* cap_h = floor(T_max / D_h).  Rows of one batch item are stored head after */
/* head: flat row = b * sum_h cap_h + sum_{h' < h} cap_{h'} + s.             */
/* Window ring: position p of (b, h) lives in row (b*H + h)*W + p mod W.     */
/* ------------------------------------------------------------------------ */
static long head_dilation(long h, long D, const unsigned char* dense_mask)
{
    return (dense_mask && dense_mask[h]) ? 1 : D;
}

long orc_cache_row(long b, long h, long s, long H, long T_max, long D,
                   const unsigned char* dense_mask)
{
    long per_b = 0, before = 0;
    for (long k = 0; k < H; ++k) {
        long cap = T_max / head_dilation(k, D, dense_mask);
        if (k < h) before += cap;
        per_b += cap;
    }
    return b * per_b + before + s;
}

long orc_cache_rows_total(long B, long H, long T_max, long D,
                          const unsigned char* dense_mask)
{
    long per_b = 0;
    for (long k = 0; k < H; ++k) per_b += T_max / head_dilation(k, D, dense_mask);
    return B * per_b;
}

long orc_ring_row(long b, long h, long p, long H, long W)
{
    return (b * H + h) * W + (p % W);
}

/* Fill the cache from prefill histories hk, hv [B][T][H][Dh] of T tokens.   */
/* Kc, Vc: [rows_total][Dh]; Kw, Vw: [B][H][W][Dh] (unused when W == 0).     */
void orc_cache_pack(const double* hk, const double* hv, long B, long T, long H,
                    long Dh, long T_max, long D, long W,
                    const unsigned char* dense_mask,
                    double* Kc, double* Vc, double* Kw, double* Vw, long* len)
{
    for (long b = 0; b < B; ++b) {
        for (long h = 0; h < H; ++h) {
            long Dd = head_dilation(h, D, dense_mask);
            for (long p = Dd - 1; p < T; p += Dd) {
                long row = orc_cache_row(b, h, p / Dd, H, T_max, D, dense_mask);
                memcpy(Kc + row * Dh, hk + ((b * T + p) * H + h) * Dh, sizeof(double) * Dh);
                memcpy(Vc + row * Dh, hv + ((b * T + p) * H + h) * Dh, sizeof(double) * Dh);
            }
            if (W > 0) {
                long lo = T - W < 0 ? 0 : T - W;
                for (long p = lo; p < T; ++p) {
                    long row = orc_ring_row(b, h, p, H, W);
                    memcpy(Kw + row * Dh, hk + ((b * T + p) * H + h) * Dh, sizeof(double) * Dh);
                    memcpy(Vw + row * Dh, hv + ((b * T + p) * H + h) * Dh, sizeof(double) * Dh);
                }
            }
        }
        len[b] = T;
    }
}

/* ------------------------------------------------------------------------ */
/* One decode step, literally: recurrence step, cache append, attention over */
/* the cache contents (dilated slots, window ring, self).                    */
/* q, xk, xv, g: [B][H][Dh]; state: [2][B][H][Dh] (k then v), in/out.       */
/* o: [B][H][Dh].  len[b] is the position t of this token; incremented.      */
/* Returns 0, or -1 when an append would exceed the capacity.                */
/* ------------------------------------------------------------------------ */
int orc_decode_step(const double* q, const double* xk, const double* xv,
                    const double* g, double* state, double* Kc, double* Vc,
                    double* Kw, double* Vw, long* len, double* o,
                    long B, long H, long Dh, long T_max, long D, long W,
                    const unsigned char* dense_mask, long L)
{
    const double scale = 1.0 / sqrt((double)Dh);
    int status = 0;
    long n_keys_max = T_max + W + 2;
    long* pos = (long*)malloc(sizeof(long) * (size_t)n_keys_max);
    const double** kr = (const double**)malloc(sizeof(double*) * (size_t)n_keys_max);
    const double** vr = (const double**)malloc(sizeof(double*) * (size_t)n_keys_max);
    double* sc = (double*)malloc(sizeof(double) * (size_t)n_keys_max);
    for (long b = 0; b < B; ++b) {
        long t = len[b];
        if (t >= T_max) { status = -1; continue; }
        for (long h = 0; h < H; ++h) {
            long Dd = head_dilation(h, D, dense_mask);
            long i0 = (b * H + h) * Dh;
            double* sk = state + i0;
            double* sv = state + B * H * Dh + i0;
            if (L > 0 && t % L == 0) {                /* chunk-local recurrence restarts */
                for (long c = 0; c < Dh; ++c) { sk[c] = 0.0; sv[c] = 0.0; }
            }
            orc_scan_step(xk + i0, g + i0, sk, Dh);
            orc_scan_step(xv + i0, g + i0, sv, Dh);
            long nk = 0;
            /* dilated slots already in the cache: positions s*Dd+Dd-1 < t */
            for (long s = 0; s * Dd + Dd - 1 < t; ++s) {
                long row = orc_cache_row(b, h, s, H, T_max, D, dense_mask);
                pos[nk] = s * Dd + Dd - 1;
                kr[nk] = Kc + row * Dh; vr[nk] = Vc + row * Dh; ++nk;
            }
            /* window positions t-W < p < t not already among the dilated ones */
            if (W > 0) {
                long lo = t - W + 1 < 0 ? 0 : t - W + 1;
                for (long p = lo; p < t; ++p) {
                    if (p % Dd == Dd - 1) continue;
                    long row = orc_ring_row(b, h, p, H, W);
                    pos[nk] = p;
                    kr[nk] = Kw + row * Dh; vr[nk] = Vw + row * Dh; ++nk;
                }
            }
            /* the query itself attends to its own new recurrent key/value */
            pos[nk] = t; kr[nk] = sk; vr[nk] = sv; ++nk;
            double m = -INFINITY;
            const double* qt = q + i0;
            for (long i = 0; i < nk; ++i) {
                double s = 0.0;
                for (long d = 0; d < Dh; ++d) s += qt[d] * kr[i][d];
                sc[i] = s * scale;
                if (sc[i] > m) m = sc[i];
            }
            double z = 0.0;
            for (long i = 0; i < nk; ++i) { sc[i] = exp(sc[i] - m); z += sc[i]; }
            for (long d = 0; d < Dh; ++d) {
                double acc = 0.0;
                for (long i = 0; i < nk; ++i) acc += sc[i] / z * vr[i][d];
                o[i0 + d] = acc;
            }
            /* append after attending (the new row is the self key above) */
            if (t % Dd == Dd - 1) {
                long s = t / Dd;
                if (s >= T_max / Dd) { status = -1; }
                else {
                    long row = orc_cache_row(b, h, s, H, T_max, D, dense_mask);
                    memcpy(Kc + row * Dh, sk, sizeof(double) * Dh);
                    memcpy(Vc + row * Dh, sv, sizeof(double) * Dh);
                }
            }
            if (W > 0) {
                long row = orc_ring_row(b, h, t, H, W);
                memcpy(Kw + row * Dh, sk, sizeof(double) * Dh);
                memcpy(Vw + row * Dh, sv, sizeof(double) * Dh);
            }
        }
        len[b] = t + 1;
    }
    free(pos); free(kr); free(vr); free(sc);
    return status;
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
