/*
 * CPU oracle for the DeepSeek-V4 compressed attention hot path (CSA and HCA).
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or call
 * this file: only the test suite, the smoke check and the benchmark's CPU
 * baseline leg use it. It shares no code, header, table or helper with the
 * CUDA library.
 *
 * Every function is the plain definition, in fp64, with the loops in the order
 * the definition states them. OpenMP only splits independent outputs between
 * threads; it never reorders a sum.
 *
 * Sources (cited by page title and section):
 *   [Notes]  "DeepSeek-V4: 迈向高效百万级上下文智能" — structured study notes on the
 *            DeepSeek-V4 report (notes.kuangjux.top), the one page whose
 *            formulas survived extraction.
 *   [Walk]   mlpod.com walk-through of "DeepSeek-V4: Towards Highly Efficient
 *            Million-Token Context Intelligence" (its inline formulas were
 *            stripped; the prose still fixes the semantics).
 *
 * Readings taken where the pages are silent:
 *   - the four compressor maps are bias-free linear maps d -> c;
 *   - ONE softmax per (block, channel) over all 2m window logits (a-part and
 *     b-part together), so the weights sum to 1;
 *   - the positional bias is B[2m][c]: rows 0..m-1 go with the a-window
 *     offsets, rows m..2m-1 with the b-window offsets;
 *   - block 0 of a sequence has no b-window (those terms are left out);
 *   - a query at 0-based position p sees compressed entry s iff s < floor(p/m);
 *   - one indexer key per entry, shared by all indexer heads; no scale;
 *   - top-k order is (score descending, index ascending), padded with -1;
 *   - MQA scale is given by the caller; an empty visible set gives out = 0
 *     and lse = -inf (or the sink logit when a sink is given);
 *   - bf16 rounding (nearest, ties to even) only where a value is stored as
 *     bf16: the compressed caches and the outputs;
 *   - RMSNorm is x / sqrt(mean(x^2) + eps) * gamma over the c channels of a
 *     row; the rotary pairs are consecutive channels of the last R, turned by
 *     p * base^(-2i/R); the output is turned back by the query's position;
 *   - the sliding window of a query at position p holds tokens p-n_win+1 .. p
 *     (itself included) and joins the selected entries in one softmax.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* bf16 storage rounding: nearest representable bf16 value, ties to even.    */
/* bf16 keeps 8 significant bits (1 implicit + 7 stored), exponent range of  */
/* fp32: normal numbers down to 2^-126, subnormals in steps of 2^-133.       */
/* ------------------------------------------------------------------------ */
static double round_half_even(double v) {
    double f = floor(v);
    double r = v - f;
    if (r > 0.5) return f + 1.0;
    if (r < 0.5) return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

double orc_bf16_round(double x) {
    if (x == 0.0 || isnan(x) || isinf(x)) return x;
    double a = fabs(x);
    int e;
    frexp(a, &e);              /* a = f * 2^e, f in [0.5, 1) */
    int q = e - 8;             /* quantum exponent for 8 significant bits */
    if (q < -133) q = -133;    /* bf16 subnormal quantum */
    double r = ldexp(round_half_even(ldexp(a, -q)), q);
    /* largest finite bf16 is (2 - 2^-7) * 2^127; beyond the halfway point to
       2^128 the value rounds to infinity */
    if (r >= ldexp(1.0, 128)) r = INFINITY;
    return x < 0 ? -r : r;
}

void orc_bf16_round_array(const double* x, int64_t n, double* y) {
    for (int64_t i = 0; i < n; ++i) y[i] = orc_bf16_round(x[i]);
}

/* ------------------------------------------------------------------------ */
/* FP8 (e4m3) storage rounding, for the low-precision indexer and KV storage */
/* [Walk §2.3.4 and Notes §1.3 "mixed-precision storage": FP8 for the KV     */
/* channels outside the rotary ones, low-precision indexer arithmetic].      */
/* e4m3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits, no          */
/* infinities; normal numbers 2^-6 .. 448, subnormals in steps of 2^-9.     */
/* Nearest value, ties to even; magnitudes beyond 448 saturate to 448 (the  */
/* saturating conversion; the format has no infinity).                      */
/* ------------------------------------------------------------------------ */
double orc_e4m3_round(double x) {
    if (x == 0.0 || isnan(x)) return x;
    double a = fabs(x);
    if (a >= 448.0) return x < 0 ? -448.0 : 448.0;
    int e;
    frexp(a, &e);              /* a = f * 2^e, f in [0.5, 1) */
    int q = e - 4;             /* quantum exponent for 4 significant bits */
    if (q < -9) q = -9;        /* subnormal quantum */
    double r = ldexp(round_half_even(ldexp(a, -q)), q);
    return x < 0 ? -r : r;
}

/* Row-wise e4m3 quantisation: each row of n values is divided by its scale  */
/* s = max|x| / 448 (1 for an all-zero row), rounded to e4m3, and the        */
/* dequantised value code * s is returned in y; scale[r] = s.               */
void orc_quantize_rows_e4m3(const double* x, int64_t rows, int64_t n, double* y, double* scale) {
    for (int64_t r = 0; r < rows; ++r) {
        double amax = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            double v = fabs(x[r * n + j]);
            if (v > amax) amax = v;
        }
        double s = amax > 0.0 ? amax / 448.0 : 1.0;
        scale[r] = s;
        for (int64_t j = 0; j < n; ++j) y[r * n + j] = orc_e4m3_round(x[r * n + j] / s) * s;
    }
}

/* ------------------------------------------------------------------------ */
/* a1. Projections [Walk §2.3.1 "KV compression"; Notes §1.1]: each of the   */
/* compressor streams is a learnable linear map of the hidden state.         */
/* W is stored as [M][d] (one row per output feature).                      */
/*   P[t][o] = sum_k X[t][k] * W[o][k]                                        */
/* ------------------------------------------------------------------------ */
void orc_project(const double* X, const double* W, int64_t n, int64_t d, int64_t M, double* P) {
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n; ++t) {
        for (int64_t o = 0; o < M; ++o) {
            double acc = 0.0;
            for (int64_t k = 0; k < d; ++k) acc += X[t * d + k] * W[o * d + k];
            P[t * M + o] = acc;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* a2. CSA overlapping compressor [Notes §1.1, equation for C^Comp_i]:        */
/*   C^Comp_i = sum_{j=mi}^{m(i+1)-1} S^a_j (.) C^a_j                          */
/*            + sum_{j=m(i-1)}^{mi-1} S^b_j (.) C^b_j                          */
/* with S the softmax (per channel) of the weight logits Z plus a learnable  */
/* positional bias [Notes §1.1, the sentence after the equation].            */
/*                                                                          */
/* proj : [n][4c], each row = C^a | C^b | Z^a | Z^b                          */
/* left : [m][4c] rows of the m tokens just before this chunk, or NULL at    */
/*        the start of a sequence (then block 0 has no b-window)             */
/* bias : [2m][c]                                                            */
/* out  : [n/m][c] (fp64, unrounded)                                         */
/* wts  : optional [n/m][2m][c] softmax weights (a-part rows 0..m-1,         */
/*        b-part rows m..2m-1; 0 where a term is absent)                     */
/* ------------------------------------------------------------------------ */
static const double* csa_row(const double* proj, const double* left, int64_t tok, int m, int c) {
    /* token index tok is relative to the chunk; -m..-1 are the left rows */
    if (tok >= 0) return proj + tok * 4 * (int64_t)c;
    return left + (tok + m) * 4 * (int64_t)c;
}

void orc_csa_compress(const double* proj, const double* left, const double* bias,
                      int64_t n, int c, int m, double* out, double* wts) {
    int64_t nb = n / m;
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nb; ++i) {
        double* logit = (double*)malloc(sizeof(double) * 2 * m);
        int* present = (int*)malloc(sizeof(int) * 2 * m);
        for (int j = 0; j < c; ++j) {
            /* gather the 2m logits of this (block, channel) */
            for (int r = 0; r < m; ++r) {
                const double* ra = csa_row(proj, left, m * i + r, m, c);
                logit[r] = ra[2 * c + j] + bias[r * c + j];          /* Z^a + B^a */
                present[r] = 1;
                int64_t tb = m * (i - 1) + r;                         /* b-window token */
                int has_b = (tb >= 0) || (left != NULL);
                present[m + r] = has_b;
                if (has_b) {
                    const double* rb = csa_row(proj, left, tb, m, c);
                    logit[m + r] = rb[3 * c + j] + bias[(m + r) * c + j]; /* Z^b + B^b */
                }
            }
            /* one softmax over all present logits (max-subtracted) */
            double mx = -INFINITY;
            for (int r = 0; r < 2 * m; ++r) if (present[r] && logit[r] > mx) mx = logit[r];
            double den = 0.0;
            for (int r = 0; r < 2 * m; ++r) if (present[r]) den += exp(logit[r] - mx);
            double acc = 0.0;
            for (int r = 0; r < 2 * m; ++r) {
                double s = present[r] ? exp(logit[r] - mx) / den : 0.0;
                if (wts) wts[(i * 2 * m + r) * c + j] = s;
                if (!present[r]) continue;
                if (r < m) {
                    const double* ra = csa_row(proj, left, m * i + r, m, c);
                    acc += s * ra[0 * c + j];                          /* S^a (.) C^a */
                } else {
                    const double* rb = csa_row(proj, left, m * (i - 1) + (r - m), m, c);
                    acc += s * rb[1 * c + j];                          /* S^b (.) C^b */
                }
            }
            out[i * c + j] = acc;
        }
        free(logit);
        free(present);
    }
}

/* ------------------------------------------------------------------------ */
/* a3. HCA compressor [Notes §1.2 and its CSA/HCA comparison table; Walk     */
/* §2.3.2]: the same weighted sum over ONE non-overlapping window of m'     */
/* tokens (no b-window), softmax per channel over the m' logits Z + B'.      */
/* proj : [n][2c], each row = C | Z ;  bias : [mp][c] ;  out : [n/mp][c]     */
/* ------------------------------------------------------------------------ */
void orc_hca_compress(const double* proj, const double* bias, int64_t n, int c, int mp,
                      double* out, double* wts) {
    int64_t nb = n / mp;
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nb; ++i) {
        double* logit = (double*)malloc(sizeof(double) * mp);
        for (int j = 0; j < c; ++j) {
            for (int r = 0; r < mp; ++r)
                logit[r] = proj[(i * mp + r) * 2 * c + c + j] + bias[r * c + j];   /* Z + B' */
            double mx = -INFINITY;
            for (int r = 0; r < mp; ++r) if (logit[r] > mx) mx = logit[r];
            double den = 0.0;
            for (int r = 0; r < mp; ++r) den += exp(logit[r] - mx);
            double acc = 0.0;
            for (int r = 0; r < mp; ++r) {
                double s = exp(logit[r] - mx) / den;
                if (wts) wts[(i * mp + r) * c + j] = s;
                acc += s * proj[(i * mp + r) * 2 * c + j];                      /* S (.) C */
            }
            out[i * c + j] = acc;
        }
        free(logit);
    }
}

/* ------------------------------------------------------------------------ */
/* a4. Lightning indexer [Notes §1.1, equation for I_{t,s}; Walk §2.3.1       */
/* "Lightning Indexer": scores only against compressed blocks that precede   */
/* the query]:                                                               */
/*   I[t][s] = sum_h w[t][h] * ReLU( q[t][h] . K[s] ),  s < floor(p_t / m)   */
/*                                                                          */
/* q      : [nq][HI][cI]      w : [nq][HI]                                   */
/* K      : [B][Nmax][cI]     (sequence b's compressed indexer keys)         */
/* pos    : [nq] 0-based query positions; seq : [nq] sequence of each query  */
/* scores : [nq][Nmax]; entries s >= floor(pos/m) are set to -inf            */
/* ------------------------------------------------------------------------ */
void orc_index_scores(const double* q, const double* w, const double* K,
                      const int32_t* pos, const int32_t* seq, int nq, int HI, int cI,
                      int64_t Nmax, int m, double* scores) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < nq; ++t) {
        int64_t vis = pos[t] / m;
        if (vis > Nmax) vis = Nmax;
        const double* Kb = K + (int64_t)seq[t] * Nmax * cI;
        for (int64_t s = 0; s < Nmax; ++s) {
            if (s >= vis) { scores[(int64_t)t * Nmax + s] = -INFINITY; continue; }
            double acc = 0.0;
            for (int h = 0; h < HI; ++h) {
                double dot = 0.0;
                for (int e = 0; e < cI; ++e)
                    dot += q[((int64_t)t * HI + h) * cI + e] * Kb[s * cI + e];
                acc += w[(int64_t)t * HI + h] * (dot > 0.0 ? dot : 0.0);
            }
            scores[(int64_t)t * Nmax + s] = acc;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* a5. Top-k selection [Walk §2.3.1: the k highest-scoring compressed blocks */
/* are kept; Notes model table: k = 512 (Flash) / 1024 (Pro)].               */
/* For row t, the first valid[t] columns are candidates. Output the          */
/* min(k, valid) best in the order (score descending, index ascending), the  */
/* rest -1. The order is a strict total order, so the result is unique.      */
/* ------------------------------------------------------------------------ */
static int better(int32_t a, int32_t b, const double* row) {
    if (row[a] != row[b]) return row[a] > row[b];
    return a < b;
}

void orc_topk(const double* scores, const int32_t* valid, int nq, int64_t ncols, int k,
              int32_t* idx) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < nq; ++t) {
        const double* row = scores + (int64_t)t * ncols;
        int64_t v = valid[t] < ncols ? valid[t] : ncols;
        if (v < 0) v = 0;
        int32_t* out = idx + (int64_t)t * k;
        int kk = (v < k) ? (int)v : k;
        /* selection by repeated "best remaining" would be O(k v); instead keep
           an array of the kk best seen so far, sorted by the order above, and
           insert each candidate in turn (insertion sort) */
        int filled = 0;
        for (int64_t s = 0; s < v; ++s) {
            if (filled == kk && !better((int32_t)s, out[kk - 1], row)) continue;
            int p = (filled < kk) ? filled++ : kk - 1;
            while (p > 0 && better((int32_t)s, out[p - 1], row)) { out[p] = out[p - 1]; --p; }
            out[p] = (int32_t)s;
        }
        for (int r = kk; r < k; ++r) out[r] = -1;
    }
}

/* ------------------------------------------------------------------------ */
/* a6/a7. Shared-KV multi-query attention [Notes §1.1 last paragraph: each   */
/* compressed entry is both key and value; Walk §2.3.2 "MQA"; sink term from */
/* Notes §1.3 equation for s_{h,i,j}]:                                       */
/*   z_s   = scale * q[h] . KV[s]                  for s in the entry set T   */
/*   P_s   = exp(z_s) / (sum_{s' in T} exp(z_s') + [sink] exp(z'_h))         */
/*   out_h = sum_s P_s KV[s]                                                  */
/*   lse_h = log of the denominator above                                    */
/* The entry set of query t is idx[t][0..k) without the -1 entries (sparse,  */
/* CSA) or all s < floor(pos_t / mp) (dense, HCA).                           */
/* ------------------------------------------------------------------------ */
static void mqa_one(const double* q, const double* KV, const int32_t* ent, int64_t ne,
                    int H, int c, double scale, const double* sink, double* out, double* lse) {
    double* z = (double*)malloc(sizeof(double) * (ne > 0 ? ne : 1));
    for (int h = 0; h < H; ++h) {
        const double* qh = q + (int64_t)h * c;
        double mx = -INFINITY;
        for (int64_t i = 0; i < ne; ++i) {
            const double* kv = KV + (int64_t)ent[i] * c;
            double dot = 0.0;
            for (int e = 0; e < c; ++e) dot += qh[e] * kv[e];
            z[i] = scale * dot;
            if (z[i] > mx) mx = z[i];
        }
        if (sink && sink[h] > mx) mx = sink[h];
        double den = 0.0;
        for (int64_t i = 0; i < ne; ++i) den += exp(z[i] - mx);
        if (sink) den += exp(sink[h] - mx);
        double* oh = out + (int64_t)h * c;
        for (int e = 0; e < c; ++e) oh[e] = 0.0;
        if (ne == 0 && !sink) { lse[h] = -INFINITY; continue; }
        for (int64_t i = 0; i < ne; ++i) {
            double p = exp(z[i] - mx) / den;
            const double* kv = KV + (int64_t)ent[i] * c;
            for (int e = 0; e < c; ++e) oh[e] += p * kv[e];
        }
        lse[h] = mx + log(den);
    }
    free(z);
}

void orc_sparse_mqa(const double* q, const double* KV, const int32_t* idx, const int32_t* seq,
                    int nq, int H, int c, int64_t Nmax, int k, double scale, const double* sink,
                    double* out, double* lse) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < nq; ++t) {
        int32_t* ent = (int32_t*)malloc(sizeof(int32_t) * (k > 0 ? k : 1));
        int64_t ne = 0;
        for (int r = 0; r < k; ++r) {
            int32_t s = idx[(int64_t)t * k + r];
            if (s >= 0) ent[ne++] = s;
        }
        mqa_one(q + (int64_t)t * H * c, KV + (int64_t)seq[t] * Nmax * c, ent, ne, H, c, scale,
                sink, out + (int64_t)t * H * c, lse + (int64_t)t * H);
        free(ent);
    }
}

void orc_dense_mqa(const double* q, const double* KV, const int32_t* pos, const int32_t* seq,
                   int nq, int H, int c, int64_t Nmax, int mp, double scale, const double* sink,
                   double* out, double* lse) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < nq; ++t) {
        int64_t vis = pos[t] / mp;
        if (vis > Nmax) vis = Nmax;
        int32_t* ent = (int32_t*)malloc(sizeof(int32_t) * (vis > 0 ? vis : 1));
        for (int64_t s = 0; s < vis; ++s) ent[s] = (int32_t)s;
        mqa_one(q + (int64_t)t * H * c, KV + (int64_t)seq[t] * Nmax * c, ent, vis, H, c, scale,
                sink, out + (int64_t)t * H * c, lse + (int64_t)t * H);
        free(ent);
    }
}

/* ------------------------------------------------------------------------ */
/* Query / KV normalisation and partial rotary encoding [Walk §2.3.3 items 1 */
/* and 2; Notes §1.3 "Partial RoPE"]: every query head and every compressed  */
/* KV entry is RMS-normalised over its c channels before the core attention; */
/* the last R channels of both are then rotated by the row's position, and   */
/* the attention output is rotated back by the query's position so that it  */
/* carries relative rather than absolute position.                           */
/* Readings (the pages give no formula):                                      */
/*   norm:   y_j = x_j / sqrt(mean_j(x_j^2) + eps) * gamma_j                  */
/*   rotary: channels (c-R+2i, c-R+2i+1), i < R/2, form a pair turned by the  */
/*           angle p * theta_i, theta_i = base^(-2i/R), in the original       */
/*           rotary form (a, b) -> (a cos - b sin, a sin + b cos); the        */
/*           inverse turns by -p.                                             */
/* Row r belongs to group r / group (the H heads of one query share its      */
/* position); pos[g] is the position of group g. gamma == NULL skips the     */
/* norm, R == 0 skips the rotation.                                           */
/* ------------------------------------------------------------------------ */
void orc_norm_rope(const double* x, int64_t rows, int group, int c, const double* gamma, double eps,
                   int R, double base, const int32_t* pos, int inverse, double* y) {
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const double* xr = x + r * c;
        double* yr = y + r * c;
        if (gamma) {
            double ss = 0.0;
            for (int j = 0; j < c; ++j) ss += xr[j] * xr[j];
            double inv = 1.0 / sqrt(ss / c + eps);
            for (int j = 0; j < c; ++j) yr[j] = xr[j] * inv * gamma[j];
        } else {
            for (int j = 0; j < c; ++j) yr[j] = xr[j];
        }
        double p = (double)pos[r / group];
        for (int i = 0; i < R / 2; ++i) {
            double theta = pow(base, -2.0 * i / R);
            double ang = (inverse ? -p : p) * theta;
            int j = c - R + 2 * i;
            double a = yr[j], b = yr[j + 1];
            yr[j] = a * cos(ang) - b * sin(ang);
            yr[j + 1] = a * sin(ang) + b * cos(ang);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Sliding-window branch [Walk §2.3.3 item 3; Notes §1.3 "sliding window     */
/* branch", n_win = 128]: besides its selected compressed entries, the query */
/* at position p attends to the uncompressed KV rows of the n_win most       */
/* recent tokens, itself included (tokens p-n_win+1 .. p that exist). The    */
/* rows live in a per-sequence window ring [Walk §5 item 2, the SWA state   */
/* cache; Notes §2.6 Fig. 6]: token tau is row ring_off + (tau mod          */
/* ring_len) of its sequence's cache block. ent[t][j] is the row of token   */
/* p_t - n_win + 1 + j, or -1 before the start of the sequence. The window  */
/* rows then join the selected entries in ONE softmax (orc_sparse_mqa over  */
/* the concatenated list).                                                   */
/* ------------------------------------------------------------------------ */
void orc_window_entries(const int32_t* pos, int nq, int n_win, int64_t ring_off, int64_t ring_len,
                        int32_t* ent) {
    for (int t = 0; t < nq; ++t) {
        for (int j = 0; j < n_win; ++j) {
            int64_t tau = (int64_t)pos[t] - n_win + 1 + j;
            ent[(int64_t)t * n_win + j] = tau < 0 ? -1 : (int32_t)(ring_off + tau % ring_len);
        }
    }
}

/* Number of OpenMP threads the oracle runs with (for the CPU baseline). */
int orc_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads for the oracle's later parallel loops (the CPU baseline is timed
   at all cores and at one). */
void orc_set_num_threads(int n) {
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    omp_set_num_threads(n > 0 ? n : 1);
#else
    (void)n;
#endif
}
