/*
 * moda_oracle.c -- plain CPU fp64 oracle for the fused MoDA attention operator.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or constant with
 * the CUDA library.
 *
 * What it computes (sources are the pages' titles and sections):
 *
 *  [OP]  "Mixture-of-Depths Attention" paper summary (arXiv 2603.15619),
 *        section "Mixture-of-Depths Attention (MoDA): The Unified Operator",
 *        the joint-softmax equation: one softmax over the concatenated key set
 *        [K_seq || K_depth], scaled by 1/sqrt(d), applied to [V_seq || V_depth].
 *  [SEQ] same section, "Sequence causal mask": key j visible iff j <= t.
 *  [DEP] same section, "Depth matching mask": a query at token t sees only the
 *        L depth rows of token t, i.e. flattened depth rows [t*L, (t+1)*L).
 *  [GQA] "moda-attention 0.1.0" PyPI page, "Key Design Choices": G query heads
 *        share one KV head, expanded by repeat_interleave, so query head h
 *        reads KV head floor(h / G).
 *  [LAY] same PyPI page, "Using the Kernel Directly": Q [B,Hq,T,d],
 *        K,V [B,Hk,T,d], K_depth,V_depth [B,Hk,T*L,d] with row t*L + l.
 *  [HW]  paper summary, "Hardware-Efficient Implementation": the natural
 *        depth cache is layer-major; the flash-compatible layout stores the L
 *        depth rows of each token contiguously at [t*L, (t+1)*L).
 *  [NC]  ByteDance-Seed/MoDA README, "TODO" (a non-causal MoDA kernel), and
 *        paper summary, "7. Implications and Future Directions" (vision
 *        use): the sequence mask is dropped (every row sees keys 0..T-1),
 *        the depth matching mask is kept.
 *  [WIN] paper summary, "6. Limitations and Trade-offs", "The Quadratic-Depth
 *        FLOPs Growth is Untested at Production Scale" (bounded depth-KV
 *        slots, sliding-window recency policy): a token attends only to the
 *        last S of its L depth rows (rows t*L + L - S .. t*L + L - 1); S = 0
 *        means all L.
 *
 * The pages give no backward formulas.  The backward here is the plain
 * derivative of the forward definition (chain rule through one softmax):
 *   P = softmax(row),  D = sum(dO * O),  dS = P * (dO . v - D),
 *   dq = scale * sum dS k,  dk_j += scale * dS q,  dv_j += P dO,
 * applied to sequence and depth keys alike.
 *
 * Every score row is materialised in full (all visible entries); there is no
 * online rescaling, blocking or reordering.  All arithmetic is double.
 * Build:  gcc -O2 -fopenmp -shared -fPIC moda_oracle.c -o libmoda_oracle.so -lm
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

static double dot(const double* a, const double* b, int d) {
    double s = 0.0;
    for (int i = 0; i < d; ++i) s += a[i] * b[i];
    return s;
}

/* Index helpers for the [LAY] layouts. */
static size_t q_off(int b, int h, int t, int Hq, int T, int d) {
    return (((size_t)b * Hq + h) * T + t) * (size_t)d;
}
static size_t kv_off(int b, int hk, int j, int Hk, int T, int d) {
    return (((size_t)b * Hk + hk) * T + j) * (size_t)d;
}
static size_t kd_off(int b, int hk, int t, int l, int Hk, int T, int L, int d) {
    return ((((size_t)b * Hk + hk) * T + t) * (size_t)L + l) * (size_t)d;
}

/*
 * One query row of the operator [OP]: one softmax over exactly the given
 * visible rows (the masks [SEQ], [DEP], [NC], [WIN] choose them; see the
 * callers below).
 *   q      : d values of the query
 *   Kseq   : n_seq visible sequence keys, row stride d
 *   Vseq   : same for values
 *   Kdep   : n_dep visible depth keys of the query's token, stride d
 *   Vdep   : same for values
 *   p_out  : optional (n_seq + n_dep) doubles; receives the normalised weights
 * Writes o[d] and *lse (natural log of the softmax denominator, plus max).
 */
void moda_oracle_row(int n_seq, int n_dep, int d, double scale,
                     const double* q, const double* Kseq, const double* Vseq,
                     const double* Kdep, const double* Vdep,
                     double* o, double* lse, double* p_out) {
    const int n = n_seq + n_dep;
    double* row = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    /* the concatenated [seq | depth] score row */
    for (int j = 0; j < n_seq; ++j) row[j] = scale * dot(q, Kseq + (size_t)j * d, d);
    for (int l = 0; l < n_dep; ++l) row[n_seq + l] = scale * dot(q, Kdep + (size_t)l * d, d);
    double m = row[0];
    for (int i = 1; i < n; ++i) if (row[i] > m) m = row[i];
    double Z = 0.0;
    for (int i = 0; i < n; ++i) { row[i] = exp(row[i] - m); Z += row[i]; }
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    for (int j = 0; j < n_seq; ++j) {
        const double w = row[j] / Z;
        for (int c = 0; c < d; ++c) o[c] += w * Vseq[(size_t)j * d + c];
    }
    for (int l = 0; l < n_dep; ++l) {
        const double w = row[n_seq + l] / Z;
        for (int c = 0; c < d; ++c) o[c] += w * Vdep[(size_t)l * d + c];
    }
    *lse = m + log(Z);
    if (p_out) for (int i = 0; i < n; ++i) p_out[i] = row[i] / Z;
    free(row);
}

/* Visible sequence keys of token t: 0..t ([SEQ]) or 0..T-1 ([NC]). */
static int seq_count(int t, int T, int causal) { return causal ? t + 1 : T; }
/* First visible depth row of a token within its L rows ([DEP], [WIN]). */
static int dep_first(int L, int window) { return (window > 0 && window < L) ? L - window : 0; }

/* Check the shape arguments shared by every entry point; 0 on success. */
static int bad_shape(int B, int Hq, int Hk, int T, int d, int L) {
    if (B < 0 || Hq <= 0 || Hk <= 0 || T < 0 || d <= 0 || L < 0) return 1;
    if (Hq % Hk != 0) return 1;
    return 0;
}
static int bad_mode(int L, int window) { return window < 0 || window > L; }

/*
 * Full forward over all (b, h, t).  Q [B,Hq,T,d], K,V [B,Hk,T,d],
 * Kd,Vd [B,Hk,T*L,d] (may be NULL when L == 0), O [B,Hq,T,d], LSE [B,Hq,T].
 * scale <= 0 selects 1/sqrt(d); causal = 0 drops the sequence mask [NC];
 * window > 0 keeps only the last `window` depth rows of each token [WIN].
 * Returns 0, or -1 on a bad shape.
 */
int moda_oracle_fwd_ex(int B, int Hq, int Hk, int T, int d, int L, double scale, int causal,
                       int window, const double* Q, const double* K, const double* V,
                       const double* Kd, const double* Vd, double* O, double* LSE) {
    if (bad_shape(B, Hq, Hk, T, d, L) || bad_mode(L, window)) return -1;
    if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
    const int G = Hq / Hk;
    const int l0 = dep_first(L, window);
    #pragma omp parallel for collapse(3) schedule(dynamic, 16)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hq; ++h)
            for (int t = 0; t < T; ++t) {
                const int hk = h / G;   /* [GQA] */
                const double* kd = L ? Kd + kd_off(b, hk, t, l0, Hk, T, L, d) : NULL;
                const double* vd = L ? Vd + kd_off(b, hk, t, l0, Hk, T, L, d) : NULL;
                moda_oracle_row(seq_count(t, T, causal), L - l0, d, scale,
                                Q + q_off(b, h, t, Hq, T, d),
                                K + kv_off(b, hk, 0, Hk, T, d), V + kv_off(b, hk, 0, Hk, T, d),
                                kd, vd, O + q_off(b, h, t, Hq, T, d),
                                LSE + ((size_t)b * Hq + h) * T + t, NULL);
            }
    return 0;
}

/* The operator as the pages define it: causal, every depth row. */
int moda_oracle_fwd(int B, int Hq, int Hk, int T, int d, int L, double scale,
                    const double* Q, const double* K, const double* V,
                    const double* Kd, const double* Vd, double* O, double* LSE) {
    return moda_oracle_fwd_ex(B, Hq, Hk, T, d, L, scale, 1, 0, Q, K, V, Kd, Vd, O, LSE);
}

/*
 * Backward over all (b, hk) slices, following the chain rule written in the
 * file header.  The forward statistics (O, LSE) are recomputed here in fp64
 * from the inputs; nothing computed elsewhere is used.
 * Outputs dQ [B,Hq,T,d], dK,dV [B,Hk,T,d], dKd,dVd [B,Hk,T*L,d] are fully
 * overwritten.  Returns 0, or -1 on a bad shape.
 */
int moda_oracle_bwd_ex(int B, int Hq, int Hk, int T, int d, int L, double scale, int causal,
                       int window, const double* Q, const double* K, const double* V,
                       const double* Kd, const double* Vd, const double* dO,
                       double* dQ, double* dK, double* dV, double* dKd, double* dVd) {
    if (bad_shape(B, Hq, Hk, T, d, L) || bad_mode(L, window)) return -1;
    if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
    const int G = Hq / Hk;
    const int l0 = dep_first(L, window);
    const size_t nrow = (size_t)B * Hq * T;
    double* O = (double*)malloc(sizeof(double) * nrow * (size_t)d);
    double* LSE = (double*)malloc(sizeof(double) * nrow);
    double* Dr = (double*)malloc(sizeof(double) * nrow);
    moda_oracle_fwd_ex(B, Hq, Hk, T, d, L, scale, causal, window, Q, K, V, Kd, Vd, O, LSE);
    /* D = rowsum(dO * O) */
    for (size_t r = 0; r < nrow; ++r) Dr[r] = dot(dO + r * d, O + r * d, d);

    /* Pass 1, per query row: dq, and the token-local depth gradients. */
    if (L) {
        memset(dKd, 0, sizeof(double) * (size_t)B * Hk * T * L * d);
        memset(dVd, 0, sizeof(double) * (size_t)B * Hk * T * L * d);
    }
    #pragma omp parallel for collapse(3) schedule(dynamic, 16)
    for (int b = 0; b < B; ++b)
        for (int hk = 0; hk < Hk; ++hk)
            for (int t = 0; t < T; ++t) {
                for (int g = 0; g < G; ++g) {
                    const int h = hk * G + g;
                    const size_t r = ((size_t)b * Hq + h) * T + t;
                    const double* q = Q + r * d;
                    const double* go = dO + r * d;
                    double* dq = dQ + r * d;
                    for (int c = 0; c < d; ++c) dq[c] = 0.0;
                    for (int j = 0; j < seq_count(t, T, causal); ++j) {
                        const double* k = K + kv_off(b, hk, j, Hk, T, d);
                        const double* v = V + kv_off(b, hk, j, Hk, T, d);
                        const double p = exp(scale * dot(q, k, d) - LSE[r]);
                        const double ds = p * (dot(go, v, d) - Dr[r]);
                        for (int c = 0; c < d; ++c) dq[c] += scale * ds * k[c];
                    }
                    for (int l = l0; l < L; ++l) {
                        const size_t o = kd_off(b, hk, t, l, Hk, T, L, d);
                        const double p = exp(scale * dot(q, Kd + o, d) - LSE[r]);
                        const double ds = p * (dot(go, Vd + o, d) - Dr[r]);
                        for (int c = 0; c < d; ++c) {
                            dq[c] += scale * ds * Kd[o + c];
                            /* token t's depth rows are touched only by this (b,hk,t) */
                            dKd[o + c] += scale * ds * q[c];
                            dVd[o + c] += p * go[c];
                        }
                    }
                }
            }

    /* Pass 2, per sequence key j: sum over every query row that sees it. */
    #pragma omp parallel for collapse(3) schedule(dynamic, 16)
    for (int b = 0; b < B; ++b)
        for (int hk = 0; hk < Hk; ++hk)
            for (int j = 0; j < T; ++j) {
                const double* k = K + kv_off(b, hk, j, Hk, T, d);
                const double* v = V + kv_off(b, hk, j, Hk, T, d);
                double* dk = dK + kv_off(b, hk, j, Hk, T, d);
                double* dv = dV + kv_off(b, hk, j, Hk, T, d);
                for (int c = 0; c < d; ++c) { dk[c] = 0.0; dv[c] = 0.0; }
                for (int g = 0; g < G; ++g) {
                    const int h = hk * G + g;
                    for (int t = causal ? j : 0; t < T; ++t) {
                        const size_t r = ((size_t)b * Hq + h) * T + t;
                        const double* q = Q + r * d;
                        const double* go = dO + r * d;
                        const double p = exp(scale * dot(q, k, d) - LSE[r]);
                        const double ds = p * (dot(go, v, d) - Dr[r]);
                        for (int c = 0; c < d; ++c) {
                            dk[c] += scale * ds * q[c];
                            dv[c] += p * go[c];
                        }
                    }
                }
            }
    free(O); free(LSE); free(Dr);
    return 0;
}

/* The backward of the operator as the pages define it: causal, all depth rows. */
int moda_oracle_bwd(int B, int Hq, int Hk, int T, int d, int L, double scale,
                    const double* Q, const double* K, const double* V,
                    const double* Kd, const double* Vd, const double* dO,
                    double* dQ, double* dK, double* dV, double* dKd, double* dVd) {
    return moda_oracle_bwd_ex(B, Hq, Hk, T, d, L, scale, 1, 0, Q, K, V, Kd, Vd, dO, dQ, dK, dV,
                              dKd, dVd);
}

/*
 * Depth repack [HW]: the layer-major cache src [L,B,Hk,T,d] becomes the
 * token-major (flash-compatible) dst [B,Hk,T*L,d] with row t*L + l.  Element
 * size is es bytes (the copy is bytewise, so any element type works).
 */
int moda_oracle_repack(int B, int Hk, int T, int d, int L, int es,
                       const void* src, void* dst) {
    if (B < 0 || Hk <= 0 || T < 0 || d <= 0 || L < 0 || es <= 0) return -1;
    const size_t rowb = (size_t)d * es;
    for (int l = 0; l < L; ++l)
        for (int b = 0; b < B; ++b)
            for (int hk = 0; hk < Hk; ++hk)
                for (int t = 0; t < T; ++t) {
                    const size_t s = (((size_t)l * B + b) * Hk + hk) * T + t;
                    const size_t o = (((size_t)b * Hk + hk) * T + t) * L + l;
                    memcpy((char*)dst + o * rowb, (const char*)src + s * rowb, rowb);
                }
    return 0;
}

/* Threads OpenMP will use for the parallel loops above. */
int moda_oracle_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
