/*
 * Retention oracle: plain, slow, fp64 CPU implementation of RetNet retention.
 *
 * TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and bench.py's
 * CPU-baseline leg may load this library. The product path (the CUDA library
 * under linear_attention_ret_b200/) never calls it and shares no code with it.
 *
 * Every function follows one passage of the source pages and cites it:
 *   [RM]   aiqz.cc, "RetNet retention mechanism" tutorial page
 *          (sections: 保留机制初识 "first look", 衰减矩阵 "decay matrix",
 *           并行训练 "parallel training", 递归推理 "recurrent inference",
 *           块级循环 "chunkwise recurrence").
 *   [RN]   171host.com, "Retentive Network (RetNet) 详解" explainer page,
 *          section 3.1 (recurrent / parallel / chunkwise forms) and 3.2 (MSR).
 *   [GR]   pwwt.cn, "unilm RetNet 技术指南 ... YOCO 中 Gated RetNet 的源码解析"
 *          page, sections on parallel_gate_retention, chunk_gate_retention,
 *          recurrent_gate_retention and the Triton kernels (cross_chunk,
 *          inner_chunk).
 *
 * Layouts (all row-major, contiguous, fp64):
 *   q, k : [B, H, N, dk]     v, o : [B, H, N, dv]
 *   gamma: [H]  (one decay per head: multi-scale retention, [RN] 3.2)
 *   g    : [B, H, N]  natural-log decay per token (gated form, [GR])
 *   state: [B, H, dk, dv]    (the K^T V matrix, [RM] 递归推理)
 *
 * Readings of points the pages leave open:
 *   - Real inputs; the "dagger" of [RN] 3.1 is a plain transpose.
 *   - No 1/sqrt(dk) scaling inside the operator.
 *   - gamma^0 = 1 (also for gamma = 0), so D_nn = 1.
 *   - Decode output uses the UPDATED state: o_n = q_n S_n ([RM] 递归推理).
 *   - Chunkwise cross term: row j (0-based inside the chunk) of chunk i gets
 *     gamma^(j+1) * q_j S_{i-1}; the state update weights key m by
 *     gamma^(L-1-m) and decays the old state by gamma^L (L = chunk length).
 *     [RM]'s printed chunkwise equation shows a single gamma^c factor; only the
 *     per-row reading makes the chunkwise form equal the parallel form, which
 *     the same page states it does. [GR]'s cross_chunk uses exactly this
 *     chunk-end key weighting, written in log space as exp(-g + g_last).
 *   - Gated: G = inclusive cumulative sum of g; D_nm = exp(G_n - G_m) for
 *     n >= m; recurrent S_n = exp(g_n) S_{n-1} + k_n^T v_n.
 *   - A ragged last chunk behaves as zero padding; its decays use its true
 *     length L.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC oracle.c -o liboracle.so -lm
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EBADARG 1
#define ORACLE_ENOMEM 2

static int bad_dims(int B, int H, int N, int dk, int dv) {
    return B <= 0 || H <= 0 || N < 0 || dk <= 0 || dv <= 0;
}

/* gamma^n for integer n >= 0 with gamma^0 = 1 (also for gamma = 0). */
static double gpow(double gamma, int n) {
    if (n == 0) return 1.0;
    return pow(gamma, (double)n);
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * [RM] 衰减矩阵 (decay matrix): D_nm = gamma^(n-m) if n >= m, else 0.
 * D is [N, N] row-major.
 */
int oracle_decay_matrix(double gamma, int N, double* D) {
    if (N < 0 || !D) return ORACLE_EBADARG;
    for (int n = 0; n < N; ++n)
        for (int m = 0; m < N; ++m)
            D[(size_t)n * N + m] = (n >= m) ? gpow(gamma, n - m) : 0.0;
    return ORACLE_OK;
}

/*
 * [RM] 保留机制初识 (first look): R_n = sum_{m<=n} gamma^(n-m) (Q_n K_m^T) V_m.
 * The definition written out as nested loops, one term at a time.
 */
int oracle_ret_brute(const double* q, const double* k, const double* v,
                     const double* gamma, double* o,
                     int B, int H, int N, int dk, int dv) {
    if (bad_dims(B, H, N, dk, dv) || !q || !k || !v || !gamma || !o) return ORACLE_EBADARG;
    #pragma omp parallel for schedule(static)
    for (int bh = 0; bh < B * H; ++bh) {
        const double gm = gamma[bh % H];
        const double* Q = q + (size_t)bh * N * dk;
        const double* K = k + (size_t)bh * N * dk;
        const double* V = v + (size_t)bh * N * dv;
        double* O = o + (size_t)bh * N * dv;
        for (int n = 0; n < N; ++n) {
            for (int c = 0; c < dv; ++c) O[(size_t)n * dv + c] = 0.0;
            for (int m = 0; m <= n; ++m) {
                double qk = 0.0;
                for (int d = 0; d < dk; ++d) qk += Q[(size_t)n * dk + d] * K[(size_t)m * dk + d];
                const double w = gpow(gm, n - m) * qk;
                for (int c = 0; c < dv; ++c) O[(size_t)n * dv + c] += w * V[(size_t)m * dv + c];
            }
        }
    }
    return ORACLE_OK;
}

/*
 * [RM] 并行训练 (parallel training) and [RN] 3.1 parallel form:
 *   R = (Q K^T (.) D) V, with D from [RM] 衰减矩阵.
 * Three steps as the page lists them: the score table Q K^T, the elementwise
 * product with D, then the product with V.
 */
int oracle_ret_parallel(const double* q, const double* k, const double* v,
                        const double* gamma, double* o,
                        int B, int H, int N, int dk, int dv) {
    if (bad_dims(B, H, N, dk, dv) || !q || !k || !v || !gamma || !o) return ORACLE_EBADARG;
    int err = ORACLE_OK;
    #pragma omp parallel
    {
        double* A = (double*)malloc(sizeof(double) * (size_t)N * N + 1);
        double* D = (double*)malloc(sizeof(double) * (size_t)N * N + 1);
        if (!A || !D) {
            #pragma omp atomic write
            err = ORACLE_ENOMEM;
        } else {
            #pragma omp for schedule(static)
            for (int bh = 0; bh < B * H; ++bh) {
                const double* Q = q + (size_t)bh * N * dk;
                const double* K = k + (size_t)bh * N * dk;
                const double* V = v + (size_t)bh * N * dv;
                double* O = o + (size_t)bh * N * dv;
                oracle_decay_matrix(gamma[bh % H], N, D);
                /* step 1: A = Q K^T */
                for (int n = 0; n < N; ++n)
                    for (int m = 0; m < N; ++m) {
                        double s = 0.0;
                        for (int d = 0; d < dk; ++d) s += Q[(size_t)n * dk + d] * K[(size_t)m * dk + d];
                        A[(size_t)n * N + m] = s;
                    }
                /* step 2: A (.) D */
                for (size_t t = 0; t < (size_t)N * N; ++t) A[t] *= D[t];
                /* step 3: (A (.) D) V */
                for (int n = 0; n < N; ++n) {
                    for (int c = 0; c < dv; ++c) O[(size_t)n * dv + c] = 0.0;
                    for (int m = 0; m < N; ++m) {
                        const double w = A[(size_t)n * N + m];
                        for (int c = 0; c < dv; ++c) O[(size_t)n * dv + c] += w * V[(size_t)m * dv + c];
                    }
                }
            }
        }
        free(A);
        free(D);
    }
    return err;
}

/*
 * [RM] 递归推理 (recurrent inference), [RN] 3.1 recurrent form:
 *   S_n = gamma S_{n-1} + K_n^T V_n,   R_n = Q_n S_n.
 * s_in: initial state (NULL = zeros); s_out: final state (NULL = not wanted).
 */
int oracle_ret_recurrent(const double* q, const double* k, const double* v,
                         const double* gamma, const double* s_in, double* s_out,
                         double* o, int B, int H, int N, int dk, int dv) {
    if (bad_dims(B, H, N, dk, dv) || !q || !k || !v || !gamma || !o) return ORACLE_EBADARG;
    int err = ORACLE_OK;
    #pragma omp parallel
    {
        double* S = (double*)malloc(sizeof(double) * (size_t)dk * dv);
        if (!S) {
            #pragma omp atomic write
            err = ORACLE_ENOMEM;
        } else {
            #pragma omp for schedule(static)
            for (int bh = 0; bh < B * H; ++bh) {
                const double gm = gamma[bh % H];
                const double* Q = q + (size_t)bh * N * dk;
                const double* K = k + (size_t)bh * N * dk;
                const double* V = v + (size_t)bh * N * dv;
                double* O = o + (size_t)bh * N * dv;
                if (s_in) memcpy(S, s_in + (size_t)bh * dk * dv, sizeof(double) * (size_t)dk * dv);
                else memset(S, 0, sizeof(double) * (size_t)dk * dv);
                for (int n = 0; n < N; ++n) {
                    /* S_n = gamma S_{n-1} + K_n^T V_n */
                    for (int a = 0; a < dk; ++a) {
                        const double kn = K[(size_t)n * dk + a];
                        for (int c = 0; c < dv; ++c)
                            S[(size_t)a * dv + c] = gm * S[(size_t)a * dv + c] + kn * V[(size_t)n * dv + c];
                    }
                    /* R_n = Q_n S_n */
                    for (int c = 0; c < dv; ++c) O[(size_t)n * dv + c] = 0.0;
                    for (int a = 0; a < dk; ++a) {
                        const double qn = Q[(size_t)n * dk + a];
                        for (int c = 0; c < dv; ++c) O[(size_t)n * dv + c] += qn * S[(size_t)a * dv + c];
                    }
                }
                if (s_out) memcpy(s_out + (size_t)bh * dk * dv, S, sizeof(double) * (size_t)dk * dv);
            }
        }
        free(S);
    }
    return err;
}

/*
 * One decode step of [RM] 递归推理 for every (b, h): S <- gamma S + k^T v, o = q S.
 * q, k: [B, H, dk]; v, o: [B, H, dv]; S: [B, H, dk, dv] updated in place.
 */
int oracle_ret_recurrent_step(const double* q, const double* k, const double* v,
                              const double* gamma, double* S, double* o,
                              int B, int H, int dk, int dv) {
    if (bad_dims(B, H, 1, dk, dv) || !S) return ORACLE_EBADARG;
    return oracle_ret_recurrent(q, k, v, gamma, S, S, o, B, H, 1, dk, dv);
}

/*
 * [RM] 块级循环 (chunkwise recurrence) and [RN] 3.1 / 4.3: split the sequence
 * into chunks; inside a chunk use the parallel form, across chunks pass the
 * state. For chunk i of length L (local positions j, m = 0..L-1):
 *   inner:  (Q_[i] K_[i]^T (.) D) V_[i]          D_jm = gamma^(j-m), j >= m
 *   cross:  gamma^(j+1) * (Q_[i] S_[i-1])_j
 *   state:  S_[i] = gamma^L S_[i-1] + sum_m gamma^(L-1-m) K_m^T V_m
 * (per-row cross factor and key weights: see the header).
 */
int oracle_ret_chunkwise(const double* q, const double* k, const double* v,
                         const double* gamma, const double* s_in, double* s_out,
                         double* o, int B, int H, int N, int dk, int dv, int chunk) {
    if (bad_dims(B, H, N, dk, dv) || chunk <= 0 || !q || !k || !v || !gamma || !o) return ORACLE_EBADARG;
    int err = ORACLE_OK;
    #pragma omp parallel
    {
        double* S = (double*)malloc(sizeof(double) * (size_t)dk * dv);
        double* A = (double*)malloc(sizeof(double) * (size_t)chunk * chunk);
        if (!S || !A) {
            #pragma omp atomic write
            err = ORACLE_ENOMEM;
        } else {
            #pragma omp for schedule(static)
            for (int bh = 0; bh < B * H; ++bh) {
                const double gm = gamma[bh % H];
                const double* Q = q + (size_t)bh * N * dk;
                const double* K = k + (size_t)bh * N * dk;
                const double* V = v + (size_t)bh * N * dv;
                double* O = o + (size_t)bh * N * dv;
                if (s_in) memcpy(S, s_in + (size_t)bh * dk * dv, sizeof(double) * (size_t)dk * dv);
                else memset(S, 0, sizeof(double) * (size_t)dk * dv);
                for (int t0 = 0; t0 < N; t0 += chunk) {
                    const int L = (N - t0 < chunk) ? (N - t0) : chunk;
                    const double* Qi = Q + (size_t)t0 * dk;
                    const double* Ki = K + (size_t)t0 * dk;
                    const double* Vi = V + (size_t)t0 * dv;
                    double* Oi = O + (size_t)t0 * dv;
                    /* inner: A = (Q_[i] K_[i]^T) (.) D */
                    for (int j = 0; j < L; ++j)
                        for (int m = 0; m < L; ++m) {
                            double s = 0.0;
                            for (int d = 0; d < dk; ++d) s += Qi[(size_t)j * dk + d] * Ki[(size_t)m * dk + d];
                            A[(size_t)j * L + m] = (j >= m) ? s * gpow(gm, j - m) : 0.0;
                        }
                    for (int j = 0; j < L; ++j) {
                        double* oj = Oi + (size_t)j * dv;
                        for (int c = 0; c < dv; ++c) oj[c] = 0.0;
                        /* inner: A V_[i] */
                        for (int m = 0; m < L; ++m) {
                            const double w = A[(size_t)j * L + m];
                            for (int c = 0; c < dv; ++c) oj[c] += w * Vi[(size_t)m * dv + c];
                        }
                        /* cross: gamma^(j+1) Q_j S_[i-1] */
                        const double r = gpow(gm, j + 1);
                        for (int a = 0; a < dk; ++a) {
                            const double qa = r * Qi[(size_t)j * dk + a];
                            for (int c = 0; c < dv; ++c) oj[c] += qa * S[(size_t)a * dv + c];
                        }
                    }
                    /* state: S_[i] = gamma^L S_[i-1] + sum_m gamma^(L-1-m) K_m^T V_m */
                    const double decay = gpow(gm, L);
                    for (size_t t = 0; t < (size_t)dk * dv; ++t) S[t] *= decay;
                    for (int m = 0; m < L; ++m) {
                        const double zeta = gpow(gm, L - 1 - m);
                        for (int a = 0; a < dk; ++a) {
                            const double ka = zeta * Ki[(size_t)m * dk + a];
                            for (int c = 0; c < dv; ++c) S[(size_t)a * dv + c] += ka * Vi[(size_t)m * dv + c];
                        }
                    }
                }
                if (s_out) memcpy(s_out + (size_t)bh * dk * dv, S, sizeof(double) * (size_t)dk * dv);
            }
        }
        free(S);
        free(A);
    }
    return err;
}

/* ------------------------------------------------------------------------ */
/* Gated retention ([GR]): the per-token log-decay g replaces log(gamma).    */
/* ------------------------------------------------------------------------ */

/*
 * Definition by products of per-step decays, read off the gated recurrence of
 * [GR] (recurrent_gate_retention: kv <- prev_kv * decay + k^T v):
 *   o_n = sum_{m<=n} exp(g_{m+1} + ... + g_n) (q_n . k_m) v_m.
 * Each weight sums its own run of g (no cumulative-sum differences).
 */
int oracle_gated_brute(const double* q, const double* k, const double* v,
                       const double* g, double* o,
                       int B, int H, int N, int dk, int dv) {
    if (bad_dims(B, H, N, dk, dv) || !q || !k || !v || !g || !o) return ORACLE_EBADARG;
    #pragma omp parallel for schedule(static)
    for (int bh = 0; bh < B * H; ++bh) {
        const double* Q = q + (size_t)bh * N * dk;
        const double* K = k + (size_t)bh * N * dk;
        const double* V = v + (size_t)bh * N * dv;
        const double* Gt = g + (size_t)bh * N;
        double* O = o + (size_t)bh * N * dv;
        for (int n = 0; n < N; ++n) {
            for (int c = 0; c < dv; ++c) O[(size_t)n * dv + c] = 0.0;
            for (int m = 0; m <= n; ++m) {
                double run = 0.0;
                for (int t = m + 1; t <= n; ++t) run += Gt[t];
                double qk = 0.0;
                for (int d = 0; d < dk; ++d) qk += Q[(size_t)n * dk + d] * K[(size_t)m * dk + d];
                const double w = exp(run) * qk;
                for (int c = 0; c < dv; ++c) O[(size_t)n * dv + c] += w * V[(size_t)m * dv + c];
            }
        }
    }
    return ORACLE_OK;
}

/*
 * [GR] parallel_gate_retention: G = cumsum(g); mask_nm = G_n - G_m for n >= m
 * (minus infinity above the diagonal, the causal mask); attn = (q k^T) * exp(mask);
 * o = attn v.
 */
int oracle_gated_parallel(const double* q, const double* k, const double* v,
                          const double* g, double* o,
                          int B, int H, int N, int dk, int dv) {
    if (bad_dims(B, H, N, dk, dv) || !q || !k || !v || !g || !o) return ORACLE_EBADARG;
    int err = ORACLE_OK;
    #pragma omp parallel
    {
        double* A = (double*)malloc(sizeof(double) * (size_t)N * N + 1);
        double* G = (double*)malloc(sizeof(double) * (size_t)N + 1);
        if (!A || !G) {
            #pragma omp atomic write
            err = ORACLE_ENOMEM;
        } else {
            #pragma omp for schedule(static)
            for (int bh = 0; bh < B * H; ++bh) {
                const double* Q = q + (size_t)bh * N * dk;
                const double* K = k + (size_t)bh * N * dk;
                const double* V = v + (size_t)bh * N * dv;
                const double* Gt = g + (size_t)bh * N;
                double* O = o + (size_t)bh * N * dv;
                double acc = 0.0;
                for (int n = 0; n < N; ++n) { acc += Gt[n]; G[n] = acc; }
                for (int n = 0; n < N; ++n)
                    for (int m = 0; m < N; ++m) {
                        double s = 0.0;
                        for (int d = 0; d < dk; ++d) s += Q[(size_t)n * dk + d] * K[(size_t)m * dk + d];
                        A[(size_t)n * N + m] = (n >= m) ? s * exp(G[n] - G[m]) : 0.0;
                    }
                for (int n = 0; n < N; ++n) {
                    for (int c = 0; c < dv; ++c) O[(size_t)n * dv + c] = 0.0;
                    for (int m = 0; m <= n; ++m) {
                        const double w = A[(size_t)n * N + m];
                        for (int c = 0; c < dv; ++c) O[(size_t)n * dv + c] += w * V[(size_t)m * dv + c];
                    }
                }
            }
        }
        free(A);
        free(G);
    }
    return err;
}

/*
 * [GR] recurrent_gate_retention: S_n = exp(g_n) S_{n-1} + k_n^T v_n, o_n = q_n S_n.
 * (The page scales k by key_dim^-0.5 inside the module; the operator here takes
 * already-scaled inputs.)
 */
int oracle_gated_recurrent(const double* q, const double* k, const double* v,
                           const double* g, const double* s_in, double* s_out,
                           double* o, int B, int H, int N, int dk, int dv) {
    if (bad_dims(B, H, N, dk, dv) || !q || !k || !v || !g || !o) return ORACLE_EBADARG;
    int err = ORACLE_OK;
    #pragma omp parallel
    {
        double* S = (double*)malloc(sizeof(double) * (size_t)dk * dv);
        if (!S) {
            #pragma omp atomic write
            err = ORACLE_ENOMEM;
        } else {
            #pragma omp for schedule(static)
            for (int bh = 0; bh < B * H; ++bh) {
                const double* Q = q + (size_t)bh * N * dk;
                const double* K = k + (size_t)bh * N * dk;
                const double* V = v + (size_t)bh * N * dv;
                const double* Gt = g + (size_t)bh * N;
                double* O = o + (size_t)bh * N * dv;
                if (s_in) memcpy(S, s_in + (size_t)bh * dk * dv, sizeof(double) * (size_t)dk * dv);
                else memset(S, 0, sizeof(double) * (size_t)dk * dv);
                for (int n = 0; n < N; ++n) {
                    const double a = exp(Gt[n]);
                    for (int r = 0; r < dk; ++r) {
                        const double kn = K[(size_t)n * dk + r];
                        for (int c = 0; c < dv; ++c)
                            S[(size_t)r * dv + c] = a * S[(size_t)r * dv + c] + kn * V[(size_t)n * dv + c];
                    }
                    for (int c = 0; c < dv; ++c) O[(size_t)n * dv + c] = 0.0;
                    for (int r = 0; r < dk; ++r) {
                        const double qn = Q[(size_t)n * dk + r];
                        for (int c = 0; c < dv; ++c) O[(size_t)n * dv + c] += qn * S[(size_t)r * dv + c];
                    }
                }
                if (s_out) memcpy(s_out + (size_t)bh * dk * dv, S, sizeof(double) * (size_t)dk * dv);
            }
        }
        free(S);
    }
    return err;
}

/*
 * [GR] chunk_gate_retention = cross_chunk + inner_chunk. With Gl the inclusive
 * cumulative sum of g restarted at each chunk (local j, m = 0..L-1):
 *   inner_chunk: (q k^T) * exp(Gl_j - Gl_m) for j >= m, times v
 *   cross:       exp(Gl_j) * (q_j S_[i-1])
 *   cross_chunk: S_[i] = exp(Gl_{L-1}) S_[i-1]
 *                        + sum_m exp(Gl_{L-1} - Gl_m) k_m^T v_m
 * (the chunk-end weighting exp(-g + g[..., -1]) of the page, in local sums).
 */
int oracle_gated_chunkwise(const double* q, const double* k, const double* v,
                           const double* g, const double* s_in, double* s_out,
                           double* o, int B, int H, int N, int dk, int dv, int chunk) {
    if (bad_dims(B, H, N, dk, dv) || chunk <= 0 || !q || !k || !v || !g || !o) return ORACLE_EBADARG;
    int err = ORACLE_OK;
    #pragma omp parallel
    {
        double* S = (double*)malloc(sizeof(double) * (size_t)dk * dv);
        double* A = (double*)malloc(sizeof(double) * (size_t)chunk * chunk);
        double* Gl = (double*)malloc(sizeof(double) * (size_t)chunk);
        if (!S || !A || !Gl) {
            #pragma omp atomic write
            err = ORACLE_ENOMEM;
        } else {
            #pragma omp for schedule(static)
            for (int bh = 0; bh < B * H; ++bh) {
                const double* Q = q + (size_t)bh * N * dk;
                const double* K = k + (size_t)bh * N * dk;
                const double* V = v + (size_t)bh * N * dv;
                const double* Gt = g + (size_t)bh * N;
                double* O = o + (size_t)bh * N * dv;
                if (s_in) memcpy(S, s_in + (size_t)bh * dk * dv, sizeof(double) * (size_t)dk * dv);
                else memset(S, 0, sizeof(double) * (size_t)dk * dv);
                for (int t0 = 0; t0 < N; t0 += chunk) {
                    const int L = (N - t0 < chunk) ? (N - t0) : chunk;
                    const double* Qi = Q + (size_t)t0 * dk;
                    const double* Ki = K + (size_t)t0 * dk;
                    const double* Vi = V + (size_t)t0 * dv;
                    double* Oi = O + (size_t)t0 * dv;
                    double acc = 0.0;
                    for (int j = 0; j < L; ++j) { acc += Gt[t0 + j]; Gl[j] = acc; }
                    for (int j = 0; j < L; ++j)
                        for (int m = 0; m < L; ++m) {
                            double s = 0.0;
                            for (int d = 0; d < dk; ++d) s += Qi[(size_t)j * dk + d] * Ki[(size_t)m * dk + d];
                            A[(size_t)j * L + m] = (j >= m) ? s * exp(Gl[j] - Gl[m]) : 0.0;
                        }
                    for (int j = 0; j < L; ++j) {
                        double* oj = Oi + (size_t)j * dv;
                        for (int c = 0; c < dv; ++c) oj[c] = 0.0;
                        for (int m = 0; m < L; ++m) {
                            const double w = A[(size_t)j * L + m];
                            for (int c = 0; c < dv; ++c) oj[c] += w * Vi[(size_t)m * dv + c];
                        }
                        const double r = exp(Gl[j]);
                        for (int a = 0; a < dk; ++a) {
                            const double qa = r * Qi[(size_t)j * dk + a];
                            for (int c = 0; c < dv; ++c) oj[c] += qa * S[(size_t)a * dv + c];
                        }
                    }
                    const double decay = exp(Gl[L - 1]);
                    for (size_t t = 0; t < (size_t)dk * dv; ++t) S[t] *= decay;
                    for (int m = 0; m < L; ++m) {
                        const double zeta = exp(Gl[L - 1] - Gl[m]);
                        for (int a = 0; a < dk; ++a) {
                            const double ka = zeta * Ki[(size_t)m * dk + a];
                            for (int c = 0; c < dv; ++c) S[(size_t)a * dv + c] += ka * Vi[(size_t)m * dv + c];
                        }
                    }
                }
                if (s_out) memcpy(s_out + (size_t)bh * dk * dv, S, sizeof(double) * (size_t)dk * dv);
            }
        }
        free(S);
        free(A);
        free(Gl);
    }
    return err;
}

/*
 * Backward pass by definition (gradients of L = sum_n dO_n . O_n from a zero
 * initial state), differentiating the first-look sum of [RM] 保留机制初识,
 * O_n = sum_{m<=n} w_nm (q_n . k_m) v_m with w_nm = gamma^(n-m):
 *   dq_n = sum_{m<=n} w_nm (dO_n . v_m) k_m
 *   dk_m = sum_{n>=m} w_nm (dO_n . v_m) q_n
 *   dv_m = sum_{n>=m} w_nm (q_n . k_m) dO_n
 *   dgamma_h = sum_{n>m} (n-m) gamma^(n-m-1) (q_n . k_m)(dO_n . v_m)
 * dgamma may be NULL.
 */
int oracle_ret_backward(const double* q, const double* k, const double* v, const double* gamma,
                        const double* dout, double* dq, double* dk_out, double* dv_out, double* dgamma,
                        int B, int H, int N, int dk, int dv) {
    if (bad_dims(B, H, N, dk, dv) || !q || !k || !v || !gamma || !dout || !dq || !dk_out || !dv_out)
        return ORACLE_EBADARG;
    if (dgamma) memset(dgamma, 0, sizeof(double) * (size_t)H);
    double* dgam_bh = (double*)calloc((size_t)B * H, sizeof(double));
    if (!dgam_bh) return ORACLE_ENOMEM;
    #pragma omp parallel for schedule(static)
    for (int bh = 0; bh < B * H; ++bh) {
        const double gm = gamma[bh % H];
        const double* Q = q + (size_t)bh * N * dk;
        const double* K = k + (size_t)bh * N * dk;
        const double* V = v + (size_t)bh * N * dv;
        const double* DO = dout + (size_t)bh * N * dv;
        double* DQ = dq + (size_t)bh * N * dk;
        double* DK = dk_out + (size_t)bh * N * dk;
        double* DV = dv_out + (size_t)bh * N * dv;
        memset(DQ, 0, sizeof(double) * (size_t)N * dk);
        memset(DK, 0, sizeof(double) * (size_t)N * dk);
        memset(DV, 0, sizeof(double) * (size_t)N * dv);
        double dg = 0.0;
        for (int n = 0; n < N; ++n) {
            for (int m = 0; m <= n; ++m) {
                const double w = gpow(gm, n - m);
                double s = 0.0, a = 0.0;
                for (int d = 0; d < dk; ++d) s += Q[(size_t)n * dk + d] * K[(size_t)m * dk + d];
                for (int c = 0; c < dv; ++c) a += DO[(size_t)n * dv + c] * V[(size_t)m * dv + c];
                for (int d = 0; d < dk; ++d) {
                    DQ[(size_t)n * dk + d] += w * a * K[(size_t)m * dk + d];
                    DK[(size_t)m * dk + d] += w * a * Q[(size_t)n * dk + d];
                }
                for (int c = 0; c < dv; ++c) DV[(size_t)m * dv + c] += w * s * DO[(size_t)n * dv + c];
                if (n > m) dg += (double)(n - m) * gpow(gm, n - m - 1) * s * a;
            }
        }
        dgam_bh[bh] = dg;
    }
    if (dgamma)
        for (int bh = 0; bh < B * H; ++bh) dgamma[bh % H] += dgam_bh[bh];
    free(dgam_bh);
    return ORACLE_OK;
}

/*
 * Gated backward by definition ([GR] parallel_gate_retention: weights
 * w_nm = exp(sum_{t=m+1..n} g_t)), from a zero initial state. dq, dk, dv as in
 * oracle_ret_backward with these weights, and, since d w_nm / d g_t = w_nm for
 * m < t <= n,
 *   dg_t = sum over pairs n >= t > m of w_nm (q_n . k_m)(dO_n . v_m).
 * dg may be NULL.
 */
int oracle_gated_backward(const double* q, const double* k, const double* v, const double* g,
                          const double* dout, double* dq, double* dk_out, double* dv_out, double* dg,
                          int B, int H, int N, int dk, int dv) {
    if (bad_dims(B, H, N, dk, dv) || !q || !k || !v || !g || !dout || !dq || !dk_out || !dv_out)
        return ORACLE_EBADARG;
    #pragma omp parallel for schedule(static)
    for (int bh = 0; bh < B * H; ++bh) {
        const double* Q = q + (size_t)bh * N * dk;
        const double* K = k + (size_t)bh * N * dk;
        const double* V = v + (size_t)bh * N * dv;
        const double* Gt = g + (size_t)bh * N;
        const double* DO = dout + (size_t)bh * N * dv;
        double* DQ = dq + (size_t)bh * N * dk;
        double* DK = dk_out + (size_t)bh * N * dk;
        double* DV = dv_out + (size_t)bh * N * dv;
        double* DG = dg ? dg + (size_t)bh * N : NULL;
        memset(DQ, 0, sizeof(double) * (size_t)N * dk);
        memset(DK, 0, sizeof(double) * (size_t)N * dk);
        memset(DV, 0, sizeof(double) * (size_t)N * dv);
        if (DG) memset(DG, 0, sizeof(double) * (size_t)N);
        for (int n = 0; n < N; ++n) {
            for (int m = 0; m <= n; ++m) {
                double run = 0.0;
                for (int t = m + 1; t <= n; ++t) run += Gt[t];
                const double w = exp(run);
                double s = 0.0, a = 0.0;
                for (int d = 0; d < dk; ++d) s += Q[(size_t)n * dk + d] * K[(size_t)m * dk + d];
                for (int c = 0; c < dv; ++c) a += DO[(size_t)n * dv + c] * V[(size_t)m * dv + c];
                for (int d = 0; d < dk; ++d) {
                    DQ[(size_t)n * dk + d] += w * a * K[(size_t)m * dk + d];
                    DK[(size_t)m * dk + d] += w * a * Q[(size_t)n * dk + d];
                }
                for (int c = 0; c < dv; ++c) DV[(size_t)m * dv + c] += w * s * DO[(size_t)n * dv + c];
                if (DG)
                    for (int t = m + 1; t <= n; ++t) DG[t] += w * s * a;
            }
        }
    }
    return ORACLE_OK;
}

/*
 * Multi-scale retention output epilogue. [RN] 3.2 adds a gate and a normalisation
 * to retention; [GR]'s GateRetention module normalises each head with subln, an
 * RMSNorm over the head dimension without affine weights, and gates with the
 * swish of the g_proj projection:
 *   y[b, n, h, :] = swish(gate[b, n, h, :]) * o[b, h, n, :] / sqrt(mean_c o[b, h, n, c]^2 + eps),
 *   swish(x) = x / (1 + exp(-x)).
 * o [B, H, N, dv] is the retention output; gate and y are token-major
 * [B, N, H, dv], the layout of the module's projections.
 */
int oracle_msr_norm_gate(const double* o, const double* gate, double* y, int B, int H, int N, int dv, double eps) {
    if (bad_dims(B, H, N, 1, dv) || !o || !gate || !y || eps < 0.0) return ORACLE_EBADARG;
    #pragma omp parallel for schedule(static)
    for (int bh = 0; bh < B * H; ++bh) {
        const int b = bh / H, h = bh % H;
        for (int n = 0; n < N; ++n) {
            const double* orow = o + ((size_t)bh * N + n) * dv;
            const size_t yoff = (((size_t)b * N + n) * H + h) * dv;
            double ms = 0.0;
            for (int c = 0; c < dv; ++c) ms += orow[c] * orow[c];
            ms /= dv;
            const double inv_rms = 1.0 / sqrt(ms + eps);
            for (int c = 0; c < dv; ++c) {
                const double x = gate[yoff + c];
                const double swish = x / (1.0 + exp(-x));
                y[yoff + c] = swish * orow[c] * inv_rms;
            }
        }
    }
    return ORACLE_OK;
}
