/*
 * Sparse Delta Memory (SDM) — CPU ORACLE.  TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, fp64 C written to be checked against the method's definition by
 * eye.  Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may
 * load this library.  It shares no code, header, table or helper with the CUDA
 * path, and nothing in the product path may call it.
 *
 * Sources (the web pages describing "Sparse Delta Memory: Scaling the State of
 * Linear RNNs through Sparsity", arXiv 2607.07386):
 *   - paperlayer.ai summary, §2 Background: "Gated DeltaNet" (retrieve, subtract,
 *     then write; decay gate alpha in (0,1), input gate beta in [0,1]) and
 *     "Product Key Memory" (top-k over N slots without forming all N scores).
 *   - same page, §3 Method: "Sparse memory updates" (gated delta updates only on
 *     the W selected slots of an N-slot table), "Sparse addressing" (top-W write
 *     slots from keys, top-R read slots from queries), "Sparse retrieval"
 *     (weighted sum of the read slots), "Connection to GDN" (all slots selected
 *     => exactly Gated DeltaNet), "Learned initial state" (memory starts at M0).
 *   - same page, §4 Experimental Setup, "SDM Configuration": read and write
 *     activations are softmax-normalised.
 *
 * The pages print no equation; the readings used here (stated once, also listed
 * in the design notes) are:
 *   score(s = i*n + j) = <x[0:h], C1[i]> + <x[h:2h], C2[j]>          (h = d_k/2)
 *   order: larger score first; equal scores -> lower slot (lower sub-index per half)
 *   weights = softmax over the selected scores, temperature 1, no scaling
 *   per token t, in this order:
 *     (i)   M <- alpha_t * M                      (every slot decays)
 *     (ii)  p  = sum_i w_i M[s_i]                 (prediction, after decay)
 *     (iii) e  = v_t - p
 *     (iv)  M[s_i] <- M[s_i] + beta_t * w_i * e   (write slots are distinct)
 *     (v)   o_t = sum_j u_j M[r_j]                (read after the write)
 *   M starts at M0 (per head, shared by the batch).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_NOMEM 2

/* ------------------------------------------------------------------------- */
/* Ordering of (score, slot) pairs: higher score first, ties to lower slot.   */
/* ------------------------------------------------------------------------- */

typedef struct {
    double score;
    int32_t id;
} scored_t;

static int cmp_scored(const void* pa, const void* pb) {
    const scored_t* a = (const scored_t*)pa;
    const scored_t* b = (const scored_t*)pb;
    if (a->score > b->score) return -1;
    if (a->score < b->score) return 1;
    if (a->id < b->id) return -1;
    if (a->id > b->id) return 1;
    return 0;
}

static double dot(const double* a, const double* b, int n) {
    double s = 0.0;
    for (int d = 0; d < n; ++d) s += a[d] * b[d];
    return s;
}

/*
 * Half scores of one vector x (length 2*hd) against one role's sub-key tables
 * sk = [2][n][hd]: s1[i] = <x[0:hd], C1[i]>, s2[j] = <x[hd:2hd], C2[j]>.
 * Product Key Memory, paperlayer.ai §2 Background.
 */
void sdm_oracle_half_scores(const double* x, const double* sk, int n, int hd,
                            double* s1, double* s2) {
    const double* c1 = sk;
    const double* c2 = sk + (size_t)n * hd;
    for (int i = 0; i < n; ++i) s1[i] = dot(x, c1 + (size_t)i * hd, hd);
    for (int j = 0; j < n; ++j) s2[j] = dot(x + hd, c2 + (size_t)j * hd, hd);
}

/* softmax of `m` scores (temperature 1), §4 "SDM Configuration". */
static void softmax(const double* sc, int m, double* w) {
    double mx = sc[0];
    for (int i = 1; i < m; ++i) if (sc[i] > mx) mx = sc[i];
    double z = 0.0;
    for (int i = 0; i < m; ++i) { w[i] = exp(sc[i] - mx); z += w[i]; }
    for (int i = 0; i < m; ++i) w[i] /= z;
}

/*
 * Top-`top` slots of one vector.
 *   mode 0 (brute force): rank all N = n*n slot scores s1[i] + s2[j].
 *   mode 1 (product key): keep the k_half best sub-keys per half, rank the
 *     k_half^2 combined candidates.  Equals mode 0 whenever k_half >= top.
 * Outputs are best-first: idx[top], score[top], w[top] (softmax of score).
 * Returns 0, or ORACLE_ERR_* on bad arguments / allocation failure.
 * §2 Background "Product Key Memory"; §3 Method "Sparse addressing".
 */
int sdm_oracle_topk_vec(const double* x, const double* sk, int n, int hd, int k_half,
                        int top, int mode, int32_t* idx, double* score, double* w) {
    if (n <= 0 || hd <= 0 || top <= 0) return ORACLE_ERR_ARG;
    double* s1 = (double*)malloc(sizeof(double) * (size_t)n);
    double* s2 = (double*)malloc(sizeof(double) * (size_t)n);
    if (!s1 || !s2) { free(s1); free(s2); return ORACLE_ERR_NOMEM; }
    sdm_oracle_half_scores(x, sk, n, hd, s1, s2);

    int rc = ORACLE_OK;
    scored_t* cand = NULL;
    int m = 0;
    if (mode == 0) {
        if (top > n * n) { rc = ORACLE_ERR_ARG; goto done; }
        m = n * n;
        cand = (scored_t*)malloc(sizeof(scored_t) * (size_t)m);
        if (!cand) { rc = ORACLE_ERR_NOMEM; goto done; }
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < n; ++j) {
                cand[i * n + j].score = s1[i] + s2[j];
                cand[i * n + j].id = i * n + j;
            }
    } else {
        if (k_half <= 0 || k_half > n || top > k_half * k_half) { rc = ORACLE_ERR_ARG; goto done; }
        scored_t* h1 = (scored_t*)malloc(sizeof(scored_t) * (size_t)n);
        scored_t* h2 = (scored_t*)malloc(sizeof(scored_t) * (size_t)n);
        if (!h1 || !h2) { free(h1); free(h2); rc = ORACLE_ERR_NOMEM; goto done; }
        for (int i = 0; i < n; ++i) { h1[i].score = s1[i]; h1[i].id = i; }
        for (int j = 0; j < n; ++j) { h2[j].score = s2[j]; h2[j].id = j; }
        qsort(h1, (size_t)n, sizeof(scored_t), cmp_scored);
        qsort(h2, (size_t)n, sizeof(scored_t), cmp_scored);
        m = k_half * k_half;
        cand = (scored_t*)malloc(sizeof(scored_t) * (size_t)m);
        if (!cand) { free(h1); free(h2); rc = ORACLE_ERR_NOMEM; goto done; }
        for (int a = 0; a < k_half; ++a)
            for (int b = 0; b < k_half; ++b) {
                int i = h1[a].id, j = h2[b].id;
                cand[a * k_half + b].score = s1[i] + s2[j];
                cand[a * k_half + b].id = i * n + j;
            }
        free(h1);
        free(h2);
    }
    qsort(cand, (size_t)m, sizeof(scored_t), cmp_scored);
    for (int r = 0; r < top; ++r) { idx[r] = cand[r].id; score[r] = cand[r].score; }
    softmax(score, top, w);
done:
    free(cand);
    free(s1);
    free(s2);
    return rc;
}

/*
 * Batched scoring of x [B][H][T][2*hd] against per-head tables sk [H][2][n][hd]
 * (one role).  Outputs [B][H][T][top].  OpenMP over (b,h,t) when available.
 */
int sdm_oracle_score(const double* x, const double* sk, int B, int H, int T, int hd,
                     int n, int k_half, int top, int mode, int32_t* idx, double* score,
                     double* w, int nthreads) {
    if (B < 0 || H < 0 || T < 0) return ORACLE_ERR_ARG;
    const long long rows = (long long)B * H * T;
    int rc = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 64)
#endif
    for (long long r = 0; r < rows; ++r) {
        const int h = (int)((r / T) % H);
        const int e = sdm_oracle_topk_vec(x + (size_t)r * 2 * hd, sk + (size_t)h * 2 * n * hd, n, hd,
                                          k_half, top, mode, idx + (size_t)r * top,
                                          score + (size_t)r * top, w + (size_t)r * top);
        if (e != ORACLE_OK) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            rc = e;
        }
    }
    (void)nthreads;
    return rc;
}

/*
 * Gradient through the scoring of `rows` vectors x [rows][2*hd] of one head against that
 * head's sub-key tables sk [2][n][hd], the selected slots idx [rows][top] held fixed:
 * with score_q = <x[0:hd], C1[i_q]> + <x[hd:2hd], C2[j_q]> (slot = i_q*n + j_q) and
 * w = softmax(score) over the selected slots (§2 Background "Product Key Memory", §3
 * Method "Sparse addressing", §4 "SDM Configuration"), for dw [rows][top]:
 *   dscore_q = w_q (dw_q - sum_r w_r dw_r)
 *   dx[0:hd] = sum_q dscore_q C1[i_q],   dx[hd:] = sum_q dscore_q C2[j_q]
 *   dsk[0][i] += sum_{q: i_q = i} dscore_q x[0:hd],   dsk[1][j] likewise with x[hd:]
 * The weights are recomputed from x and the tables.  dx [rows][2*hd] is written; dsk
 * [2][n][hd] is added to.
 */
int sdm_oracle_score_backward(const double* x, const double* sk, int rows, int n, int hd,
                              int top, const int32_t* idx, const double* dw, double* dx,
                              double* dsk) {
    if (rows < 0 || n <= 0 || hd <= 0 || top <= 0) return ORACLE_ERR_ARG;
    double* sc = (double*)malloc(sizeof(double) * (size_t)top);
    double* w = (double*)malloc(sizeof(double) * (size_t)top);
    double* ds = (double*)malloc(sizeof(double) * (size_t)top);
    if (!sc || !w || !ds) { free(sc); free(w); free(ds); return ORACLE_ERR_NOMEM; }
    const double* c1 = sk;
    const double* c2 = sk + (size_t)n * hd;
    for (int r = 0; r < rows; ++r) {
        const double* xr = x + (size_t)r * 2 * hd;
        const int32_t* id = idx + (size_t)r * top;
        for (int q = 0; q < top; ++q) {
            if (id[q] < 0 || id[q] >= n * n) { free(sc); free(w); free(ds); return ORACLE_ERR_ARG; }
            const int i = id[q] / n, j = id[q] % n;
            sc[q] = dot(xr, c1 + (size_t)i * hd, hd) + dot(xr + hd, c2 + (size_t)j * hd, hd);
        }
        softmax(sc, top, w);
        double s = 0.0;
        for (int q = 0; q < top; ++q) s += w[q] * dw[(size_t)r * top + q];
        for (int q = 0; q < top; ++q) ds[q] = w[q] * (dw[(size_t)r * top + q] - s);
        double* dxr = dx + (size_t)r * 2 * hd;
        for (int d = 0; d < 2 * hd; ++d) dxr[d] = 0.0;
        for (int q = 0; q < top; ++q) {
            const int i = id[q] / n, j = id[q] % n;
            for (int d = 0; d < hd; ++d) {
                dxr[d] += ds[q] * c1[(size_t)i * hd + d];
                dxr[hd + d] += ds[q] * c2[(size_t)j * hd + d];
                dsk[(size_t)i * hd + d] += ds[q] * xr[d];
                dsk[(size_t)n * hd + (size_t)j * hd + d] += ds[q] * xr[hd + d];
            }
        }
    }
    free(sc); free(w); free(ds);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------- */
/* Recurrence for one (b,h).                                                  */
/* ------------------------------------------------------------------------- */

static int check_slots(const int32_t* s, int m, int N) {
    for (int i = 0; i < m; ++i) if (s[i] < 0 || s[i] >= N) return 0;
    return 1;
}

/*
 * Dense-decay recurrence: steps (i)-(v) above, taken literally, with decay
 * applied to every one of the N slots at every token.  M [N][dv] is the state
 * in/out (caller initialises it to M0 for a fresh sequence); out [T][dv].
 * §2 Background "Gated DeltaNet"; §3 Method "Sparse memory updates",
 * "Sparse retrieval", "Learned initial state".
 */
int sdm_oracle_recur_dense(int T, int N, int dv, int W, int R, const double* v,
                           const double* alpha, const double* beta, const int32_t* widx,
                           const double* ww, const int32_t* ridx, const double* rw,
                           double* M, double* out) {
    if (T < 0 || N <= 0 || dv <= 0 || W <= 0 || R <= 0) return ORACLE_ERR_ARG;
    double* p = (double*)malloc(sizeof(double) * (size_t)dv);
    double* e = (double*)malloc(sizeof(double) * (size_t)dv);
    if (!p || !e) { free(p); free(e); return ORACLE_ERR_NOMEM; }
    int rc = ORACLE_OK;
    for (int t = 0; t < T; ++t) {
        const int32_t* ws = widx + (size_t)t * W;
        const int32_t* rs = ridx + (size_t)t * R;
        if (!check_slots(ws, W, N) || !check_slots(rs, R, N)) { rc = ORACLE_ERR_ARG; break; }
        /* (i) decay every slot */
        for (size_t q = 0; q < (size_t)N * dv; ++q) M[q] *= alpha[t];
        /* (ii) prediction */
        for (int c = 0; c < dv; ++c) p[c] = 0.0;
        for (int i = 0; i < W; ++i)
            for (int c = 0; c < dv; ++c) p[c] += ww[(size_t)t * W + i] * M[(size_t)ws[i] * dv + c];
        /* (iii) error */
        for (int c = 0; c < dv; ++c) e[c] = v[(size_t)t * dv + c] - p[c];
        /* (iv) gated delta write on the W slots */
        for (int i = 0; i < W; ++i)
            for (int c = 0; c < dv; ++c)
                M[(size_t)ws[i] * dv + c] += beta[t] * ww[(size_t)t * W + i] * e[c];
        /* (v) read after the write */
        for (int c = 0; c < dv; ++c) {
            double o = 0.0;
            for (int j = 0; j < R; ++j) o += rw[(size_t)t * R + j] * M[(size_t)rs[j] * dv + c];
            out[(size_t)t * dv + c] = o;
        }
    }
    free(p);
    free(e);
    return rc;
}

/*
 * Touched-slots decay: the other reading of §3 Method "Sparse memory updates"
 * (the gated delta update, its decay gate included, acts only on the W slots the
 * keys select).  Per token t:
 *   (i')  M[s_i] <- alpha_t * M[s_i]             (the W write slots only)
 *   (ii)  p  = sum_i w_i M[s_i]
 *   (iii) e  = v_t - p
 *   (iv)  M[s_i] <- M[s_i] + beta_t * w_i * e
 *   (v)   o_t = sum_j u_j M[r_j]                (read after the write)
 * Every other slot keeps its value, so a slot never written still holds M0.  With
 * every slot written at every token (W = N) this is the dense form above (Gated
 * DeltaNet, "Connection to GDN"); with alpha = 1 the two readings coincide.
 * M [N][dv] in/out; out [T][dv].
 */
int sdm_oracle_recur_touched(int T, int N, int dv, int W, int R, const double* v,
                             const double* alpha, const double* beta, const int32_t* widx,
                             const double* ww, const int32_t* ridx, const double* rw,
                             double* M, double* out) {
    if (T < 0 || N <= 0 || dv <= 0 || W <= 0 || R <= 0) return ORACLE_ERR_ARG;
    double* p = (double*)malloc(sizeof(double) * (size_t)dv);
    double* e = (double*)malloc(sizeof(double) * (size_t)dv);
    if (!p || !e) { free(p); free(e); return ORACLE_ERR_NOMEM; }
    int rc = ORACLE_OK;
    for (int t = 0; t < T; ++t) {
        const int32_t* ws = widx + (size_t)t * W;
        const int32_t* rs = ridx + (size_t)t * R;
        if (!check_slots(ws, W, N) || !check_slots(rs, R, N)) { rc = ORACLE_ERR_ARG; break; }
        /* (i') decay the write slots */
        for (int i = 0; i < W; ++i)
            for (int c = 0; c < dv; ++c) M[(size_t)ws[i] * dv + c] *= alpha[t];
        /* (ii) prediction */
        for (int c = 0; c < dv; ++c) p[c] = 0.0;
        for (int i = 0; i < W; ++i)
            for (int c = 0; c < dv; ++c) p[c] += ww[(size_t)t * W + i] * M[(size_t)ws[i] * dv + c];
        /* (iii) error */
        for (int c = 0; c < dv; ++c) e[c] = v[(size_t)t * dv + c] - p[c];
        /* (iv) gated delta write on the W slots */
        for (int i = 0; i < W; ++i)
            for (int c = 0; c < dv; ++c)
                M[(size_t)ws[i] * dv + c] += beta[t] * ww[(size_t)t * W + i] * e[c];
        /* (v) read after the write */
        for (int c = 0; c < dv; ++c) {
            double o = 0.0;
            for (int j = 0; j < R; ++j) o += rw[(size_t)t * R + j] * M[(size_t)rs[j] * dv + c];
            out[(size_t)t * dv + c] = o;
        }
    }
    free(p);
    free(e);
    return rc;
}

/*
 * Gradients of the recurrence of one (b,h) with respect to its inputs, for a loss whose
 * gradient with respect to the outputs is dout [T][dv]; the slot selections are fixed
 * (they are not differentiated).  touched = 0: steps (i)-(v) of the dense form (every slot
 * decays); touched = 1: step (i') instead (only the write slots decay).  Plain
 * reverse-mode differentiation, token by token, from every state M_0..M_T kept in memory
 * (small cases only); the pages' appendix A.3 ("Memory-Efficient Backward") recovers the
 * states by undoing the in-place updates instead.  Per token t, backwards:
 *   (v)   o = sum_j u_j M_t[r_j]:        du_j = <G, M_t[r_j]>,  dM[r_j] += u_j G
 *   (iv)  M_t[s_i] = Mt[s_i] + beta w_i e  (Mt = the decayed state):
 *         de = beta sum_i w_i dM[s_i],  dbeta = sum_i w_i <dM[s_i], e>,
 *         dw_i = beta <dM[s_i], e>
 *   (iii) e = v - p:                       dv = de,  dp = -de
 *   (ii)  p = sum_i w_i Mt[s_i]:           dw_i += <dp, Mt[s_i]>,  dMt[s_i] = dM[s_i] + w_i dp
 *   (i)   Mt = alpha M_{t-1}:              dalpha = <dMt, M_{t-1}> over every slot (the
 *         write slots only when touched),   dM_{t-1} = alpha dMt (those slots only)
 * G = dout[t].  dM_end [N][dv] (may be NULL: zero) is the loss's gradient with respect to
 * the memory after the last token, for a loss that also reads the final state (a sequence
 * processed in several calls: the next call's gradient of its start state); the sweep
 * starts from it.  Outputs: dv [T][dv], dalpha [T], dbeta [T], dww [T][W], drw [T][R] and
 * dM0 [N][dv], the gradient with respect to the state at the start of the call.
 * §2 Background "Gated DeltaNet"; §3 Method "Sparse memory updates", "Sparse retrieval".
 */
int sdm_oracle_recur_backward(int T, int N, int dv, int W, int R, int touched, const double* v,
                              const double* alpha, const double* beta, const int32_t* widx,
                              const double* ww, const int32_t* ridx, const double* rw,
                              const double* M0, const double* dout, const double* dM_end,
                              double* dvv, double* dalpha, double* dbeta, double* dww,
                              double* drw, double* dM0) {
    if (T < 0 || N <= 0 || dv <= 0 || W <= 0 || R <= 0) return ORACLE_ERR_ARG;
    const size_t ND = (size_t)N * dv;
    double* S = (double*)malloc(sizeof(double) * ND * (size_t)(T + 1));  /* S[t] = M_t */
    double* dM = (double*)calloc(ND, sizeof(double));
    double* Mt = (double*)malloc(sizeof(double) * (size_t)W * dv);       /* decayed write rows */
    double* p = (double*)malloc(sizeof(double) * (size_t)dv);
    double* e = (double*)malloc(sizeof(double) * (size_t)dv);
    double* de = (double*)malloc(sizeof(double) * (size_t)dv);
    if (!S || !dM || !Mt || !p || !e || !de) {
        free(S); free(dM); free(Mt); free(p); free(e); free(de);
        return ORACLE_ERR_NOMEM;
    }
    int rc = ORACLE_OK;
    memcpy(S, M0, sizeof(double) * ND);
    if (dM_end) memcpy(dM, dM_end, sizeof(double) * ND);
    for (int t = 0; t < T && rc == ORACLE_OK; ++t) {
        const int32_t* ws = widx + (size_t)t * W;
        const int32_t* rs = ridx + (size_t)t * R;
        if (!check_slots(ws, W, N) || !check_slots(rs, R, N)) { rc = ORACLE_ERR_ARG; break; }
        double* M = S + ND * (size_t)(t + 1);
        memcpy(M, S + ND * (size_t)t, sizeof(double) * ND);
        if (touched) {
            for (int i = 0; i < W; ++i)
                for (int c = 0; c < dv; ++c) M[(size_t)ws[i] * dv + c] *= alpha[t];
        } else {
            for (size_t q = 0; q < ND; ++q) M[q] *= alpha[t];
        }
        for (int c = 0; c < dv; ++c) {
            double pc = 0.0;
            for (int i = 0; i < W; ++i) pc += ww[(size_t)t * W + i] * M[(size_t)ws[i] * dv + c];
            e[c] = v[(size_t)t * dv + c] - pc;
        }
        for (int i = 0; i < W; ++i)
            for (int c = 0; c < dv; ++c)
                M[(size_t)ws[i] * dv + c] += beta[t] * ww[(size_t)t * W + i] * e[c];
    }
    for (int t = T - 1; t >= 0 && rc == ORACLE_OK; --t) {
        const int32_t* ws = widx + (size_t)t * W;
        const int32_t* rs = ridx + (size_t)t * R;
        const double* Mnow = S + ND * (size_t)(t + 1);
        const double* Mprev = S + ND * (size_t)t;
        const double* G = dout + (size_t)t * dv;
        const double* wt = ww + (size_t)t * W;
        /* (v) the read */
        for (int j = 0; j < R; ++j) {
            const double u = rw[(size_t)t * R + j];
            drw[(size_t)t * R + j] = dot(G, Mnow + (size_t)rs[j] * dv, dv);
            for (int c = 0; c < dv; ++c) dM[(size_t)rs[j] * dv + c] += u * G[c];
        }
        /* recompute the decayed write rows, p and e of this token */
        for (int i = 0; i < W; ++i)
            for (int c = 0; c < dv; ++c)
                Mt[(size_t)i * dv + c] = alpha[t] * Mprev[(size_t)ws[i] * dv + c];
        for (int c = 0; c < dv; ++c) {
            double pc = 0.0;
            for (int i = 0; i < W; ++i) pc += wt[i] * Mt[(size_t)i * dv + c];
            p[c] = pc;
            e[c] = v[(size_t)t * dv + c] - pc;
        }
        /* (iv) the write */
        double db = 0.0;
        for (int c = 0; c < dv; ++c) {
            double s = 0.0;
            for (int i = 0; i < W; ++i) s += wt[i] * dM[(size_t)ws[i] * dv + c];
            de[c] = beta[t] * s;
        }
        for (int i = 0; i < W; ++i) {
            const double ge = dot(dM + (size_t)ws[i] * dv, e, dv);
            db += wt[i] * ge;
            dww[(size_t)t * W + i] = beta[t] * ge;
        }
        dbeta[t] = db;
        /* (iii), (ii) */
        for (int c = 0; c < dv; ++c) dvv[(size_t)t * dv + c] = de[c];
        for (int i = 0; i < W; ++i) {
            dww[(size_t)t * W + i] -= dot(de, Mt + (size_t)i * dv, dv);
            for (int c = 0; c < dv; ++c) dM[(size_t)ws[i] * dv + c] -= wt[i] * de[c];
        }
        /* (i) the decay */
        double da = 0.0;
        if (touched) {
            for (int i = 0; i < W; ++i) {
                da += dot(dM + (size_t)ws[i] * dv, Mprev + (size_t)ws[i] * dv, dv);
                for (int c = 0; c < dv; ++c) dM[(size_t)ws[i] * dv + c] *= alpha[t];
            }
        } else {
            for (size_t q = 0; q < ND; ++q) da += dM[q] * Mprev[q];
            for (size_t q = 0; q < ND; ++q) dM[q] *= alpha[t];
        }
        dalpha[t] = da;
    }
    if (rc == ORACLE_OK) memcpy(dM0, dM, sizeof(double) * ND);
    free(S); free(dM); free(Mt); free(p); free(e); free(de);
    return rc;
}

/*
 * Lazy-decay recurrence, the same steps with decay applied only when a slot is
 * touched.  State: Mraw [N][dv], stamp [N] (log-decay prefix at the slot's last
 * write), *Lambda (running log-decay prefix).  The true slot value at the current
 * prefix is Mraw[s] * exp(Lambda - stamp[s]).  A fresh state is Mraw = M0,
 * stamp = 0, Lambda = 0.  Equal to the dense form up to rounding because
 * prod_{u in (a,b]} alpha_u = exp(Lambda_b - Lambda_a).
 */
int sdm_oracle_recur_lazy(int T, int N, int dv, int W, int R, const double* v,
                          const double* alpha, const double* beta, const int32_t* widx,
                          const double* ww, const int32_t* ridx, const double* rw,
                          double* Mraw, double* stamp, double* Lambda, double* out) {
    if (T < 0 || N <= 0 || dv <= 0 || W <= 0 || R <= 0) return ORACLE_ERR_ARG;
    double* seen = (double*)malloc(sizeof(double) * (size_t)W * dv); /* decayed write rows */
    double* e = (double*)malloc(sizeof(double) * (size_t)dv);
    if (!seen || !e) { free(seen); free(e); return ORACLE_ERR_NOMEM; }
    int rc = ORACLE_OK;
    double L = *Lambda;
    for (int t = 0; t < T; ++t) {
        const int32_t* ws = widx + (size_t)t * W;
        const int32_t* rs = ridx + (size_t)t * R;
        if (!check_slots(ws, W, N) || !check_slots(rs, R, N)) { rc = ORACLE_ERR_ARG; break; }
        /* (i) advance the prefix: every slot is now implicitly scaled by alpha_t */
        L += log(alpha[t]);
        /* (ii) prediction from the decayed write rows */
        for (int i = 0; i < W; ++i) {
            const double f = exp(L - stamp[ws[i]]);
            for (int c = 0; c < dv; ++c) seen[(size_t)i * dv + c] = Mraw[(size_t)ws[i] * dv + c] * f;
        }
        for (int c = 0; c < dv; ++c) {
            double p = 0.0;
            for (int i = 0; i < W; ++i) p += ww[(size_t)t * W + i] * seen[(size_t)i * dv + c];
            /* (iii) error */
            e[c] = v[(size_t)t * dv + c] - p;
        }
        /* (iv) write back the updated rows, stamped with the current prefix */
        for (int i = 0; i < W; ++i) {
            for (int c = 0; c < dv; ++c)
                Mraw[(size_t)ws[i] * dv + c] =
                    seen[(size_t)i * dv + c] + beta[t] * ww[(size_t)t * W + i] * e[c];
            stamp[ws[i]] = L;
        }
        /* (v) read after the write */
        for (int c = 0; c < dv; ++c) {
            double o = 0.0;
            for (int j = 0; j < R; ++j)
                o += rw[(size_t)t * R + j] * Mraw[(size_t)rs[j] * dv + c] * exp(L - stamp[rs[j]]);
            out[(size_t)t * dv + c] = o;
        }
    }
    *Lambda = L;
    free(seen);
    free(e);
    return rc;
}

/* Dense memory from a lazy state: M[s] = Mraw[s] * exp(Lambda - stamp[s]). */
void sdm_oracle_materialize(int N, int dv, const double* Mraw, const double* stamp,
                            double Lambda, double* M) {
    for (int s = 0; s < N; ++s) {
        const double f = exp(Lambda - stamp[s]);
        for (int c = 0; c < dv; ++c) M[(size_t)s * dv + c] = Mraw[(size_t)s * dv + c] * f;
    }
}

/*
 * Whole prefill for a list of (b,h) pairs: score both roles (product-key mode)
 * and run the lazy recurrence from a fresh state (M0 of head h).  Used to time
 * the CPU baseline.  Inputs are full [B][H][T][.] arrays; only the listed pairs
 * are processed; out is [npairs][T][dv].  OpenMP over pairs.
 */
int sdm_oracle_prefill_pairs(int B, int H, int T, int hd, int n, int dv, int k_half,
                             int W, int R, const double* q, const double* k, const double* v,
                             const double* alpha, const double* beta, const double* skw,
                             const double* skr, const double* M0, int npairs,
                             const int32_t* pairs, double* out, int nthreads) {
    const int N = n * n;
    int rc = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int pi = 0; pi < npairs; ++pi) {
        const int b = pairs[2 * pi], h = pairs[2 * pi + 1];
        if (b < 0 || b >= B || h < 0 || h >= H) { rc = ORACLE_ERR_ARG; continue; }
        const size_t bh = (size_t)b * H + h;
        int32_t* widx = (int32_t*)malloc(sizeof(int32_t) * (size_t)T * W);
        int32_t* ridx = (int32_t*)malloc(sizeof(int32_t) * (size_t)T * R);
        double* ww = (double*)malloc(sizeof(double) * (size_t)T * W);
        double* rw = (double*)malloc(sizeof(double) * (size_t)T * R);
        double* wsc = (double*)malloc(sizeof(double) * (size_t)W);
        double* rsc = (double*)malloc(sizeof(double) * (size_t)R);
        double* Mraw = (double*)malloc(sizeof(double) * (size_t)N * dv);
        double* stamp = (double*)calloc((size_t)N, sizeof(double));
        if (!widx || !ridx || !ww || !rw || !wsc || !rsc || !Mraw || !stamp) {
            rc = ORACLE_ERR_NOMEM;
        } else {
            for (int t = 0; t < T; ++t) {
                const size_t row = bh * T + t;
                int e1 = sdm_oracle_topk_vec(k + row * 2 * hd, skw + (size_t)h * 2 * n * hd, n, hd,
                                             k_half, W, 1, widx + (size_t)t * W, wsc,
                                             ww + (size_t)t * W);
                int e2 = sdm_oracle_topk_vec(q + row * 2 * hd, skr + (size_t)h * 2 * n * hd, n, hd,
                                             k_half, R, 1, ridx + (size_t)t * R, rsc,
                                             rw + (size_t)t * R);
                if (e1 || e2) rc = e1 ? e1 : e2;
            }
            memcpy(Mraw, M0 + (size_t)h * N * dv, sizeof(double) * (size_t)N * dv);
            double L = 0.0;
            int e3 = sdm_oracle_recur_lazy(T, N, dv, W, R, v + bh * T * dv, alpha + bh * T,
                                           beta + bh * T, widx, ww, ridx, rw, Mraw, stamp, &L,
                                           out + (size_t)pi * T * dv);
            if (e3) rc = e3;
        }
        free(widx); free(ridx); free(ww); free(rw); free(wsc); free(rsc); free(Mraw); free(stamp);
    }
    (void)nthreads;
    return rc;
}

/*
 * Memory-utilisation diagnostics over post-softmax selected-slot weights (pages:
 * Appendix D.1 "Memory Utilization and Access": cumulative top-k mass and an
 * entropy-based effective-key measure, summarised by the mean and by token-level
 * quantiles over batch, head and time).  For each of `rows` weight vectors of length
 * K, given best first (the order sdm_oracle_topk_vec returns):
 *   cum[r][k] = w[r][0] + ... + w[r][k]                 (mass of the k+1 largest)
 *   eff[r]    = exp(H_r) / K,  H_r = -sum_i w[r][i] ln w[r][i]   (0 ln 0 = 0)
 * eff = 1 for uniform weights, 1/K for a one-hot vector.  Summary: mean_cum[k] =
 * mean over rows of cum[r][k]; mean_eff = mean of eff; quant[q] = the order
 * statistic of eff at index floor(probs[q] * (rows - 1)) of the ascending sort.
 * cum and eff may be NULL.
 */
static int cmp_double_asc(const void* pa, const void* pb) {
    const double a = *(const double*)pa, b = *(const double*)pb;
    return a < b ? -1 : (a > b ? 1 : 0);
}

int sdm_oracle_weight_stats(int rows, int K, const double* w, double* cum, double* eff,
                            double* mean_cum, double* mean_eff, int nprobs,
                            const double* probs, double* quant) {
    if (rows < 1 || K < 1 || !w || !mean_cum || !mean_eff) return ORACLE_ERR_ARG;
    double* e = (double*)malloc(sizeof(double) * (size_t)rows);
    if (!e) return ORACLE_ERR_NOMEM;
    for (int k = 0; k < K; ++k) mean_cum[k] = 0.0;
    double sum_eff = 0.0;
    for (int r = 0; r < rows; ++r) {
        const double* wr = w + (size_t)r * K;
        double c = 0.0, H = 0.0;
        for (int k = 0; k < K; ++k) {
            c += wr[k];
            if (cum) cum[(size_t)r * K + k] = c;
            mean_cum[k] += c;
            if (wr[k] > 0.0) H -= wr[k] * log(wr[k]);
        }
        e[r] = exp(H) / K;
        if (eff) eff[r] = e[r];
        sum_eff += e[r];
    }
    for (int k = 0; k < K; ++k) mean_cum[k] /= rows;
    *mean_eff = sum_eff / rows;
    if (nprobs > 0) {
        if (!probs || !quant) { free(e); return ORACLE_ERR_ARG; }
        qsort(e, (size_t)rows, sizeof(double), cmp_double_asc);
        for (int q = 0; q < nprobs; ++q) {
            if (!(probs[q] >= 0.0 && probs[q] <= 1.0)) { free(e); return ORACLE_ERR_ARG; }
            quant[q] = e[(size_t)floor(probs[q] * (rows - 1))];
        }
    }
    free(e);
    return ORACLE_OK;
}

/*
 * Output side of an SDM layer (paperlayer.ai §3 Method "Sparse retrieval": the read result
 * is RMS-normalised, elementwise gated and mixed across heads by the output projection).
 * Readings: RMS-norm over each head's d_v values with one weight vector wn shared by the
 * heads, x / sqrt(mean x^2 + eps); the gate is swish(z) = z * sigmoid(z) of a given
 * pre-activation g; the mix is the output projection Wo (given transposed).
 *   o [B][H][T][dv], g [B][T][H*dv], wn [dv], Wo_t [dm][H*dv]  ->  y [B][T][dm]
 * Only the rows listed in `rows` (indices b*T + t, nrows of them) are computed; y is then
 * [nrows][dm].  OpenMP over rows.
 */
int sdm_oracle_layer_out(int B, int H, int T, int dv, int dm, const double* o, const double* g,
                         const double* wn, double eps, const double* Wo_t, int nrows,
                         const int64_t* rows, double* y) {
    const int K = H * dv;
    int rc = ORACLE_OK;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int ri = 0; ri < nrows; ++ri) {
        const int64_t bt = rows[ri];
        if (bt < 0 || bt >= (int64_t)B * T) { rc = ORACLE_ERR_ARG; continue; }
        const int b = (int)(bt / T), t = (int)(bt % T);
        double* a = (double*)malloc(sizeof(double) * (size_t)K);
        if (!a) { rc = ORACLE_ERR_NOMEM; continue; }
        for (int h = 0; h < H; ++h) {
            const double* x = o + (((size_t)b * H + h) * T + t) * dv;
            double ms = 0.0;
            for (int c = 0; c < dv; ++c) ms += x[c] * x[c];
            const double r = 1.0 / sqrt(ms / dv + eps);
            for (int c = 0; c < dv; ++c) {
                const double z = g[(size_t)bt * K + (size_t)h * dv + c];
                const double sw = z / (1.0 + exp(-z));
                a[h * dv + c] = x[c] * r * wn[c] * sw;
            }
        }
        for (int n = 0; n < dm; ++n) {
            double acc = 0.0;
            for (int k = 0; k < K; ++k) acc += a[k] * Wo_t[(size_t)n * K + k];
            y[(size_t)ri * dm + n] = acc;
        }
        free(a);
    }
    return rc;
}

/*
 * Input side of an SDM layer: the projections of the layer input x into the per-head query,
 * key, value, output-gate pre-activation and the two gates (paperlayer.ai §2 Background
 * "Gated DeltaNet": decay gate alpha_t in (0,1), input gate beta_t in [0,1]; §4 "SDM
 * Configuration": forget gate and time-step bias as in GDN/FLA; appendix "Gate dynamics":
 * the forget gate is exp(g), the input gate sigma(b)).  Readings: per head h, the columns
 * of P = x Win (Win given transposed, Win_t [Nin][dm]) are laid out as
 *   [q (dk) | k (dk) | v (dv) | g (dv) | a | b],  Nin = H (2 dk + 2 dv + 2),
 * alpha = exp(-exp(A_log[h]) * softplus(a + dt_bias[h])), beta = sigmoid(b);
 * no short convolution and no q/k normalisation.
 *   x [B][T][dm]  ->  q, k [B][H][T][dk], v [B][H][T][dv], g [B][T][H*dv],
 *                     alpha, beta [B][H][T]
 * Only the rows listed (b*T + t) are computed; outputs are then indexed by list position
 * in place of (b, t): q [nrows][H][dk], v [nrows][H][dv], g [nrows][H*dv], alpha/beta
 * [nrows][H].  OpenMP over rows.
 */
static double softplus_d(double z) { return z > 30.0 ? z : log1p(exp(z)); }

int sdm_oracle_layer_in(int B, int H, int T, int dk, int dv, int dm, const double* x,
                        const double* Win_t, const double* A_log, const double* dt_bias,
                        int nrows, const int64_t* rows, double* q, double* k, double* v,
                        double* g, double* alpha, double* beta) {
    const int hs = 2 * dk + 2 * dv + 2, Nin = H * hs;
    int rc = ORACLE_OK;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (int ri = 0; ri < nrows; ++ri) {
        const int64_t bt = rows[ri];
        if (bt < 0 || bt >= (int64_t)B * T) { rc = ORACLE_ERR_ARG; continue; }
        double* P = (double*)malloc(sizeof(double) * (size_t)Nin);
        if (!P) { rc = ORACLE_ERR_NOMEM; continue; }
        const double* xr = x + (size_t)bt * dm;
        for (int n = 0; n < Nin; ++n) P[n] = dot(xr, Win_t + (size_t)n * dm, dm);
        for (int h = 0; h < H; ++h) {
            const double* ph = P + (size_t)h * hs;
            for (int c = 0; c < dk; ++c) {
                q[((size_t)ri * H + h) * dk + c] = ph[c];
                k[((size_t)ri * H + h) * dk + c] = ph[dk + c];
            }
            for (int c = 0; c < dv; ++c) {
                v[((size_t)ri * H + h) * dv + c] = ph[2 * dk + c];
                g[(size_t)ri * H * dv + (size_t)h * dv + c] = ph[2 * dk + dv + c];
            }
            const double a = ph[2 * dk + 2 * dv], bb = ph[2 * dk + 2 * dv + 1];
            alpha[(size_t)ri * H + h] = exp(-exp(A_log[h]) * softplus_d(a + dt_bias[h]));
            beta[(size_t)ri * H + h] = 1.0 / (1.0 + exp(-bb));
        }
        free(P);
    }
    return rc;
}

int sdm_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
