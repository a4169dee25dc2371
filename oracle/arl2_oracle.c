/*
 * ARL2 hybrid attention layer: plain CPU oracle in fp64.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file; only the tests, the smoke check and the benchmark's CPU
 * baseline do.  It shares no code with the CUDA library.
 *
 * Method ("Attend Locally, Remember Linearly", gist.science technical
 * summary, section 2.1 Hybrid Attention Decomposition and section 2.2
 * Memory State Management).  For every stream b and head h of one frame N:
 *
 *   intra  : O_intra = softmax(Q K^T * scale) V, bidirectional over the
 *            frame's L tokens (2.1, item 1 "Intra-Frame Branch")
 *   maps   : Q' = Q W_q[h], K' = rownorm(K W_k[h]), V' = V W_v[h]; the
 *            per-head grouped 1x1 feature maps phi_q, phi_k, phi_v of 2.1
 *            ("Adaptation") are plain d x d linear maps; only k' rows are
 *            L2-normalised
 *   read   : O_inter = Q' S_{N-1} (2.1 "Output"); every token reads the
 *            same pre-update state (2.2 "Frame-Level Access")
 *   output : O = O_intra + O_inter
 *   update : clean pass only (2.2 "Clean-Pass Updates"), after the read:
 *            S_N = alpha S_{N-1} + K'^T diag(beta) (V' - K' S_{N-1})
 *            (2.1 "State Update", read with the transpose and diag(beta)
 *            that make it well formed for L tokens)
 *
 * Layouts (all dense, row-major, double):
 *   q, k, v, out : [B][L][H][d]    token-major, as a DiT's QKV output
 *   w_q, w_k, w_v: [H][d][d]       row = input feature, column = output
 *   alpha        : [B][H]          forget gate of the frame (headwise), or
 *                  [B][H][d]       one per key feature (elementwise gating)
 *   beta         : [B][H][L]       per-token rate
 *   S            : [B][H][d][d]    row = key feature, column = value feature
 *
 * Every entry returns 0 on success and -1 on a bad argument or a failed
 * allocation.  Streams and heads are independent, so the loops over (b, h)
 * run in parallel with OpenMP; the arithmetic inside each (b, h) is done in
 * the order written.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#define IDX4(a, b, c, e, B1, C1, E1) ((((size_t)(a) * (B1) + (b)) * (C1) + (c)) * (E1) + (e))

static int bad_dims(int B, int H, int d, int L) {
    return B < 1 || H < 1 || d < 1 || L < 1;
}

/* x'[t] = x[t] W  for the L rows of head h of stream b; x' is [L][d]. */
static void phi_map_head(int H, int d, int L, int b, int h, const double* x,
                         const double* w, int l2norm, double* xp) {
    const double* W = w + (size_t)h * d * d;
    for (int t = 0; t < L; ++t) {
        const double* xr = x + IDX4(b, t, h, 0, L, H, d);
        double* yr = xp + (size_t)t * d;
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int a = 0; a < d; ++a) acc += xr[a] * W[(size_t)a * d + c];
            yr[c] = acc;
        }
        if (l2norm) {
            double ss = 0.0;
            for (int c = 0; c < d; ++c) ss += yr[c] * yr[c];
            double n = sqrt(ss);
            if (n < 1e-6) n = 1e-6;
            for (int c = 0; c < d; ++c) yr[c] /= n;
        }
    }
}

/* Softmax attention of one query row over all L keys of (b, h).
 * s_j = scale * q.k_j ; p_j = exp(s_j - max_j s_j) ; o = sum_j p_j v_j / sum_j p_j */
static void intra_row(int H, int d, int L, int b, int h, int i, double scale,
                      const double* q, const double* k, const double* v,
                      double* s /* [L] scratch */, double* o /* [d] */) {
    const double* qi = q + IDX4(b, i, h, 0, L, H, d);
    double m = -INFINITY;
    for (int j = 0; j < L; ++j) {
        const double* kj = k + IDX4(b, j, h, 0, L, H, d);
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += qi[c] * kj[c];
        s[j] = scale * dot;
        if (s[j] > m) m = s[j];
    }
    double l = 0.0;
    for (int j = 0; j < L; ++j) {
        s[j] = exp(s[j] - m);
        l += s[j];
    }
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    for (int j = 0; j < L; ++j) {
        const double* vj = v + IDX4(b, j, h, 0, L, H, d);
        for (int c = 0; c < d; ++c) o[c] += s[j] * vj[c];
    }
    for (int c = 0; c < d; ++c) o[c] /= l;
}

/* o += (q W_q) S for one row q of head h; S is the pre-update state. */
static void inter_row(int d, const double* qi, const double* Wq, const double* S, double* o) {
    double* qp = (double*)malloc(sizeof(double) * (size_t)d);
    for (int c = 0; c < d; ++c) {
        double acc = 0.0;
        for (int a = 0; a < d; ++a) acc += qi[a] * Wq[(size_t)a * d + c];
        qp[c] = acc;
    }
    for (int n = 0; n < d; ++n) {
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += qp[c] * S[(size_t)c * d + n];
        o[n] += acc;
    }
    free(qp);
}

/* Gated delta update of one (b, h) state, clean pass only:
 * S <- alpha S + K'^T diag(beta) (V' - K' S), with the residual taken
 * against the pre-update S for every token (frame-level access). */
static int update_head(int B, int H, int d, int L, int b, int h, const double* k,
                       const double* v, const double* w_k, const double* w_v,
                       const double* alpha, int alpha_per_key, const double* beta, double* S_all) {
    (void)B;
    double* kp = (double*)malloc(sizeof(double) * (size_t)L * d);
    double* vp = (double*)malloc(sizeof(double) * (size_t)L * d);
    double* r = (double*)malloc(sizeof(double) * (size_t)L * d);
    double* dS = (double*)malloc(sizeof(double) * (size_t)d * d);
    if (!kp || !vp || !r || !dS) {
        free(kp); free(vp); free(r); free(dS);
        return -1;
    }
    double* S = S_all + IDX4(b, h, 0, 0, H, d, d);
    phi_map_head(H, d, L, b, h, k, w_k, 1, kp);
    phi_map_head(H, d, L, b, h, v, w_v, 0, vp);
    /* r_t = v'_t - k'_t S */
    for (int t = 0; t < L; ++t) {
        for (int n = 0; n < d; ++n) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c) acc += kp[(size_t)t * d + c] * S[(size_t)c * d + n];
            r[(size_t)t * d + n] = vp[(size_t)t * d + n] - acc;
        }
    }
    /* dS = sum_t beta_t k'_t^T r_t */
    const double* bt = beta + IDX4(0, b, h, 0, 1, H, L);
    for (int c = 0; c < d; ++c) {
        for (int n = 0; n < d; ++n) {
            double acc = 0.0;
            for (int t = 0; t < L; ++t) acc += bt[t] * kp[(size_t)t * d + c] * r[(size_t)t * d + n];
            dS[(size_t)c * d + n] = acc;
        }
    }
    /* headwise gate: one alpha for the whole state; elementwise gate: one
     * alpha per key feature c, i.e. diag(alpha) S (row c of S scaled) */
    for (int c = 0; c < d; ++c) {
        const double a = alpha_per_key ? alpha[((size_t)b * H + h) * d + c] : alpha[(size_t)b * H + h];
        for (int n = 0; n < d; ++n)
            S[(size_t)c * d + n] = a * S[(size_t)c * d + n] + dS[(size_t)c * d + n];
    }
    free(kp); free(vp); free(r); free(dS);
    return 0;
}

/* phi map of a whole [B][L][H][d] tensor: out = x W[h] per head, with an
 * optional L2 normalisation of each output row (used for k'). */
int arl2_oracle_phi(int B, int H, int d, int L, const double* x, const double* w,
                    int l2norm, double* out) {
    if (bad_dims(B, H, d, L) || !x || !w || !out) return -1;
    int err = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : err)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            double* xp = (double*)malloc(sizeof(double) * (size_t)L * d);
            if (!xp) { err |= 1; continue; }
            phi_map_head(H, d, L, b, h, x, w, l2norm, xp);
            for (int t = 0; t < L; ++t)
                for (int c = 0; c < d; ++c) out[IDX4(b, t, h, c, L, H, d)] = xp[(size_t)t * d + c];
            free(xp);
        }
    }
    return err ? -1 : 0;
}

/* Outputs O = O_intra + O_inter of selected rows.  Row r is token rows_t[r]
 * of stream rows_b[r]; out_rows is [nrows][H][d].  S is only read. */
int arl2_oracle_rows(int B, int H, int d, int L, double scale, const double* q,
                     const double* k, const double* v, const double* w_q, const double* S,
                     int nrows, const int* rows_b, const int* rows_t, double* out_rows) {
    if (bad_dims(B, H, d, L) || nrows < 0 || !q || !k || !v || !w_q || !S || !out_rows) return -1;
    if (nrows > 0 && (!rows_b || !rows_t)) return -1;
    for (int r = 0; r < nrows; ++r)
        if (rows_b[r] < 0 || rows_b[r] >= B || rows_t[r] < 0 || rows_t[r] >= L) return -1;
    int err = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : err)
    for (int r = 0; r < nrows; ++r) {
        for (int h = 0; h < H; ++h) {
            double* s = (double*)malloc(sizeof(double) * (size_t)L);
            if (!s) { err |= 1; continue; }
            const int b = rows_b[r], i = rows_t[r];
            double* o = out_rows + ((size_t)r * H + h) * d;
            intra_row(H, d, L, b, h, i, scale, q, k, v, s, o);
            inter_row(d, q + IDX4(b, i, h, 0, L, H, d), w_q + (size_t)h * d * d,
                      S + IDX4(b, h, 0, 0, H, d, d), o);
            free(s);
        }
    }
    return err ? -1 : 0;
}

/* Clean-pass state update of every (b, h), in place.  alpha_per_key = 0:
 * alpha is [B][H] (headwise gating, the form the pages adopt); 1: alpha is
 * [B][H][d], one gate per key feature, S_N = diag(alpha) S_{N-1} + ... (the
 * elementwise gating the pages compare it with, atlas summary "Surprising
 * findings"). */
int arl2_oracle_state_update_gated(int B, int H, int d, int L, const double* k, const double* v,
                                   const double* w_k, const double* w_v, const double* alpha,
                                   int alpha_per_key, const double* beta, double* S) {
    if (bad_dims(B, H, d, L) || !k || !v || !w_k || !w_v || !alpha || !beta || !S) return -1;
    int err = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : err)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            if (update_head(B, H, d, L, b, h, k, v, w_k, w_v, alpha, alpha_per_key, beta, S)) err |= 1;
    return err ? -1 : 0;
}

int arl2_oracle_state_update(int B, int H, int d, int L, const double* k, const double* v,
                             const double* w_k, const double* w_v, const double* alpha,
                             const double* beta, double* S) {
    return arl2_oracle_state_update_gated(B, H, d, L, k, v, w_k, w_v, alpha, 0, beta, S);
}

/* One full pass: out for every token, then (clean != 0) the state update.
 * The output of a clean pass reads the pre-update state. */
int arl2_oracle_pass(int B, int H, int d, int L, double scale, const double* q,
                     const double* k, const double* v, const double* w_q, const double* w_k,
                     const double* w_v, const double* alpha, const double* beta, int clean,
                     double* S, double* out) {
    if (bad_dims(B, H, d, L) || !q || !k || !v || !w_q || !S || !out) return -1;
    if (clean && (!w_k || !w_v || !alpha || !beta)) return -1;
    int err = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : err)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            double* s = (double*)malloc(sizeof(double) * (size_t)L);
            if (!s) { err |= 1; continue; }
            for (int i = 0; i < L; ++i) {
                double* o = out + IDX4(b, i, h, 0, L, H, d);
                intra_row(H, d, L, b, h, i, scale, q, k, v, s, o);
                inter_row(d, q + IDX4(b, i, h, 0, L, H, d), w_q + (size_t)h * d * d,
                          S + IDX4(b, h, 0, 0, H, d, d), o);
            }
            free(s);
        }
    }
    if (err) return -1;
    if (clean) return arl2_oracle_state_update(B, H, d, L, k, v, w_k, w_v, alpha, beta, S);
    return 0;
}

/* Token-level (sequential) state access: the ablation the pages compare with
 * frame-level access (technical summary section 2.2 "Frame-Level Access";
 * atlas summary "Surprising findings").  Within the frame, token i reads the
 * state left by tokens 0..i-1 and then updates it with the delta rule; the
 * frame's forget gate acts once, with token 0's update:
 *   S^(0)   = S_{N-1}
 *   o_i     = intra_i + q'_i S^(i)
 *   S^(i+1) = G_i S^(i) + beta_i k'_i^T (v'_i - k'_i S^(i)),
 *             G_0 = alpha (diag(alpha) with per-key gates), G_i = I for i > 0
 * With one token per frame this is the frame-level rule.  Every pass reads
 * through its own sequential states; only the clean pass keeps S^(L) as S_N
 * ("Clean-Pass Updates").  Tokens are taken in their order in the frame. */
static int token_level_head(int H, int d, int L, int b, int h, double scale, const double* q,
                            const double* k, const double* v, const double* w_q, const double* w_k,
                            const double* w_v, const double* alpha, int alpha_per_key,
                            const double* beta, int clean, double* S_all, double* out) {
    double* qp = (double*)malloc(sizeof(double) * (size_t)L * d);
    double* kp = (double*)malloc(sizeof(double) * (size_t)L * d);
    double* vp = (double*)malloc(sizeof(double) * (size_t)L * d);
    double* St = (double*)malloc(sizeof(double) * (size_t)d * d);
    double* u = (double*)malloc(sizeof(double) * (size_t)d);
    double* s = (double*)malloc(sizeof(double) * (size_t)L);
    if (!qp || !kp || !vp || !St || !u || !s) {
        free(qp); free(kp); free(vp); free(St); free(u); free(s);
        return -1;
    }
    double* S = S_all + IDX4(b, h, 0, 0, H, d, d);
    phi_map_head(H, d, L, b, h, q, w_q, 0, qp);
    phi_map_head(H, d, L, b, h, k, w_k, 1, kp);
    phi_map_head(H, d, L, b, h, v, w_v, 0, vp);
    for (size_t e = 0; e < (size_t)d * d; ++e) St[e] = S[e];
    const double* bt = beta + IDX4(0, b, h, 0, 1, H, L);
    for (int i = 0; i < L; ++i) {
        double* o = out + IDX4(b, i, h, 0, L, H, d);
        intra_row(H, d, L, b, h, i, scale, q, k, v, s, o);
        /* read the state before this token's update */
        for (int n = 0; n < d; ++n) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c) acc += qp[(size_t)i * d + c] * St[(size_t)c * d + n];
            o[n] += acc;
        }
        /* u = v'_i - k'_i S^(i) */
        for (int n = 0; n < d; ++n) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c) acc += kp[(size_t)i * d + c] * St[(size_t)c * d + n];
            u[n] = vp[(size_t)i * d + n] - acc;
        }
        for (int c = 0; c < d; ++c) {
            double g = 1.0;
            if (i == 0) g = alpha_per_key ? alpha[((size_t)b * H + h) * d + c] : alpha[(size_t)b * H + h];
            for (int n = 0; n < d; ++n)
                St[(size_t)c * d + n] = g * St[(size_t)c * d + n] + bt[i] * kp[(size_t)i * d + c] * u[n];
        }
    }
    if (clean)
        for (size_t e = 0; e < (size_t)d * d; ++e) S[e] = St[e];
    free(qp); free(kp); free(vp); free(St); free(u); free(s);
    return 0;
}

int arl2_oracle_pass_token_level(int B, int H, int d, int L, double scale, const double* q,
                                 const double* k, const double* v, const double* w_q,
                                 const double* w_k, const double* w_v, const double* alpha,
                                 int alpha_per_key, const double* beta, int clean, double* S,
                                 double* out) {
    if (bad_dims(B, H, d, L) || !q || !k || !v || !w_q || !w_k || !w_v || !alpha || !beta || !S ||
        !out)
        return -1;
    int err = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : err)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            if (token_level_head(H, d, L, b, h, scale, q, k, v, w_q, w_k, w_v, alpha, alpha_per_key,
                                 beta, clean, S, out))
                err |= 1;
    return err ? -1 : 0;
}

/* ------------------------------------------------------------------------
 * Softmax teacher layer with a KV cache: the attention the hybrid layer
 * replaces, kept by the layers of the stack that stay softmax (technical
 * summary section 1 "KV Cache Growth"; section 4 "Efficiency", where the
 * speedup grows with video length as the cache comes to dominate).  The
 * pages fix the cache's role, not its arithmetic; the reading taken here is
 * chunk-causal attention at frame granularity:
 *   O = softmax([Q Kc^T, Q K^T] * scale) [Vc; V]
 * for the L query rows of frame N, where (Kc, Vc) hold, in frame order, the
 * keys and values of the clean passes of frames 0..N-1 (the same passes
 * that update the hybrid layer's state, section 2.2 "Clean-Pass Updates"),
 * and (K, V) are the current pass's own, attended bidirectionally.  A clean
 * pass then appends its K and V to the cache; the caller does that by
 * concatenation, nothing here keeps state.
 *
 * kc, vc: [B][Lc][H][d] (Lc = N L; Lc = 0 for the first frame, when kc and
 * vc may be NULL).  q, k, v, out: [B][L][H][d]. */

/* One query row: cached keys j < Lc first, then the frame's own keys. */
static void teacher_row(int H, int d, int L, int Lc, int b, int h, int i, double scale,
                        const double* q, const double* k, const double* v, const double* kc,
                        const double* vc, double* s /* [Lc + L] */, double* o /* [d] */) {
    const double* qi = q + IDX4(b, i, h, 0, L, H, d);
    const int n = Lc + L;
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) {
        const double* kj = j < Lc ? kc + IDX4(b, j, h, 0, Lc, H, d)
                                  : k + IDX4(b, j - Lc, h, 0, L, H, d);
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += qi[c] * kj[c];
        s[j] = dot * scale;
        if (s[j] > m) m = s[j];
    }
    double l = 0.0;
    for (int j = 0; j < n; ++j) {
        s[j] = exp(s[j] - m);
        l += s[j];
    }
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    for (int j = 0; j < n; ++j) {
        const double* vj = j < Lc ? vc + IDX4(b, j, h, 0, Lc, H, d)
                                  : v + IDX4(b, j - Lc, h, 0, L, H, d);
        for (int c = 0; c < d; ++c) o[c] += s[j] * vj[c];
    }
    for (int c = 0; c < d; ++c) o[c] = o[c] / l;
}

static int teacher_args_bad(int B, int H, int d, int L, int Lc, const double* q, const double* k,
                            const double* v, const double* kc, const double* vc) {
    if (bad_dims(B, H, d, L) || Lc < 0 || !q || !k || !v) return 1;
    return Lc > 0 && (!kc || !vc);
}

/* Every row of the frame. */
int arl2_oracle_teacher_pass(int B, int H, int d, int L, int Lc, double scale, const double* q,
                             const double* k, const double* v, const double* kc, const double* vc,
                             double* out) {
    if (teacher_args_bad(B, H, d, L, Lc, q, k, v, kc, vc) || !out) return -1;
    int err = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : err)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            double* s = (double*)malloc(sizeof(double) * ((size_t)Lc + L));
            if (!s) { err |= 1; continue; }
            for (int i = 0; i < L; ++i)
                teacher_row(H, d, L, Lc, b, h, i, scale, q, k, v, kc, vc, s,
                            out + IDX4(b, i, h, 0, L, H, d));
            free(s);
        }
    }
    return err ? -1 : 0;
}

/* Selected rows only (row r: token rows_t[r] of stream rows_b[r]); out_rows
 * is [nrows][H][d].  For long caches, where the whole frame is too slow. */
int arl2_oracle_teacher_rows(int B, int H, int d, int L, int Lc, double scale, const double* q,
                             const double* k, const double* v, const double* kc, const double* vc,
                             int nrows, const int* rows_b, const int* rows_t, double* out_rows) {
    if (teacher_args_bad(B, H, d, L, Lc, q, k, v, kc, vc) || nrows < 0 || !out_rows) return -1;
    if (nrows > 0 && (!rows_b || !rows_t)) return -1;
    for (int r = 0; r < nrows; ++r)
        if (rows_b[r] < 0 || rows_b[r] >= B || rows_t[r] < 0 || rows_t[r] >= L) return -1;
    int err = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : err)
    for (int r = 0; r < nrows; ++r) {
        for (int h = 0; h < H; ++h) {
            double* s = (double*)malloc(sizeof(double) * ((size_t)Lc + L));
            if (!s) { err |= 1; continue; }
            teacher_row(H, d, L, Lc, rows_b[r], h, rows_t[r], scale, q, k, v, kc, vc, s,
                        out_rows + ((size_t)r * H + h) * d);
            free(s);
        }
    }
    return err ? -1 : 0;
}

/* ------------------------------------------------------------------------
 * Gate projections.  The technical summary (section 2.1 "State Update")
 * calls alpha (forget gate) and beta (learning rate) learned per-token
 * projections and gives no form; the reading taken here:
 *   per token i and head h, two logits from the token's hidden state x_i:
 *     a_ih = x_i . w[:, h]     + bias[h]
 *     g_ih = x_i . w[:, H + h] + bias[H + h]
 *   beta_ih = sigmoid(g_ih)                 (one rate per token)
 *   alpha_h = sigmoid((1/L) sum_i a_ih)     (one forget gate per frame and
 *             head: the frame updates the state once, section 2.2
 *             "Frame-Level Access", and headwise gating is the form the
 *             ablations adopt, section 4)
 * x: [B][L][D] (the layer's input hidden states); w: [D][2H]; bias: [2H];
 * alpha: [B][H]; beta: [B][H][L]. */
static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

int arl2_oracle_gate_projection(int B, int L, int D, int H, const double* x, const double* w,
                                const double* bias, double* alpha, double* beta) {
    if (B < 1 || L < 1 || D < 1 || H < 1 || !x || !w || !bias || !alpha || !beta) return -1;
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            double a_sum = 0.0;
            for (int i = 0; i < L; ++i) {
                const double* xi = x + ((size_t)b * L + i) * D;
                double a = bias[h], g = bias[H + h];
                for (int e = 0; e < D; ++e) {
                    a += xi[e] * w[(size_t)e * 2 * H + h];
                    g += xi[e] * w[(size_t)e * 2 * H + H + h];
                }
                beta[((size_t)b * H + h) * L + i] = sigmoid(g);
                a_sum += a;
            }
            alpha[(size_t)b * H + h] = sigmoid(a_sum / L);
        }
    }
    return 0;
}
