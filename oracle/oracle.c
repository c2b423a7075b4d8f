/*
 * fp64 CPU oracle for the four token mixers of the Super Apriel supernet.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the slow, plain reference that the CUDA kernels are
 * checked against. Only the tests, the smoke check and the benchmark's CPU-baseline leg load
 * it; the library's product path never does. It shares no code, header or constant with the
 * CUDA sources.
 *
 * What the pages fix: every decoder layer offers four mixers, full attention (FA, O(n^2)),
 * sliding-window attention (SWA, O(n*w)), Kimi Delta Attention (KDA, a recurrence with
 * channel-wise gating, O(n)) and Gated DeltaNet (GDN, a recurrence with a scalar gate, O(n));
 * a placement picks one per layer ("Super Apriel: One Checkpoint, Many Speeds", abstract;
 * gist.science technical summary of the same paper, section 2a "Supernet architecture").
 * The pages give no equations, so the standard published definitions are used:
 *
 *   GDN (Gated DeltaNet):  S_t = g_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T,  o_t = S_t q_t
 *                          S is d_v x d_k, g_t in (0,1) one scalar per token-head.
 *   KDA (Kimi Delta Attn): S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T,
 *                          o_t = S_t^T q_t;  S is d_k x d_v, a_t in (0,1)^{d_k}.
 *   FA:  o = softmax(q K^T / sqrt(d)) V over every cached key of the sequence.
 *   SWA: the same over the last w keys (the window includes the current token).
 *
 * Conventions (the pages are silent on these; see the design notes):
 *   - States are stored as M[d_k][d_v] for both kinds, i.e. M = S^T for GDN and M = S for KDA.
 *   - Gates arrive as logarithms: g = exp(log_g), a = exp(log_a).
 *   - o is multiplied by `scale` (1.0 in every workload; the definitions have no scale).
 *   - Attention scale 1/sqrt(d); GQA query head h reads kv-head h / (Hq/Hkv).
 *   - Paged KV: logical position p lives at (page_table[b][p / PT], p % PT) for FA, and at ring
 *     index r = p mod (R*PT), R = ceil(w / PT), i.e. (page_table[b][r / PT], r % PT), for SWA.
 *
 * Arithmetic is fp64 in plain loops, token by token, no fast-math. OpenMP threads split only
 * independent (batch, head) pairs, so results do not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_FA = 0, OR_SWA = 1, OR_KDA = 2, OR_GDN = 3 };

static void set_threads(int n_threads) {
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
}

/* bf16 bit pattern -> double (exact: bf16 is the top half of an IEEE binary32). */
static double bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------------------------ */
/* Recurrent form, token by token (GDN and KDA definitions written out as above).              */
/* ------------------------------------------------------------------------------------------ */

/* One GDN token on one head, in the definition's own orientation S[j][i] (d_v x d_k):
 *   S_new = g S (I - b k k^T) + b v k^T
 *         = g S - g b (S k) k^T + b v k^T,   o = S_new q.                                       */
static void gdn_token(int dk, int dv, double *S /* [dv][dk] */, const double *q,
                      const double *k, const double *v, double beta, double log_g, double scale,
                      double *o, double *Sk /* scratch [dv] */) {
    const double g = exp(log_g);
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += S[(size_t)j * dk + i] * k[i];
        Sk[j] = acc;
    }
    for (int j = 0; j < dv; ++j)
        for (int i = 0; i < dk; ++i)
            S[(size_t)j * dk + i] = g * S[(size_t)j * dk + i] - g * beta * Sk[j] * k[i]
                                    + beta * v[j] * k[i];
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += S[(size_t)j * dk + i] * q[i];
        o[j] = scale * acc;
    }
}

/* One KDA token on one head, S[i][j] (d_k x d_v):
 *   S_new = (I - b k k^T) Diag(a) S + b k v^T
 *         = Diag(a) S - b k (k^T Diag(a) S) + b k v^T,   o = S_new^T q.                         */
static void kda_token(int dk, int dv, double *S /* [dk][dv] */, const double *q,
                      const double *k, const double *v, double beta, const double *log_a,
                      double scale, double *o, double *kaS /* scratch [dv] */,
                      double *a /* scratch [dk] */) {
    for (int i = 0; i < dk; ++i) a[i] = exp(log_a[i]);
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += k[i] * a[i] * S[(size_t)i * dv + j];
        kaS[j] = acc;
    }
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j)
            S[(size_t)i * dv + j] = a[i] * S[(size_t)i * dv + j] - beta * k[i] * kaS[j]
                                    + beta * k[i] * v[j];
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * q[i];
        o[j] = scale * acc;
    }
}

/* Token-by-token GDN / KDA over T tokens.
 *   q, k [B][T][H][dk]; v [B][T][H][dv]; beta [B][T][H];
 *   log_gate [B][T][H] (GDN) or [B][T][H][dk] (KDA);
 *   state [B][H][dk][dv] in/out (M = S^T for GDN, M = S for KDA); o [B][T][H][dv].
 * Returns 0, or -1 on a bad kind / allocation failure.                                          */
int oracle_delta_recurrent(int kind, int B, int T, int H, int dk, int dv, const double *q,
                           const double *k, const double *v, const double *beta,
                           const double *log_gate, double scale, double *state, double *o,
                           int n_threads) {
    if (kind != OR_GDN && kind != OR_KDA) return -1;
    set_threads(n_threads);
    int bad = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : bad)
    for (int bh = 0; bh < B * H; ++bh) {
        const int b = bh / H, h = bh % H;
        double *M = state + (size_t)bh * dk * dv;
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        double *s1 = (double *)malloc(sizeof(double) * (size_t)(dk > dv ? dk : dv));
        double *s2 = (double *)malloc(sizeof(double) * (size_t)(dk > dv ? dk : dv));
        if (!S || !s1 || !s2) { bad |= 1; free(S); free(s1); free(s2); continue; }
        /* Load the stored state into the definition's orientation. */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j)
                if (kind == OR_GDN) S[(size_t)j * dk + i] = M[(size_t)i * dv + j];
                else S[(size_t)i * dv + j] = M[(size_t)i * dv + j];
        for (int t = 0; t < T; ++t) {
            const size_t th = ((size_t)b * T + t) * H + h;
            const double *qt = q + th * dk, *kt = k + th * dk, *vt = v + th * dv;
            double *ot = o + th * dv;
            if (kind == OR_GDN)
                gdn_token(dk, dv, S, qt, kt, vt, beta[th], log_gate[th], scale, ot, s1);
            else
                kda_token(dk, dv, S, qt, kt, vt, beta[th], log_gate + th * dk, scale, ot, s1, s2);
        }
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j)
                M[(size_t)i * dv + j] = (kind == OR_GDN) ? S[(size_t)j * dk + i]
                                                         : S[(size_t)i * dv + j];
        free(S); free(s1); free(s2);
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------------------------ */
/* Chunked (WY / UT-transform) form. The pages only name the recurrences; this is the standard */
/* chunkwise rewriting of the gated delta rule, derived here for M = S^T (GDN) / S (KDA):       */
/*                                                                                             */
/* Within a chunk of C tokens starting from state M0, with per-channel cumulative log-gates    */
/* G[r][i] = sum_{s<=r} log a_{s,i} (a scalar gate is broadcast over i):                       */
/*   A[r][s] = b_r sum_i k_{r,i} k_{s,i} exp(G[r][i]-G[s][i])        (s < r, else 0)           */
/*   T       = (I + A)^{-1} Diag(b)                                  (forward substitution)    */
/*   Kt[r][i]= exp(G[r][i]) k_{r,i};  Qt[r][i] = exp(G[r][i]) q_{r,i}                          */
/*   W = T Kt;  Ut = T V;  U = Ut - W M0                              (U[r] = u_r of the token) */
/*   P[r][s] = sum_i q_{r,i} k_{s,i} exp(G[r][i]-G[s][i])            (s <= r, else 0)          */
/*   O = Qt M0 + P U                                                                           */
/*   M_C[i][j] = exp(G[C-1][i]) M0[i][j] + sum_s k_{s,i} exp(G[C-1][i]-G[s][i]) U[s][j]        */
/* The exponent differences are formed directly so nothing overflows in fp64.                  */
/* ------------------------------------------------------------------------------------------ */
int oracle_delta_chunked(int kind, int B, int T, int H, int dk, int dv, int C, const double *q,
                         const double *k, const double *v, const double *beta,
                         const double *log_gate, double scale, double *state, double *o,
                         int n_threads) {
    if ((kind != OR_GDN && kind != OR_KDA) || C < 1) return -1;
    set_threads(n_threads);
    int bad = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : bad)
    for (int bh = 0; bh < B * H; ++bh) {
        const int b = bh / H, h = bh % H;
        double *M = state + (size_t)bh * dk * dv;
        double *G = (double *)malloc(sizeof(double) * (size_t)C * dk);
        double *A = (double *)malloc(sizeof(double) * (size_t)C * C);
        double *Tm = (double *)malloc(sizeof(double) * (size_t)C * C);
        double *P = (double *)malloc(sizeof(double) * (size_t)C * C);
        double *W = (double *)malloc(sizeof(double) * (size_t)C * dk);
        double *U = (double *)malloc(sizeof(double) * (size_t)C * dv);
        double *Mn = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        if (!G || !A || !Tm || !P || !W || !U || !Mn) {
            bad |= 1;
            free(G); free(A); free(Tm); free(P); free(W); free(U); free(Mn);
            continue;
        }
        for (int t0 = 0; t0 < T; t0 += C) {
            const int n = (T - t0) < C ? (T - t0) : C; /* the last chunk may be partial */
#define TH(r) (((size_t)b * T + (size_t)(t0 + (r))) * H + h)
#define LG(r, i) (kind == OR_GDN ? log_gate[TH(r)] : log_gate[TH(r) * dk + (i)])
            /* cumulative log-gates */
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int r = 0; r < n; ++r) { acc += LG(r, i); G[(size_t)r * dk + i] = acc; }
            }
            /* A (strictly lower) and P (lower incl. diagonal) */
            for (int r = 0; r < n; ++r)
                for (int s = 0; s < n; ++s) {
                    double a = 0.0, p = 0.0;
                    for (int i = 0; i < dk; ++i) {
                        const double e = exp(G[(size_t)r * dk + i] - G[(size_t)s * dk + i]);
                        a += k[TH(r) * dk + i] * k[TH(s) * dk + i] * e;
                        p += q[TH(r) * dk + i] * k[TH(s) * dk + i] * e;
                    }
                    A[(size_t)r * C + s] = (s < r) ? beta[TH(r)] * a : 0.0;
                    P[(size_t)r * C + s] = (s <= r) ? p : 0.0;
                }
            /* T = (I + A)^{-1} Diag(beta): solve (I + A) T = Diag(beta) row by row */
            for (int r = 0; r < n; ++r)
                for (int c = 0; c < n; ++c) {
                    double x = (r == c) ? beta[TH(r)] : 0.0;
                    for (int s = 0; s < r; ++s) x -= A[(size_t)r * C + s] * Tm[(size_t)s * C + c];
                    Tm[(size_t)r * C + c] = x;
                }
            /* W = T Kt,  U = T V - W M0 */
            for (int r = 0; r < n; ++r) {
                for (int i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int s = 0; s < n; ++s)
                        acc += Tm[(size_t)r * C + s] * exp(G[(size_t)s * dk + i]) * k[TH(s) * dk + i];
                    W[(size_t)r * dk + i] = acc;
                }
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int s = 0; s < n; ++s) acc += Tm[(size_t)r * C + s] * v[TH(s) * dv + j];
                    for (int i = 0; i < dk; ++i) acc -= W[(size_t)r * dk + i] * M[(size_t)i * dv + j];
                    U[(size_t)r * dv + j] = acc;
                }
            }
            /* O = Qt M0 + P U */
            for (int r = 0; r < n; ++r)
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i)
                        acc += exp(G[(size_t)r * dk + i]) * q[TH(r) * dk + i] * M[(size_t)i * dv + j];
                    for (int s = 0; s < n; ++s) acc += P[(size_t)r * C + s] * U[(size_t)s * dv + j];
                    o[TH(r) * dv + j] = scale * acc;
                }
            /* state at the end of the chunk */
            for (int i = 0; i < dk; ++i) {
                const double gC = G[(size_t)(n - 1) * dk + i];
                for (int j = 0; j < dv; ++j) {
                    double acc = exp(gC) * M[(size_t)i * dv + j];
                    for (int s = 0; s < n; ++s)
                        acc += k[TH(s) * dk + i] * exp(gC - G[(size_t)s * dk + i]) * U[(size_t)s * dv + j];
                    Mn[(size_t)i * dv + j] = acc;
                }
            }
            memcpy(M, Mn, sizeof(double) * (size_t)dk * dv);
#undef LG
#undef TH
        }
        free(G); free(A); free(Tm); free(P); free(W); free(U); free(Mn);
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------------------------ */
/* Paged KV indexing and decode attention.                                                     */
/* ------------------------------------------------------------------------------------------ */

/* Where logical position `pos` of a sequence lives: writes the physical page and the offset in
 * it. FA: page_row[pos / PT], pos % PT. SWA: ring index r = pos mod (R*PT) with
 * R = ceil(window / PT), then page_row[r / PT], r % PT. Returns 0, or -1 on bad arguments.     */
int oracle_kv_slot(int kind, int window, int page_tokens, const int32_t *page_row, int max_pages,
                   int pos, int32_t *page, int32_t *offset) {
    if (page_tokens < 1 || pos < 0) return -1;
    long idx = pos;
    if (kind == OR_SWA) {
        if (window < 1) return -1;
        const long R = (window + page_tokens - 1) / page_tokens;
        idx = pos % (R * page_tokens);
    } else if (kind != OR_FA) {
        return -1;
    }
    const long lp = idx / page_tokens;
    if (lp >= max_pages) return -1;
    *page = page_row[lp];
    *offset = (int32_t)(idx % page_tokens);
    return 0;
}

/* One decode step of FA or SWA for every (sequence, query head).
 *   q [B][Hq][d] (double); new_k, new_v [B][Hkv][d] (double) are the token being decoded, at
 *   logical position L-1 where L = seq_lens[b] counts it; k_pool, v_pool are bf16 bits
 *   [P][Hkv][PT][d] holding positions 0..L-2; page_table [B][max_pages].
 *   The keys attended are j in [lo, L-1] with lo = 0 (FA) or max(0, L - window) (SWA).
 *   o [B][Hq][d] (double). Returns 0, or -1 on bad arguments or a bad page id.               */
int oracle_attn_decode(int kind, int window, int B, int Hq, int Hkv, int d, int page_tokens,
                       int n_pages, const double *q, const double *new_k, const double *new_v,
                       const uint16_t *k_pool, const uint16_t *v_pool, const int32_t *page_table,
                       int max_pages, const int32_t *seq_lens, double *o, int n_threads) {
    if ((kind != OR_FA && kind != OR_SWA) || Hkv < 1 || Hq % Hkv) return -1;
    if (kind == OR_SWA && window < 1) return -1;
    set_threads(n_threads);
    const int group = Hq / Hkv;
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    int bad = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : bad)
    for (int bh = 0; bh < B * Hq; ++bh) {
        const int b = bh / Hq, h = bh % Hq, g = h / group;
        const int L = seq_lens[b];
        if (L < 1) { bad |= 1; continue; }
        const int lo = (kind == OR_SWA && L > window) ? L - window : 0;
        const int n = L - lo;
        double *s = (double *)malloc(sizeof(double) * (size_t)n);
        if (!s) { bad |= 1; continue; }
        const double *qv = q + ((size_t)b * Hq + h) * d;
        double mx = -INFINITY;
        for (int j = lo; j < L; ++j) {
            double acc = 0.0;
            if (j == L - 1) {
                const double *kv = new_k + ((size_t)b * Hkv + g) * d;
                for (int c = 0; c < d; ++c) acc += qv[c] * kv[c];
            } else {
                int32_t pg, off;
                if (oracle_kv_slot(kind, window, page_tokens, page_table + (size_t)b * max_pages,
                                   max_pages, j, &pg, &off) || pg < 0 || pg >= n_pages) {
                    bad |= 1; acc = 0.0;
                } else {
                    const uint16_t *kv = k_pool + (((size_t)pg * Hkv + g) * page_tokens + off) * d;
                    for (int c = 0; c < d; ++c) acc += qv[c] * bf16_to_double(kv[c]);
                }
            }
            s[j - lo] = acc * inv_sqrt_d;
            if (s[j - lo] > mx) mx = s[j - lo];
        }
        double denom = 0.0;
        for (int j = 0; j < n; ++j) { s[j] = exp(s[j] - mx); denom += s[j]; }
        double *ov = o + ((size_t)b * Hq + h) * d;
        for (int c = 0; c < d; ++c) ov[c] = 0.0;
        for (int j = lo; j < L; ++j) {
            const double p = s[j - lo] / denom;
            if (j == L - 1) {
                const double *vv = new_v + ((size_t)b * Hkv + g) * d;
                for (int c = 0; c < d; ++c) ov[c] += p * vv[c];
            } else {
                int32_t pg, off;
                if (oracle_kv_slot(kind, window, page_tokens, page_table + (size_t)b * max_pages,
                                   max_pages, j, &pg, &off) || pg < 0 || pg >= n_pages) {
                    bad |= 1;
                } else {
                    const uint16_t *vv = v_pool + (((size_t)pg * Hkv + g) * page_tokens + off) * d;
                    for (int c = 0; c < d; ++c) ov[c] += p * bf16_to_double(vv[c]);
                }
            }
        }
        free(s);
    }
    return bad ? -1 : 0;
}

/* Prefill of FA or SWA over T new tokens per sequence, starting from an empty cache. Token t
 * sits at logical position t and attends keys j in [lo_t, t], lo_t = 0 (FA) or
 * max(0, t + 1 - window) (SWA): the decode step above with L = t + 1, for every t at once.
 *   q [B][T][Hq][d], k, v [B][T][Hkv][d], o [B][T][Hq][d] (double).
 * Returns 0, or -1 on bad arguments.                                                          */
int oracle_attn_prefill(int kind, int window, int B, int T, int Hq, int Hkv, int d,
                        const double *q, const double *k, const double *v, double *o,
                        int n_threads) {
    if ((kind != OR_FA && kind != OR_SWA) || Hkv < 1 || Hq % Hkv || T < 0 || d < 1) return -1;
    if (kind == OR_SWA && window < 1) return -1;
    set_threads(n_threads);
    const int group = Hq / Hkv;
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    int bad = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : bad)
    for (int bh = 0; bh < B * Hq; ++bh) {
        const int b = bh / Hq, h = bh % Hq, kvh = h / group;
        double *s = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
        if (!s) { bad |= 1; continue; }
        for (int t = 0; t < T; ++t) {
            const int lo = (kind == OR_SWA && t + 1 > window) ? t + 1 - window : 0;
            const double *qv = q + (((size_t)b * T + t) * Hq + h) * d;
            double mx = -INFINITY;
            for (int j = lo; j <= t; ++j) {
                const double *kv = k + (((size_t)b * T + j) * Hkv + kvh) * d;
                double acc = 0.0;
                for (int c = 0; c < d; ++c) acc += qv[c] * kv[c];
                s[j - lo] = inv_sqrt_d * acc;
                if (s[j - lo] > mx) mx = s[j - lo];
            }
            double denom = 0.0;
            for (int j = lo; j <= t; ++j) {
                s[j - lo] = exp(s[j - lo] - mx);
                denom += s[j - lo];
            }
            double *ov = o + (((size_t)b * T + t) * Hq + h) * d;
            for (int c = 0; c < d; ++c) ov[c] = 0.0;
            for (int j = lo; j <= t; ++j) {
                const double p = s[j - lo] / denom;
                const double *vv = v + (((size_t)b * T + j) * Hkv + kvh) * d;
                for (int c = 0; c < d; ++c) ov[c] += p * vv[c];
            }
        }
        free(s);
    }
    return bad ? -1 : 0;
}

/* Cache slot of logical position pos when SWA keeps a ring of ring_pages pages (a verifier of
 * n_q tokens needs at least window + n_q - 1 positions in its ring, see below). FA ignores
 * ring_pages. Returns 0, or -1 on bad arguments.                                              */
int oracle_kv_slot_ring(int kind, int ring_pages, int page_tokens, const int32_t *page_row,
                        int max_pages, int pos, int32_t *page, int32_t *offset) {
    if (page_tokens < 1 || pos < 0) return -1;
    long ring_idx = pos;
    if (kind == OR_SWA) {
        if (ring_pages < 1) return -1;
        ring_idx = pos % ((long)ring_pages * page_tokens);
    } else if (kind != OR_FA) {
        return -1;
    }
    const long logical_page = ring_idx / page_tokens;
    if (logical_page >= max_pages) return -1;
    *page = page_row[logical_page];
    *offset = (int32_t)(ring_idx % page_tokens);
    return 0;
}

/* Verification pass of speculative decoding: n_q new tokens per sequence, which is exactly n_q
 * decode steps in a row (each appends its token, then attends). Token i of sequence b sits at
 * logical position P = L - n_q + i (L = seq_lens[b] counts all n_q) and query head h attends
 * keys j in [lo, P], lo = 0 (FA) or max(0, P + 1 - window) (SWA), with kv-head h / (Hq / Hkv).
 * Keys j < L - n_q are read from the pools (bf16 bits [P][Hkv][PT][d], SWA ring of ring_pages
 * pages); keys j >= L - n_q are the new tokens themselves.
 *   q [B][n_q][Hq][d]; new_k, new_v [B][n_q][Hkv][d]; o [B][n_q][Hq][d] (double).
 * Returns 0, or -1 on bad arguments or a bad page id.                                          */
int oracle_attn_verify(int kind, int window, int ring_pages, int n_q, int B, int Hq, int Hkv,
                       int d, int page_tokens, int n_pages, const double *q, const double *new_k,
                       const double *new_v, const uint16_t *k_pool, const uint16_t *v_pool,
                       const int32_t *page_table, int max_pages, const int32_t *seq_lens,
                       double *o, int n_threads) {
    if ((kind != OR_FA && kind != OR_SWA) || Hkv < 1 || Hq % Hkv || n_q < 1) return -1;
    if (kind == OR_SWA && window < 1) return -1;
    set_threads(n_threads);
    const int heads_per_kv = Hq / Hkv;
    const double rsqrt_d = 1.0 / sqrt((double)d);
    int bad = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : bad)
    for (int row = 0; row < B * n_q * Hq; ++row) {
        const int b = row / (n_q * Hq), i = (row / Hq) % n_q, h = row % Hq;
        const int kvh_v = h / heads_per_kv;
        const int L = seq_lens[b];
        const int first_new = L - n_q;  /* logical position of new token 0 */
        const int P_pos = first_new + i;
        if (first_new < 0) { bad |= 1; continue; }
        const int lo = (kind == OR_SWA && P_pos + 1 > window) ? P_pos + 1 - window : 0;
        double *sc = (double *)malloc(sizeof(double) * (size_t)(P_pos - lo + 1));
        if (!sc) { bad |= 1; continue; }
        const double *qv = q + (size_t)row * d;
        double mx = -INFINITY;
        for (int j = lo; j <= P_pos; ++j) {
            double dot = 0.0;
            if (j >= first_new) {
                const double *kv = new_k + (((size_t)b * n_q + (j - first_new)) * Hkv + kvh_v) * d;
                for (int c = 0; c < d; ++c) dot += qv[c] * kv[c];
            } else {
                int32_t pg, off;
                if (oracle_kv_slot_ring(kind, ring_pages, page_tokens,
                                        page_table + (size_t)b * max_pages, max_pages, j, &pg,
                                        &off) || pg < 0 || pg >= n_pages) {
                    bad |= 1;
                } else {
                    const uint16_t *kv = k_pool + (((size_t)pg * Hkv + kvh_v) * page_tokens + off) * d;
                    for (int c = 0; c < d; ++c) dot += qv[c] * bf16_to_double(kv[c]);
                }
            }
            sc[j - lo] = dot * rsqrt_d;
            if (sc[j - lo] > mx) mx = sc[j - lo];
        }
        double denom = 0.0;
        for (int j = lo; j <= P_pos; ++j) {
            sc[j - lo] = exp(sc[j - lo] - mx);
            denom += sc[j - lo];
        }
        double *ov = o + (size_t)row * d;
        for (int c = 0; c < d; ++c) ov[c] = 0.0;
        for (int j = lo; j <= P_pos; ++j) {
            const double w = sc[j - lo] / denom;
            if (j >= first_new) {
                const double *vv = new_v + (((size_t)b * n_q + (j - first_new)) * Hkv + kvh_v) * d;
                for (int c = 0; c < d; ++c) ov[c] += w * vv[c];
            } else {
                int32_t pg, off;
                if (oracle_kv_slot_ring(kind, ring_pages, page_tokens,
                                        page_table + (size_t)b * max_pages, max_pages, j, &pg,
                                        &off) || pg < 0 || pg >= n_pages) {
                    bad |= 1;
                } else {
                    const uint16_t *vv = v_pool + (((size_t)pg * Hkv + kvh_v) * page_tokens + off) * d;
                    for (int c = 0; c < d; ++c) ov[c] += w * bf16_to_double(vv[c]);
                }
            }
        }
        free(sc);
    }
    return bad ? -1 : 0;
}

/* The input activations of the GDN / KDA mixers, from the projections' raw outputs (the
 * pages name the mixers but not their parameterisation; this is the standard one of the
 * published GDN and KDA layers):
 *   q = q_raw / sqrt(sum(q_raw^2) + eps), k likewise (L2 over d_k, per token and head);
 *   beta = 1 / (1 + exp(-beta_logit));
 *   log_gate = -exp(A_log[h]) * softplus(gate_logit + dt_bias),  softplus(x) = log(1 + exp(x)),
 *   with dt_bias [H] and gate_logit [N][H] for GDN, dt_bias [H][dk] and gate_logit [N][H][dk]
 *   for KDA. N counts the token rows (B*T, or B for one decode step).
 *   q_raw, k_raw [N][H][dk] in, q, k out; beta_logit [N][H] in, beta out; log_gate out.
 * Returns 0, or -1 on bad arguments.                                                          */
int oracle_delta_activations(int kind, int N, int H, int dk, double eps, const double *q_raw,
                             const double *k_raw, const double *beta_logit,
                             const double *gate_logit, const double *A_log, const double *dt_bias,
                             double *q, double *k, double *beta, double *log_gate) {
    if ((kind != OR_GDN && kind != OR_KDA) || N < 0 || H < 1 || dk < 1 || !(eps >= 0.0))
        return -1;
    for (long row = 0; row < (long)N * H; ++row) {
        const int h = (int)(row % H);
        double sq = 0.0, sk = 0.0;
        for (int i = 0; i < dk; ++i) {
            sq += q_raw[row * dk + i] * q_raw[row * dk + i];
            sk += k_raw[row * dk + i] * k_raw[row * dk + i];
        }
        const double nq = sqrt(sq + eps), nk = sqrt(sk + eps);
        for (int i = 0; i < dk; ++i) {
            q[row * dk + i] = q_raw[row * dk + i] / nq;
            k[row * dk + i] = k_raw[row * dk + i] / nk;
        }
        beta[row] = 1.0 / (1.0 + exp(-beta_logit[row]));
        const double decay_rate = exp(A_log[h]);
        if (kind == OR_GDN) {
            const double x = gate_logit[row] + dt_bias[h];
            log_gate[row] = -decay_rate * log1p(exp(x));
        } else {
            for (int i = 0; i < dk; ++i) {
                const double x = gate_logit[row * dk + i] + dt_bias[(size_t)h * dk + i];
                log_gate[row * dk + i] = -decay_rate * log1p(exp(x));
            }
        }
    }
    return 0;
}

/* The oracle's thread count after set-up (for reporting). */
int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
