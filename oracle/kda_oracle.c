/*
 * kda_oracle.c -- fp64 CPU oracle for Kimi Delta Attention (KDA).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct
 * definition that the CUDA library is checked against.  It shares no code,
 * header, table or helper with the CUDA path, and nothing in the product
 * path may load it: only the tests, the smoke check and the benchmark's CPU
 * baseline leg do.
 *
 * What it computes (KimiLinear: A Next-Generation Linear Attention
 * Architecture for Long-Context LLMs, section 2.3, the KDA state-update rule):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(a_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = scale * S_t^T q_t
 *
 * with S_t a d_k x d_v matrix (row index = key channel, column index = value
 * channel), a_t = exp(g_t) the per-channel forget gate acting on the ROWS of
 * the state (the same section gives each row of the state, one latent
 * feature per key channel, its own forgetting rate), and beta_t a scalar
 * write strength per token and head.
 * Readings taken where the page is silent or garbled (each also listed in the
 * design notes):
 *   - orientation: the page writes the write term as v k^T but left-multiplies
 *     by a d_k x d_k matrix; we keep S in d_k x d_v form, write k v^T and read
 *     o = S^T q (the transpose of the page's convention, identical o);
 *   - the output o_t is read from the state AFTER token t has been written;
 *   - scale multiplies the output only, never the state;
 *   - the gate is supplied as its logarithm g_t, a_t = exp(g_t).
 *
 * Expanding the product gives the sequential form used below:
 *     S'  = Diag(a_t) S_{t-1}                  (decay rows)
 *     u   = beta_t (v_t - S'^T k_t)            (delta-rule correction)
 *     S_t = S' + k_t u^T                       (rank-1 write)
 * because (I - b k k^T) S' + b k v^T = S' + k (b (v - S'^T k))^T.
 *
 * mode == KDA_ORACLE_LINEAR drops the delta correction (u = beta_t v_t), which
 * turns the update into gated linear attention; with a == 1 and beta == 1 it
 * is plain linear attention, S_t = S_{t-1} + k_t v_t^T (same article, section
 * 2.1).  That mode exists only so the oracle's decay/output machinery can be
 * pinned against a closed form.
 *
 * Layouts (row-major, contiguous):
 *   q, k, g : [B, T, H, dk]     v, o : [B, T, H, dv]     beta : [B, T, H]
 *   s0, sT  : [B, H, dk, dv]    (s0 may be NULL => zero initial state;
 *                                sT may be NULL => final state not written)
 * Parallelism: OpenMP over (b, h, column block); the columns of S evolve
 * independently, so splitting them changes no arithmetic.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define KDA_ORACLE_DELTA 0
#define KDA_ORACLE_LINEAR 1

static int oracle_col_block(int dv) { return dv < 16 ? dv : 16; }

/* One (b, h, column block [j0, j1)) chain, token by token. */
static void oracle_chain(const double* q, const double* k, const double* v, const double* g,
                         const double* beta, double scale, const double* s0, double* o,
                         double* sT, int b, int h, int j0, int j1, int T, int H, int dk, int dv,
                         int mode) {
  const int nc = j1 - j0;
  double* S = (double*)malloc(sizeof(double) * (size_t)dk * nc);  /* S[i][j-j0] */
  double* a = (double*)malloc(sizeof(double) * (size_t)dk);
  double* u = (double*)malloc(sizeof(double) * (size_t)nc);
  for (int i = 0; i < dk; ++i)
    for (int j = 0; j < nc; ++j)
      S[(size_t)i * nc + j] =
          s0 ? s0[(((size_t)b * H + h) * dk + i) * dv + j0 + j] : 0.0;

  for (int t = 0; t < T; ++t) {
    const size_t tok = ((size_t)b * T + t) * H + h;  /* (b, t, h) */
    const double* qt = q + tok * dk;
    const double* kt = k + tok * dk;
    const double* gt = g + tok * dk;
    const double* vt = v + tok * dv;
    const double bt = beta[tok];

    /* S' = Diag(exp(g_t)) S : every key-channel row i scaled by a_i. */
    for (int i = 0; i < dk; ++i) a[i] = exp(gt[i]);
    for (int i = 0; i < dk; ++i)
      for (int j = 0; j < nc; ++j) S[(size_t)i * nc + j] *= a[i];

    /* u = beta (v - S'^T k), or u = beta v without the delta correction. */
    for (int j = 0; j < nc; ++j) {
      double pred = 0.0;
      if (mode == KDA_ORACLE_DELTA)
        for (int i = 0; i < dk; ++i) pred += S[(size_t)i * nc + j] * kt[i];
      u[j] = bt * (vt[j0 + j] - pred);
    }

    /* S = S' + k u^T */
    for (int i = 0; i < dk; ++i)
      for (int j = 0; j < nc; ++j) S[(size_t)i * nc + j] += kt[i] * u[j];

    /* o_t = scale * S_t^T q_t */
    for (int j = 0; j < nc; ++j) {
      double acc = 0.0;
      for (int i = 0; i < dk; ++i) acc += S[(size_t)i * nc + j] * qt[i];
      o[tok * dv + j0 + j] = scale * acc;
    }
  }

  if (sT)
    for (int i = 0; i < dk; ++i)
      for (int j = 0; j < nc; ++j)
        sT[(((size_t)b * H + h) * dk + i) * dv + j0 + j] = S[(size_t)i * nc + j];
  free(S);
  free(a);
  free(u);
}

/*
 * Runs the recurrence over all (b, h).  Returns 0 on success, -1 on a bad
 * argument.  nthreads <= 0 lets OpenMP choose.
 */
int kda_oracle_forward(const double* q, const double* k, const double* v, const double* g,
                       const double* beta, double scale, const double* s0, double* o, double* sT,
                       int B, int T, int H, int dk, int dv, int mode, int nthreads) {
  if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
  if (mode != KDA_ORACLE_DELTA && mode != KDA_ORACLE_LINEAR) return -1;
  if (T > 0 && (!q || !k || !v || !g || !beta || !o)) return -1;
  const int cb = oracle_col_block(dv);
  const int nblk = (dv + cb - 1) / cb;
  const long total = (long)B * H * nblk;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
  for (long w = 0; w < total; ++w) {
    const int blk = (int)(w % nblk);
    const int h = (int)((w / nblk) % H);
    const int b = (int)(w / ((long)nblk * H));
    const int j0 = blk * cb;
    const int j1 = j0 + cb < dv ? j0 + cb : dv;
    oracle_chain(q, k, v, g, beta, scale, s0, o, sT, b, h, j0, j1, T, H, dk, dv, mode);
  }
  return 0;
}

/* Number of threads OpenMP would use (for reporting the CPU baseline). */
int kda_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/*
 * Backward pass: the gradients of a scalar loss L through the recurrence
 * above, given dL/do (dO, [B,T,H,dv]) and dL/dS_T (dST, [B,H,dk,dv] or NULL
 * for zero).  Outputs, in the layouts of the inputs: dq, dk, dg ([B,T,H,dk]),
 * dv ([B,T,H,dv]), dbeta ([B,T,H]) and dS0 = dL/dS_0 ([B,H,dk,dv]).
 *
 * Reverse-mode differentiation of the sequential form, one state column j at
 * a time (a column of S evolves on its own: s' = a_t .* s, w = v_t[j] - s'.k_t,
 * u = beta_t w, s = s' + k_t u, o_t[j] = scale s.q_t).  With G = dL/dS_t[:, j],
 * starting from dST[:, j], for t = T-1 .. 0:
 *   G += scale q_t dO_t[j];   dq_t += scale s_t dO_t[j]          (o_t reads S_t)
 *   du = G.k_t;   dk_t += G u;   dv_t[j] = beta_t du;   dbeta_t += du w
 *   G -= beta_t k_t du;   dk_t -= beta_t s'_t du                   (G = dL/dS'_t)
 *   dg_t += G .* s'_t                 (dL/da_t .* a_t, since s' = a_t .* s_{t-1})
 *   G = a_t .* G                                                   (dL/dS_{t-1})
 * and dS0[:, j] = G.  The per-token sums over j (dq, dk, dg, dbeta) collect
 * over the columns of one (b, h) in column order.
 */
static void oracle_chain_bwd(const double* q, const double* k, const double* v, const double* g,
                             const double* beta, double scale, const double* s0, const double* dO,
                             const double* dST, double* dq, double* dk, double* dvv, double* dg,
                             double* dbeta, double* dS0, int b, int h, int T, int H, int nk, int nv) {
  double* sp = (double*)malloc(sizeof(double) * ((size_t)T * nk + 1));  /* s'_t, all t */
  double* w = (double*)malloc(sizeof(double) * ((size_t)T + 1));
  double* s = (double*)malloc(sizeof(double) * (size_t)nk);
  double* G = (double*)malloc(sizeof(double) * (size_t)nk);
  const size_t st0 = ((size_t)b * H + h) * nk * nv;
  for (int t = 0; t < T; ++t) {  /* zero this (b, h)'s per-token sums */
    const size_t tok = ((size_t)b * T + t) * H + h;
    for (int i = 0; i < nk; ++i) dq[tok * nk + i] = dk[tok * nk + i] = dg[tok * nk + i] = 0.0;
    dbeta[tok] = 0.0;
  }
  for (int j = 0; j < nv; ++j) {
    /* forward over column j, keeping s'_t and w_t */
    for (int i = 0; i < nk; ++i) s[i] = s0 ? s0[st0 + (size_t)i * nv + j] : 0.0;
    for (int t = 0; t < T; ++t) {
      const size_t tok = ((size_t)b * T + t) * H + h;
      const double* kt = k + tok * nk;
      const double* gt = g + tok * nk;
      double* spt = sp + (size_t)t * nk;
      double pred = 0.0;
      for (int i = 0; i < nk; ++i) {
        spt[i] = exp(gt[i]) * s[i];
        pred += spt[i] * kt[i];
      }
      w[t] = v[tok * nv + j] - pred;
      const double u = beta[tok] * w[t];
      for (int i = 0; i < nk; ++i) s[i] = spt[i] + kt[i] * u;
    }
    /* reverse */
    for (int i = 0; i < nk; ++i) G[i] = dST ? dST[st0 + (size_t)i * nv + j] : 0.0;
    for (int t = T - 1; t >= 0; --t) {
      const size_t tok = ((size_t)b * T + t) * H + h;
      const double* qt = q + tok * nk;
      const double* kt = k + tok * nk;
      const double* gt = g + tok * nk;
      const double* spt = sp + (size_t)t * nk;
      const double bt = beta[tok], u = bt * w[t], dot = dO[tok * nv + j];
      double du = 0.0;
      for (int i = 0; i < nk; ++i) {
        const double st = spt[i] + kt[i] * u;           /* S_t[i][j] */
        G[i] += scale * qt[i] * dot;
        dq[tok * nk + i] += scale * st * dot;
        du += G[i] * kt[i];
      }
      dvv[tok * nv + j] = bt * du;
      dbeta[tok] += du * w[t];
      for (int i = 0; i < nk; ++i) {
        dk[tok * nk + i] += G[i] * u - bt * spt[i] * du;
        G[i] -= bt * kt[i] * du;
        dg[tok * nk + i] += G[i] * spt[i];
        G[i] *= exp(gt[i]);
      }
    }
    if (dS0)
      for (int i = 0; i < nk; ++i) dS0[st0 + (size_t)i * nv + j] = G[i];
  }
  free(sp);
  free(w);
  free(s);
  free(G);
}

/* Backward over all (b, h) (OpenMP over them).  0 on success, -1 on a bad argument. */
int kda_oracle_backward(const double* q, const double* k, const double* v, const double* g,
                        const double* beta, double scale, const double* s0, const double* dO,
                        const double* dST, double* dq, double* dk, double* dv_out, double* dg,
                        double* dbeta, double* dS0, int B, int T, int H, int nk, int nv, int nthreads) {
  if (B < 0 || T < 0 || H < 0 || nk <= 0 || nv <= 0) return -1;
  if (T > 0 && (!q || !k || !v || !g || !beta || !dO || !dq || !dk || !dv_out || !dg || !dbeta)) return -1;
  const long total = (long)B * H;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
  for (long wk = 0; wk < total; ++wk) {
    const int h = (int)(wk % H), b = (int)(wk / H);
    oracle_chain_bwd(q, k, v, g, beta, scale, s0, dO, dST, dq, dk, dv_out, dg, dbeta, dS0, b, h, T, H, nk, nv);
  }
  return 0;
}
