/*
 * kda_oracle.c -- plain fp64 CPU oracle for the Kimi Delta Attention (KDA)
 * operator.  TEST INFRASTRUCTURE: only the test suite, the smoke check and
 * the CPU-baseline leg of the benchmark load this library.  It shares no code,
 * header or constant with the CUDA library under gated_delta_rule_110_b200/.
 *
 * What it computes (per sequence n and head h, token by token, in order):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t                 alpha_t = exp(log_alpha_t), per channel
 *
 * S is a dk x dv matrix (row index = key channel, column = value channel).
 * Sources (the pages' titles and sections):
 *   - "Kimi Linear" news summary (pt.news.hada.io), section "Da atencao linear
 *     ao Gated DeltaNet": the delta rule is online gradient descent on the
 *     reconstruction loss; each rank-1 update is a generalised Householder
 *     transform; GDN adds a scalar forget gate.
 *   - same page, section "Controle fino de memoria no Kimi Delta Attention":
 *     KDA replaces the scalar gate by a per-channel (diagonal) gate and the
 *     transition is a specialised Diagonal-Plus-Low-Rank matrix.
 *   The update equation itself is not printed on the pages; the form above is
 *   the plainest one consistent with that prose (decay first, then the delta
 *   correction; output read from the post-update state).
 *
 * Evaluated literally:
 *     S~   = Diag(alpha_t) S                 (decay each key channel row)
 *     kS   = S~^T k_t                         (what the memory recalls for k)
 *     d    = beta_t (v_t - kS)                (delta-rule error, scaled)
 *     S    = S~ + k_t d^T                     (rank-1 correction)
 *     o_t  = S^T q_t
 * which equals the transition form above by distributing the product.
 *
 * Parity is pinned by the CPU tests (brute-force transition products,
 * DeltaNet / Gated DeltaNet reductions, the pure-decay closed form,
 * Householder identities and structural invariances); the `mutation`
 * argument exists only so those tests can plant known mistakes here and
 * check that some pin catches each one.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Planted mistakes, used only by the pin-strength tests. 0 = the oracle. */
enum {
  MUT_NONE = 0,
  MUT_DECAY_AFTER_DELTA = 1,   /* apply Diag(alpha) after the rank-1 step   */
  MUT_OUTPUT_PRE_UPDATE = 2,   /* o_t read from S_{t-1} (decayed)           */
  MUT_OUTPUT_TRANSPOSED = 3,   /* o_t = S q_t instead of S^T q_t            */
  MUT_DELTA_SIGN = 4,          /* d = beta (kS - v)                         */
  MUT_DROP_BETA_ERASE = 5,     /* S~ + beta k v^T - k kS^T (beta on v only)  */
  MUT_GATE_ON_VALUES = 6,      /* Diag(alpha) scales value columns          */
  MUT_IGNORE_S0 = 7,           /* start from zeros whatever S0 holds        */
  MUT_KS_UNDECAYED = 8,        /* error term uses S_{t-1}, not S~           */
  MUT_COUNT = 9
};

static void run_one(int64_t t0, int64_t t1, int h, int H, int dk, int dv,
                    const double* q, const double* k, const double* v,
                    const double* la, const double* beta, const double* S0,
                    double* o, double* ST, int mutation,
                    double* S, double* Sprev, double* tmp)
{
  const size_t dd = (size_t)dk * dv;
  if (S0 && mutation != MUT_IGNORE_S0)
    memcpy(S, S0, dd * sizeof(double));
  else
    memset(S, 0, dd * sizeof(double));

  for (int64_t t = t0; t < t1; ++t) {
    const double* qt = q + ((size_t)t * H + h) * dk;
    const double* kt = k + ((size_t)t * H + h) * dk;
    const double* vt = v + ((size_t)t * H + h) * dv;
    const double* lt = la + ((size_t)t * H + h) * dk;
    const double bt = beta[(size_t)t * H + h];
    double* ot = o + ((size_t)t * H + h) * dv;

    if (mutation == MUT_KS_UNDECAYED || mutation == MUT_DECAY_AFTER_DELTA)
      memcpy(Sprev, S, dd * sizeof(double));

    /* S~ = Diag(alpha) S */
    if (mutation != MUT_DECAY_AFTER_DELTA) {
      for (int c = 0; c < dk; ++c)
        for (int j = 0; j < dv; ++j) {
          const double a = (mutation == MUT_GATE_ON_VALUES) ? exp(lt[j % dk]) : exp(lt[c]);
          S[(size_t)c * dv + j] *= a;
        }
    }

    /* kS = S~^T k  (the value the memory returns for key k) */
    const double* Sread = (mutation == MUT_KS_UNDECAYED) ? Sprev : S;
    for (int j = 0; j < dv; ++j) {
      double acc = 0.0;
      for (int c = 0; c < dk; ++c) acc += kt[c] * Sread[(size_t)c * dv + j];
      tmp[j] = acc;
    }

    /* o from the pre-update state, if that mistake is planted */
    if (mutation == MUT_OUTPUT_PRE_UPDATE) {
      for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int c = 0; c < dk; ++c) acc += qt[c] * S[(size_t)c * dv + j];
        ot[j] = acc;
      }
    }

    /* S = S~ + k d^T,  d = beta (v - kS) */
    for (int c = 0; c < dk; ++c)
      for (int j = 0; j < dv; ++j) {
        double d;
        if (mutation == MUT_DELTA_SIGN)
          d = bt * (tmp[j] - vt[j]);
        else if (mutation == MUT_DROP_BETA_ERASE)
          d = bt * vt[j] - tmp[j];
        else
          d = bt * (vt[j] - tmp[j]);
        S[(size_t)c * dv + j] += kt[c] * d;
      }

    if (mutation == MUT_DECAY_AFTER_DELTA) {
      for (int c = 0; c < dk; ++c) {
        const double a = exp(lt[c]);
        for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] *= a;
      }
    }

    /* o_t = S^T q_t */
    if (mutation == MUT_OUTPUT_TRANSPOSED) {
      /* o_j = sum_c S[j][c] q_c -- only meaningful when dk == dv */
      for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int c = 0; c < dk; ++c) acc += S[(size_t)(j % dk) * dv + (c % dv)] * qt[c];
        ot[j] = acc;
      }
    } else if (mutation != MUT_OUTPUT_PRE_UPDATE) {
      for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int c = 0; c < dk; ++c) acc += qt[c] * S[(size_t)c * dv + j];
        ot[j] = acc;
      }
    }
  }
  memcpy(ST, S, dd * sizeof(double));
}

/*
 * kda_oracle_forward_mut -- the oracle with an optional planted mistake.
 *
 *   n_seqs      number of packed sequences N
 *   cu_seqlens  N+1 non-decreasing token offsets, cu[0] = 0 (host memory)
 *   H, dk, dv   heads, key and value head dimensions
 *   q, k        [T_total, H, dk] fp64, token-major       (host memory)
 *   v           [T_total, H, dv]
 *   log_alpha   [T_total, H, dk]  natural log of the per-channel gate
 *   beta        [T_total, H]
 *   S0          [N, H, dk, dv] initial states, or NULL for zeros
 *   o           [T_total, H, dv] output
 *   S_T         [N, H, dk, dv] final states
 *   n_threads   OpenMP threads over (sequence, head); <= 0 = runtime default
 *   mutation    0 for the oracle; a MUT_* code plants one mistake
 * Returns 0, or -1 on bad arguments / allocation failure.
 */
int kda_oracle_forward_mut(int n_seqs, const int64_t* cu_seqlens, int H, int dk, int dv,
                           const double* q, const double* k, const double* v,
                           const double* log_alpha, const double* beta, const double* S0,
                           double* o, double* S_T, int n_threads, int mutation)
{
  if (n_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0 || !cu_seqlens || !S_T) return -1;
  if (mutation < 0 || mutation >= MUT_COUNT) return -1;
  for (int n = 0; n < n_seqs; ++n)
    if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
  const int64_t total = (int64_t)n_seqs * H;
  const size_t dd = (size_t)dk * dv;
  int failed = 0;

#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel
#endif
  {
    double* S = (double*)malloc(dd * sizeof(double));
    double* Sprev = (double*)malloc(dd * sizeof(double));
    double* tmp = (double*)malloc((size_t)dv * sizeof(double));
    if (!S || !Sprev || !tmp) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
      failed = 1;
    } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
      for (int64_t nh = 0; nh < total; ++nh) {
        const int n = (int)(nh / H), h = (int)(nh % H);
        run_one(cu_seqlens[n], cu_seqlens[n + 1], h, H, dk, dv, q, k, v, log_alpha, beta,
                S0 ? S0 + ((size_t)n * H + h) * dd : NULL, o,
                S_T + ((size_t)n * H + h) * dd, mutation, S, Sprev, tmp);
      }
    }
    free(S);
    free(Sprev);
    free(tmp);
  }
  return failed ? -1 : 0;
}

/* The oracle proper: kda_oracle_forward_mut with no planted mistake. */
int kda_oracle_forward(int n_seqs, const int64_t* cu_seqlens, int H, int dk, int dv,
                       const double* q, const double* k, const double* v,
                       const double* log_alpha, const double* beta, const double* S0,
                       double* o, double* S_T, int n_threads)
{
  return kda_oracle_forward_mut(n_seqs, cu_seqlens, H, dk, dv, q, k, v, log_alpha, beta, S0,
                                o, S_T, n_threads, MUT_NONE);
}

/*
 * kda_oracle_decode -- one recurrent step for N independent (sequence, head)
 * states, updated in place: the same arithmetic as one token of
 * kda_oracle_forward.  q, k, log_alpha: [N, H, dk]; v, o: [N, H, dv];
 * beta: [N, H]; S: [N, H, dk, dv].
 */
int kda_oracle_decode(int N, int H, int dk, int dv, const double* q, const double* k,
                      const double* v, const double* log_alpha, const double* beta,
                      double* S, double* o, int n_threads)
{
  if (N < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
  int64_t* cu = (int64_t*)malloc(((size_t)N + 1) * sizeof(int64_t));
  if (!cu) return -1;
  for (int n = 0; n <= N; ++n) cu[n] = n;
  /* one token per sequence: token index n is sequence n, so the packed
     [T=N, H, d] layout is exactly the decode layout [N, H, d]. */
  int rc = kda_oracle_forward(N, cu, H, dk, dv, q, k, v, log_alpha, beta, S, o, S, n_threads);
  free(cu);
  return rc;
}

int kda_oracle_mutation_count(void) { return MUT_COUNT; }

/*
 * kda_oracle_output_gate -- the per-head output normalisation and gate that
 * the "Kimi Linear" summary (section "Configuracao do modelo Kimi Linear")
 * places after the operator and before the output projection: an RMSNorm per
 * head and a data-dependent output gate.  The page gives no formula; taken
 * here in its plainest form, per token t and head h over the dv channels:
 *
 *     rms     = sqrt( (1/dv) * sum_j o[j]^2 + eps )
 *     out[j]  = o[j] / rms * w[j] * sigmoid(g[j]),   sigmoid(x) = 1 / (1 + e^-x)
 *
 * w (dv values) is the RMSNorm weight, shared by all heads; g is the gate's
 * pre-activation for this token and head (the low-rank projection that
 * produces it belongs to the model, not to the operator).
 * o, g, out: [rows, dv] (rows = tokens x heads, one row per (token, head)).
 */
int kda_oracle_output_gate(int64_t rows, int dv, const double* o, const double* g, const double* w, double eps,
                           double* out) {
  if (rows < 0 || dv <= 0 || !o || !g || !w || !out || !(eps >= 0.0)) return -1;
  for (int64_t r = 0; r < rows; ++r) {
    const double* x = o + r * dv;
    double ss = 0.0;
    for (int j = 0; j < dv; ++j) ss += x[j] * x[j];
    const double rms = sqrt(ss / dv + eps);
    for (int j = 0; j < dv; ++j) {
      const double gate = 1.0 / (1.0 + exp(-g[r * dv + j]));
      out[r * dv + j] = x[j] / rms * w[j] * gate;
    }
  }
  return 0;
}

/*
 * kda_oracle_l2norm -- the L2 normalisation of the query and the key that the
 * "Kimi Linear" summary (section "Configuração do modelo Kimi Linear") adds
 * for the stability of the transition's eigenvalues.  Per row (one token and
 * head) of d values:
 *
 *     out[j] = x[j] / sqrt( sum_i x[i]^2 + eps )
 *
 * eps >= 0 keeps a zero row at zero (the page names no epsilon).
 */
int kda_oracle_l2norm(int64_t rows, int d, const double* x, double eps, double* out) {
  if (rows < 0 || d <= 0 || !x || !out || !(eps >= 0.0)) return -1;
  for (int64_t r = 0; r < rows; ++r) {
    double ss = 0.0;
    for (int j = 0; j < d; ++j) ss += x[r * d + j] * x[r * d + j];
    const double n = sqrt(ss + eps);
    for (int j = 0; j < d; ++j) out[r * d + j] = n > 0.0 ? x[r * d + j] / n : 0.0;
  }
  return 0;
}

/* log(1 + e^x) without overflow */
static double softplus(double x) { return x > 0.0 ? x + log1p(exp(-x)) : log1p(exp(x)); }

/*
 * kda_oracle_decay_gate -- the channel-wise decay gate.  The same page
 * parametrises it by a low-rank projection (its output f, one value per key
 * channel) and a decay function "like GDN's and Mamba's": a positive step
 * size softplus(f + bias) times a negative per-head rate -exp(A_log).  Per
 * token t, head h, channel c:
 *
 *     log alpha[t][h][c] = -exp(A_log[h]) * softplus(f[t][h][c] + dt_bias[h][c])
 *
 * f, out: [tokens, H, dk]; A_log: [H]; dt_bias: [H, dk].
 */
int kda_oracle_decay_gate(int64_t tokens, int H, int dk, const double* f, const double* A_log,
                          const double* dt_bias, double* out) {
  if (tokens < 0 || H <= 0 || dk <= 0 || !f || !A_log || !dt_bias || !out) return -1;
  for (int64_t t = 0; t < tokens; ++t)
    for (int h = 0; h < H; ++h) {
      const double rate = exp(A_log[h]);
      for (int c = 0; c < dk; ++c) {
        const int64_t e = (t * H + h) * dk + c;
        out[e] = -rate * softplus(f[e] + dt_bias[h * dk + c]);
      }
    }
  return 0;
}

/*
 * kda_oracle_backward -- gradients of the operator (no page prints them; the
 * chunkwise algorithm section of the "Kimi Linear" summary mentions the UT
 * transform's use in training).  Reverse-mode differentiation of the token
 * recurrence above, written out by hand, per (sequence, head):
 *
 *   forward, token t (S_prev the state before it):
 *     S~ = Diag(alpha) S_prev,  u = v - S~^T k,  S = S~ + beta k u^T,  o = S^T q
 *   backward, with dS the gradient reaching S_t from later tokens (dS_T at
 *   the end) and do = dL/do_t:
 *     dq   = S do                      dS  += q do^T
 *     dbeta = k^T dS u                 du   = beta dS^T k
 *     dk   = beta dS u - S~ du         dv   = du
 *     dS~  = dS - k du^T
 *     dlog_alpha[i] = sum_j dS~[i][j] S~[i][j]     (d alpha = alpha d log alpha)
 *     dS_prev = Diag(alpha) dS~
 *   and dS0 = the gradient reaching the initial state.
 *
 * Layouts as kda_oracle_forward; dO like o, dS_T like S_T (either may be
 * NULL: no gradient from it).  Outputs dq, dk, dlog_alpha like q; dv like v;
 * dbeta like beta; dS0 like S0 (always written).  The forward states are
 * recomputed and kept for the whole sequence (test sizes only).
 */
int kda_oracle_backward(int n_seqs, const int64_t* cu_seqlens, int H, int dk, int dv,
                        const double* q, const double* k, const double* v, const double* log_alpha,
                        const double* beta, const double* S0, const double* dO, const double* dS_T,
                        double* dq, double* dk_out, double* dv_out, double* dla, double* dbeta, double* dS0)
{
  if (n_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0 || !cu_seqlens) return -1;
  const size_t dd = (size_t)dk * dv;
  for (int n = 0; n < n_seqs; ++n) {
    const int64_t t0 = cu_seqlens[n], t1 = cu_seqlens[n + 1];
    if (t1 < t0) return -1;
    const int64_t L = t1 - t0;
    for (int h = 0; h < H; ++h) {
      /* states[i] = state after i tokens of this sequence (states[0] = S0) */
      double* states = (double*)calloc((size_t)(L + 1) * dd, sizeof(double));
      double* dS = (double*)calloc(dd, sizeof(double));
      double* St = (double*)malloc(dd * sizeof(double));
      double* u = (double*)malloc((size_t)dv * sizeof(double));
      double* du = (double*)malloc((size_t)dv * sizeof(double));
      if (!states || !dS || !St || !u || !du) {
        free(states); free(dS); free(St); free(u); free(du);
        return -1;
      }
      if (S0) memcpy(states, S0 + ((size_t)n * H + h) * dd, dd * sizeof(double));
      for (int64_t i = 0; i < L; ++i) {
        const int64_t row = (t0 + i) * H + h;
        const double* kt = k + row * dk;
        const double* vt = v + row * dv;
        const double b = beta[row];
        const double* Sp = states + (size_t)i * dd;
        double* Sn = states + (size_t)(i + 1) * dd;
        for (int a = 0; a < dk; ++a) {
          const double al = exp(log_alpha[row * dk + a]);
          for (int j = 0; j < dv; ++j) St[a * dv + j] = al * Sp[a * dv + j];
        }
        for (int j = 0; j < dv; ++j) {
          double r = 0.0;
          for (int a = 0; a < dk; ++a) r += St[a * dv + j] * kt[a];
          u[j] = vt[j] - r;
        }
        for (int a = 0; a < dk; ++a)
          for (int j = 0; j < dv; ++j) Sn[a * dv + j] = St[a * dv + j] + b * kt[a] * u[j];
      }
      if (dS_T) memcpy(dS, dS_T + ((size_t)n * H + h) * dd, dd * sizeof(double));
      for (int64_t i = L - 1; i >= 0; --i) {
        const int64_t row = (t0 + i) * H + h;
        const double* qt = q + row * dk;
        const double* kt = k + row * dk;
        const double* vt = v + row * dv;
        const double b = beta[row];
        const double* Sp = states + (size_t)i * dd;
        const double* Sn = states + (size_t)(i + 1) * dd;
        /* o = S^T q */
        for (int a = 0; a < dk; ++a) {
          double g = 0.0;
          if (dO)
            for (int j = 0; j < dv; ++j) g += Sn[a * dv + j] * dO[row * dv + j];
          dq[row * dk + a] = g;
        }
        if (dO)
          for (int a = 0; a < dk; ++a)
            for (int j = 0; j < dv; ++j) dS[a * dv + j] += qt[a] * dO[row * dv + j];
        /* recompute S~ and u of this token */
        for (int a = 0; a < dk; ++a) {
          const double al = exp(log_alpha[row * dk + a]);
          for (int j = 0; j < dv; ++j) St[a * dv + j] = al * Sp[a * dv + j];
        }
        for (int j = 0; j < dv; ++j) {
          double r = 0.0;
          for (int a = 0; a < dk; ++a) r += St[a * dv + j] * kt[a];
          u[j] = vt[j] - r;
        }
        /* S = S~ + beta k u^T */
        double db = 0.0;
        for (int a = 0; a < dk; ++a)
          for (int j = 0; j < dv; ++j) db += kt[a] * dS[a * dv + j] * u[j];
        dbeta[row] = db;
        for (int j = 0; j < dv; ++j) {
          double r = 0.0;
          for (int a = 0; a < dk; ++a) r += dS[a * dv + j] * kt[a];
          du[j] = b * r;
          dv_out[row * dv + j] = du[j];  /* u = v - S~^T k */
        }
        for (int a = 0; a < dk; ++a) {
          double g1 = 0.0, g2 = 0.0;
          for (int j = 0; j < dv; ++j) {
            g1 += dS[a * dv + j] * u[j];
            g2 += St[a * dv + j] * du[j];
          }
          dk_out[row * dk + a] = b * g1 - g2;
        }
        /* dS~ = dS - k du^T; then through the decay */
        for (int a = 0; a < dk; ++a) {
          const double al = exp(log_alpha[row * dk + a]);
          double gl = 0.0;
          for (int j = 0; j < dv; ++j) {
            const double g = dS[a * dv + j] - kt[a] * du[j];
            gl += g * St[a * dv + j];
            dS[a * dv + j] = al * g;
          }
          dla[row * dk + a] = gl;
        }
      }
      if (dS0) memcpy(dS0 + ((size_t)n * H + h) * dd, dS, dd * sizeof(double));
      free(states); free(dS); free(St); free(u); free(du);
    }
  }
  return 0;
}
