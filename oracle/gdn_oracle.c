/*
 * Plain fp64 CPU oracle for the gated delta rule decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker the CUDA library is
 * compared against.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark may load it; the library never calls it and
 * shares no code, header or table with it.
 *
 * Sources (page titles as printed or as named by their address):
 *   [P1] "GDN tuning limits on Kunlun XPU" (buru.work), section 二 背景:
 *        a GDN layer runs input projection GEMM -> short conv (kernel size 4)
 *        -> gating -> recurrent update of a 128x128 state per head -> output
 *        projection; the recurrent update is a per-token rank-1 update of the
 *        state together with a decay term.
 *   The step itself (the pages never print it as an equation) is the gated
 *   delta rule, read in the plainest way that fits "rank-1 update + decay":
 *        alpha = exp(g),  beta = sigmoid(b_logit)
 *        S     <- alpha * S                      (decay)
 *        delta  = beta * (v - S^T k)             (prediction on decayed S)
 *        S     <- S + k delta^T                  (rank-1 update)
 *        o      = scale * S^T q                  (read-out on updated S)
 *   with q, k L2-normalised over dk.  S is dk x dv.
 *
 * Everything is computed in double precision, sequentially over b, h, t, in
 * exactly the order above; there is no blocking, fusion or algebraic
 * rewriting.  Compile with -O2 -fno-fast-math -ffp-contract=off.
 *
 * Storage layout shared with the library's ABI (a layout, not arithmetic):
 *   state[slot][h][j][i] = S_ij   (j in [0,dv), i in [0,dk): dk contiguous)
 *   q, k [B][T][Hk][dk];  v, out [B][T][H][dv];  g, beta [B][T][H]
 *   v-head h reads q/k head h / (H/Hk) (contiguous groups).
 *   slot_idx[b] = -1 marks a padding row: out rows are zero, no state touched.
 *
 * Pins (tests/test_oracle_pins.py): identity (alpha=1, beta=0), projection
 * (beta=1, unit k => S^T k = v), decay-only closed form, the unrolled product
 * form on tiny sizes, a hand-derived worked example (tests/golden), conv and
 * gate special cases, RMSNorm of constant vectors.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_SLOT_RANGE 2

/* ---- scalar functions ------------------------------------------------- */

/* logistic sigmoid, beta = sigmoid(b_logit) */
double oracle_sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* softplus(x) = log(1 + e^x), written in the overflow-free identity
 * softplus(x) = x + log1p(e^-x) for x > 0. */
double oracle_softplus(double x) {
  if (x > 0.0) return x + log1p(exp(-x));
  return log1p(exp(x));
}

/* SiLU(x) = x * sigmoid(x) */
double oracle_silu(double x) { return x * oracle_sigmoid(x); }

/* gate of the fused front: g = -exp(A_log) * softplus(a + dt_bias) */
double oracle_gate_g(double a, double A_log, double dt_bias) {
  return -exp(A_log) * oracle_softplus(a + dt_bias);
}

/* ---- storage rounding --------------------------------------------------- */

/* Round x to the nearest value of a binary floating-point format with p
 * significand bits (the leading one included) and smallest normal 2^emin,
 * ties to even; magnitudes above maxv become infinite.  A normal value in
 * [2^E, 2^(E+1)) has spacing 2^(E-p+1); below 2^emin the spacing stays
 * 2^(emin-p+1) (subnormals).  rint() rounds half to even in the default
 * rounding mode. */
double oracle_round_to(double x, int p, int emin, double maxv) {
  if (x == 0.0 || !isfinite(x)) return x;
  int e;
  (void)frexp(x, &e); /* |x| in [2^(e-1), 2^e) */
  int E = e - 1;
  if (E < emin) E = emin;
  const int u = E - p + 1; /* exponent of one unit in the last place */
  const double r = ldexp(rint(ldexp(x, -u)), u);
  if (fabs(r) > maxv) return copysign(INFINITY, x);
  return r;
}

/* Storage kinds of the state pool: 0 none (keep fp64), 1 fp32, 2 bf16,
 * 3 fp16 (IEEE binary16). */
double oracle_round_storage(double x, int kind) {
  switch (kind) {
    case 1: return oracle_round_to(x, 24, -126, 3.4028234663852886e38);
    case 2: return oracle_round_to(x, 8, -126, 3.3895313892515355e38);
    case 3: return oracle_round_to(x, 11, -14, 65504.0);
    default: return x;
  }
}

/* ---- vector functions ------------------------------------------------- */

/* y = x / sqrt(sum x^2 + eps) over n elements (y may alias x) */
void oracle_l2norm(const double* x, int n, double eps, double* y) {
  double ss = 0.0;
  for (int i = 0; i < n; ++i) ss += x[i] * x[i];
  double inv = 1.0 / sqrt(ss + eps);
  for (int i = 0; i < n; ++i) y[i] = x[i] * inv;
}

/* One channel of the causal depthwise conv of kernel size 4 ([P1] 二 背景):
 * the window is the three previous inputs, oldest first, then the new x.
 * w[0] multiplies the oldest input, w[3] the new one.  No bias. */
double oracle_conv4(const double* cs, double x, const double* w) {
  return w[0] * cs[0] + w[1] * cs[1] + w[2] * cs[2] + w[3] * x;
}

/* Gated RMSNorm over dv: y_j = o_j / sqrt(mean(o^2) + eps) * w_j * silu(z_j) */
void oracle_gated_rmsnorm(const double* o, const double* z, const double* w,
                          int dv, double eps, double* y) {
  double ss = 0.0;
  for (int j = 0; j < dv; ++j) ss += o[j] * o[j];
  double inv = 1.0 / sqrt(ss / (double)dv + eps);
  for (int j = 0; j < dv; ++j) y[j] = o[j] * inv * w[j] * oracle_silu(z[j]);
}

/* ---- the recurrence --------------------------------------------------- */

/* One token of the gated delta rule on one head, in the definition's order.
 * S is one head's state in storage layout S[j*dk + i] = S_ij.
 * q, k must already be normalised (or not, if the caller so chooses). */
void oracle_gdn_token(double* S, int dk, int dv, const double* q,
                      const double* k, const double* v, double alpha,
                      double beta, double scale, double* o) {
  /* decay: S <- alpha * S */
  for (int j = 0; j < dv; ++j)
    for (int i = 0; i < dk; ++i) S[(size_t)j * dk + i] *= alpha;
  /* prediction p = S^T k and delta = beta (v - p), per column j */
  double* delta = (double*)malloc(sizeof(double) * (size_t)dv);
  for (int j = 0; j < dv; ++j) {
    double p = 0.0;
    for (int i = 0; i < dk; ++i) p += S[(size_t)j * dk + i] * k[i];
    delta[j] = beta * (v[j] - p);
  }
  /* rank-1 update: S <- S + k delta^T */
  for (int j = 0; j < dv; ++j)
    for (int i = 0; i < dk; ++i) S[(size_t)j * dk + i] += k[i] * delta[j];
  /* read-out on the updated state: o = scale * S^T q */
  for (int j = 0; j < dv; ++j) {
    double acc = 0.0;
    for (int i = 0; i < dk; ++i) acc += S[(size_t)j * dk + i] * q[i];
    o[j] = scale * acc;
  }
  free(delta);
}

/* The batched decode step over T tokens per sequence.  After the T tokens
 * of a (sequence, head) the state is rounded once to the pool's storage
 * kind (oracle_round_storage; 0 keeps fp64).
 * Returns ORACLE_OK, or ORACLE_SLOT_RANGE if some slot was outside
 * [-1, n_slots) (such rows are treated as padding), or ORACLE_BAD_ARG. */
int oracle_decode_step(const double* q, const double* k, const double* v,
                       const double* g, const double* beta, double* state,
                       const int32_t* slot_idx, double* out, int B, int T,
                       int Hk, int H, int dk, int dv, int n_slots,
                       double scale, int qk_l2norm, double eps,
                       int state_round) {
  if (B < 0 || T < 1 || Hk < 1 || H < 1 || dk < 1 || dv < 1 || H % Hk != 0)
    return ORACLE_BAD_ARG;
  int rc = ORACLE_OK;
  int group = H / Hk;
  double* qn = (double*)malloc(sizeof(double) * (size_t)dk);
  double* kn = (double*)malloc(sizeof(double) * (size_t)dk);
  for (int b = 0; b < B; ++b) {
    int s = slot_idx[b];
    if (s < 0 || s >= n_slots) {
      if (s != -1) rc = ORACLE_SLOT_RANGE;
      for (int t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h)
          for (int j = 0; j < dv; ++j)
            out[(((size_t)b * T + t) * H + h) * dv + j] = 0.0;
      continue;
    }
    for (int h = 0; h < H; ++h) {
      int kh = h / group;
      double* S = state + ((size_t)s * H + h) * (size_t)dv * dk;
      for (int t = 0; t < T; ++t) {
        const double* qt = q + (((size_t)b * T + t) * Hk + kh) * dk;
        const double* kt = k + (((size_t)b * T + t) * Hk + kh) * dk;
        const double* vt = v + (((size_t)b * T + t) * H + h) * dv;
        size_t gi = ((size_t)b * T + t) * H + h;
        if (qk_l2norm) {
          oracle_l2norm(qt, dk, eps, qn);
          oracle_l2norm(kt, dk, eps, kn);
        } else {
          memcpy(qn, qt, sizeof(double) * (size_t)dk);
          memcpy(kn, kt, sizeof(double) * (size_t)dk);
        }
        double alpha = exp(g[gi]);
        oracle_gdn_token(S, dk, dv, qn, kn, vt, alpha, beta[gi], scale,
                         out + (((size_t)b * T + t) * H + h) * dv);
      }
      for (size_t e = 0; e < (size_t)dv * dk; ++e)
        S[e] = oracle_round_storage(S[e], state_round);
    }
  }
  free(qn);
  free(kn);
  return rc;
}

/* The decode step with speculative-decoding state handling.  Each
 * (sequence, head) starts from pool slot slot_idx[b] and applies its T
 * tokens in order to a working copy; every output is produced as in
 * oracle_decode_step.  Where the state goes:
 *   token_slots != NULL ([B][T]): after token t the working state is
 *       stored (rounded to the storage kind) in pool slot token_slots[b][t]
 *       when that entry is >= 0; slot_idx[b] itself is not written;
 *   n_accept != NULL ([B]): after token n_accept[b]-1 the working state is
 *       stored in slot_idx[b]; n_accept[b] == 0 stores nothing; a value
 *       outside [0, T] stores nothing and is reported;
 *   neither: after the last token, as in oracle_decode_step.
 * Returns ORACLE_OK, ORACLE_SLOT_RANGE (a slot outside its range: the row
 * is padding / the snapshot is skipped), ORACLE_ACCEPT_RANGE, or
 * ORACLE_BAD_ARG (both modes at once). */
#define ORACLE_ACCEPT_RANGE 4
int oracle_decode_step_spec(const double* q, const double* k, const double* v,
                            const double* g, const double* beta, double* state,
                            const int32_t* slot_idx, const int32_t* n_accept,
                            const int32_t* token_slots, double* out, int B, int T,
                            int Hk, int H, int dk, int dv, int n_slots, double scale,
                            int qk_l2norm, double eps, int state_round) {
  if (B < 0 || T < 1 || Hk < 1 || H < 1 || dk < 1 || dv < 1 || H % Hk != 0)
    return ORACLE_BAD_ARG;
  if (n_accept != NULL && token_slots != NULL) return ORACLE_BAD_ARG;
  int rc = ORACLE_OK;
  const int group = H / Hk;
  const size_t hsz = (size_t)dv * dk;
  double* work = (double*)malloc(sizeof(double) * hsz);
  double* qn = (double*)malloc(sizeof(double) * (size_t)dk);
  double* kn = (double*)malloc(sizeof(double) * (size_t)dk);
  for (int b = 0; b < B; ++b) {
    const int s = slot_idx[b];
    if (s < 0 || s >= n_slots) {
      if (s != -1) rc |= ORACLE_SLOT_RANGE;
      for (size_t e = 0; e < (size_t)T * H * dv; ++e) out[(size_t)b * T * H * dv + e] = 0.0;
      continue;
    }
    int na = T;
    if (n_accept != NULL) {
      na = n_accept[b];
      if (na < 0 || na > T) {
        rc |= ORACLE_ACCEPT_RANGE;
        na = 0;
      }
    }
    for (int h = 0; h < H; ++h) {
      const int kh = h / group;
      memcpy(work, state + ((size_t)s * H + h) * hsz, sizeof(double) * hsz);
      for (int t = 0; t < T; ++t) {
        const double* qt = q + (((size_t)b * T + t) * Hk + kh) * dk;
        const double* kt = k + (((size_t)b * T + t) * Hk + kh) * dk;
        const double* vt = v + (((size_t)b * T + t) * H + h) * dv;
        const size_t gi = ((size_t)b * T + t) * H + h;
        if (qk_l2norm) {
          oracle_l2norm(qt, dk, eps, qn);
          oracle_l2norm(kt, dk, eps, kn);
        } else {
          memcpy(qn, qt, sizeof(double) * (size_t)dk);
          memcpy(kn, kt, sizeof(double) * (size_t)dk);
        }
        oracle_gdn_token(work, dk, dv, qn, kn, vt, exp(g[gi]), beta[gi], scale,
                         out + (((size_t)b * T + t) * H + h) * dv);
        int dst = -1;
        if (token_slots != NULL) {
          const int ts = token_slots[(size_t)b * T + t];
          if (ts >= n_slots || ts < -1) rc |= ORACLE_SLOT_RANGE;
          else dst = ts;
        } else if (n_accept != NULL) {
          if (t + 1 == na) dst = s;
        } else if (t + 1 == T) {
          dst = s;
        }
        if (dst >= 0) {
          double* d = state + ((size_t)dst * H + h) * hsz;
          for (size_t e = 0; e < hsz; ++e) d[e] = oracle_round_storage(work[e], state_round);
        }
      }
    }
  }
  free(work);
  free(qn);
  free(kn);
  return rc;
}

/* Prefill: the same recurrence over whole prompts.  N sequences are packed
 * along the token axis; sequence n owns tokens [cu_seqlens[n],
 * cu_seqlens[n+1]).  Each (sequence, head) starts from pool slot
 * slot_idx[n] (or from zeros when initial_state == 0), applies its tokens in
 * order exactly as the decode step does, and stores the final state back in
 * that slot (rounded to the storage kind).  slot_idx[n] == -1 skips the
 * sequence (outputs zero).  Layouts: q, k [total][Hk][dk]; v, out
 * [total][H][dv]; g, beta [total][H]. */
int oracle_prefill(const double* q, const double* k, const double* v,
                   const double* g, const double* beta, double* state,
                   const int32_t* slot_idx, const int32_t* cu_seqlens, double* out,
                   int N, int Hk, int H, int dk, int dv, int n_slots, double scale,
                   int qk_l2norm, double eps, int initial_state, int state_round) {
  if (N < 0 || Hk < 1 || H < 1 || dk < 1 || dv < 1 || H % Hk != 0) return ORACLE_BAD_ARG;
  int rc = ORACLE_OK;
  const int group = H / Hk;
  const size_t hsz = (size_t)dv * dk;
  double* work = (double*)malloc(sizeof(double) * hsz);
  double* qn = (double*)malloc(sizeof(double) * (size_t)dk);
  double* kn = (double*)malloc(sizeof(double) * (size_t)dk);
  for (int n = 0; n < N; ++n) {
    const int s = slot_idx[n];
    const int t0 = cu_seqlens[n], t1 = cu_seqlens[n + 1];
    if (t1 < t0) return ORACLE_BAD_ARG;
    if (s < 0 || s >= n_slots) {
      if (s != -1) rc |= ORACLE_SLOT_RANGE;
      for (size_t e = (size_t)t0 * H * dv; e < (size_t)t1 * H * dv; ++e) out[e] = 0.0;
      continue;
    }
    for (int h = 0; h < H; ++h) {
      const int kh = h / group;
      double* S = state + ((size_t)s * H + h) * hsz;
      if (initial_state) memcpy(work, S, sizeof(double) * hsz);
      else memset(work, 0, sizeof(double) * hsz);
      for (int t = t0; t < t1; ++t) {
        const double* qt = q + ((size_t)t * Hk + kh) * dk;
        const double* kt = k + ((size_t)t * Hk + kh) * dk;
        if (qk_l2norm) {
          oracle_l2norm(qt, dk, eps, qn);
          oracle_l2norm(kt, dk, eps, kn);
        } else {
          memcpy(qn, qt, sizeof(double) * (size_t)dk);
          memcpy(kn, kt, sizeof(double) * (size_t)dk);
        }
        const size_t gi = (size_t)t * H + h;
        oracle_gdn_token(work, dk, dv, qn, kn, v + gi * dv, exp(g[gi]), beta[gi], scale,
                         out + gi * dv);
      }
      for (size_t e = 0; e < hsz; ++e) S[e] = oracle_round_storage(work[e], state_round);
    }
  }
  free(work);
  free(qn);
  free(kn);
  return rc;
}

/* One token of the low-rank window of one head (definition below): K [r][dk],
 * U [r][dv], c [r] and *count are the head's window; qn, kn the token's
 * (normalised) q and k, vt its v; p is scratch of dv doubles; o receives the
 * dv outputs. */
void oracle_lowrank_token(double* K, double* U, double* c, int32_t* count, const double* qn,
                          const double* kn, const double* vt, double alpha, double bb, int dk,
                          int dv, int R, double scale, double* p, double* o) {
  const int filled = *count < R ? *count : R;
  /* decay */
  for (int j = 0; j < filled; ++j) c[j] *= alpha;
  /* prediction over the current window */
  for (int i = 0; i < dv; ++i) p[i] = 0.0;
  for (int j = 0; j < filled; ++j) {
    double d = 0.0;
    for (int i = 0; i < dk; ++i) d += K[(size_t)j * dk + i] * kn[i];
    for (int i = 0; i < dv; ++i) p[i] += c[j] * d * U[(size_t)j * dv + i];
  }
  /* the new update replaces ring position count % R */
  const int slot_e = *count % R;
  for (int i = 0; i < dv; ++i) U[(size_t)slot_e * dv + i] = bb * (vt[i] - p[i]);
  for (int i = 0; i < dk; ++i) K[(size_t)slot_e * dk + i] = kn[i];
  c[slot_e] = 1.0;
  *count += 1;
  /* read-out over the new window */
  const int filled2 = *count < R ? *count : R;
  for (int i = 0; i < dv; ++i) o[i] = 0.0;
  for (int j = 0; j < filled2; ++j) {
    double d = 0.0;
    for (int i = 0; i < dk; ++i) d += K[(size_t)j * dk + i] * qn[i];
    for (int i = 0; i < dv; ++i) o[i] += c[j] * d * U[(size_t)j * dv + i];
  }
  for (int i = 0; i < dv; ++i) o[i] *= scale;
}

/* Low-rank sliding-window decode ("GDN tuning limits on Kunlun XPU",
 * section 三.3: the low-rank "UV state" is a cache of the most recent r
 * rank-1 updates, not a matrix factorisation).  Reading taken for the decay,
 * which the page leaves open: every cached update keeps the decay
 * accumulated since it was made, so the state the window stands for is
 *     S = sum_{j in window} c_j k_j u_j^T,   c_j = product of alpha since j.
 * Per token (q, k normalised as in the full-rank step):
 *     c_j <- alpha c_j                       (decay)
 *     p = S^T k = sum_j c_j (k_j . k) u_j    (prediction)
 *     delta = beta (v - p)
 *     push (k, delta) with c = 1; a full window (r entries) first drops its
 *     oldest entry
 *     o = scale S^T q over the new window.
 * Storage (per slot and head): win_k [r][dk], win_u [r][dv], win_c [r] and
 * the number of updates made so far, win_count; the update made as number
 * n (0-based) lives in ring position n % r.  Rows of padding sequences
 * (slot -1) are zero; T tokens per sequence are applied in order. */
int oracle_lowrank_decode_step(const double* q, const double* k, const double* v,
                               const double* g, const double* beta, double* win_k,
                               double* win_u, double* win_c, int32_t* win_count,
                               const int32_t* slot_idx, double* out, int B, int T, int Hk,
                               int H, int dk, int dv, int R, int n_slots, double scale,
                               int qk_l2norm, double eps) {
  if (B < 0 || T < 1 || Hk < 1 || H < 1 || dk < 1 || dv < 1 || R < 1 || H % Hk != 0)
    return ORACLE_BAD_ARG;
  int rc = ORACLE_OK;
  const int group = H / Hk;
  double* qn = (double*)malloc(sizeof(double) * (size_t)dk);
  double* kn = (double*)malloc(sizeof(double) * (size_t)dk);
  double* p = (double*)malloc(sizeof(double) * (size_t)dv);
  for (int b = 0; b < B; ++b) {
    const int s = slot_idx[b];
    if (s < 0 || s >= n_slots) {
      if (s != -1) rc |= ORACLE_SLOT_RANGE;
      for (size_t e = 0; e < (size_t)T * H * dv; ++e) out[(size_t)b * T * H * dv + e] = 0.0;
      continue;
    }
    for (int h = 0; h < H; ++h) {
      const int kh = h / group;
      const size_t sh = (size_t)s * H + h;
      for (int t = 0; t < T; ++t) {
        const size_t bt = (size_t)b * T + t;
        const double* qt = q + (bt * Hk + kh) * dk;
        const double* kt = k + (bt * Hk + kh) * dk;
        const double* vt = v + (bt * H + h) * dv;
        if (qk_l2norm) {
          oracle_l2norm(qt, dk, eps, qn);
          oracle_l2norm(kt, dk, eps, kn);
        } else {
          memcpy(qn, qt, sizeof(double) * (size_t)dk);
          memcpy(kn, kt, sizeof(double) * (size_t)dk);
        }
        oracle_lowrank_token(win_k + sh * R * dk, win_u + sh * R * dv, win_c + sh * R,
                             win_count + sh, qn, kn, vt, exp(g[bt * H + h]), beta[bt * H + h],
                             dk, dv, R, scale, p, out + (bt * H + h) * dv);
      }
    }
  }
  free(qn);
  free(kn);
  free(p);
  return rc;
}

/* The low-rank window over whole prompts: the low-rank prefill ("GDN tuning
 * limits on Kunlun XPU", section 三.3, runs the low-rank chain over a prompt
 * in chunks; its result is defined by the per-token window above).  N
 * sequences are packed along the token axis, sequence n owning tokens
 * [cu_seqlens[n], cu_seqlens[n+1]); the window of (slot_idx[n], h) takes
 * the sequence's tokens one at a time in order (oracle_lowrank_token), from
 * the window stored in the slot (initial_window = 1) or from an empty one
 * (0: count 0).  Layouts as in oracle_prefill: q, k [total][Hk][dk];
 * v, out [total][H][dv]; g, beta [total][H].  Rows of padding sequences
 * (slot -1) are zero and touch no window. */
int oracle_lowrank_prefill(const double* q, const double* k, const double* v,
                           const double* g, const double* beta, double* win_k, double* win_u,
                           double* win_c, int32_t* win_count, const int32_t* slot_idx,
                           const int32_t* cu_seqlens, double* out, int N, int Hk, int H, int dk,
                           int dv, int R, int n_slots, double scale, int qk_l2norm, double eps,
                           int initial_window) {
  if (N < 0 || Hk < 1 || H < 1 || dk < 1 || dv < 1 || R < 1 || H % Hk != 0)
    return ORACLE_BAD_ARG;
  int rc = ORACLE_OK;
  const int group = H / Hk;
  double* qn = (double*)malloc(sizeof(double) * (size_t)dk);
  double* kn = (double*)malloc(sizeof(double) * (size_t)dk);
  double* p = (double*)malloc(sizeof(double) * (size_t)dv);
  for (int n = 0; n < N; ++n) {
    const int s = slot_idx[n];
    const int t0 = cu_seqlens[n], t1 = cu_seqlens[n + 1];
    if (t1 < t0) {
      rc = ORACLE_BAD_ARG;
      break;
    }
    if (s < 0 || s >= n_slots) {
      if (s != -1) rc |= ORACLE_SLOT_RANGE;
      for (size_t e = (size_t)t0 * H * dv; e < (size_t)t1 * H * dv; ++e) out[e] = 0.0;
      continue;
    }
    for (int h = 0; h < H; ++h) {
      const int kh = h / group;
      const size_t sh = (size_t)s * H + h;
      if (!initial_window) win_count[sh] = 0;
      for (int t = t0; t < t1; ++t) {
        const double* qt = q + ((size_t)t * Hk + kh) * dk;
        const double* kt = k + ((size_t)t * Hk + kh) * dk;
        if (qk_l2norm) {
          oracle_l2norm(qt, dk, eps, qn);
          oracle_l2norm(kt, dk, eps, kn);
        } else {
          memcpy(qn, qt, sizeof(double) * (size_t)dk);
          memcpy(kn, kt, sizeof(double) * (size_t)dk);
        }
        const size_t gi = (size_t)t * H + h;
        oracle_lowrank_token(win_k + sh * R * dk, win_u + sh * R * dv, win_c + sh * R,
                             win_count + sh, qn, kn, v + gi * dv, exp(g[gi]), beta[gi], dk, dv,
                             R, scale, p, out + gi * dv);
      }
    }
  }
  free(qn);
  free(kn);
  free(p);
  return rc;
}

/* The fused decode step (T = 1): conv k=4 + SiLU over the mixed projection
 * row [q (Hk*dk) | k (Hk*dk) | v (H*dv)], conv-state shift, L2-norm of q/k,
 * gates g = -exp(A_log) softplus(a + dt_bias), beta = sigmoid(b), the
 * recurrence, and the gated RMSNorm o' = RMSNorm(o) * w * silu(z).
 *   mixed_x [B][C]; conv_state [n_slots][C][3] (oldest first);
 *   conv_w [C][4]; a, b [B][H]; A_log, dt_bias [H]; z [B][H*dv];
 *   norm_w [dv]; state as above; out [B][H][dv].
 * Padding rows (slot -1) zero their out rows and touch no state. */
int oracle_fused_step(const double* mixed_x, double* conv_state,
                      const double* conv_w, const double* a,
                      const double* b_logit, const double* A_log,
                      const double* dt_bias, const double* z,
                      const double* norm_w, double norm_eps, double* state,
                      const int32_t* slot_idx, double* out, int B, int Hk,
                      int H, int dk, int dv, int n_slots, double scale,
                      double l2_eps) {
  if (B < 0 || Hk < 1 || H < 1 || dk < 1 || dv < 1 || H % Hk != 0)
    return ORACLE_BAD_ARG;
  int rc = ORACLE_OK;
  int group = H / Hk;
  size_t C = (size_t)2 * Hk * dk + (size_t)H * dv;
  double* xc = (double*)malloc(sizeof(double) * C);
  double* qn = (double*)malloc(sizeof(double) * (size_t)dk);
  double* kn = (double*)malloc(sizeof(double) * (size_t)dk);
  double* o = (double*)malloc(sizeof(double) * (size_t)dv);
  for (int b = 0; b < B; ++b) {
    int s = slot_idx[b];
    if (s < 0 || s >= n_slots) {
      if (s != -1) rc = ORACLE_SLOT_RANGE;
      for (int h = 0; h < H; ++h)
        for (int j = 0; j < dv; ++j) out[((size_t)b * H + h) * dv + j] = 0.0;
      continue;
    }
    /* short conv + SiLU over every channel, then shift the conv state */
    for (size_t c = 0; c < C; ++c) {
      double* cs = conv_state + ((size_t)s * C + c) * 3;
      double x = mixed_x[(size_t)b * C + c];
      xc[c] = oracle_silu(oracle_conv4(cs, x, conv_w + c * 4));
      cs[0] = cs[1];
      cs[1] = cs[2];
      cs[2] = x;
    }
    for (int h = 0; h < H; ++h) {
      int kh = h / group;
      oracle_l2norm(xc + (size_t)kh * dk, dk, l2_eps, qn);
      oracle_l2norm(xc + (size_t)Hk * dk + (size_t)kh * dk, dk, l2_eps, kn);
      const double* vh = xc + (size_t)2 * Hk * dk + (size_t)h * dv;
      size_t bh = (size_t)b * H + h;
      double g = oracle_gate_g(a[bh], A_log[h], dt_bias[h]);
      double beta = oracle_sigmoid(b_logit[bh]);
      double* S = state + ((size_t)s * H + h) * (size_t)dv * dk;
      oracle_gdn_token(S, dk, dv, qn, kn, vh, exp(g), beta, scale, o);
      oracle_gated_rmsnorm(o, z + bh * dv, norm_w, dv, norm_eps,
                           out + bh * dv);
    }
  }
  free(xc);
  free(qn);
  free(kn);
  free(o);
  return rc;
}
