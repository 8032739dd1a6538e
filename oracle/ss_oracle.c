/*
 * ss_oracle.c -- plain, slow, sequential fp64 oracle for the selective scan (S6).
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  The
 * product path (selective_state_space_11_b200 + libss.so) never calls it, and
 * this file shares no code, header, table or helper with the CUDA path.
 *
 * What it computes, and where the pages define it:
 *   "Mamba" (stanleyjacob.dev/oss/mamba), Part IV Stage 3: Delta is a softplus
 *     of a per-channel projection; A = -exp(A_log) is stored by the caller.
 *   same page, Part IV Stage 4: zero-order hold for A, Abar = exp(Delta*A)
 *     elementwise; B discretised by the simplified (Euler) rule Bbar = Delta*B;
 *     h_t = Abar_t * h_{t-1} + Bbar_t * x_t, readout y_t = C_t * h_t.
 *   same page, Part IV Stage 5: selective_scan_fn(u, delta, A, B, C, D, z,
 *     delta_bias, delta_softplus) shapes: u, delta, z (B, D, L); A (D, N);
 *     B, C (B, N, L); D (D,).
 *   same page, Part IV Stage 6: skip then gate, y = (y + D*u) * SiLU(z).
 *   same page, Part V "the hardware-aware scan kernel": the per-thread sketch
 *     adds delta_bias inside the softplus and reads out with the state AFTER
 *     the step's update.
 *   same page, Part IV Stage 7: backward recomputes the states and yields
 *     gradients for u, Delta, A, B, C, D and z; decode applies one recurrence
 *     step to a cached state in place.
 *   "Mamba, on a laptop GPU." (anamaya.fyi), section "The state lives in
 *     registers": a checkpoint of the state every 64 steps.
 *   "mamba-metal" README, "Long-context prompts (parallel prefill)": the scan
 *     writes the final state, and decode continues from it.
 *   niverel-mamba README, "seq_idx strict reset": with packed documents, at
 *     every change of seq_idx both the convolution state and the SSM state
 *     restart from zero, so a packed run equals the documents run one by one.
 *   "Mamba", Part V "Deep dive: Mamba-2 and state-space duality": SSD keeps
 *     one scalar A per head (A times the identity), a state of N ~ 64..128
 *     per channel, multi-head with B and C shared by groups of heads; the
 *     same operation as a recurrence or as a masked quadratic form.  Its
 *     backward (oracle_ssd_bwd) is the adjoint of that recurrence, as in
 *     Part IV Stage 7 for S6.
 *   "Mamba", Part IV Stage 2: before the scan, a depthwise causal 1-D
 *     convolution of width d_conv (4) and a SiLU; position t sees t-3 .. t.
 *     Part II and Part IV Stage 7: decoding keeps the small convolution window
 *     and advances it one token at a time.
 *
 * Readings where the pages are silent (the plainest reading in each case):
 *   - initial state h_{-1} = 0 unless h0 is given (the kernel sketch zeroes it);
 *   - softplus is the exact log(1 + e^x), written in a cancellation-free form;
 *   - with delta_softplus = 0, Delta = delta + bias (the bias is still added);
 *   - checkpoint k holds the state after the last step of chunk k (steps
 *     64k .. 64k+63); the last checkpoint of a ragged L is the final state;
 *   - the loss is <dy, y>; the final state carries no incoming gradient.
 *
 * Every array is dense, row-major, float64.  Nullable arguments are marked.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* softplus(x) = log(1 + exp(x)) -- "Mamba" Part IV Stage 3 (Delta through a
 * softplus).  Written as max(x,0) + log1p(exp(-|x|)), which is the same real
 * number without overflow or cancellation. */
static double sp(double x) { return (x > 0 ? x : 0.0) + log1p(exp(-fabs(x))); }

/* logistic sigmoid; d softplus / dx = sigmoid(x), and SiLU(z) = z*sigmoid(z). */
static double sg(double x) {
  if (x >= 0) return 1.0 / (1.0 + exp(-x));
  double e = exp(x);
  return e / (1.0 + e);
}

static double at(const double* p, size_t i, double dflt) { return p ? p[i] : dflt; }

/* seq_idx (Bsz, L) or NULL: the state restarts before step t when the id
 * changes between t-1 and t (t = 0 keeps the given initial state). */
static int reset_before(const int32_t* seq_idx, int64_t b, int64_t L, int64_t t) {
  return seq_idx && t > 0 && seq_idx[b * L + t] != seq_idx[b * L + t - 1];
}

/*
 * Forward scan ("Mamba" Part IV Stages 4-6; Part V kernel sketch).
 *   u, delta, z: (Bsz, D, L); A: (D, N); Bm, Cm: (Bsz, N, L); Dskip, bias: (D,)
 *   h0: (Bsz, D, N) or NULL (zero initial state)
 *   y: (Bsz, D, L) out; final_state: (Bsz, D, N) out or NULL;
 *   ckpt: (Bsz, D, ceil(L/chunk), N) out or NULL.
 */
void oracle_ss_fwd(int64_t Bsz, int64_t D, int64_t N, int64_t L,
                   const double* u, const double* delta, const double* z,
                   const double* A, const double* Bm, const double* Cm,
                   const double* Dskip, const double* bias, int softplus,
                   const double* h0, const int32_t* seq_idx, double* y,
                   double* final_state, double* ckpt, int64_t chunk) {
  double* h = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
  int64_t nchunk = chunk > 0 ? (L + chunk - 1) / chunk : 0;
  for (int64_t b = 0; b < Bsz; ++b) {
    for (int64_t d = 0; d < D; ++d) {
      size_t row = (size_t)(b * D + d);
      for (int64_t n = 0; n < N; ++n) h[n] = h0 ? h0[row * N + n] : 0.0;
      for (int64_t t = 0; t < L; ++t) {
        if (reset_before(seq_idx, b, L, t))
          for (int64_t n = 0; n < N; ++n) h[n] = 0.0;  /* a new document */
        size_t i = row * (size_t)L + (size_t)t;
        double x = delta[i] + at(bias, (size_t)d, 0.0);
        double dt = softplus ? sp(x) : x;
        double ys = 0.0;
        for (int64_t n = 0; n < N; ++n) {
          size_t bi = ((size_t)b * N + n) * (size_t)L + (size_t)t;
          double abar = exp(dt * A[d * N + n]);          /* ZOH for A      */
          h[n] = abar * h[n] + dt * Bm[bi] * u[i];        /* Euler for B    */
          ys += Cm[bi] * h[n];                            /* readout, h_t   */
        }
        double out = ys + at(Dskip, (size_t)d, 0.0) * u[i]; /* D skip       */
        y[i] = z ? out * z[i] * sg(z[i]) : out;            /* SiLU(z) gate */
        if (ckpt && (t % chunk == chunk - 1 || t == L - 1)) {
          double* c = ckpt + (row * (size_t)nchunk + (size_t)(t / chunk)) * (size_t)N;
          for (int64_t n = 0; n < N; ++n) c[n] = h[n];
        }
      }
      if (final_state)
        for (int64_t n = 0; n < N; ++n) final_state[row * N + n] = h[n];
    }
  }
  free(h);
}

/*
 * Backward: the adjoint of oracle_ss_fwd for the loss <dy, y> ("Mamba" Part IV
 * Stage 7: recompute the states, then accumulate gradients for u, Delta, A, B,
 * C, D, z).  States are recomputed in full per (b, d) -- no checkpointing, no
 * chunking.  With g_t = dloss/dh_t:
 *   g_t     = Abar_{t+1} g_{t+1} + dout_t C_t,      dout_t = dy_t SiLU(z_t)
 *   dC_t   += dout_t h_t          dB_t += g_t Delta_t u_t
 *   du_t    = dout_t D + Delta_t sum_n g_t B_t
 *   dDelta  = u_t sum_n g_t B_t + sum_n g_t A Abar_t h_{t-1}
 *   dA     += g_t Delta_t Abar_t h_{t-1}
 *   ddelta  = dDelta * sigmoid(delta + bias) (softplus on), else dDelta
 *   dz      = dy (C h + D u) SiLU'(z),  dD += dout u,  dbias = sum ddelta
 * dB, dC, dA, dD, dbias are overwritten (not accumulated into).
 * z == NULL: no gate (dz not written).  dD, dbias, dz, dh0 may be NULL.
 * h0 as in the forward; dh0 (Bsz, D, N) receives dloss/dh0 when non-NULL.
 * dfinal (Bsz, D, N) or NULL: the gradient arriving at the final state
 * h_{L-1} from whatever consumes it (the next piece of a split sequence);
 * the loss is then <dy, y> + <dfinal, h_{L-1}>, so g_{L-1} gains dfinal.
 * seq_idx as in the forward: a restart before step t makes Abar_t zero, so
 * neither the carry nor the A and Delta terms cross a document boundary.
 */
void oracle_ss_bwd(int64_t Bsz, int64_t D, int64_t N, int64_t L,
                   const double* u, const double* delta, const double* z,
                   const double* A, const double* Bm, const double* Cm,
                   const double* Dskip, const double* bias, int softplus,
                   const double* h0, const int32_t* seq_idx, const double* dy,
                   const double* dfinal, double* du, double* ddelta, double* dz, double* dA, double* dB,
                   double* dC, double* dD, double* dbias, double* dh0) {
  size_t LN = (size_t)(L + 1) * (size_t)N;
  double* H = (double*)malloc(sizeof(double) * (LN > 0 ? LN : 1));   /* h_{t-1}, t=0..L */
  double* Ab = (double*)malloc(sizeof(double) * ((size_t)L * N + 1)); /* Abar_t          */
  double* g = (double*)malloc(sizeof(double) * (size_t)(N + 1));
  memset(dA, 0, sizeof(double) * (size_t)(D * N));
  memset(dB, 0, sizeof(double) * (size_t)(Bsz * N * L));
  memset(dC, 0, sizeof(double) * (size_t)(Bsz * N * L));
  if (dD) memset(dD, 0, sizeof(double) * (size_t)D);
  if (dbias) memset(dbias, 0, sizeof(double) * (size_t)D);
  for (int64_t b = 0; b < Bsz; ++b) {
    for (int64_t d = 0; d < D; ++d) {
      size_t row = (size_t)(b * D + d);
      double Dd = at(Dskip, (size_t)d, 0.0), bd = at(bias, (size_t)d, 0.0);
      /* forward recompute: H[t*N + n] = h_{t-1}[n] */
      for (int64_t n = 0; n < N; ++n) H[n] = h0 ? h0[row * N + n] : 0.0;
      for (int64_t t = 0; t < L; ++t) {
        size_t i = row * (size_t)L + (size_t)t;
        double x = delta[i] + bd;
        double dt = softplus ? sp(x) : x;
        int rst = reset_before(seq_idx, b, L, t); /* h_{t-1} does not reach h_t */
        for (int64_t n = 0; n < N; ++n) {
          size_t bi = ((size_t)b * N + n) * (size_t)L + (size_t)t;
          double a = rst ? 0.0 : exp(dt * A[d * N + n]);
          Ab[(size_t)t * N + n] = a;
          H[(size_t)(t + 1) * N + n] = a * H[(size_t)t * N + n] + dt * Bm[bi] * u[i];
        }
      }
      /* reverse sweep; nothing after step L-1 except what reaches the final state */
      for (int64_t n = 0; n < N; ++n) g[n] = dfinal ? dfinal[row * N + n] : 0.0;
      for (int64_t t = L - 1; t >= 0; --t) {
        size_t i = row * (size_t)L + (size_t)t;
        double x = delta[i] + bd;
        double dt = softplus ? sp(x) : x;
        double gate = 1.0, out = 0.0;
        const double* ht = H + (size_t)(t + 1) * N;  /* h_t     */
        const double* hp = H + (size_t)t * N;        /* h_{t-1} */
        if (z) {
          double ys = 0.0;
          for (int64_t n = 0; n < N; ++n)
            ys += Cm[((size_t)b * N + n) * (size_t)L + (size_t)t] * ht[n];
          out = ys + Dd * u[i];
          double s = sg(z[i]);
          gate = z[i] * s;
          if (dz) dz[i] = dy[i] * out * s * (1.0 + z[i] * (1.0 - s));
        }
        double dout = dy[i] * gate;
        if (dD) dD[d] += dout * u[i];
        double sgb = 0.0, sga = 0.0;
        for (int64_t n = 0; n < N; ++n) {
          size_t bi = ((size_t)b * N + n) * (size_t)L + (size_t)t;
          /* g[n] holds Abar_{t+1} g_{t+1} on entry */
          g[n] += dout * Cm[bi];
          dC[bi] += dout * ht[n];
          dB[bi] += g[n] * dt * u[i];
          sgb += g[n] * Bm[bi];
          double a = Ab[(size_t)t * N + n];
          double q = g[n] * a * hp[n];
          dA[d * N + n] += q * dt;
          sga += q * A[d * N + n];
          g[n] *= a; /* becomes Abar_t g_t for step t-1 */
        }
        du[i] = dout * Dd + dt * sgb;
        double dDelta = u[i] * sgb + sga;
        double dx = softplus ? dDelta * sg(x) : dDelta;
        ddelta[i] = dx;
        if (dbias) dbias[d] += dx;
      }
      if (dh0)
        for (int64_t n = 0; n < N; ++n) dh0[row * N + n] = g[n];
    }
  }
  free(H);
  free(Ab);
  free(g);
}

/*
 * One decode step on a cached state, in place ("Mamba" Part IV Stage 7: one
 * token in, a fixed-size state updated in place, one token out; "mamba-metal"
 * README, "O(1) per token via state caching").  It is exactly one iteration of
 * the forward loop body.
 *   state: (Bsz, D, N) in/out; u, delta, z, y: (Bsz, D); Bm, Cm: (Bsz, N).
 */
void oracle_ss_state_update(int64_t Bsz, int64_t D, int64_t N, double* state,
                            const double* u, const double* delta,
                            const double* z, const double* A,
                            const double* Bm, const double* Cm,
                            const double* Dskip, const double* bias,
                            int softplus, double* y) {
  for (int64_t b = 0; b < Bsz; ++b) {
    for (int64_t d = 0; d < D; ++d) {
      size_t i = (size_t)(b * D + d);
      double x = delta[i] + at(bias, (size_t)d, 0.0);
      double dt = softplus ? sp(x) : x;
      double ys = 0.0;
      for (int64_t n = 0; n < N; ++n) {
        double a = exp(dt * A[d * N + n]);
        double* h = state + i * N + n;
        *h = a * *h + dt * Bm[b * N + n] * u[i];
        ys += Cm[b * N + n] * *h;
      }
      double out = ys + at(Dskip, (size_t)d, 0.0) * u[i];
      y[i] = z ? out * z[i] * sg(z[i]) : out;
    }
  }
}

/*
 * Causal depthwise conv1d + SiLU ("Mamba" Part IV Stage 2).  For each (b, d):
 *   pre_t = bias[d] + sum_{k=0}^{W-1} w[d,k] * xin(t - (W-1) + k)
 *   u_t   = silu ? pre_t * sigmoid(pre_t) : pre_t
 * where xin(s) = x[b,d,s] for s >= 0 and, for s < 0, the incoming window
 * state_in[b,d, W-1+s] (the W-1 inputs before t = 0, oldest first), or 0 when
 * state_in is NULL.  state_out (nullable) receives the last W-1 inputs
 * xin(L-(W-1)) .. xin(L-1), oldest first: the window a continuation (the next
 * piece of the sequence, or decode) starts from.  With seq_idx (Bsz, L) the
 * window restarts from zero at every document start: input s reaches output
 * t only when no document starts in (s, t]; state_out keeps only the last
 * document's inputs.
 * x, u: (Bsz, D, L); w: (D, W); bias (D) or NULL; state_in/out (Bsz, D, W-1).
 */
static double conv_in(const double* x, const double* st, int64_t W, size_t row,
                      int64_t L, int64_t s) {
  if (s >= 0) return x[row * (size_t)L + (size_t)s];
  return st ? st[row * (size_t)(W - 1) + (size_t)(W - 1 + s)] : 0.0;
}

/* input s reaches output t (s <= t) only inside one document: no change of
 * seq_idx in (max(s, 0), t]; the incoming window (s < 0) belongs to the
 * document at t = 0 */
static int same_doc(const int32_t* seq_idx, int64_t b, int64_t L, int64_t s, int64_t t) {
  for (int64_t r = (s > 0 ? s : 0) + 1; r <= t; ++r)
    if (reset_before(seq_idx, b, L, r)) return 0;
  return 1;
}

void oracle_conv1d_fwd(int64_t Bsz, int64_t D, int64_t L, int64_t W,
                       const double* x, const double* w, const double* bias,
                       const double* state_in, const int32_t* seq_idx, int silu,
                       double* u, double* state_out) {
  for (int64_t b = 0; b < Bsz; ++b) {
    for (int64_t d = 0; d < D; ++d) {
      size_t row = (size_t)(b * D + d);
      for (int64_t t = 0; t < L; ++t) {
        double pre = at(bias, (size_t)d, 0.0);
        for (int64_t k = 0; k < W; ++k)
          if (same_doc(seq_idx, b, L, t - (W - 1) + k, t))
            pre += w[d * W + k] * conv_in(x, state_in, W, row, L, t - (W - 1) + k);
        u[row * (size_t)L + (size_t)t] = silu ? pre * sg(pre) : pre;
      }
      if (state_out) /* the window a continuation of the last document sees */
        for (int64_t j = 0; j < W - 1; ++j)
          state_out[row * (size_t)(W - 1) + (size_t)j] =
              same_doc(seq_idx, b, L, L - (W - 1) + j, L - 1)
                  ? conv_in(x, state_in, W, row, L, L - (W - 1) + j) : 0.0;
    }
  }
}

/*
 * Adjoint of oracle_conv1d_fwd for the loss <du, u> + <dstate_out, state_out>.
 *   dpre_t = du_t * (silu ? sigmoid(pre_t) (1 + pre_t (1 - sigmoid(pre_t))) : 1)
 *   d xin(s) = sum_k w[d,k] dpre_{s + (W-1) - k}     (targets inside [0, L))
 *              + dstate_out[s - (L-(W-1))]            (if s is in the out window)
 *   dw[d,k]  = sum_{b,t} dpre_t xin(t - (W-1) + k),   dbias[d] = sum_{b,t} dpre_t
 * dx receives d xin(s) for s >= 0; dstate_in (nullable) for s < 0.
 * dw, dbias are overwritten.  dbias, dstate_out, dstate_in may be NULL.
 */
void oracle_conv1d_bwd(int64_t Bsz, int64_t D, int64_t L, int64_t W,
                       const double* x, const double* w, const double* bias,
                       const double* state_in, const int32_t* seq_idx, int silu,
                       const double* du,
                       const double* dstate_out, double* dx, double* dw,
                       double* dbias, double* dstate_in) {
  double* dp = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
  double* dxin = (double*)malloc(sizeof(double) * (size_t)(L + W));
  memset(dw, 0, sizeof(double) * (size_t)(D * W));
  if (dbias) memset(dbias, 0, sizeof(double) * (size_t)D);
  for (int64_t b = 0; b < Bsz; ++b) {
    for (int64_t d = 0; d < D; ++d) {
      size_t row = (size_t)(b * D + d);
      for (int64_t t = 0; t < L; ++t) {
        double pre = at(bias, (size_t)d, 0.0);
        for (int64_t k = 0; k < W; ++k)
          if (same_doc(seq_idx, b, L, t - (W - 1) + k, t))
            pre += w[d * W + k] * conv_in(x, state_in, W, row, L, t - (W - 1) + k);
        double g = du[row * (size_t)L + (size_t)t];
        if (silu) {
          double s = sg(pre);
          g *= s * (1.0 + pre * (1.0 - s));
        }
        dp[t] = g;
        if (dbias) dbias[d] += g;
        for (int64_t k = 0; k < W; ++k)
          if (same_doc(seq_idx, b, L, t - (W - 1) + k, t))
            dw[d * W + k] += g * conv_in(x, state_in, W, row, L, t - (W - 1) + k);
      }
      /* dxin[s + W - 1] = gradient of xin(s), s = -(W-1) .. L-1 */
      for (int64_t s = -(W - 1); s < L; ++s) {
        double g = 0.0;
        for (int64_t k = 0; k < W; ++k) {
          int64_t t = s + (W - 1) - k;
          if (t >= 0 && t < L && same_doc(seq_idx, b, L, s, t)) g += w[d * W + k] * dp[t];
        }
        int64_t j = s - (L - (W - 1));
        if (dstate_out && j >= 0 && j < W - 1) g += dstate_out[row * (size_t)(W - 1) + (size_t)j];
        dxin[s + W - 1] = g;
      }
      for (int64_t t = 0; t < L; ++t) dx[row * (size_t)L + (size_t)t] = dxin[t + W - 1];
      if (dstate_in)
        for (int64_t j = 0; j < W - 1; ++j)
          dstate_in[row * (size_t)(W - 1) + (size_t)j] = dxin[j];
    }
  }
  free(dp);
  free(dxin);
}

/*
 * One decode step of the convolution ("Mamba" Part IV Stage 7: the step path
 * advances the small convolution window): u_t from the window
 * [state (W-1 oldest-first inputs), x_t], then the window drops its oldest
 * input and appends x_t.  state (Bsz, D, W-1) in/out; x, u (Bsz, D).
 */
void oracle_conv1d_step(int64_t Bsz, int64_t D, int64_t W, double* state,
                        const double* x, const double* w, const double* bias,
                        int silu, double* u) {
  for (int64_t b = 0; b < Bsz; ++b) {
    for (int64_t d = 0; d < D; ++d) {
      size_t i = (size_t)(b * D + d);
      double* st = state + i * (size_t)(W - 1);
      double pre = at(bias, (size_t)d, 0.0);
      for (int64_t k = 0; k < W - 1; ++k) pre += w[d * W + k] * st[k];
      pre += w[d * W + W - 1] * x[i];
      u[i] = silu ? pre * sg(pre) : pre;
      for (int64_t k = 0; k + 1 < W - 1; ++k) st[k] = st[k + 1];
      if (W > 1) st[W - 2] = x[i];
    }
  }
}

/*
 * Mamba-2 SSD forward ("Mamba" Part V, "Mamba-2 and state-space duality"),
 * the plain recurrence.  Per batch b and head h, with scalar A_h and the
 * B, C of the head's group g = h / (nh / ng):
 *   Delta_t = softplus(dt_t + dt_bias_h)   (dt_t + dt_bias_h when softplus = 0)
 *   H_t     = exp(Delta_t A_h) H_{t-1} + Delta_t x_t B_t^T          H: P x N
 *   y_t     = (H_t C_t + D_h x_t) * SiLU(z_t)                       (no gate: z NULL)
 * Time-major layouts as in Mamba-2: x, z, y (Bsz, L, nh, P); dt (Bsz, L, nh);
 * A, D, dt_bias (nh); B, C (Bsz, L, ng, N); h0, final_state (Bsz, nh, P, N).
 * D, z, dt_bias, h0, final_state may be NULL.
 */
void oracle_ssd_fwd(int64_t Bsz, int64_t L, int64_t nh, int64_t P, int64_t ng, int64_t N,
                    const double* x, const double* dt, const double* A, const double* Bm,
                    const double* Cm, const double* Dskip, const double* z,
                    const double* dt_bias, int softplus, const double* h0, double* y,
                    double* final_state) {
  double* H = (double*)malloc(sizeof(double) * (size_t)(P * N > 0 ? P * N : 1));
  int64_t hpg = nh / ng;  /* heads per group */
  for (int64_t b = 0; b < Bsz; ++b) {
    for (int64_t h = 0; h < nh; ++h) {
      int64_t g = h / hpg;
      size_t sidx = ((size_t)b * nh + h) * (size_t)(P * N);
      for (int64_t i = 0; i < P * N; ++i) H[i] = h0 ? h0[sidx + i] : 0.0;
      for (int64_t t = 0; t < L; ++t) {
        double v = dt[((size_t)b * L + t) * nh + h] + at(dt_bias, (size_t)h, 0.0);
        double Dt = softplus ? sp(v) : v;
        double a = exp(Dt * A[h]);
        const double* Bt = Bm + (((size_t)b * L + t) * ng + g) * (size_t)N;
        const double* Ct = Cm + (((size_t)b * L + t) * ng + g) * (size_t)N;
        size_t xo = (((size_t)b * L + t) * nh + h) * (size_t)P;
        for (int64_t p = 0; p < P; ++p) {
          double xp = x[xo + p];
          double acc = 0.0;
          for (int64_t n = 0; n < N; ++n) {
            double* hp = H + p * N + n;
            *hp = a * *hp + Dt * xp * Bt[n];  /* update, then read out */
            acc += *hp * Ct[n];
          }
          double out = acc + at(Dskip, (size_t)h, 0.0) * xp;
          y[xo + p] = z ? out * z[xo + p] * sg(z[xo + p]) : out;
        }
      }
      if (final_state)
        for (int64_t i = 0; i < P * N; ++i) final_state[sidx + i] = H[i];
    }
  }
  free(H);
}

/* Mamba-2 SSD backward for the loss <dy, y> + <dfinal, H_{L-1}>: the adjoint
 * of oracle_ssd_fwd ("Mamba", Part IV Stage 7, applied to the Part V
 * recurrence H_t = a_t H_{t-1} + Delta_t x_t B_t^T with a_t = exp(Delta_t A_h),
 * y_t = (H_t C_t + D_h x_t) SiLU(z_t)).  The forward states are kept for every
 * step, then with G = dloss/dH_t walked backwards:
 *   dout   = dy SiLU(z)                     dz = dy (H_t C_t + D x_t) sigma(z)(1 + z(1 - sigma(z)))
 *   G     += dout C_t^T                     dC_t += H_t^T dout   (summed over the group's heads)
 *   dx_t   = Delta_t G B_t + D dout         dB_t += Delta_t G^T x_t
 *   dDelta = x_t^T G B_t + A_h <G, a_t H_{t-1}>,   dA_h += Delta_t <G, a_t H_{t-1}>
 *   ddt    = dDelta sigma(dt + dt_bias) (softplus on),   ddt_bias_h += ddt,   dD_h += <dout, x_t>
 *   G     <- a_t G   (the gradient reaching H_{t-1});   dh0 = G after step 0.
 * Outputs are overwritten: dx, dz (b, L, nh, P); ddt (b, L, nh); dB, dC
 * (b, L, ng, N); dA, dD, ddt_bias (nh,); dh0 (b, nh, P, N) or NULL.  dz may be
 * NULL when z is. */
void oracle_ssd_bwd(int64_t Bsz, int64_t L, int64_t nh, int64_t P, int64_t ng, int64_t N,
                    const double* x, const double* dt, const double* A, const double* Bm,
                    const double* Cm, const double* Dskip, const double* z,
                    const double* dt_bias, int softplus, const double* h0, const double* dy,
                    const double* dfinal, double* dx, double* ddt, double* dA, double* dB,
                    double* dC, double* dD, double* dz, double* ddt_bias, double* dh0) {
  const int64_t PN = P * N;
  int64_t hpg = nh / ng;
  double* Hs = (double*)malloc(sizeof(double) * (size_t)((L + 1) * PN > 0 ? (L + 1) * PN : 1));
  double* G = (double*)malloc(sizeof(double) * (size_t)(PN > 0 ? PN : 1));
  double* dout = (double*)malloc(sizeof(double) * (size_t)(P > 0 ? P : 1));
  memset(dB, 0, sizeof(double) * (size_t)(Bsz * L * ng * N));
  memset(dC, 0, sizeof(double) * (size_t)(Bsz * L * ng * N));
  for (int64_t h = 0; h < nh; ++h) {
    dA[h] = 0.0;
    dD[h] = 0.0;
    ddt_bias[h] = 0.0;
  }
  for (int64_t b = 0; b < Bsz; ++b) {
    for (int64_t h = 0; h < nh; ++h) {
      const int64_t grp = h / hpg;
      size_t sidx = ((size_t)b * nh + h) * (size_t)PN;
      double Dh = at(Dskip, (size_t)h, 0.0);
      /* forward: Hs[t + 1] = H_t, Hs[0] = the initial state */
      for (int64_t i = 0; i < PN; ++i) Hs[i] = h0 ? h0[sidx + i] : 0.0;
      for (int64_t t = 0; t < L; ++t) {
        double v = dt[((size_t)b * L + t) * nh + h] + at(dt_bias, (size_t)h, 0.0);
        double Dt = softplus ? sp(v) : v;
        const double af = exp(A[h] * Dt);
        const double* Bt = Bm + (((size_t)b * L + t) * ng + grp) * (size_t)N;
        size_t xo = (((size_t)b * L + t) * nh + h) * (size_t)P;
        const double* Hp = Hs + (size_t)t * PN;
        double* Hn = Hs + (size_t)(t + 1) * PN;
        for (int64_t p = 0; p < P; ++p)
          for (int64_t n = 0; n < N; ++n)
            Hn[p * N + n] = af * Hp[p * N + n] + Dt * x[xo + p] * Bt[n];
      }
      /* backward */
      for (int64_t i = 0; i < PN; ++i) G[i] = dfinal ? dfinal[sidx + i] : 0.0;
      for (int64_t t = L - 1; t >= 0; --t) {
        size_t ti = ((size_t)b * L + t) * nh + h;
        double v = dt[ti] + at(dt_bias, (size_t)h, 0.0);
        double Dt = softplus ? sp(v) : v;
        double a = exp(A[h] * Dt);
        size_t bo = (((size_t)b * L + t) * ng + grp) * (size_t)N;
        const double* Bt = Bm + bo;
        const double* Ct = Cm + bo;
        size_t xo = ti * (size_t)P;
        const double* Ht = Hs + (size_t)(t + 1) * PN;
        const double* Hp = Hs + (size_t)t * PN;
        for (int64_t p = 0; p < P; ++p) {
          double hc = 0.0;  /* (H_t C_t)_p */
          for (int64_t n = 0; n < N; ++n) hc += Ht[p * N + n] * Ct[n];
          double out = hc + Dh * x[xo + p];
          if (z) {
            double zz = z[xo + p], s = sg(zz);
            dout[p] = dy[xo + p] * zz * s;
            dz[xo + p] = dy[xo + p] * out * s * (1.0 + zz * (1.0 - s));
          } else {
            dout[p] = dy[xo + p];
          }
          dD[h] += dout[p] * x[xo + p];
        }
        double gbx = 0.0, q = 0.0;  /* x^T G B, <G, a H_{t-1}> */
        for (int64_t p = 0; p < P; ++p) {
          double gb = 0.0;
          for (int64_t n = 0; n < N; ++n) {
            double* gp = G + p * N + n;
            *gp += dout[p] * Ct[n];
            dC[bo + n] += Ht[p * N + n] * dout[p];
            dB[bo + n] += Dt * *gp * x[xo + p];
            gb += *gp * Bt[n];
            q += *gp * a * Hp[p * N + n];
          }
          dx[xo + p] = Dt * gb + Dh * dout[p];
          gbx += x[xo + p] * gb;
        }
        double dDelta = gbx + A[h] * q;
        dA[h] += Dt * q;
        double dd = softplus ? dDelta * sg(v) : dDelta;
        ddt[ti] = dd;
        ddt_bias[h] += dd;
        for (int64_t i = 0; i < PN; ++i) G[i] *= a;
      }
      if (dh0)
        for (int64_t i = 0; i < PN; ++i) dh0[sidx + i] = G[i];
    }
  }
  free(dout);
  free(G);
  free(Hs);
}
