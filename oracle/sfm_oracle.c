/*
 * sfm_oracle.c -- plain, slow, fp64 CPU definition of the SF-Mamba mixer hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this library.  It shares no code, header, table or
 * helper with the CUDA library; it is compiled with gcc from this file alone.
 *
 * Every routine is the plain definition written out, one sample at a time, in the
 * order the pages describe the method:
 *   - selective SSM recurrence h_t = Abar_t h_{t-1} + Bbar_t x_t, y_t = C_t h_t
 *     ("Seeing Both Ways, Running One Way", sungsoo.github.io, section 3.1, the recurrence);
 *   - discretisation Abar = exp(Delta*A), Bbar = Delta*B, D skip, SiLU(z) gate and
 *     Delta = softplus(dt + dt_bias): the standard Mamba convention (Gu & Dao, cited
 *     as background source 4 on the same page); the pages do not spell it out;
 *   - auxiliary head/tail tokens initialised to avg(X) and swapped head<->tail between
 *     layers (sungsoo.github.io section 3.2 equations; techloop.online
 *     "Auxiliary Patch Swapping");
 *   - batch folding [B,D,T] -> [B1,D,B2*T] with the transition factor forced to zero
 *     at every sample start (sungsoo.github.io section 3.3 equations; techloop.online
 *     "Batch Folding with Periodic State Reset");
 *   - a depthwise conv1d that never reads across sample boundaries (techloop.online,
 *     the paragraph on convolution boundaries; sungsoo.github.io section 8.1 item 5).
 *
 * Readings where the pages are silent (kept identical on the CUDA side):
 *   - reset: the DISCRETE factor Abar is set to 0 at folded position p with
 *     p mod L == 0 (the first token of each sample, L = T + 2 with aux tokens);
 *     the folded mode applies it as a select, so a non-finite value in one sample
 *     cannot reach the next one through 0*Inf;
 *   - softplus(v) = log1p(exp(v)), returning v itself for v > 20;
 *   - SiLU(v) = v / (1 + exp(-v));
 *   - conv: out[t] = bias + sum_k w[k] * in[t + k - pad_left], zero outside [0, L)
 *     of the same sample (cross-correlation, as in a deep-learning conv layer).
 *
 * Layouts (all contiguous, row-major): x [B,D,T]; xa, u, dt, z, y [B,D,L];
 * Bm, Cm [B,N,L]; A [D,N]; Dskip, dt_bias, conv_b [D]; conv_w [D,K];
 * final_state [B,D,N].
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

double ora_softplus(double v) { return v > 20.0 ? v : log1p(exp(v)); }
double ora_silu(double v) { return v / (1.0 + exp(-v)); }
static double ora_sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

/* Aux init: xa[b,d,0] = xa[b,d,L-1] = mean_t x[b,d,t]; xa[b,d,1..T] = x[b,d,0..T-1]. */
void ora_aux_init(const double* x, double* xa, long B, long D, long T) {
  const long L = T + 2;
  for (long b = 0; b < B; ++b)
    for (long d = 0; d < D; ++d) {
      const double* xr = x + (b * D + d) * T;
      double* ar = xa + (b * D + d) * L;
      double s = 0.0;
      for (long t = 0; t < T; ++t) s += xr[t];
      const double m = s / (double)T;
      ar[0] = m;
      for (long t = 0; t < T; ++t) ar[t + 1] = xr[t];
      ar[L - 1] = m;
    }
}

/* Aux swap between consecutive layers: the next head is this tail, the next tail this head. */
void ora_aux_swap(double* y, long B, long D, long L) {
  for (long r = 0; r < B * D; ++r) {
    double* yr = y + r * L;
    const double h = yr[0];
    yr[0] = yr[L - 1];
    yr[L - 1] = h;
  }
}

/* Depthwise conv1d with zero padding per sample (never reads a neighbouring sample). */
void ora_conv1d(const double* xa, const double* w, const double* bias, double* u,
                long B, long D, long L, int K, int pad_left, int silu) {
  for (long b = 0; b < B; ++b)
    for (long d = 0; d < D; ++d) {
      const double* xr = xa + (b * D + d) * L;
      double* ur = u + (b * D + d) * L;
      for (long t = 0; t < L; ++t) {
        double acc = bias ? bias[d] : 0.0;
        for (int k = 0; k < K; ++k) {
          const long s = t + k - pad_left;
          const double v = (s >= 0 && s < L) ? xr[s] : 0.0;
          acc += w[d * K + k] * v;
        }
        ur[t] = silu ? ora_silu(acc) : acc;
      }
    }
}

/* Per-sample (unfolded) selective scan with D skip and SiLU(z) gate, samples [b_lo, b_hi).
 * h starts at zero for every sample; this is the definition the folded run must equal. */
void ora_scan(const double* u, const double* dt, const double* z,
              const double* Bm, const double* Cm, const double* A,
              const double* Dskip, const double* dt_bias,
              double* y, double* final_state,
              long B, long D, long L, long N, int dt_softplus, long b_lo, long b_hi) {
  (void)B;
  double* h = (double*)malloc(sizeof(double) * (size_t)N);
  for (long b = b_lo; b < b_hi; ++b)
    for (long d = 0; d < D; ++d) {
      const long row = (b * D + d) * L;
      for (long n = 0; n < N; ++n) h[n] = 0.0;
      for (long t = 0; t < L; ++t) {
        double delta = dt[row + t] + (dt_bias ? dt_bias[d] : 0.0);
        if (dt_softplus) delta = ora_softplus(delta);
        const double ut = u[row + t];
        double yt = 0.0;
        for (long n = 0; n < N; ++n) {
          const double abar = exp(delta * A[d * N + n]);
          const double bbar = delta * Bm[(b * N + n) * L + t];
          h[n] = abar * h[n] + bbar * ut;
          yt += Cm[(b * N + n) * L + t] * h[n];
        }
        if (Dskip) yt += Dskip[d] * ut;
        if (z) yt *= ora_silu(z[row + t]);
        y[row + t] = yt;
      }
      if (final_state)
        for (long n = 0; n < N; ++n) final_state[(b * D + d) * N + n] = h[n];
    }
  free(h);
}

/* Literal batch-folded scan: physically re-lays [B,D,L] as [B1,D,B2*L] (sample
 * b = b1*B2 + b2 occupies folded positions b2*L .. b2*L+L-1), runs ONE recurrence per
 * folded row with the transition factor selected to 0 where p mod L == 0, then
 * un-folds the output.  Exists to check that folding with reset equals the per-sample
 * definition above. */
void ora_scan_folded(const double* u, const double* dt, const double* z,
                     const double* Bm, const double* Cm, const double* A,
                     const double* Dskip, const double* dt_bias,
                     double* y, double* final_state,
                     long B, long D, long L, long N, int dt_softplus, long B2) {
  const long B1 = B / B2, P = B2 * L;
  double* fu = (double*)malloc(sizeof(double) * (size_t)(B1 * D * P));
  double* fdt = (double*)malloc(sizeof(double) * (size_t)(B1 * D * P));
  double* fz = z ? (double*)malloc(sizeof(double) * (size_t)(B1 * D * P)) : NULL;
  double* fB = (double*)malloc(sizeof(double) * (size_t)(B1 * N * P));
  double* fC = (double*)malloc(sizeof(double) * (size_t)(B1 * N * P));
  double* fy = (double*)malloc(sizeof(double) * (size_t)(B1 * D * P));
  double* h = (double*)malloc(sizeof(double) * (size_t)N);
  /* fold */
  for (long b1 = 0; b1 < B1; ++b1)
    for (long b2 = 0; b2 < B2; ++b2) {
      const long b = b1 * B2 + b2;
      for (long d = 0; d < D; ++d)
        for (long t = 0; t < L; ++t) {
          const long src = (b * D + d) * L + t, dst = (b1 * D + d) * P + b2 * L + t;
          fu[dst] = u[src];
          fdt[dst] = dt[src];
          if (z) fz[dst] = z[src];
        }
      for (long n = 0; n < N; ++n)
        for (long t = 0; t < L; ++t) {
          const long src = (b * N + n) * L + t, dst = (b1 * N + n) * P + b2 * L + t;
          fB[dst] = Bm[src];
          fC[dst] = Cm[src];
        }
    }
  /* one long recurrence per folded row */
  for (long b1 = 0; b1 < B1; ++b1)
    for (long d = 0; d < D; ++d) {
      const long row = (b1 * D + d) * P;
      for (long n = 0; n < N; ++n) h[n] = 0.0;
      for (long p = 0; p < P; ++p) {
        double delta = fdt[row + p] + (dt_bias ? dt_bias[d] : 0.0);
        if (dt_softplus) delta = ora_softplus(delta);
        const double ut = fu[row + p];
        const int reset = (p % L) == 0;
        double yt = 0.0;
        for (long n = 0; n < N; ++n) {
          const double abar = exp(delta * A[d * N + n]);
          const double carry = reset ? 0.0 : abar * h[n];
          const double bbar = delta * fB[(b1 * N + n) * P + p];
          h[n] = carry + bbar * ut;
          yt += fC[(b1 * N + n) * P + p] * h[n];
        }
        if (Dskip) yt += Dskip[d] * ut;
        if (z) yt *= ora_silu(fz[row + p]);
        fy[row + p] = yt;
        if (final_state && (p % L) == L - 1) {
          const long b = b1 * B2 + p / L;
          for (long n = 0; n < N; ++n) final_state[(b * D + d) * N + n] = h[n];
        }
      }
    }
  /* un-fold */
  for (long b1 = 0; b1 < B1; ++b1)
    for (long b2 = 0; b2 < B2; ++b2)
      for (long d = 0; d < D; ++d)
        for (long t = 0; t < L; ++t)
          y[((b1 * B2 + b2) * D + d) * L + t] = fy[(b1 * D + d) * P + b2 * L + t];
  free(fu); free(fdt); free(fz); free(fB); free(fC); free(fy); free(h);
}

/* Backward of ora_scan (gate included) by a reverse adjoint sweep, fp64.
 * Given dout = dLoss/dy (gated output), produces
 *   du, ddt, dz [B,D,L]; dA [D,N]; dDskip, ddt_bias [D]; dB, dC [B,N,L].
 * Reduced gradients (dA, dDskip, ddt_bias over b and t; dB, dC over d) are
 * accumulated into the output arrays, which this routine zeroes first.
 * The adjoint of h obeys g_t = C_t*dy_t + Abar_{t+1}*g_{t+1} inside a sample and
 * never crosses a sample start, where the transition factor is the constant 0. */
void ora_scan_bwd(const double* u, const double* dt, const double* z,
                  const double* Bm, const double* Cm, const double* A,
                  const double* Dskip, const double* dt_bias, const double* dout,
                  double* du, double* ddt, double* dz, double* dA, double* dDskip,
                  double* ddt_bias, double* dB, double* dC,
                  long B, long D, long L, long N, int dt_softplus) {
  double* h = (double*)malloc(sizeof(double) * (size_t)(L * N));    /* h[t][n] */
  double* abar = (double*)malloc(sizeof(double) * (size_t)(L * N)); /* Abar[t][n] */
  double* delta = (double*)malloc(sizeof(double) * (size_t)L);
  double* g = (double*)malloc(sizeof(double) * (size_t)N);
  memset(dA, 0, sizeof(double) * (size_t)(D * N));
  if (dDskip) memset(dDskip, 0, sizeof(double) * (size_t)D);
  if (ddt_bias) memset(ddt_bias, 0, sizeof(double) * (size_t)D);
  memset(dB, 0, sizeof(double) * (size_t)(B * N * L));
  memset(dC, 0, sizeof(double) * (size_t)(B * N * L));
  for (long b = 0; b < B; ++b)
    for (long d = 0; d < D; ++d) {
      const long row = (b * D + d) * L;
      /* forward, keeping every state */
      for (long t = 0; t < L; ++t) {
        double s = dt[row + t] + (dt_bias ? dt_bias[d] : 0.0);
        delta[t] = dt_softplus ? ora_softplus(s) : s;
        for (long n = 0; n < N; ++n) {
          const double prev = t > 0 ? h[(t - 1) * N + n] : 0.0;
          abar[t * N + n] = exp(delta[t] * A[d * N + n]);
          h[t * N + n] = abar[t * N + n] * prev + delta[t] * Bm[(b * N + n) * L + t] * u[row + t];
        }
      }
      /* reverse sweep */
      for (long n = 0; n < N; ++n) g[n] = 0.0;
      for (long t = L - 1; t >= 0; --t) {
        const double ut = u[row + t];
        double yt = 0.0;
        for (long n = 0; n < N; ++n) yt += Cm[(b * N + n) * L + t] * h[t * N + n];
        if (Dskip) yt += Dskip[d] * ut;
        double dy = dout[row + t];
        if (z) {
          const double zt = z[row + t], sg = ora_sigmoid(zt);
          dz[row + t] = dout[row + t] * yt * (sg * (1.0 + zt * (1.0 - sg)));
          dy = dout[row + t] * ora_silu(zt);
        }
        double du_t = Dskip ? dy * Dskip[d] : 0.0;
        if (Dskip) dDskip[d] += dy * ut;
        double ddelta = 0.0;
        for (long n = 0; n < N; ++n) {
          const double Bv = Bm[(b * N + n) * L + t], Cv = Cm[(b * N + n) * L + t];
          /* adjoint of h_t: direct read-out plus the carry into t+1 (none past the sample end) */
          const double carry = (t + 1 < L) ? abar[(t + 1) * N + n] * g[n] : 0.0;
          g[n] = dy * Cv + carry;
          dC[(b * N + n) * L + t] += dy * h[t * N + n];
          dB[(b * N + n) * L + t] += g[n] * delta[t] * ut;
          du_t += g[n] * delta[t] * Bv;
          ddelta += g[n] * Bv * ut;
          if (t > 0) {
            const double da = g[n] * h[(t - 1) * N + n]; /* dLoss/dAbar_t */
            ddelta += da * abar[t * N + n] * A[d * N + n];
            dA[d * N + n] += da * abar[t * N + n] * delta[t];
          }
        }
        du[row + t] = du_t;
        double s = dt[row + t] + (dt_bias ? dt_bias[d] : 0.0);
        const double ds = dt_softplus ? ddelta * (s > 20.0 ? 1.0 : ora_sigmoid(s)) : ddelta;
        ddt[row + t] = ds;
        if (ddt_bias) ddt_bias[d] += ds;
      }
    }
  free(h); free(abar); free(delta); free(g);
}

/* Backward of ora_conv1d (+ SiLU when silu != 0) given du = dLoss/du:
 *   pre = bias + sum_k w[k] * xa[t+k-pad_left] (zero outside the sample), u = act(pre);
 *   dpre[t] = du[t] * act'(pre[t]);  dxa[s] = sum_k w[k] * dpre[s-k+pad_left] (inside the sample);
 *   dw[d,k] = sum_{b,t} dpre[b,d,t] * xa[b,d,t+k-pad_left];  dbias[d] = sum_{b,t} dpre[b,d,t].
 * dw and dbias (if not NULL) are zeroed and accumulated. */
void ora_conv1d_bwd(const double* xa, const double* w, const double* bias, const double* du,
                    double* dxa, double* dw, double* dbias,
                    long B, long D, long L, int K, int pad_left, int silu) {
  double* dpre = (double*)malloc(sizeof(double) * (size_t)L);
  memset(dw, 0, sizeof(double) * (size_t)(D * K));
  if (dbias) memset(dbias, 0, sizeof(double) * (size_t)D);
  for (long b = 0; b < B; ++b)
    for (long d = 0; d < D; ++d) {
      const double* xr = xa + (b * D + d) * L;
      const double* dur = du + (b * D + d) * L;
      double* dxr = dxa + (b * D + d) * L;
      for (long t = 0; t < L; ++t) {
        double pre = bias ? bias[d] : 0.0;
        for (int k = 0; k < K; ++k) {
          const long s = t + k - pad_left;
          if (s >= 0 && s < L) pre += w[d * K + k] * xr[s];
        }
        double g = 1.0;
        if (silu) {
          const double sg = ora_sigmoid(pre);
          g = sg * (1.0 + pre * (1.0 - sg));
        }
        dpre[t] = dur[t] * g;
      }
      for (long s = 0; s < L; ++s) {
        double acc = 0.0;
        for (int k = 0; k < K; ++k) {
          const long t = s - k + pad_left;
          if (t >= 0 && t < L) acc += w[d * K + k] * dpre[t];
        }
        dxr[s] = acc;
      }
      for (long t = 0; t < L; ++t) {
        for (int k = 0; k < K; ++k) {
          const long s = t + k - pad_left;
          if (s >= 0 && s < L) dw[d * K + k] += dpre[t] * xr[s];
        }
        if (dbias) dbias[d] += dpre[t];
      }
    }
  free(dpre);
}

/* Backward of ora_aux_init: xa = [m, x_0..x_{T-1}, m] with m the mean of x, so
 * dx[t] = dxa[t+1] + (dxa[0] + dxa[T+1]) / T. */
void ora_aux_init_bwd(const double* dxa, double* dx, long B, long D, long T) {
  const long L = T + 2;
  for (long r = 0; r < B * D; ++r) {
    const double* g = dxa + r * L;
    const double share = (g[0] + g[L - 1]) / (double)T;
    for (long t = 0; t < T; ++t) dx[r * T + t] = g[t + 1] + share;
  }
}
