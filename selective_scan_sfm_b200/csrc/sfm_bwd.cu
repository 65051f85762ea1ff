// sfm_bwd.cu -- backward of the folded selective scan (from its input u to the gated
// output), sm_100a.
//
// Per sample b, channel d and state n, the adjoint of the state obeys
//   g_t = C_t * dy_t + Abar_(t+1) * g_(t+1)   (no carry past the sample's last token)
// where dy_t = dout_t * SiLU(z_t).  At a sample start the transition factor is the
// constant 0 (the reset of "Seeing Both Ways, Running One Way", sungsoo.github.io,
// section 3.3), so no gradient crosses samples and none flows into A, Delta or the
// previous state through that token.
//
// Schedule (every sum in a fixed order, so results are reproducible bit for bit):
//   bwd_pair_kernel (N <= 16, B and C of a sample within 64 KB of shared memory): all
//     states in registers, two threads per channel, one forward and one reverse sweep.
//   bwd_main_kernel (other shapes): grid (channel tiles, B); one thread per channel.  It first lays out
//     u, Delta and the gated output gradient per token (once), then loops over the N
//     states: a forward sweep stores h_t, a reverse sweep accumulates du, dDelta and dA
//     and writes each channel's dB/dC contribution; the CTA then sums those over its
//     channels in a fixed order into per-tile partials.  Every per-token array of the
//     workspace is time-major [B, L, D], so the channels of a warp read and write one
//     contiguous run per token; the caller's row-major outputs are written once at the end.
//   bwd_reduce_bc_kernel: dB, dC = sum of the tile partials, in tile order.
//   bwd_reduce_param_kernel: dA, dDskip, ddt_bias = sum over samples, in sample order.
#include <mutex>

#include "sfm_device.cuh"
#include "sfm_internal.h"

namespace sfm {

__device__ __forceinline__ float sigmoid(float v) { return rcp(1.0f + ex2(-v * kLog2e)); }

// xa at position s of row `xr` (aux: the mean at 0 and L-1, x shifted by one inside);
// zero outside the sample.
template <typename TI>
__device__ __forceinline__ float xa_row(const TI* xr, int s, int L, bool aux, float mean) {
  if (s < 0 || s >= L) return 0.0f;
  if (aux) return (s == 0 || s == L - 1) ? mean : to_f(xr[s - 1]);
  return to_f(xr[s]);
}

template <typename TI>
__device__ __forceinline__ float conv_pre(const BwdParams& p, const TI* xr, int t, int d, float mean) {
  float acc = p.conv_b ? p.conv_b[d] : 0.0f;
  for (int k = 0; k < p.K; ++k) acc = fmaf(p.conv_w[(size_t)d * p.K + k], xa_row(xr, t + k - p.pad_left, p.L, p.aux, mean), acc);
  return acc;
}

// Register-resident backward: states per channel at most, states per thread, tokens per
// dB/dC buffer, and the buffer's rows per token (B and C of each half's kHalfN states).
constexpr int kFastN = 16, kHalfN = kFastN / 2, kRedT = 2, kRedRows = 2 * kFastN;

static int bwd_fast_smem(int N, int L, int d_tile) {
  // bc [L][2N] + red: kRedT tokens x kRedRows rows of d_tile + 1 (the pad keeps the row sums
  // off one bank)
  return (int)(((size_t)L * 2 * N + (size_t)kRedT * kRedRows * (d_tile + 1)) * sizeof(float));
}

template <typename TI, typename TD, bool MIXER>
__global__ void __launch_bounds__(128) bwd_main_kernel(const BwdParams p) {
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int tile = blockIdx.x, b = blockIdx.y;
  const int d0 = tile * p.d_tile;
  const int dcount = min(p.d_tile, p.D - d0);
  const bool active = tid < dcount;
  const int d = d0 + (active ? tid : 0);
  const int L = p.L, N = p.N;
  const bool gate = p.z != nullptr, use_sp = p.softplus;
  const size_t row = ((size_t)b * p.D + d) * L;

  const TI* u = MIXER ? nullptr : static_cast<const TI*>(p.u) + row;
  const TI* dt = static_cast<const TI*>(p.dt) + row;
  const TI* z = gate ? static_cast<const TI*>(p.z) + row : nullptr;
  const TD* dout = static_cast<const TD*>(p.dout) + row;
  const TI* Bm = static_cast<const TI*>(p.Bm) + (size_t)b * N * L;
  const TI* Cm = static_cast<const TI*>(p.Cm) + (size_t)b * N * L;
  const float dsk = p.Dskip ? p.Dskip[d] : 0.0f;
  const float dtb = p.dt_bias ? p.dt_bias[d] : 0.0f;
  float* du = p.du + row;
  float* ddt = p.ddt + row;
  float* dz = gate ? p.dz + row : nullptr;
  // time-major workspace: element (b, t, this channel)
  const size_t tm0 = (size_t)b * L * p.D + d, tD = (size_t)p.D;
  float* tu = p.tm_u + tm0;
  float* tdl = p.tm_dl + tm0;   // Delta_t
  float* tgy = p.tm_gy + tm0;   // dLoss/dy_t through the gate
  float* tdu = p.tm_du + tm0;   // dLoss/du_t, accumulated over the states
  float* tdd = p.tm_dd + tm0;   // dLoss/dDelta_t, accumulated over the states
  float* ty = p.tm_y + tm0;     // the pre-gate output y_t (for dz)
  float* hb = p.hbuf + tm0;
  float* cB = p.cB + tm0;
  float* cC = p.cC + tm0;

  auto delta_at = [&](int t) {
    const float v = to_f(dt[t]) + dtb;
    return use_sp ? softplus(v) : v;
  };
  // the layer output was swapped head<->tail: read its gradient through the same map
  auto dout_at = [&](int t) {
    const int i = (MIXER && p.swap_dout) ? (t == 0 ? L - 1 : (t == L - 1 ? 0 : t)) : t;
    return to_f(dout[i]);
  };

  // per token, once: u (the layer's scan input, u = SiLU(conv(xa)) in mixer mode), Delta
  // and the output gradient through the gate, each laid out time-major
  float sum_dsk = 0.0f;
  if (active) {
    const TI* xr = MIXER ? static_cast<const TI*>(p.x) + ((size_t)b * p.D + d) * p.Tx : nullptr;
    float mean = 0.0f;
    if (MIXER && p.aux) {
      for (int t = 0; t < p.Tx; ++t) mean += to_f(xr[t]);
      mean /= (float)p.Tx;
    }
    for (int t = 0; t < L; ++t) {
      float ut;
      if constexpr (MIXER)
        ut = p.conv ? silu(conv_pre(p, xr, t, d, mean)) : xa_row(xr, t, L, p.aux, mean);
      else
        ut = to_f(u[t]);
      const float gy = gate ? dout_at(t) * silu(to_f(z[t])) : dout_at(t);
      tu[t * tD] = ut;
      tdl[t * tD] = delta_at(t);
      tgy[t * tD] = gy;
      tdu[t * tD] = gy * dsk;
      tdd[t * tD] = 0.0f;
      if (gate) ty[t * tD] = dsk * ut;
      sum_dsk = fmaf(gy, ut, sum_dsk);
    }
  }

  for (int n = 0; n < N; ++n) {
    if (active) {
      const float an = p.A[(size_t)d * N + n];
      const TI* Bn = Bm + (size_t)n * L;
      const TI* Cn = Cm + (size_t)n * L;
      // forward sweep: h_t (the reset token starts from 0)
      float h = 0.0f;
      for (int t = 0; t < L; ++t) {
        const float delta = tdl[t * tD];
        const float bu = delta * to_f(Bn[t]) * tu[t * tD];
        h = t == 0 ? bu : fmaf(ex2(delta * an * kLog2e), h, bu);
        hb[t * tD] = h;
        if (gate) ty[t * tD] = fmaf(to_f(Cn[t]), h, ty[t * tD]);
      }
      // reverse sweep
      float g = 0.0f, a_next = 0.0f, dA = 0.0f;
      for (int t = L - 1; t >= 0; --t) {
        const float delta = tdl[t * tD], gy = tgy[t * tD], ut = tu[t * tD], Bv = to_f(Bn[t]);
        g = fmaf(gy, to_f(Cn[t]), t + 1 < L ? a_next * g : 0.0f);
        cC[t * tD] = gy * hb[t * tD];
        cB[t * tD] = g * delta * ut;
        tdu[t * tD] = fmaf(g * delta, Bv, tdu[t * tD]);
        float dd = g * Bv * ut;
        float a_t = 0.0f;
        if (t > 0) {
          a_t = ex2(delta * an * kLog2e);
          const float gha = g * hb[(t - 1) * tD] * a_t;  // dLoss/dAbar_t * Abar_t
          dd = fmaf(gha, an, dd);
          dA = fmaf(gha, delta, dA);
        }
        tdd[t * tD] += dd;
        a_next = a_t;
      }
      p.partA[((size_t)b * p.D + d) * N + n] = dA;
    }
    __syncthreads();
    // this tile's share of dB[b,n,:] and dC[b,n,:], summed over its channels in order
    for (int t = tid; t < L; t += nthr) {
      float sb = 0.0f, sc = 0.0f;
      const size_t base = ((size_t)b * L + t) * p.D + d0;
      for (int c = 0; c < dcount; ++c) {
        sb += p.cB[base + c];
        sc += p.cC[base + c];
      }
      const size_t o = (((size_t)b * p.ntiles + tile) * 2) * N * L + (size_t)n * L + t;
      p.partBC[o] = sb;
      p.partBC[o + (size_t)N * L] = sc;
    }
    __syncthreads();
  }

  if (active) {  // the caller's row-major outputs, once
    float sum_bias = 0.0f;
    for (int t = 0; t < L; ++t) {
      const float v = to_f(dt[t]) + dtb;
      const float dd = tdd[t * tD];
      const float ds = use_sp ? dd * (v > 20.0f ? 1.0f : sigmoid(v)) : dd;
      ddt[t] = ds;
      du[t] = tdu[t * tD];
      sum_bias += ds;
      if (gate) {
        const float zt = to_f(z[t]), sg = sigmoid(zt);
        dz[t] = dout_at(t) * ty[t * tD] * (sg * (1.0f + zt * (1.0f - sg)));
      }
    }
    p.partD[(size_t)b * p.D + d] = sum_dsk;
    p.partBias[(size_t)b * p.D + d] = sum_bias;
  }
}

// The backward with all N (<= 16) states in registers, two threads per channel.  Lanes
// 0-15 of a warp hold states 0 .. ceil(N/2)-1 of 16 channels and lanes 16-31 the other
// states of the same channels; every sum over the states adds the two halves' partial
// sums (lane ^ 16).  Half the registers per thread buys twice the warps per SM, which
// hide the latency of the per-token loads.
//   prologue: per token (split by parity between a channel's two threads), u, Delta and
//     the output gradient through the gate, laid out time-major;
//   forward sweep: every state's h_t (stored [B, L, N, D], so a warp's channels store one
//     contiguous run per (token, state)) and the pre-gate output;
//   reverse sweep: every state's adjoint, with h_t and h_(t-1) in registers and the next
//     token's states and inputs loaded one step ahead;
//   dB/dC: each token's contributions go to a shared buffer of kRedT tokens, summed over
//     the tile's channels in channel order when it fills.
// B and C of the sample are staged in shared memory as fp32 [t][2N].  A lane past the
// tile's last channel computes on the tile's first channel and stores nothing, so every
// lane takes part in the shuffles.

template <typename TI, typename TD, bool MIXER>
__global__ void __launch_bounds__(128, MIXER ? 5 : 4) bwd_pair_kernel(const BwdParams p) {
  extern __shared__ float bsm[];
  constexpr unsigned kAll = 0xffffffffu;
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int lane = tid & 31, half = lane >> 4;
  const int cl = (tid >> 5) * 16 + (lane & 15);  // channel within the tile
  const int tile = blockIdx.x, b = blockIdx.y;
  const int d0 = tile * p.d_tile;
  const int dcount = min(p.d_tile, p.D - d0);
  const bool active = cl < dcount;
  const int d = d0 + (active ? cl : 0);
  const int L = p.L, N = p.N, N2 = 2 * p.N;
  const int nh = (N + 1) / 2, n0 = half * nh, ncount = half ? N - nh : nh;  // this thread's states
  const bool gate = p.z != nullptr, use_sp = p.softplus;
  const size_t row = ((size_t)b * p.D + d) * L;
  float* bc = bsm;                    // [L][2N]: B then C of token t
  // [kRedT][kRedRows][d_tile + 1]: half h's B rows at 16h .. 16h+7, its C rows at 16h+8 ..
  // 16h+15, so the two halves' stores of one state index land 16 banks apart
  float* red = bsm + (size_t)L * N2;
  const int rstride = p.d_tile + 1;

  const TI* u = MIXER ? nullptr : static_cast<const TI*>(p.u) + row;
  const TI* dt = static_cast<const TI*>(p.dt) + row;
  const TI* z = gate ? static_cast<const TI*>(p.z) + row : nullptr;
  const TD* dout = static_cast<const TD*>(p.dout) + row;
  const TI* Bm = static_cast<const TI*>(p.Bm) + (size_t)b * N * L;
  const TI* Cm = static_cast<const TI*>(p.Cm) + (size_t)b * N * L;
  const float dsk = p.Dskip ? p.Dskip[d] : 0.0f;
  const float dtb = p.dt_bias ? p.dt_bias[d] : 0.0f;
  const size_t tm0 = (size_t)b * L * p.D + d, tD = (size_t)p.D;
  float* tu = p.tm_u + tm0;
  float* tdl = p.tm_dl + tm0;
  float* tgy = p.tm_gy + tm0;
  float* tdu = p.tm_du + tm0;
  float* tdd = p.tm_dd + tm0;
  float* ty = p.tm_y + tm0;
  // h of (t, state n0 + k) at hs[t * N * D + k * D]
  float* hs = p.hstore + (size_t)b * L * N * p.D + (size_t)n0 * p.D + d;

  for (int e = tid; e < L * N2; e += nthr) {
    const int t = e / N2, j = e - t * N2;
    bc[e] = j < N ? to_f(Bm[(size_t)j * L + t]) : to_f(Cm[(size_t)(j - N) * L + t]);
  }
  auto delta_at = [&](int t) {
    const float v = to_f(dt[t]) + dtb;
    return use_sp ? softplus(v) : v;
  };
  auto dout_at = [&](int t) {
    const int i = (MIXER && p.swap_dout) ? (t == 0 ? L - 1 : (t == L - 1 ? 0 : t)) : t;
    return to_f(dout[i]);
  };
  // prologue: this thread's tokens t = half, half + 2, ...
  float sum_dsk = 0.0f;
  {
    const TI* xr = MIXER ? static_cast<const TI*>(p.x) + ((size_t)b * p.D + d) * p.Tx : nullptr;
    float mean = 0.0f;
    if (MIXER && p.aux) {
      float s = 0.0f;
      for (int t = half; t < p.Tx; t += 2) s += to_f(xr[t]);
      const float so = __shfl_xor_sync(kAll, s, 16);
      mean = (half ? so + s : s + so) / (float)p.Tx;  // (even tokens) + (odd tokens) in both
    }
    for (int t = half; t < L; t += 2) {
      float ut;
      if constexpr (MIXER)
        ut = p.conv ? silu(conv_pre(p, xr, t, d, mean)) : xa_row(xr, t, L, p.aux, mean);
      else
        ut = to_f(u[t]);
      const float gy = gate ? dout_at(t) * silu(to_f(z[t])) : dout_at(t);
      if (active) {
        tu[t * tD] = ut;
        tdl[t * tD] = delta_at(t);
        tgy[t * tD] = gy;
        if (gate) ty[t * tD] = dsk * ut;
      }
      sum_dsk = fmaf(gy, ut, sum_dsk);
    }
  }
  __syncthreads();

  float An[kHalfN];
#pragma unroll
  for (int k = 0; k < kHalfN; ++k) An[k] = k < ncount ? p.A[(size_t)d * N + n0 + k] : 0.0f;
  const size_t hstep = (size_t)N * tD;  // h of the next token

  // forward sweep: this thread's states' h_t; the pre-gate output adds both halves
  {
    float h[kHalfN];
#pragma unroll
    for (int k = 0; k < kHalfN; ++k) h[k] = 0.0f;
    float* hp = hs;
    const float* bt = bc + n0;  // B of state n0 + k at bt[k], its C at bt[N + k]
    float nd = tdl[0], nu = tu[0], ny = gate ? ty[0] : 0.0f;
    for (int t = 0; t < L; ++t, hp += hstep, bt += N2) {
      const float delta = nd, ut = nu, y0 = ny;
      if (t + 1 < L) {
        const size_t o = (size_t)(t + 1) * tD;
        nd = tdl[o];
        nu = tu[o];
        if (gate) ny = ty[o];
      }
      float yp = 0.0f;
#pragma unroll
      for (int k = 0; k < kHalfN; ++k) {
        if (k < ncount) {
          const float bu = delta * bt[k] * ut;
          h[k] = t == 0 ? bu : fmaf(ex2(delta * An[k] * kLog2e), h[k], bu);
          if (active) hp[k * tD] = h[k];
          yp = fmaf(bt[N + k], h[k], yp);
        }
      }
      if (gate) {
        const float yo = __shfl_xor_sync(kAll, yp, 16);
        if (active && half == 0) ty[(size_t)t * tD] = y0 + (yp + yo);
      }
    }
  }

  // reverse sweep: this thread's states' adjoints; du and dDelta add both halves
  float g[kHalfN], a_next[kHalfN], dA[kHalfN];
#pragma unroll
  for (int k = 0; k < kHalfN; ++k) g[k] = a_next[k] = dA[k] = 0.0f;
  const size_t pbc = (((size_t)b * p.ntiles + tile) * 2) * N * L;
  float hc[kHalfN], hq[kHalfN];  // h_t and h_(t-1); h_(t-2) and the next inputs load one step ahead
  float nd, ngy, nu;
  {
    const size_t o = (size_t)(L - 1) * tD;
    nd = tdl[o];
    ngy = tgy[o];
    nu = tu[o];
#pragma unroll
    for (int k = 0; k < kHalfN; ++k) {
      hc[k] = k < ncount ? hs[(size_t)(L - 1) * hstep + k * tD] : 0.0f;
      hq[k] = (k < ncount && L > 1) ? hs[(size_t)(L - 2) * hstep + k * tD] : 0.0f;
    }
  }
  for (int t = L - 1; t >= 0; --t) {
    const int slot = (L - 1 - t) % kRedT;
    const float delta = nd, gy = ngy, ut = nu;
    if (t >= 1) {
      const size_t o1 = (size_t)(t - 1) * tD;
      nd = tdl[o1];
      ngy = tgy[o1];
      nu = tu[o1];
    }
    float hn[kHalfN];  // h_(t-2), for the next step
#pragma unroll
    for (int k = 0; k < kHalfN; ++k) hn[k] = (k < ncount && t >= 2) ? hs[(size_t)(t - 2) * hstep + k * tD] : 0.0f;
    const float* bt = bc + (size_t)t * N2 + n0;
    float* rs = red + ((size_t)slot * kRedRows + 2 * kHalfN * half) * rstride + cl;
    float dup = 0.0f, ddp = 0.0f;
#pragma unroll
    for (int k = 0; k < kHalfN; ++k) {
      if (k < ncount) {
        const float Bv = bt[k], Cv = bt[N + k];
        g[k] = fmaf(gy, Cv, t + 1 < L ? a_next[k] * g[k] : 0.0f);
        rs[(kHalfN + k) * rstride] = gy * hc[k];
        rs[k * rstride] = g[k] * delta * ut;
        dup = fmaf(g[k] * delta, Bv, dup);
        float dd = g[k] * Bv * ut;
        float a_t = 0.0f;
        if (t > 0) {
          a_t = ex2(delta * An[k] * kLog2e);
          const float gha = g[k] * hq[k] * a_t;
          dd = fmaf(gha, An[k], dd);
          dA[k] = fmaf(gha, delta, dA[k]);
        }
        ddp += dd;
        a_next[k] = a_t;
      }
    }
    const float dupo = __shfl_xor_sync(kAll, dup, 16), ddpo = __shfl_xor_sync(kAll, ddp, 16);
    if (active && half == 0) {  // du_t = dy_t Dskip + the states' share; dDelta_t = the states' share
      const size_t o = (size_t)t * tD;
      tdu[o] = fmaf(gy, dsk, dup + dupo);
      tdd[o] = ddp + ddpo;
    }
#pragma unroll
    for (int k = 0; k < kHalfN; ++k) {
      hc[k] = hq[k];
      hq[k] = hn[k];
    }
    if (slot == kRedT - 1 || t == 0) {  // the buffered tokens t .. t + slot: sum over channels in order
      __syncthreads();
      for (int e = tid; e < (slot + 1) * kRedRows; e += nthr) {
        const int k = e / kRedRows, j = e - k * kRedRows;  // buffer slot k holds token t + slot - k
        const int hh = j / (2 * kHalfN), kk = j % kHalfN, n = hh * nh + kk;
        const bool is_c = (j / kHalfN) & 1;
        if (kk >= (hh ? N - nh : nh)) continue;  // a row of no state
        const float* r = red + ((size_t)k * kRedRows + j) * rstride;
        float sum = 0.0f;
        for (int c = 0; c < dcount; ++c) sum += r[c];
        const int tt = t + slot - k;
        p.partBC[pbc + (is_c ? (size_t)N * L : 0) + (size_t)n * L + tt] = sum;
      }
      __syncthreads();
    }
  }

  // epilogue: this thread's tokens; the last barrier above ordered every tdu/tdd write
  if (active)
#pragma unroll
    for (int k = 0; k < kHalfN; ++k)
      if (k < ncount) p.partA[((size_t)b * p.D + d) * N + n0 + k] = dA[k];
  float* du = p.du + row;
  float* ddt = p.ddt + row;
  float* dz = gate ? p.dz + row : nullptr;
  float sum_bias = 0.0f;
  for (int t = half; t < L; t += 2) {
    const float v = to_f(dt[t]) + dtb;
    const float dd = tdd[t * tD];
    const float ds = use_sp ? dd * (v > 20.0f ? 1.0f : sigmoid(v)) : dd;
    if (active) {
      ddt[t] = ds;
      du[t] = tdu[t * tD];
      if (gate) {
        const float zt = to_f(z[t]), sg = sigmoid(zt);
        dz[t] = dout_at(t) * ty[t * tD] * (sg * (1.0f + zt * (1.0f - sg)));
      }
    }
    sum_bias += ds;
  }
  const float sdo = __shfl_xor_sync(kAll, sum_dsk, 16), sbo = __shfl_xor_sync(kAll, sum_bias, 16);
  if (active && half == 0) {
    p.partD[(size_t)b * p.D + d] = sum_dsk + sdo;
    p.partBias[(size_t)b * p.D + d] = sum_bias + sbo;
  }
}

// The register-resident kernels cover N <= 16 with B and C of a sample in 64 KB of
// shared memory; other shapes take bwd_main_kernel.
static bool bwd_fast_ok(int N, int L, int d_tile) {
  return N <= kFastN && d_tile <= 64 && bwd_fast_smem(N, L, d_tile) <= 64 * 1024;
}

// dB[b,n,t] / dC[b,n,t]: sum over channel tiles in tile order.
__global__ void bwd_reduce_bc_kernel(const BwdParams p) {
  const size_t NL = (size_t)p.N * p.L;
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (size_t)p.B * NL) return;
  const size_t b = i / NL, r = i % NL;
  float sb = 0.0f, sc = 0.0f;
  for (int k = 0; k < p.ntiles; ++k) {
    const size_t o = ((b * p.ntiles + k) * 2) * NL + r;
    sb += p.partBC[o];
    sc += p.partBC[o + NL];
  }
  p.dB[i] = sb;
  p.dC[i] = sc;
}

// dA[d,n], dDskip[d], ddt_bias[d]: sum over samples in sample order.
__global__ void bwd_reduce_param_kernel(const BwdParams p) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t DN = (size_t)p.D * p.N;
  if (i < DN) {
    float s = 0.0f;
    for (int b = 0; b < p.B; ++b) s += p.partA[(size_t)b * DN + i];
    p.dA[i] = s;
  }
  if (i < (size_t)p.D) {
    float s0 = 0.0f, s1 = 0.0f;
    for (int b = 0; b < p.B; ++b) {
      s0 += p.partD[(size_t)b * p.D + i];
      s1 += p.partBias[(size_t)b * p.D + i];
    }
    if (p.dDskip) p.dDskip[i] = s0;
    if (p.ddt_bias) p.ddt_bias[i] = s1;
  }
}

// Workspace carve-up: each region starts on a 256-byte boundary.
static size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

size_t bwd_workspace_bytes(int B, int D, int L, int N, int d_tile) {
  const size_t bdl = (size_t)B * D * L, ntiles = (size_t)((D + d_tile - 1) / d_tile);
  size_t s = 0;
  s += 9 * align256(bdl * 4);                           // hbuf, cB, cC, tm_u, tm_dl, tm_gy, tm_du, tm_dd, tm_y
  if (bwd_fast_ok(N, L, d_tile)) s += align256(bdl * N * 4);  // hstore
  s += align256((size_t)B * ntiles * 2 * N * L * 4);    // partBC
  s += align256((size_t)B * D * N * 4);                 // partA
  s += 2 * align256((size_t)B * D * 4);                 // partD, partBias
  return s;
}

void bwd_carve(BwdParams& p, char* ws) {
  const size_t bdl = (size_t)p.B * p.D * p.L;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    float* r = reinterpret_cast<float*>(ws + o);
    o += align256(bytes);
    return r;
  };
  p.hbuf = take(bdl * 4);
  p.cB = take(bdl * 4);
  p.cC = take(bdl * 4);
  p.tm_u = take(bdl * 4);
  p.tm_dl = take(bdl * 4);
  p.tm_gy = take(bdl * 4);
  p.tm_du = take(bdl * 4);
  p.tm_dd = take(bdl * 4);
  p.tm_y = take(bdl * 4);
  p.hstore = bwd_fast_ok(p.N, p.L, p.d_tile) ? take(bdl * p.N * 4) : nullptr;
  p.partBC = take((size_t)p.B * p.ntiles * 2 * p.N * p.L * 4);
  p.partA = take((size_t)p.B * p.D * p.N * 4);
  p.partD = take((size_t)p.B * p.D * 4);
  p.partBias = take((size_t)p.B * p.D * 4);
}

// Built-in workspace of sfm_selective_scan_fold_bwd_noalloc: a file-scope device array
// that every GPU loading this library holds until the process exits.  Host code must not
// pass its name to a kernel (on the host it is only a stand-in); noalloc_scratch() looks
// up its device address once per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SFM_NOALLOC_SCRATCH_BYTES];

cudaError_t noalloc_scratch(void** out) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {  // first call on this device (which is current): take the array's address
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *out = addr[dev];
  return cudaSuccess;
}

template <typename TI, typename TD, bool MIXER>
static cudaError_t launch_main(const BwdParams& p, cudaStream_t s) {
  const int threads = (p.d_tile + 31) & ~31;
  if (p.hstore) {  // two threads per channel, 16 channels per warp
    const int bytes = bwd_fast_smem(p.N, p.L, p.d_tile);
    static SmemLimit lim;
    cudaError_t e = raise_smem_limit(bwd_pair_kernel<TI, TD, MIXER>, bytes, lim);
    if (e != cudaSuccess) return e;
    bwd_pair_kernel<TI, TD, MIXER><<<dim3(p.ntiles, p.B), 2 * ((p.d_tile + 15) & ~15), bytes, s>>>(p);
  } else {
    bwd_main_kernel<TI, TD, MIXER><<<dim3(p.ntiles, p.B), threads, 0, s>>>(p);
  }
  return cudaGetLastError();
}

template <typename TI, typename TD>
static cudaError_t launch_bwd_t(const BwdParams& p, cudaStream_t s) {
  cudaError_t e = launch_main<TI, TD, false>(p, s);
  if (e != cudaSuccess) return e;
  const size_t nbc = (size_t)p.B * p.N * p.L;
  bwd_reduce_bc_kernel<<<(unsigned)((nbc + 255) / 256), 256, 0, s>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t np = (size_t)p.D * p.N > (size_t)p.D ? (size_t)p.D * p.N : (size_t)p.D;
  bwd_reduce_param_kernel<<<(unsigned)((np + 255) / 256), 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_bwd(const BwdParams& p, sfm_dtype in_dtype, sfm_dtype dout_dtype, cudaStream_t s) {
  if (in_dtype == SFM_F32 && dout_dtype == SFM_F32) return launch_bwd_t<float, float>(p, s);
  if (in_dtype == SFM_BF16 && dout_dtype == SFM_BF16) return launch_bwd_t<__nv_bfloat16, __nv_bfloat16>(p, s);
  if (in_dtype == SFM_BF16 && dout_dtype == SFM_F32) return launch_bwd_t<__nv_bfloat16, float>(p, s);
  return cudaErrorInvalidValue;
}

// Conv + SiLU (+ aux init) backward, one warp per (b, d) row: dpre = du * SiLU'(pre) (pre
// recomputed from x), dxa = transposed conv of dpre inside the sample, dx = dxa shifted by
// the aux token plus the mean's share (dxa[0] + dxa[L-1]) / T; per-row partials of dw, db.
template <typename TI>
__global__ void conv_bwd_kernel(const BwdParams p) {
  const int lane = threadIdx.x & 31;
  const long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= (long long)p.B * p.D) return;
  const int d = (int)(r % p.D), L = p.L, Tx = p.Tx, K = p.conv ? p.K : 1, pl = p.conv ? p.pad_left : 0;
  const TI* xr = static_cast<const TI*>(p.x) + r * Tx;
  float mean = 0.0f;
  if (p.aux) {
    for (int t = lane; t < Tx; t += 32) mean += to_f(xr[t]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mean += __shfl_xor_sync(0xffffffffu, mean, o);
    mean /= (float)Tx;
  }
  float* dp = p.u_ws + r * L;      // u is no longer needed: the row holds dpre
  const float* du = p.du + r * L;
  float dw[SFM_MAX_K] = {0.f, 0.f, 0.f, 0.f}, db = 0.0f;
  for (int t = lane; t < L; t += 32) {
    float g = du[t];
    if (p.conv) {
      const float pre = conv_pre(p, xr, t, d, mean), sg = rcp(1.0f + ex2(-pre * kLog2e));
      g *= sg * (1.0f + pre * (1.0f - sg));
#pragma unroll
      for (int k = 0; k < SFM_MAX_K; ++k)
        if (k < K) dw[k] = fmaf(g, xa_row(xr, t + k - pl, L, p.aux, mean), dw[k]);
      db += g;
    }
    dp[t] = g;
  }
  __syncwarp();
  auto dxa = [&](int s) {
    if (!p.conv) return dp[s];
    float acc = 0.0f;
    for (int k = 0; k < K; ++k) {
      const int t = s - k + pl;
      if (t >= 0 && t < L) acc = fmaf(p.conv_w[(size_t)d * K + k], dp[t], acc);
    }
    return acc;
  };
  float* dx = p.dx + r * Tx;
  const float share = p.aux ? (dxa(0) + dxa(L - 1)) / (float)Tx : 0.0f;
  for (int t = lane; t < Tx; t += 32) dx[t] = dxa(p.aux ? t + 1 : t) + share;
  if (p.conv) {
#pragma unroll
    for (int k = 0; k < SFM_MAX_K; ++k)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dw[k] += __shfl_xor_sync(0xffffffffu, dw[k], o);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) db += __shfl_xor_sync(0xffffffffu, db, o);
    if (lane == 0) {
      for (int k = 0; k < K; ++k) p.dw_part[r * K + k] = dw[k];
      p.db_part[r] = db;
    }
  }
}

// dconv_w[d,k], dconv_b[d]: sum of the per-sample partials in sample order.
__global__ void conv_reduce_kernel(const BwdParams p) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t DK = (size_t)p.D * p.K;
  if (i < DK) {
    float s = 0.0f;
    for (int b = 0; b < p.B; ++b) s += p.dw_part[(size_t)b * DK + i];
    p.dconv_w[i] = s;
  }
  if (i < (size_t)p.D && p.dconv_b) {
    float s = 0.0f;
    for (int b = 0; b < p.B; ++b) s += p.db_part[(size_t)b * p.D + i];
    p.dconv_b[i] = s;
  }
}

size_t mixer_bwd_workspace_bytes(int B, int D, int L, int N, int K, int d_tile) {
  const size_t bdl = (size_t)B * D * L;
  return bwd_workspace_bytes(B, D, L, N, d_tile) + 2 * align256(bdl * 4) + align256((size_t)B * D * K * 4) +
         align256((size_t)B * D * 4);
}

void mixer_bwd_carve(BwdParams& p, char* ws) {
  bwd_carve(p, ws);
  size_t o = bwd_workspace_bytes(p.B, p.D, p.L, p.N, p.d_tile);
  const size_t bdl = (size_t)p.B * p.D * p.L;
  p.u_ws = reinterpret_cast<float*>(ws + o);
  o += align256(bdl * 4);
  p.du = reinterpret_cast<float*>(ws + o);  // the scan input's gradient stays internal
  o += align256(bdl * 4);
  p.dw_part = reinterpret_cast<float*>(ws + o);
  o += align256((size_t)p.B * p.D * (p.K > 0 ? p.K : 1) * 4);
  p.db_part = reinterpret_cast<float*>(ws + o);
}

template <typename TI, typename TD>
static cudaError_t launch_mixer_bwd_t(const BwdParams& p, cudaStream_t s) {
  cudaError_t e = launch_main<TI, TD, true>(p, s);
  if (e != cudaSuccess) return e;
  const size_t nbc = (size_t)p.B * p.N * p.L;
  bwd_reduce_bc_kernel<<<(unsigned)((nbc + 255) / 256), 256, 0, s>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t np = (size_t)p.D * p.N > (size_t)p.D ? (size_t)p.D * p.N : (size_t)p.D;
  bwd_reduce_param_kernel<<<(unsigned)((np + 255) / 256), 256, 0, s>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const long long rows = (long long)p.B * p.D;
  conv_bwd_kernel<TI><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (p.conv) {
    const size_t nc = (size_t)p.D * p.K > (size_t)p.D ? (size_t)p.D * p.K : (size_t)p.D;
    conv_reduce_kernel<<<(unsigned)((nc + 255) / 256), 256, 0, s>>>(p);
    e = cudaGetLastError();
  }
  return e;
}

cudaError_t launch_mixer_bwd(const BwdParams& p, sfm_dtype in_dtype, sfm_dtype dout_dtype, cudaStream_t s) {
  if (in_dtype == SFM_F32 && dout_dtype == SFM_F32) return launch_mixer_bwd_t<float, float>(p, s);
  if (in_dtype == SFM_BF16 && dout_dtype == SFM_BF16) return launch_mixer_bwd_t<__nv_bfloat16, __nv_bfloat16>(p, s);
  if (in_dtype == SFM_BF16 && dout_dtype == SFM_F32) return launch_mixer_bwd_t<__nv_bfloat16, float>(p, s);
  return cudaErrorInvalidValue;
}

}  // namespace sfm
