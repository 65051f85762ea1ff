// sfm_fwd.cu -- fused forward of the SF-Mamba mixer hot path on B200 (sm_100a).
//
// One launch computes, for a tile of channels and one folded row of B2 samples:
//   [aux init] -> depthwise conv (zero outside the sample) + SiLU -> Delta = softplus
//   -> selective scan with the state restarted at every sample start -> D skip
//   -> SiLU(z) gate -> [head<->tail swap] -> store.
// Sources: "Seeing Both Ways, Running One Way" (sungsoo.github.io) sections 3.1-3.3 and 8.1;
// "SF-Mamba：重新思考视觉 Mamba 的信息流与并行效率" (techloop.online), Auxiliary Patch Swapping and
// Batch Folding with Periodic State Reset.
//
// Schedule.  Grid = (channel tiles, B1 folded rows).  Each thread owns one channel and
// walks the folded row p = 0 .. B2*L-1 in order with its N fp32 states in registers
// (packed in pairs for the f32x2 FMA pipe).  The reset at p mod L == 0 makes the
// transition factor of every sample's first token 0: the state restarts there and no
// exp is evaluated.  The work is bound by the transcendental unit (N exp2 per token),
// so the inner loop is built to keep it fed: interior tokens are processed in unrolled
// groups with branch-free conv windows, so that one token's exps overlap the previous
// token's state updates; tokens whose conv window touches an aux token or the
// sample's zero padding (at most K per sample) take a general path.
//
// Staging, two modes:
//  * whole-sample: when a sample's rows fit in shared memory and every slab is 16-byte
//    aligned, the CTA's slab of each tensor -- [b, d0:d0+Dt, :], contiguous in memory --
//    arrives with ONE bulk asynchronous copy (the TMA engine, no multicast) completing
//    on an mbarrier, and the output slab leaves with one bulk store.
//  * chunked: tokens are staged in chunks; each row segment is copied with 16-byte
//    cp.async granules starting at the granule that holds its first element (rows of
//    odd length are never 16-byte aligned, which rules out tensor maps and per-row bulk
//    copies), and each thread reads its row at that row's byte offset.
// B and C of the staged tokens are transposed once per CTA into fp32 [token][2N] so a
// thread reads the N values of a token as 128-bit broadcast loads.
#include <type_traits>

#include "sfm_device.cuh"
#include "sfm_internal.h"

namespace sfm {

__device__ unsigned int g_device_error = 0;

#ifndef SFM_FWD_GROUP
#define SFM_FWD_GROUP 4
#endif
constexpr int kGroup = SFM_FWD_GROUP;  // tokens per unrolled group

__host__ __device__ inline int round16(int v) { return (v + 15) & ~15; }

// Row stride (bytes) of a staged row of `cnt` elements (chunked mode): room for the
// up-to-15 head bytes of the granule copy, and an odd number of 16-byte units.
__host__ __device__ inline int stage_row_bytes(int cnt, int esize) {
  int b = round16(cnt * esize + 15);
  if (((b >> 4) & 1) == 0) b += 16;
  return b;
}

// Output row stride when the output cannot overwrite the dt row in place (chunked mode).
__host__ __device__ inline int out_row_bytes(int cnt, int esize) {
  int b = (cnt * esize + 3) & ~3;
  if (((b >> 2) & 1) == 0) b += 4;
  return b;
}

// ------------------------------------------------------------------ bulk copy

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void bulk_s2g(void* dst, const void* src, unsigned bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;\n" ::"l"(dst), "r"(smem_u32(src)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }

// ------------------------------------------------------------------ per-token arithmetic

// Per-channel constants and state.  NH = pairs of states (N padded to an even count;
// padded states have A = B = C = 0 and stay 0).
template <int NH>
struct Chan {
  float2 h[NH];
  float2 A2[NH];  // A * log2(e)
  float w[4];
  float cb, dsk, dtb, mean;
};

// State update and read-out of one token:
//   h = Abar*h + Delta*B*u (Abar = 0 on a reset token), returns sum_n C_n h_n.
// The exp2 of the first PE state pairs runs on the FMA pipe (exp2_fma2), the rest on the
// transcendental unit, so that both pipes share the N exponentials.
template <int NH, bool RESET, int PE>
__device__ __forceinline__ float scan_token(Chan<NH>& c, const float* __restrict__ bc, float delta, float dbu) {
  const float2 d2 = make_float2(delta, delta), u2 = make_float2(dbu, dbu);
  float2 ya = make_float2(0.f, 0.f), yb = make_float2(0.f, 0.f);
#pragma unroll
  for (int k = 0; k < NH; k += (NH % 2 == 0 ? 2 : 1)) {
    float2 Bp[2], Cp[2];
    if constexpr (NH % 2 == 0) {
      const float4 b4 = *reinterpret_cast<const float4*>(bc + 2 * k);
      const float4 c4 = *reinterpret_cast<const float4*>(bc + 2 * NH + 2 * k);
      Bp[0] = make_float2(b4.x, b4.y);
      Bp[1] = make_float2(b4.z, b4.w);
      Cp[0] = make_float2(c4.x, c4.y);
      Cp[1] = make_float2(c4.z, c4.w);
    } else {
      Bp[0] = *reinterpret_cast<const float2*>(bc + 2 * k);
      Cp[0] = *reinterpret_cast<const float2*>(bc + 2 * NH + 2 * k);
    }
#pragma unroll
    for (int j = 0; j < (NH % 2 == 0 ? 2 : 1); ++j) {
      const float2 bu = __fmul2_rn(Bp[j], u2);
      if constexpr (RESET) {
        c.h[k + j] = bu;
      } else {
        float2 a = __fmul2_rn(d2, c.A2[k + j]);
        if (k + j < PE) {
          a = exp2_fma2(a);
        } else {
          a.x = ex2(a.x);
          a.y = ex2(a.y);
        }
        c.h[k + j] = __ffma2_rn(a, c.h[k + j], bu);
      }
      if (j == 0)
        ya = __ffma2_rn(Cp[j], c.h[k + j], ya);
      else
        yb = __ffma2_rn(Cp[j], c.h[k + j], yb);
    }
  }
  const float2 s = __fadd2_rn(ya, yb);
  return s.x + s.y;
}

// Runtime options of the general path.
struct Opts {
  int L, K, pl, off, Tx;  // off = 1 with aux tokens
  bool conv, gate, sp, aux;
};

// Output of one token from its conv taps (xw[0..3] = xa[t-pl .. t-pl+3]), raw dt and z.
// STD: conv (K = 4) + softplus + gate, all compile-time; else the runtime options.
// FAST: one-transcendental SiLU and softplus (used when the output is rounded to bf16).
template <typename TI, int NH, bool STD, bool RESET, bool FAST, int PE>
__device__ __forceinline__ float token_out(Chan<NH>& c, const Opts& o, const float* xw, TI dtv, TI zv,
                                           const float* __restrict__ bc) {
  float u;
  if (STD || o.conv) {
    float acc = c.cb;
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (STD || q < o.K) acc = fmaf(c.w[q], xw[q], acc);
    u = FAST ? silu_fast(acc) : silu(acc);
  } else {
    u = xw[0];
  }
  const float v = to_f(dtv) + c.dtb;
  const float delta = (STD || o.sp) ? (FAST ? softplus_fast(v) : softplus(v)) : v;
  float yv = scan_token<NH, RESET, PE>(c, bc, delta, delta * u);
  yv = fmaf(c.dsk, u, yv);
  if (STD || o.gate) {
    const float zf = to_f(zv);
    yv *= FAST ? silu_fast(zf) : silu(zf);
  }
  return yv;
}

// CPT channels of one thread, one token: the B and C loads of the token are shared.
template <int NH, bool RESET, int PE, int CPT>
__device__ __forceinline__ void scan_token_multi(Chan<NH> (&c)[CPT], const float* __restrict__ bc,
                                                 const float (&delta)[CPT], const float (&dbu)[CPT],
                                                 float (&y)[CPT]) {
  float2 ya[CPT], yb[CPT];
#pragma unroll
  for (int ch = 0; ch < CPT; ++ch) ya[ch] = yb[ch] = make_float2(0.f, 0.f);
#pragma unroll
  for (int k = 0; k < NH; k += (NH % 2 == 0 ? 2 : 1)) {
    float2 Bp[2], Cp[2];
    if constexpr (NH % 2 == 0) {
      const float4 b4 = *reinterpret_cast<const float4*>(bc + 2 * k);
      const float4 c4 = *reinterpret_cast<const float4*>(bc + 2 * NH + 2 * k);
      Bp[0] = make_float2(b4.x, b4.y);
      Bp[1] = make_float2(b4.z, b4.w);
      Cp[0] = make_float2(c4.x, c4.y);
      Cp[1] = make_float2(c4.z, c4.w);
    } else {
      Bp[0] = *reinterpret_cast<const float2*>(bc + 2 * k);
      Cp[0] = *reinterpret_cast<const float2*>(bc + 2 * NH + 2 * k);
    }
#pragma unroll
    for (int j = 0; j < (NH % 2 == 0 ? 2 : 1); ++j) {
#pragma unroll
      for (int ch = 0; ch < CPT; ++ch) {
        const float2 bu = __fmul2_rn(Bp[j], make_float2(dbu[ch], dbu[ch]));
        if constexpr (RESET) {
          c[ch].h[k + j] = bu;
        } else {
          float2 a = __fmul2_rn(make_float2(delta[ch], delta[ch]), c[ch].A2[k + j]);
          if (k + j < PE) {
            a = exp2_fma2(a);
          } else {
            a.x = ex2(a.x);
            a.y = ex2(a.y);
          }
          c[ch].h[k + j] = __ffma2_rn(a, c[ch].h[k + j], bu);
        }
        if (j == 0)
          ya[ch] = __ffma2_rn(Cp[j], c[ch].h[k + j], ya[ch]);
        else
          yb[ch] = __ffma2_rn(Cp[j], c[ch].h[k + j], yb[ch]);
      }
    }
  }
#pragma unroll
  for (int ch = 0; ch < CPT; ++ch) {
    const float2 s2 = __fadd2_rn(ya[ch], yb[ch]);
    y[ch] = s2.x + s2.y;
  }
}

// CPT channels, one interior token (standard mixer path); xw[ch][0..3] are the taps.
template <typename TI, int NH, bool STD, bool FAST, int PE, int CPT>
__device__ __forceinline__ void token_out_multi(Chan<NH> (&c)[CPT], const Opts& o, const float* const (&xw)[CPT],
                                                const TI (&dtv)[CPT], const TI (&zv)[CPT],
                                                const float* __restrict__ bc, float (&yo)[CPT]) {
  float u[CPT], delta[CPT], dbu[CPT];
#pragma unroll
  for (int ch = 0; ch < CPT; ++ch) {
    if (STD || o.conv) {
      float acc = c[ch].cb;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (STD || q < o.K) acc = fmaf(c[ch].w[q], xw[ch][q], acc);
      u[ch] = FAST ? silu_fast(acc) : silu(acc);
    } else {
      u[ch] = xw[ch][0];
    }
    const float v = to_f(dtv[ch]) + c[ch].dtb;
    delta[ch] = (STD || o.sp) ? (FAST ? softplus_fast(v) : softplus(v)) : v;
    dbu[ch] = delta[ch] * u[ch];
  }
  float ys[CPT];
  scan_token_multi<NH, false, PE, CPT>(c, bc, delta, dbu, ys);
#pragma unroll
  for (int ch = 0; ch < CPT; ++ch) {
    float yv = fmaf(c[ch].dsk, u[ch], ys[ch]);
    if (STD || o.gate) {
      const float zf = to_f(zv[ch]);
      yv *= FAST ? silu_fast(zf) : silu(zf);
    }
    yo[ch] = yv;
  }
}

// xa at position s of the sample from the x row `xr` (x index q at xr[q - xlo]); aux
// tokens are the mean; zero outside the sample or outside the staged window.
template <typename TI>
__device__ __forceinline__ float xa_at(const Opts& o, const TI* xr, int xlo, int xhi, float mean, int s) {
  if (s < 0 || s >= o.L) return 0.0f;
  if (o.aux) {
    if (s == 0 || s == o.L - 1) return mean;
    s -= 1;
  }
  if (s < xlo || s >= xhi) return 0.0f;
  return to_f(xr[s - xlo]);
}

// General path for token t (chunk-relative i): conv taps with explicit boundary handling.
template <typename TI, typename TO, int NH, bool STD, bool FAST, int PE>
__device__ __forceinline__ float general_token(Chan<NH>& c, const Opts& o, const TI* xr, int xlo, int xhi, int t,
                                               TI dtv, TI zv, const float* bc) {
  float xw[4];
  const int K = (STD || o.conv) ? 4 : 1, pl = (STD || o.conv) ? o.pl : 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) xw[q] = q < K ? xa_at<TI>(o, xr, xlo, xhi, c.mean, t - pl + q) : 0.0f;
  if (t == 0) return token_out<TI, NH, STD, true, FAST, PE>(c, o, xw, dtv, zv, bc);
  return token_out<TI, NH, STD, false, FAST, PE>(c, o, xw, dtv, zv, bc);
}

// G interior tokens of CPT channels starting at chunk-relative index i: loads first (x
// windows, dt, z), then the token computations, then the stores, so the compiler can
// overlap tokens and channels.  xb[ch][i + q] is conv tap q of token i of channel ch.
template <typename TI, typename TO, int NH, bool STD, bool FAST, int PE, int G, int CPT>
__device__ __forceinline__ void fast_group(Chan<NH> (&c)[CPT], const Opts& o, const TI* const (&xb)[CPT],
                                           const TI* const (&dtr)[CPT], const TI* const (&zr)[CPT],
                                           TO* const (&yr)[CPT], int i, const float* __restrict__ bct) {
  constexpr int NP2 = 4 * NH;  // floats per token in bct
  float xv[CPT][G + 3];
  TI dv[CPT][G], zv[CPT][G];
#pragma unroll
  for (int ch = 0; ch < CPT; ++ch) {
#pragma unroll
    for (int q = 0; q < G + 3; ++q) xv[ch][q] = (q < G || STD || o.conv) ? to_f(xb[ch][i + q]) : 0.0f;
#pragma unroll
    for (int k = 0; k < G; ++k) {
      dv[ch][k] = dtr[ch][i + k];
      zv[ch][k] = (STD || o.gate) ? zr[ch][i + k] : dv[ch][k];
    }
  }
  float yv[G][CPT];
#pragma unroll
  for (int k = 0; k < G; ++k) {
    const float* xw[CPT];
    TI d1[CPT], z1[CPT];
#pragma unroll
    for (int ch = 0; ch < CPT; ++ch) {
      xw[ch] = xv[ch] + k;
      d1[ch] = dv[ch][k];
      z1[ch] = zv[ch][k];
    }
    token_out_multi<TI, NH, STD, FAST, PE, CPT>(c, o, xw, d1, z1, bct + (i + k) * NP2, yv[k]);
  }
#pragma unroll
  for (int k = 0; k < G; ++k)
#pragma unroll
    for (int ch = 0; ch < CPT; ++ch) yr[ch][i + k] = from_f<TO>(yv[k][ch]);
}

// Walks tokens [t0, t0 + cnt) of one sample for the thread's CPT channels.  xr[ch]: x
// row holding x indices [xlo, xhi); dtr/zr/yr: rows indexed chunk-relative; bct:
// transposed B/C of the chunk.  Edge tokens take the general path channel by channel.
template <typename TI, typename TO, int NH, bool STD, bool FAST, int PE, int CPT>
__device__ __forceinline__ void walk(Chan<NH> (&c)[CPT], const Opts& o, const TI* const (&xr)[CPT], int xlo,
                                     int xhi, const TI* const (&dtr)[CPT], const TI* const (&zr)[CPT],
                                     TO* const (&yr)[CPT], const float* bct, int t0, int cnt) {
  constexpr int NP2 = 4 * NH;
  // interior tokens: every conv tap on a plain x token; never the reset token
  int ta = 1, tb = 0;
  if (STD) {
    ta = max(o.off + o.pl, 1);
    tb = o.off + o.Tx - 4 + o.pl + 1;
  }
  const int tend = t0 + cnt;
  const int e1 = min(tend, max(t0, ta));
  const int e2 = max(e1, min(tend, tb));
  for (int t = t0; t < e1; ++t) {
    const int i = t - t0;
#pragma unroll
    for (int ch = 0; ch < CPT; ++ch)
      yr[ch][i] = from_f<TO>(general_token<TI, TO, NH, STD, FAST, PE>(c[ch], o, xr[ch], xlo, xhi, t, dtr[ch][i],
                                                                       zr[ch][i], bct + i * NP2));
  }
  if (e2 > e1) {
    // x index of tap 0 of token t is t - pl - off; xb[i + q] must be that + q
    const TI* xb[CPT];
#pragma unroll
    for (int ch = 0; ch < CPT; ++ch) xb[ch] = xr[ch] + (t0 - o.pl - o.off - xlo);
    int i = e1 - t0;
    const int iend = e2 - t0;
    for (; i + kGroup <= iend; i += kGroup)
      fast_group<TI, TO, NH, STD, FAST, PE, kGroup, CPT>(c, o, xb, dtr, zr, yr, i, bct);
    for (; i < iend; ++i) fast_group<TI, TO, NH, STD, FAST, PE, 1, CPT>(c, o, xb, dtr, zr, yr, i, bct);
  }
  for (int t = e2; t < tend; ++t) {
    const int i = t - t0;
#pragma unroll
    for (int ch = 0; ch < CPT; ++ch)
      yr[ch][i] = from_f<TO>(general_token<TI, TO, NH, STD, FAST, PE>(c[ch], o, xr[ch], xlo, xhi, t, dtr[ch][i],
                                                                       zr[ch][i], bct + i * NP2));
  }
}

template <int NH>
__device__ __forceinline__ void load_chan(Chan<NH>& c, const FwdParams& p, int d, bool conv) {
  const int N = p.N;
#pragma unroll
  for (int k = 0; k < NH; ++k) {
    const int n0 = 2 * k, n1 = 2 * k + 1;
    c.A2[k] = make_float2(n0 < N ? p.A[(size_t)d * N + n0] * kLog2e : 0.f,
                          n1 < N ? p.A[(size_t)d * N + n1] * kLog2e : 0.f);
    c.h[k] = make_float2(0.f, 0.f);
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) c.w[q] = (conv && q < p.K) ? p.conv_w[(size_t)d * p.K + q] : 0.0f;
  c.cb = (conv && p.conv_b) ? p.conv_b[d] : 0.0f;
  c.dsk = p.Dskip ? p.Dskip[d] : 0.0f;
  c.dtb = p.dt_bias ? p.dt_bias[d] : 0.0f;
  c.mean = 0.0f;
}

// B, C [N][cnt] (raw, element (n,i) at src + head_n + i*si) -> fp32 [cnt][4*NH] (B pairs
// then C pairs), zero for padded states.
template <typename TI, int NH>
__device__ __forceinline__ void transpose_bc(float* bct, const char* bs, const char* cs, int row_bytes,
                                             unsigned e0_base, unsigned L, int N, int cnt, int tid, int nthr,
                                             bool per_row_head) {
  constexpr int NP = 2 * NH, si = sizeof(TI);
  for (int e = tid; e < cnt * NP; e += nthr) {
    const int i = e / NP, n = e % NP;
    float bv = 0.0f, cv = 0.0f;
    if (n < N) {
      // only the low 4 bits of the byte offset matter: 32-bit arithmetic is exact there
      const int hb = per_row_head ? (int)(((e0_base + (unsigned)n * L) * si) & 15u) : 0;
      const int off = n * row_bytes + hb + i * si;
      bv = to_f(*reinterpret_cast<const TI*>(bs + off));
      cv = to_f(*reinterpret_cast<const TI*>(cs + off));
    }
    bct[i * 2 * NP + n] = bv;
    bct[i * 2 * NP + NP + n] = cv;
  }
}

template <typename TI>
__device__ __forceinline__ float row_mean(const TI* xr, int Tx) {
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
  int t = 0;
  for (; t + 4 <= Tx; t += 4) {
    s0 += to_f(xr[t]);
    s1 += to_f(xr[t + 1]);
    s2 += to_f(xr[t + 2]);
    s3 += to_f(xr[t + 3]);
  }
  for (; t < Tx; ++t) s0 += to_f(xr[t]);
  return ((s0 + s1) + (s2 + s3)) / (float)Tx;
}

__device__ __forceinline__ Opts make_opts(const FwdParams& p) {
  Opts o;
  o.L = p.L;
  o.conv = p.flags & kConv;
  o.gate = p.flags & kGate;
  o.sp = p.flags & kSoftplus;
  o.aux = p.flags & kAuxInit;
  o.K = o.conv ? p.K : 1;
  o.pl = o.conv ? p.pad_left : 0;
  o.off = o.aux ? 1 : 0;
  o.Tx = p.Tx;
  return o;
}

// ------------------------------------------------------------------ whole-sample mode

// Shared memory: [barrier 16 B][x slab][dt slab][z slab][B][C][bct][y slab if not in place]
// Thread tid owns the CPT adjacent channels CPT*tid .. CPT*tid + CPT-1 of the tile.
template <typename TI, typename TO, int NH, bool STD, int PE, int CPT>
__global__ void __launch_bounds__(128) fwd_whole_kernel(const FwdParams p) {
  constexpr bool kInPlace = std::is_same<TI, TO>::value;
  constexpr bool kFast = std::is_same<TO, __nv_bfloat16>::value;
  constexpr int si = sizeof(TI), so = sizeof(TO), NP = 2 * NH;
  extern __shared__ __align__(16) char smem[];

  const int tid = threadIdx.x, nthr = blockDim.x;
  const int d0 = blockIdx.x * p.d_tile;
  const int dcount = min(p.d_tile, p.D - d0);
  const int b1 = blockIdx.y;
  const int c0 = tid * CPT;          // first channel of this thread within the tile
  const bool active = c0 < dcount;   // the host keeps dcount a multiple of CPT
  const int L = p.L, N = p.N, Tx = p.Tx;
  const Opts o = make_opts(p);
  const bool swap = p.flags & kSwapOut;

  uint64_t* bar = reinterpret_cast<uint64_t*>(smem);
  volatile int& abort_flag = *reinterpret_cast<int*>(smem + 8);
  char* xs = smem + 16;
  char* dts = xs + round16(p.d_tile * Tx * si);
  char* zs = dts + round16(p.d_tile * L * si);
  char* bs = zs + (o.gate ? round16(p.d_tile * L * si) : 0);
  char* cs = bs + round16(N * L * si);
  float* bct = reinterpret_cast<float*>(cs + round16(N * L * si));
  char* ys = reinterpret_cast<char*>(bct + L * 2 * NP);

  if (tid == 0) {
    mbar_init(bar, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  __syncthreads();

  Chan<NH> c[CPT];
#pragma unroll
  for (int ch = 0; ch < CPT; ++ch) load_chan(c[ch], p, d0 + (active ? c0 + ch : 0), o.conv);

  const unsigned xbytes = (unsigned)(dcount * Tx * si), iobytes = (unsigned)(dcount * L * si);
  const unsigned bcbytes = (unsigned)(N * L * si), ybytes = (unsigned)(dcount * L * so);
  const char* xg = static_cast<const char*>(p.x);
  const char* dtg = static_cast<const char*>(p.dt);
  const char* zg = static_cast<const char*>(p.z);
  const char* bg = static_cast<const char*>(p.Bm);
  const char* cg = static_cast<const char*>(p.Cm);
  char* yg = static_cast<char*>(p.y);

  for (int j = 0; j < p.B2; ++j) {
    const int b = b1 * p.B2 + j;
    const long long row0 = (long long)b * p.D + d0;
    if (tid == 0) {
      if (j > 0) bulk_wait_read0();  // the previous output slab has been read out of smem
      fence_proxy_async();
      mbar_expect_tx(bar, xbytes + iobytes * (o.gate ? 2u : 1u) + 2u * bcbytes);
      bulk_g2s(xs, xg + row0 * Tx * si, xbytes, bar);
      bulk_g2s(dts, dtg + row0 * L * si, iobytes, bar);
      if (o.gate) bulk_g2s(zs, zg + row0 * L * si, iobytes, bar);
      bulk_g2s(bs, bg + (long long)b * N * L * si, bcbytes, bar);
      bulk_g2s(cs, cg + (long long)b * N * L * si, bcbytes, bar);
      if (!mbar_wait_bounded(bar, j & 1)) {
        atomicExch(&g_device_error, (unsigned)SFM_ERR_TIMEOUT);
        mbar_wait_bounded(bar, j & 1);  // give the copies in flight one more bounded chance
        abort_flag = 1;
      }
    }
    __syncthreads();
    if (abort_flag) {
      if (tid == 0) bulk_wait0();
      return;
    }
    mbar_try_wait(bar, j & 1);  // completed: acquire the copied bytes in every thread

    transpose_bc<TI, NH>(bct, bs, cs, L * si, 0u, (unsigned)L, N, L, tid, nthr, false);
    if (active && o.aux)
#pragma unroll
      for (int ch = 0; ch < CPT; ++ch) c[ch].mean = row_mean(reinterpret_cast<const TI*>(xs) + (c0 + ch) * Tx, Tx);
    __syncthreads();

    if (active) {
      const TI* xr[CPT];
      const TI* dtr[CPT];
      const TI* zr[CPT];
      TO* yr[CPT];
#pragma unroll
      for (int ch = 0; ch < CPT; ++ch) {
        xr[ch] = reinterpret_cast<const TI*>(xs) + (c0 + ch) * Tx;
        dtr[ch] = reinterpret_cast<const TI*>(dts) + (c0 + ch) * L;
        zr[ch] = o.gate ? reinterpret_cast<const TI*>(zs) + (c0 + ch) * L : dtr[ch];
        yr[ch] = kInPlace ? reinterpret_cast<TO*>(dts) + (c0 + ch) * L : reinterpret_cast<TO*>(ys) + (c0 + ch) * L;
#pragma unroll
        for (int k = 0; k < NH; ++k) c[ch].h[k] = make_float2(0.f, 0.f);
      }
      walk<TI, TO, NH, STD, kFast, PE, CPT>(c, o, xr, 0, Tx, dtr, zr, yr, bct, 0, L);
#pragma unroll
      for (int ch = 0; ch < CPT; ++ch) {
        if (swap) {
          const TO h0 = yr[ch][0];
          yr[ch][0] = yr[ch][L - 1];
          yr[ch][L - 1] = h0;
        }
        if (p.final_state) {
          float* fs = p.final_state + ((size_t)b * p.D + d0 + c0 + ch) * N;
#pragma unroll
          for (int k = 0; k < NH; ++k) {
            if (2 * k < N) fs[2 * k] = c[ch].h[k].x;
            if (2 * k + 1 < N) fs[2 * k + 1] = c[ch].h[k].y;
          }
        }
      }
    }
    __syncthreads();
    if (tid == 0) {
      fence_proxy_async();  // the threads' smem writes become visible to the bulk store
      bulk_s2g(yg + row0 * L * so, kInPlace ? dts : ys, ybytes);
      bulk_commit();
    }
  }
  if (tid == 0) bulk_wait0();
}

// ------------------------------------------------------------------ chunked mode

// Two staging buffers: while the threads work on step s (a chunk of one sample), the
// copies of step s+1 (the next chunk, or the first chunk of the next sample of the folded
// row) are in flight.  Buffer layout per stage: [x rows][dt rows][z rows][B rows][C rows];
// after both stages: [bct][y rows if not in place].
//
// The samples of a folded row are either the fixed [B,D,L] layout (sample s at element
// s*D*L, every sample L long) or the ragged packed layout (sample s at packed offset
// cu_seqlens[s] of rows that are the packed length long, its own length
// cu_seqlens[s+1] - cu_seqlens[s]); in both the state restarts at each sample's first
// token and the conv never reads across a sample boundary.
template <typename TI, typename TO, int NH, bool STD, int PE, int CPT>
__global__ void __launch_bounds__(128) fwd_chunk_kernel(const FwdParams p) {
  constexpr bool kInPlace = std::is_same<TI, TO>::value;
  constexpr bool kFast = std::is_same<TO, __nv_bfloat16>::value;
  constexpr int si = sizeof(TI), so = sizeof(TO), NP = 2 * NH;
  extern __shared__ __align__(16) char smem[];

  const int tid = threadIdx.x, nthr = blockDim.x;
  const int lane = tid & 31, warp = tid >> 5, nwarps = nthr >> 5;
  const int d0 = blockIdx.x * p.d_tile;
  const int dcount = min(p.d_tile, p.D - d0);
  const int c0 = tid * CPT;
  const bool active = c0 < dcount;
  const int N = p.N, S = p.chunk;
  Opts o = make_opts(p);  // o.L and o.Tx follow the sample being walked
  const bool swap = p.flags & kSwapOut;
  const int K = o.conv ? o.K : 1, pl = o.pl;
  const int s0 = blockIdx.y * p.B2, ns = min(p.B2, p.B - s0);  // this folded row's samples

  const int stage_bytes = p.d_tile * p.x_row + p.d_tile * p.io_row * (o.gate ? 2 : 1) + 2 * N * p.io_row;
  float* bct = reinterpret_cast<float*>(smem + 2 * stage_bytes);
  char* ys = reinterpret_cast<char*>(bct + S * 2 * NP);
  auto xs_of = [&](int st) { return smem + st * stage_bytes; };
  auto dts_of = [&](int st) { return xs_of(st) + p.d_tile * p.x_row; };
  auto zs_of = [&](int st) { return dts_of(st) + p.d_tile * p.io_row; };
  auto bs_of = [&](int st) { return zs_of(st) + (o.gate ? p.d_tile * p.io_row : 0); };
  auto cs_of = [&](int st) { return bs_of(st) + N * p.io_row; };

  Chan<NH> c[CPT];
#pragma unroll
  for (int ch = 0; ch < CPT; ++ch) load_chan(c[ch], p, d0 + (active ? c0 + ch : 0), o.conv);

  const long long x_bytes = p.x_elems * si, io_bytes = p.io_elems * si, bc_bytes = p.bc_elems * si;
  const char* xg = static_cast<const char*>(p.x);
  const char* dtg = static_cast<const char*>(p.dt);
  const char* zg = static_cast<const char*>(p.z);
  const char* bg = static_cast<const char*>(p.Bm);
  const char* cg = static_cast<const char*>(p.Cm);
  TO* yg = static_cast<TO*>(p.y);

  // One step = chunk kc of sample s0 + j.  len/tx: the sample's tokens (with aux) and x
  // tokens; xb, ib, bb: element offsets of its channel-0 x row, channel-0 dt/z/y row and
  // state-0 B/C row.  A sample with len 0 has no steps.
  struct Step {
    int j, kc, len, tx;
    long long xb, ib, bb;
  };
  auto load_sample = [&](Step& q) {
    const int s = s0 + q.j;
    if (!p.cu_seqlens) {
      q.len = p.L;
      q.tx = p.Tx;
      q.xb = (long long)s * p.D * p.Tx;
      q.ib = (long long)s * p.D * p.L;
      q.bb = (long long)s * N * p.L;
      return;
    }
    const int a = p.cu_seqlens[s], e = p.cu_seqlens[s + 1];
    // offsets out of order or out of the packed rows, or an aux sample without a patch
    // token: reported in the device error word; the sample is skipped, nothing is read
    const bool bad = a < 0 || e < a || e > p.L ||
                     (o.aux && (e - a < 3 || a - 2LL * s < 0 || e - 2LL * s - 2 > p.Tx));
    if (bad) {
      if (tid == 0) atomicExch(&g_device_error, (unsigned)SFM_ERR_INVALID_ARG);
      q.len = 0;
      return;
    }
    q.len = e - a;
    q.tx = o.aux ? q.len - 2 : q.len;
    q.xb = o.aux ? a - 2LL * s : a;
    q.ib = a;
    q.bb = a;
  };
  // moves q to the first step at or after (q.j, q.kc) that has tokens
  auto settle = [&](Step& q) {
    while (q.j < ns) {
      if (q.kc == 0) load_sample(q);
      if (q.kc * S < q.len) return;
      ++q.j;
      q.kc = 0;
    }
  };

  // x tokens a chunk needs: xa positions [t0-pl, t0+cnt-1+K-1-pl], clamped to the sample
  auto x_window = [&](int t0, int cnt, int tx, int& xlo, int& xhi) {
    const int slo = t0 - pl - o.off, shi = t0 + cnt - 1 + (K - 1 - pl) - o.off;
    xlo = max(slo, 0);
    xhi = min(shi + 1, tx);
  };
  // issues the copies of step q into buffer `buf` (each thread its own rows; threads
  // 0..2N-1 the B and C rows) and commits them as one group
  auto stage = [&](const Step& q, int buf) {
    const int t0 = q.kc * S, cnt = min(S, q.len - t0);
    int xlo, xhi;
    x_window(t0, cnt, q.tx, xlo, xhi);
    if (active) {
#pragma unroll
      for (int ch = 0; ch < CPT; ++ch) {
        const int r = c0 + ch;
        const long long xrow = q.xb + (d0 + r) * p.x_cs, iorow = q.ib + (d0 + r) * p.io_cs;
        copy_span_async(xs_of(buf) + r * p.x_row, xg, xrow + xlo, xhi - xlo, si, x_bytes, 0, 1);
        copy_span_async(dts_of(buf) + r * p.io_row, dtg, iorow + t0, cnt, si, io_bytes, 0, 1);
        if (o.gate) copy_span_async(zs_of(buf) + r * p.io_row, zg, iorow + t0, cnt, si, io_bytes, 0, 1);
      }
    }
    for (int r = tid; r < 2 * N; r += nthr) {
      const int n = r % N;
      const long long e0 = q.bb + n * p.bc_cs + t0;
      copy_span_async((r < N ? bs_of(buf) : cs_of(buf)) + n * p.io_row, r < N ? bg : cg, e0, cnt, si, bc_bytes, 0,
                      1);
    }
    cp_async_commit();
  };

  TO head_val[CPT];
  Step cur{0, 0, 0, 0, 0, 0, 0};
  settle(cur);
  if (cur.j < ns) stage(cur, 0);
  for (int it = 0; cur.j < ns; ++it) {
    const int buf = it & 1;
    Step nxt = cur;
    ++nxt.kc;
    settle(nxt);
    const int s = s0 + cur.j, kc = cur.kc;
    const int t0 = kc * S, cnt = min(S, cur.len - t0);
    const bool last = t0 + cnt == cur.len;
    o.L = cur.len;
    o.Tx = cur.tx;
    int xlo, xhi;
    x_window(t0, cnt, cur.tx, xlo, xhi);
    if (kc == 0) {  // a new sample: the state restarts; the aux mean needs the whole x row
#pragma unroll
      for (int ch = 0; ch < CPT; ++ch) {
        c[ch].mean = (o.aux && active) ? row_mean(reinterpret_cast<const TI*>(xg) + cur.xb +
                                                      (d0 + c0 + ch) * p.x_cs, cur.tx)
                                       : 0.0f;
#pragma unroll
        for (int k = 0; k < NH; ++k) c[ch].h[k] = make_float2(0.f, 0.f);
      }
    }
    if (nxt.j < ns) {
      stage(nxt, buf ^ 1);
      cp_async_wait<1>();  // this step's group has landed; the next one stays in flight
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();

    transpose_bc<TI, NH>(bct, bs_of(buf), cs_of(buf), p.io_row, (unsigned)(cur.bb + t0), (unsigned)p.bc_cs, N, cnt,
                         tid, nthr, true);
    __syncthreads();

    if (active) {
      const TI* xr[CPT];
      const TI* dtr[CPT];
      const TI* zr[CPT];
      TO* yr[CPT];
#pragma unroll
      for (int ch = 0; ch < CPT; ++ch) {
        const int r = c0 + ch;
        const long long xrow = cur.xb + (d0 + r) * p.x_cs, iorow = cur.ib + (d0 + r) * p.io_cs;
        xr[ch] = reinterpret_cast<const TI*>(xs_of(buf) + r * p.x_row + span_head(xrow + xlo, si));
        const int hd = span_head(iorow + t0, si);
        dtr[ch] = reinterpret_cast<const TI*>(dts_of(buf) + r * p.io_row + hd);
        zr[ch] = o.gate ? reinterpret_cast<const TI*>(zs_of(buf) + r * p.io_row + hd) : dtr[ch];
        yr[ch] = kInPlace ? reinterpret_cast<TO*>(dts_of(buf) + r * p.io_row + hd)
                          : reinterpret_cast<TO*>(ys + r * p.y_row);
      }
      walk<TI, TO, NH, STD, kFast, PE, CPT>(c, o, xr, xlo, xhi, dtr, zr, yr, bct, t0, cnt);
      if (swap) {
#pragma unroll
        for (int ch = 0; ch < CPT; ++ch) {
          if (t0 == 0) head_val[ch] = yr[ch][0];  // goes to the sample's last position
          if (last) {
            yg[cur.ib + (d0 + c0 + ch) * p.io_cs] = yr[ch][cnt - 1];  // the tail output becomes the next head
            yr[ch][cnt - 1] = head_val[ch];
          }
        }
      }
      // in place: each thread writes its own rows back, 16-byte stores where aligned
      if (kInPlace)
#pragma unroll
        for (int ch = 0; ch < CPT; ++ch)
          store_row<TO>(yg, cur.ib + (d0 + c0 + ch) * p.io_cs + t0, dts_of(buf) + (c0 + ch) * p.io_row, cnt,
                        swap && t0 == 0);
      if (p.final_state && last) {
#pragma unroll
        for (int ch = 0; ch < CPT; ++ch) {
          float* fs = p.final_state + ((size_t)s * p.D + d0 + c0 + ch) * N;
#pragma unroll
          for (int k = 0; k < NH; ++k) {
            if (2 * k < N) fs[2 * k] = c[ch].h[k].x;
            if (2 * k + 1 < N) fs[2 * k + 1] = c[ch].h[k].y;
          }
        }
      }
    }
    __syncthreads();  // the buffer of this step is free for the copies of step it + 2
    if (!kInPlace) {  // separate output rows: coalesced element stores by rows
      for (int r = warp; r < dcount; r += nwarps) {
        const char* src = ys + r * p.y_row;
        TO* dst = yg + cur.ib + (d0 + r) * p.io_cs + t0;
        for (int i = lane; i < cnt; i += 32)
          if (!(swap && t0 + i == 0)) dst[i] = *reinterpret_cast<const TO*>(src + i * so);
      }
      __syncthreads();  // ys is rewritten by the next step's walk
    }
    cur = nxt;
  }
}

// ------------------------------------------------------------------ lanes mode (P > 1)
//
// For long samples and few channels (B*D too small to fill the GPU with one thread per
// channel), and for more than 16 states, P lanes share a channel and split each chunk of
// S = P*J tokens: lane l owns tokens [l*J, (l+1)*J).  Per pair of states each lane
//   1. runs its J tokens from a zero state, keeping the decays Abar_j and accumulating the
//      aggregate (A, B): A the product of the decays, B the state reached from zero;
//   2. combines the aggregates of the P lanes with a warp-shuffle inclusive scan under
//        (A1, B1) o (A2, B2) = (A1*A2, A2*B1 + B2),
//      to get the state entering its tokens from the chunk's carry;
//   3. replays its J tokens from that state with the kept decays (no second exp) and
//      accumulates C*h into the outputs.
// A reset is simply A = 0 on the sample's first token.  The carry between chunks lives
// in shared memory; staging is double-buffered over (sample, chunk) steps like the
// chunked mode.  The number of state pairs is a run-time value, so one instance serves
// every N up to SFM_MAX_N.
constexpr int kLaneJ = kLaneTokens;  // tokens per lane per chunk

template <typename TI, typename TO>
__global__ void __launch_bounds__(256) fwd_lanes_kernel(const FwdParams p) {
  constexpr bool kInPlace = std::is_same<TI, TO>::value;
  constexpr bool kFast = std::is_same<TO, __nv_bfloat16>::value;
  constexpr int si = sizeof(TI), so = sizeof(TO), J = kLaneJ;
  extern __shared__ __align__(16) char smem[];

  const int NP = p.np, NH = NP / 2;
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int P = p.lanes, lane = tid % P, c = tid / P;
  const int nch = nthr / P;
  const int d0 = blockIdx.x * p.d_tile;
  const int dcount = min(p.d_tile, p.D - d0);
  const int b1 = blockIdx.y;
  const bool active = c < dcount;
  const int d = d0 + (active ? c : 0);
  const int L = p.L, N = p.N, S = p.chunk, Tx = p.Tx;
  const Opts o = make_opts(p);
  const bool swap = p.flags & kSwapOut;
  const int K = o.conv ? o.K : 1, pl = o.pl;
  // every thread of a warp runs the lane scan (channels past D compute on staged rows that
  // are never stored), so the shuffles take the full mask
  constexpr unsigned gmask = 0xffffffffu;

  const int stage_bytes = p.d_tile * p.x_row + p.d_tile * p.io_row * (o.gate ? 2 : 1) + 2 * N * p.io_row;
  // B and C in fp32, pair-interleaved per lane: [2][NH][P][LS] with (state 2k, state 2k+1) adjacent
  // for each token, so a lane's J tokens of one state pair are 2J consecutive floats; the
  // 4-float pad per lane segment spreads the lanes of a channel over distinct banks.
  constexpr int LS = 2 * J + 4;
  float* bcn = reinterpret_cast<float*>(smem + 2 * stage_bytes);
  float* a_s = bcn + 2 * NH * P * LS;                              // [d_tile][NP]: A * log2(e)
  float* carry = a_s + p.d_tile * NP;                              // [d_tile][NP]: state entering the chunk
  char* ys = reinterpret_cast<char*>(carry + p.d_tile * NP);
  auto xs_of = [&](int st) { return smem + st * stage_bytes; };
  auto dts_of = [&](int st) { return xs_of(st) + p.d_tile * p.x_row; };
  auto zs_of = [&](int st) { return dts_of(st) + p.d_tile * p.io_row; };
  auto bs_of = [&](int st) { return zs_of(st) + (o.gate ? p.d_tile * p.io_row : 0); };
  auto cs_of = [&](int st) { return bs_of(st) + N * p.io_row; };

  for (int e = tid; e < p.d_tile * NP; e += nthr) {
    const int cc = e / NP, n = e % NP;
    a_s[e] = (cc < dcount && n < N) ? p.A[(size_t)(d0 + cc) * N + n] * kLog2e : 0.0f;
  }
  float w[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) w[q] = (o.conv && q < p.K) ? p.conv_w[(size_t)d * p.K + q] : 0.0f;
  const float cb = (o.conv && p.conv_b) ? p.conv_b[d] : 0.0f;
  const float dsk = p.Dskip ? p.Dskip[d] : 0.0f;
  const float dtb = p.dt_bias ? p.dt_bias[d] : 0.0f;

  const long long x_bytes = (long long)p.B * p.D * Tx * si;
  const long long io_bytes = (long long)p.B * p.D * L * si;
  const long long bc_bytes = (long long)p.B * N * L * si;
  const char* xg = static_cast<const char*>(p.x);
  const char* dtg = static_cast<const char*>(p.dt);
  const char* zg = static_cast<const char*>(p.z);
  const char* bg = static_cast<const char*>(p.Bm);
  const char* cg = static_cast<const char*>(p.Cm);
  TO* yg = static_cast<TO*>(p.y);
  const int nchunks = (L + S - 1) / S;
  const int nsteps = p.B2 * nchunks;

  auto x_window = [&](int t0, int cnt, int& xlo, int& xhi) {
    const int slo = t0 - pl - o.off, shi = t0 + cnt - 1 + (K - 1 - pl) - o.off;
    xlo = max(slo, 0);
    xhi = min(shi + 1, Tx);
  };
  // the lanes of a channel share its rows' granules; channel groups share the B, C rows
  auto stage = [&](int st, int buf) {
    const int b = b1 * p.B2 + st / nchunks, t0 = (st % nchunks) * S, cnt = min(S, L - t0);
    const long long myrow = (long long)b * p.D + d0 + c;
    int xlo, xhi;
    x_window(t0, cnt, xlo, xhi);
    if (active) {
      copy_span_async(xs_of(buf) + c * p.x_row, xg, myrow * Tx + xlo, xhi - xlo, si, x_bytes, lane, P);
      copy_span_async(dts_of(buf) + c * p.io_row, dtg, myrow * L + t0, cnt, si, io_bytes, lane, P);
      if (o.gate) copy_span_async(zs_of(buf) + c * p.io_row, zg, myrow * L + t0, cnt, si, io_bytes, lane, P);
    }
    for (int r = c; r < 2 * N; r += nch) {
      const int n = r % N;
      const long long e0 = ((long long)b * N + n) * L + t0;
      copy_span_async((r < N ? bs_of(buf) : cs_of(buf)) + n * p.io_row, r < N ? bg : cg, e0, cnt, si, bc_bytes,
                      lane, P);
    }
    cp_async_commit();
  };

  float mean = 0.0f, head_val = 0.0f;
  stage(0, 0);
  for (int st = 0; st < nsteps; ++st) {
    const int buf = st & 1;
    const int jsam = st / nchunks, kc = st % nchunks;
    const int b = b1 * p.B2 + jsam;
    const long long row0 = (long long)b * p.D + d0;
    const long long myrow = row0 + c;
    const int t0 = kc * S, cnt = min(S, L - t0);
    int xlo, xhi;
    x_window(t0, cnt, xlo, xhi);
    if (kc == 0) {  // a new sample: zero carry; the aux mean from the whole x row
      if (o.aux) {
        float s0 = 0.0f, s1 = 0.0f;
        if (active) {
          const TI* xr = reinterpret_cast<const TI*>(xg) + myrow * Tx;
          int t = lane;
          for (; t + P < Tx; t += 2 * P) {
            s0 += to_f(xr[t]);
            s1 += to_f(xr[t + P]);
          }
          if (t < Tx) s0 += to_f(xr[t]);
        }
        s0 += s1;
        for (int off = P / 2; off > 0; off >>= 1) s0 += __shfl_xor_sync(gmask, s0, off, P);
        mean = s0 / (float)Tx;
      }
      for (int e = tid; e < p.d_tile * NP; e += nthr) carry[e] = 0.0f;
    }
    if (st + 1 < nsteps) {
      stage(st + 1, buf ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    // ---- B, C -> fp32, one warp per row; zero past the chunk end and for padded states
    for (int r = tid / 32; r < 2 * NP; r += nthr / 32) {
      const int side = r >= NP, n = r - side * NP;
      float* dst = bcn + (side * NH + (n >> 1)) * P * LS + (n & 1);
      const char* raw = nullptr;
      if (n < N) {
        const long long e0 = ((long long)b * N + n) * L + t0;
        raw = (side ? cs_of(buf) : bs_of(buf)) + n * p.io_row + span_head(e0, si);
      }
      for (int i = tid % 32; i < S; i += 32) {
        const float v = (raw && i < cnt) ? to_f(reinterpret_cast<const TI*>(raw)[i]) : 0.0f;
        dst[(i / J) * LS + 2 * (i % J)] = v;
      }
    }
    __syncthreads();

    {
      const TI* xr = reinterpret_cast<const TI*>(xs_of(buf) + c * p.x_row + span_head(myrow * Tx + xlo, si));
      const int hd = span_head(myrow * L + t0, si);
      char* dtrow = dts_of(buf) + c * p.io_row;  // the granule row: element 0 at byte hd
      const TI* dtr = reinterpret_cast<const TI*>(dtrow + hd);
      const TI* zr = o.gate ? reinterpret_cast<const TI*>(zs_of(buf) + c * p.io_row + hd) : dtr;
      TO* yr = kInPlace ? reinterpret_cast<TO*>(dtrow + hd) : reinterpret_cast<TO*>(ys + c * p.y_row);
      const int i0 = lane * J;  // chunk-relative first token of this lane

      // ---- per-token inputs of the lane's J tokens (identity (a,b) = (1,0) past the end);
      // delta and delta*u are kept duplicated, the form the paired FP32 instructions take
      float2 dl2[J], du2[J], yacc[J];
      float sdl = 0.0f;
      {
        float xw[J + 3];
#pragma unroll
        for (int q = 0; q < J + 3; ++q)
          xw[q] = (q < J || o.conv) ? xa_at<TI>(o, xr, xlo, xhi, mean, t0 + i0 + q - pl) : 0.0f;
#pragma unroll
        for (int jj = 0; jj < J; ++jj) {
          const bool valid = i0 + jj < cnt;
          float u;
          if (o.conv) {
            float acc = cb;
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (q < K) acc = fmaf(w[q], xw[jj + q], acc);
            u = kFast ? silu_fast(acc) : silu(acc);
          } else {
            u = xw[jj];
          }
          const float v = valid ? to_f(dtr[i0 + jj]) + dtb : 0.0f;
          const float delta = valid ? (o.sp ? (kFast ? softplus_fast(v) : softplus(v)) : v) : 0.0f;
          const float dus = valid ? delta * u : 0.0f;
          sdl += delta;
          dl2[jj] = make_float2(delta, delta);
          du2[jj] = make_float2(dus, dus);
          yacc[jj] = make_float2(dsk * u, 0.0f);
        }
      }
      const bool reset0 = (t0 + i0 == 0);  // the sample's first token lives in lane 0 of chunk 0

#pragma unroll 1
      for (int k = 0; k < NH; ++k) {
        const float2 A2 = *reinterpret_cast<const float2*>(a_s + c * NP + 2 * k);
        const float* Bk = bcn + (k * P + lane) * LS;
        const float* Ck = Bk + NH * P * LS;
        // 1. the lane's decays and inputs, and its aggregate (Ar, Br) from a zero state;
        //    Ar = exp2(A * sum(delta)) is the product of the decays, 0 across a reset
        float2 a[J], bj[J];
        float2 Br = make_float2(0.f, 0.f);
#pragma unroll
        for (int q = 0; q < J; q += 2) {
          const float4 u = *reinterpret_cast<const float4*>(Bk + 2 * q);
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int jj = q + e;
            float2 aj = __fmul2_rn(dl2[jj], A2);
            aj.x = ex2(aj.x);
            aj.y = ex2(aj.y);
            if (jj == 0 && reset0) aj = make_float2(0.f, 0.f);
            const float2 bv = e ? make_float2(u.z, u.w) : make_float2(u.x, u.y);
            bj[jj] = __fmul2_rn(bv, du2[jj]);
            Br = __ffma2_rn(aj, Br, bj[jj]);
            a[jj] = aj;
          }
        }
        float2 Ar = __fmul2_rn(make_float2(sdl, sdl), A2);
        Ar.x = reset0 ? 0.f : ex2(Ar.x);
        Ar.y = reset0 ? 0.f : ex2(Ar.y);
        // 2. inclusive scan of the lanes' aggregates within the channel's P lanes
        float2 Ai = Ar, Bi = Br;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          if (off < P) {
            const float2 Ap = make_float2(__shfl_up_sync(gmask, Ai.x, off, P), __shfl_up_sync(gmask, Ai.y, off, P));
            const float2 Bp = make_float2(__shfl_up_sync(gmask, Bi.x, off, P), __shfl_up_sync(gmask, Bi.y, off, P));
            if (lane >= off) {
              Bi = __ffma2_rn(Ai, Bp, Bi);
              Ai = __fmul2_rn(Ai, Ap);
            }
          }
        }
        float2 Ae = make_float2(__shfl_up_sync(gmask, Ai.x, 1, P), __shfl_up_sync(gmask, Ai.y, 1, P));
        float2 Be = make_float2(__shfl_up_sync(gmask, Bi.x, 1, P), __shfl_up_sync(gmask, Bi.y, 1, P));
        if (lane == 0) {
          Ae = make_float2(1.f, 1.f);
          Be = make_float2(0.f, 0.f);
        }
        const float2 hc = *reinterpret_cast<const float2*>(carry + c * NP + 2 * k);
        float2 h = __ffma2_rn(Ae, hc, Be);  // the state entering this lane's tokens
        __syncwarp(gmask);
        if (lane == P - 1) *reinterpret_cast<float2*>(carry + c * NP + 2 * k) = __ffma2_rn(Ai, hc, Bi);
        // 3. replay from the entering state with the kept decays and inputs
#pragma unroll
        for (int q = 0; q < J; q += 2) {
          const float4 cv = *reinterpret_cast<const float4*>(Ck + 2 * q);
          h = __ffma2_rn(a[q], h, bj[q]);
          yacc[q] = __ffma2_rn(make_float2(cv.x, cv.y), h, yacc[q]);
          h = __ffma2_rn(a[q + 1], h, bj[q + 1]);
          yacc[q + 1] = __ffma2_rn(make_float2(cv.z, cv.w), h, yacc[q + 1]);
        }
      }
#pragma unroll
      for (int jj = 0; jj < J; ++jj) {
        const int i = i0 + jj;
        if (i >= cnt) continue;
        float yo = yacc[jj].x + yacc[jj].y;
        if (o.gate) {
          const float zf = to_f(zr[i]);
          yo *= kFast ? silu_fast(zf) : silu(zf);
        }
        const int t = t0 + i;
        if (swap && t == 0) head_val = yo;
        if (swap && t == L - 1) {
          if (active) yg[myrow * L] = from_f<TO>(yo);  // the tail output becomes the next head
        } else {
          yr[i] = from_f<TO>(yo);
        }
      }
      if (swap && t0 + cnt == L) {
        // token 0's output sits in lane 0; the lane that owns token L-1 stores it there
        const float hv = __shfl_sync(gmask, head_val, 0, P);
        if (lane == (cnt - 1) / J) yr[cnt - 1] = from_f<TO>(hv);
      }
      __syncwarp(gmask);
      if (kInPlace && active && i0 < cnt) {  // each lane writes its own tokens back, 16-byte stores where aligned
        const int off = hd + i0 * si;
        store_row<TO>(yg, myrow * L + t0 + i0, dtrow + (off & ~15), min(J, cnt - i0), swap && t0 + i0 == 0);
      }
      if (p.final_state && kc == nchunks - 1) {
        __syncwarp(gmask);
        if (active && lane == 0) {
          float* fs = p.final_state + ((size_t)b * p.D + d) * N;
          for (int n = 0; n < N; ++n) fs[n] = carry[c * NP + n];
        }
      }
    }
    __syncthreads();  // this step's buffer and bcn are free for the next steps
    if (!kInPlace) {
      for (int r = tid / 32; r < dcount; r += nthr / 32) {
        const char* src = ys + r * p.y_row;
        TO* dst = yg + (row0 + r) * L + t0;
        for (int i = tid % 32; i < cnt; i += 32)
          if (!(swap && t0 + i == 0)) dst[i] = *reinterpret_cast<const TO*>(src + i * so);
      }
      __syncthreads();
    }
  }
}

// ------------------------------------------------------------------ host side

int fwd_whole_smem(const FwdParams& p, int si, int so, int NP) {
  const bool gate = p.flags & kGate;
  long long s = 16;
  s += round16(p.d_tile * p.Tx * si);
  s += (long long)round16(p.d_tile * p.L * si) * (gate ? 2 : 1);
  s += 2LL * round16(p.N * p.L * si);
  s += (long long)p.L * 2 * NP * 4;
  if (si != so) s += round16(p.d_tile * p.L * so);
  return s > (1LL << 30) ? (1 << 30) : (int)s;
}

int fwd_chunk_smem(const FwdParams& p, int si, int so, int NP) {
  const bool gate = p.flags & kGate;
  long long s = 0;
  s += (long long)p.d_tile * p.x_row;
  s += (long long)p.d_tile * p.io_row * (gate ? 2 : 1);
  s += 2LL * p.N * p.io_row;
  s *= 2;  // two staging buffers
  s += (long long)p.chunk * 2 * NP * 4;
  if (si != so) s += (long long)p.d_tile * p.y_row;
  return s > (1LL << 30) ? (1 << 30) : (int)s;
}

int fwd_lanes_smem(const FwdParams& p, int si, int so, int NP) {
  const bool gate = p.flags & kGate;
  long long s = 0;
  s += (long long)p.d_tile * p.x_row;
  s += (long long)p.d_tile * p.io_row * (gate ? 2 : 1);
  s += 2LL * p.N * p.io_row;
  s *= 2;                          // two staging buffers
  s += (long long)NP * p.lanes * (2 * kLaneTokens + 4) * 4;  // B, C in fp32, pair-interleaved
  s += 2LL * p.d_tile * NP * 4;                               // A * log2(e), carry
  if (si != so) s += (long long)p.d_tile * p.y_row;
  return s > (1LL << 30) ? (1 << 30) : (int)s;
}

int fwd_max_smem() { return 227 * 1024; }

int fwd_x_row(int chunk, int K, int esize) { return stage_row_bytes(chunk + K - 1 + 1, esize); }
int fwd_io_row(int chunk, int esize) { return stage_row_bytes(chunk, esize); }
int fwd_y_row(int chunk, int esize) { return out_row_bytes(chunk, esize); }

template <typename TI, typename TO>
static cudaError_t launch_lanes(const FwdParams& p, cudaStream_t s) {
  static SmemLimit lim;
  cudaError_t e = raise_smem_limit(fwd_lanes_kernel<TI, TO>, p.smem_bytes, lim);
  if (e != cudaSuccess) return e;
  dim3 grid((p.D + p.d_tile - 1) / p.d_tile, p.B / p.B2);
  fwd_lanes_kernel<TI, TO><<<grid, p.d_tile * p.lanes, p.smem_bytes, s>>>(p);
  return cudaGetLastError();
}

template <typename TI, typename TO, int NH, bool STD, int PE, int CPT>
static cudaError_t launch_cpt(const FwdParams& p, cudaStream_t s) {
  static SmemLimit whole_lim, chunk_lim;
  const int threads = ((p.d_tile + CPT - 1) / CPT + 31) & ~31;
  dim3 grid((p.D + p.d_tile - 1) / p.d_tile, p.B / p.B2);
  cudaError_t e;
  if (p.mode == kModeWhole) {
    if ((e = raise_smem_limit(fwd_whole_kernel<TI, TO, NH, STD, PE, CPT>, p.smem_bytes, whole_lim)) != cudaSuccess)
      return e;
    fwd_whole_kernel<TI, TO, NH, STD, PE, CPT><<<grid, threads, p.smem_bytes, s>>>(p);
  } else {
    if ((e = raise_smem_limit(fwd_chunk_kernel<TI, TO, NH, STD, PE, CPT>, p.smem_bytes, chunk_lim)) != cudaSuccess)
      return e;
    fwd_chunk_kernel<TI, TO, NH, STD, PE, CPT><<<grid, threads, p.smem_bytes, s>>>(p);
  }
  return cudaGetLastError();
}

// Two channels per thread are built for the standard mixer at N = 16 only.
template <typename TI, typename TO, int NH, bool STD, int PE>
static cudaError_t launch_t(const FwdParams& p, cudaStream_t s) {
  if constexpr (STD && NH == 8) {
    if (p.cpt == 2) return launch_cpt<TI, TO, NH, STD, PE, 2>(p, s);
  }
  return launch_cpt<TI, TO, NH, STD, PE, 1>(p, s);
}

// The standard mixer (conv K=4 + softplus + gate) gets the specialised path and, at
// N = 16, a choice of how many state pairs take exp2 on the FMA pipe.
template <typename TI, typename TO, int NH>
static cudaError_t launch_std(const FwdParams& p, cudaStream_t s) {
  const bool std_path = (p.flags & kConv) && (p.flags & kGate) && (p.flags & kSoftplus) && p.K == 4;
  if (!std_path) return launch_t<TI, TO, NH, false, 0>(p, s);
  if constexpr (NH == 8) {
    switch (p.exp2_fma_pairs) {
      case 1: return launch_t<TI, TO, NH, true, 1>(p, s);
      case 2: return launch_t<TI, TO, NH, true, 2>(p, s);
      case 3: return launch_t<TI, TO, NH, true, 3>(p, s);
      default: break;
    }
  }
  return launch_t<TI, TO, NH, true, 0>(p, s);
}

template <typename TI, typename TO>
static cudaError_t launch_np(const FwdParams& p, int NP, cudaStream_t s) {
  if (p.mode == kModeLanes) return launch_lanes<TI, TO>(p, s);
  switch (NP) {
    case 2: return launch_std<TI, TO, 1>(p, s);
    case 4: return launch_std<TI, TO, 2>(p, s);
    case 8: return launch_std<TI, TO, 4>(p, s);
    case 16: return launch_std<TI, TO, 8>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_fwd(const FwdParams& p, sfm_dtype in_dtype, sfm_dtype out_dtype, int NP, cudaStream_t s) {
  if (in_dtype == SFM_F32 && out_dtype == SFM_F32) return launch_np<float, float>(p, NP, s);
  if (in_dtype == SFM_BF16 && out_dtype == SFM_BF16) return launch_np<__nv_bfloat16, __nv_bfloat16>(p, NP, s);
  if (in_dtype == SFM_BF16 && out_dtype == SFM_F32) return launch_np<__nv_bfloat16, float>(p, NP, s);
  return cudaErrorInvalidValue;
}

cudaError_t read_device_error(cudaStream_t s, int clear, unsigned* value) {
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return e;
  e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(unsigned));
  if (e != cudaSuccess || !clear) return e;
  const unsigned zero = 0;
  return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned));
}

}  // namespace sfm
