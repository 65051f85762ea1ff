// sfm_api.cu -- the C ABI of libsfm (declared in include/sfm.h): argument validation,
// the adaptive-B1 chooser, and dispatch to the sm_100a kernels.
//
// Validation is complete before any CUDA call, so every argument error returns
// synchronously and leaves the device untouched.  The library keeps no mutable state
// besides the once-per-kernel shared-memory attribute and the device error word.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>

#include "sfm.h"
#include "sfm_internal.h"

using namespace sfm;

namespace {

constexpr int kAbiVersion = 4;
constexpr int kMaxDTile = 128;
constexpr int kMaxChunk = 256;
constexpr int kMaxB1 = 65535;  // grid.y
constexpr int kMaxNFused = 16;
constexpr int kWholeSmemCap = 80 * 1024;  // whole-sample staging only while 2+ CTAs fit an SM

struct LutEntry {
  int T, B, D, N, B2, lanes, d_tile, chunk, exp2_pairs, cpt;
};
const LutEntry kLut[] = {
#include "sfm_lut.inc"
};

thread_local const char* t_last_cuda_error = "none";

// Maps a launch result to a status, remembering the CUDA error name for sfm_last_cuda_error.
sfm_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SFM_OK;
  t_last_cuda_error = cudaGetErrorName(e);
  return SFM_ERR_CUDA;
}

bool fault_injected() {
  const char* v = std::getenv("SFM_FAULT_INJECT");
  return v && std::strcmp(v, "launch") == 0;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int esize_of(sfm_dtype t) { return t == SFM_F32 ? 4 : 2; }
bool dtype_ok(int t) { return t == SFM_F32 || t == SFM_BF16; }

bool overlaps(const void* a, long long abytes, const void* b, long long bbytes) {
  if (!a || !b) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + (uintptr_t)bbytes && b0 < a0 + (uintptr_t)abytes;
}

int largest_divisor_at_most(int B, int cap) {
  if (cap < 1) cap = 1;
  for (int v = cap < B ? cap : B; v >= 1; --v)
    if (B % v == 0) return v;
  return 1;
}

int round_up(int v, int m) { return (v + m - 1) / m * m; }

// Chunk length: at most `cap` tokens, balanced so that the last chunk is not a sliver,
// rounded up to a multiple of 8.
int balanced_chunk(int L, int cap) {
  const int n = (L + cap - 1) / cap;
  return round_up((L + n - 1) / n, 8);
}

// Nearest table row in log space of (T, B*D, N), then adapted to the actual sizes.
sfm_variant choose(int B, int T, int D, int N) {
  const LutEntry* best = &kLut[0];
  double bestd = 1e300;
  for (const LutEntry& e : kLut) {
    const double dT = std::log2((double)T / e.T), dW = std::log2((double)B * D / ((double)e.B * e.D)),
                 dN = std::log2((double)N / e.N);
    const double dist = 4.0 * dT * dT + dW * dW + 2.0 * dN * dN;
    if (dist < bestd) {
      bestd = dist;
      best = &e;
    }
  }
  sfm_variant v;
  int B2 = largest_divisor_at_most(B, best->B2);
  while (B / B2 > kMaxB1) {  // more samples per folded row until the grid fits
    int next = B2 + 1;
    while (B % next) ++next;
    B2 = next;
  }
  v.B1 = B / B2;
  v.lanes = best->lanes > 1 ? best->lanes : 1;
  int dt = best->d_tile;
  if (v.lanes > 1) {  // lanes mode: d_tile * lanes threads, a multiple of 32, at most 256
    if (dt * v.lanes > 256) dt = 256 / v.lanes;
    if (dt * v.lanes < 32) dt = 32 / v.lanes;
  } else if (dt > round_up(D, 32)) {
    dt = round_up(D, 32);
  }
  v.d_tile = dt;
  // the measured chunk for the row's own token count; re-balanced for other lengths
  v.chunk = T == best->T ? best->chunk : balanced_chunk(T + 2, best->chunk);
  v.exp2_pairs = N > 14 ? best->exp2_pairs : 0;
  v.chans_per_thread = (best->cpt == 2 && N > 8 && N <= 16 && D % 2 == 0 && v.lanes == 1) ? 2 : 1;
  return v;
}

sfm_status validate_scan(const sfm_scan_args* a, bool bwd) {
  if (!a || a->size != sizeof(sfm_scan_args)) return SFM_ERR_INVALID_ARG;
  if (!a->x || !a->dt || !a->Bm || !a->Cm || !a->A) return SFM_ERR_INVALID_ARG;
  if (!bwd && !a->y) return SFM_ERR_INVALID_ARG;
  if (a->B < 1 || a->D < 1 || a->L < 1 || a->N < 1) return SFM_ERR_INVALID_ARG;
  if (a->N > SFM_MAX_N || a->L > SFM_MAX_L) return SFM_ERR_UNSUPPORTED;
  if ((a->dt_softplus | a->aux_init | a->swap_out) & ~1) return SFM_ERR_INVALID_ARG;
  if (a->aux_init && a->L < 3) return SFM_ERR_INVALID_ARG;
  if (a->conv_w && (a->K < 1 || a->K > SFM_MAX_K || a->pad_left < 0 || a->pad_left >= a->K))
    return SFM_ERR_INVALID_ARG;
  if (a->B1 < 0 || (a->B1 > 0 && a->B % a->B1 != 0)) return SFM_ERR_INVALID_ARG;
  if (a->B1 > kMaxB1) return SFM_ERR_UNSUPPORTED;
  if (a->reset_period != 0 && a->reset_period != a->L) return SFM_ERR_UNSUPPORTED;
  if (!dtype_ok(a->in_dtype) || !dtype_ok(a->out_dtype)) return SFM_ERR_INVALID_ARG;
  if (a->in_dtype == SFM_F32 && a->out_dtype == SFM_BF16) return SFM_ERR_UNSUPPORTED;
  if (a->lanes < 0 || a->lanes > 32 || (a->lanes & (a->lanes - 1)) != 0) return SFM_ERR_UNSUPPORTED;
  if (a->lanes > 1 && a->d_tile && (a->d_tile * a->lanes > 256 || (a->d_tile * a->lanes) % 32 != 0))
    return SFM_ERR_UNSUPPORTED;
  if (a->d_tile < 0 || a->d_tile > kMaxDTile) return SFM_ERR_UNSUPPORTED;
  if (a->chunk < 0 || a->chunk > kMaxChunk || (a->chunk % 8) != 0) return SFM_ERR_UNSUPPORTED;
  if (a->exp2_split < 0 || a->exp2_split > 4) return SFM_ERR_UNSUPPORTED;
  if (a->chans_per_thread < 0 || a->chans_per_thread > 2) return SFM_ERR_UNSUPPORTED;
  const void* acts[] = {a->x, a->dt, a->z, a->Bm, a->Cm, a->y};
  for (const void* p : acts)
    if (p && !aligned16(p)) return SFM_ERR_MISALIGNED;
  const long long si = esize_of(a->in_dtype), so = esize_of(a->out_dtype);
  const long long bdl = (long long)a->B * a->D * a->L;
  const long long xbytes = (long long)a->B * a->D * (a->aux_init ? a->L - 2 : a->L) * si;
  const long long bcbytes = (long long)a->B * a->N * a->L * si;
  if (!bwd) {
    const long long ybytes = bdl * so;
    if (overlaps(a->y, ybytes, a->x, xbytes) || overlaps(a->y, ybytes, a->dt, bdl * si) ||
        overlaps(a->y, ybytes, a->z, bdl * si) || overlaps(a->y, ybytes, a->Bm, bcbytes) ||
        overlaps(a->y, ybytes, a->Cm, bcbytes))
      return SFM_ERR_INVALID_ARG;
  }
  return SFM_OK;
}

// The ragged forward: B samples packed along time in rows of L (the packed total)
// positions; the per-sample offsets live on the device and are checked by the kernel.
sfm_status validate_varlen(const sfm_scan_args* a, const int* cu_seqlens) {
  if (!a || a->size != sizeof(sfm_scan_args) || !cu_seqlens) return SFM_ERR_INVALID_ARG;
  if (!a->x || !a->dt || !a->Bm || !a->Cm || !a->A || !a->y) return SFM_ERR_INVALID_ARG;
  if (a->B < 1 || a->D < 1 || a->L < 1 || a->N < 1) return SFM_ERR_INVALID_ARG;
  if (a->N > kMaxNFused) return SFM_ERR_UNSUPPORTED;
  if ((a->dt_softplus | a->aux_init | a->swap_out) & ~1) return SFM_ERR_INVALID_ARG;
  if (a->aux_init && (long long)a->L < 3LL * a->B) return SFM_ERR_INVALID_ARG;  // >= 3 tokens per sample
  if (a->conv_w && (a->K < 1 || a->K > SFM_MAX_K || a->pad_left < 0 || a->pad_left >= a->K))
    return SFM_ERR_INVALID_ARG;
  if (a->B1 < 0 || (a->B1 > 0 && a->B % a->B1 != 0)) return SFM_ERR_INVALID_ARG;
  if (a->B1 > kMaxB1) return SFM_ERR_UNSUPPORTED;
  if (a->reset_period != 0) return SFM_ERR_UNSUPPORTED;  // the resets follow cu_seqlens
  if (!dtype_ok(a->in_dtype) || !dtype_ok(a->out_dtype)) return SFM_ERR_INVALID_ARG;
  if (a->in_dtype == SFM_F32 && a->out_dtype == SFM_BF16) return SFM_ERR_UNSUPPORTED;
  if (a->lanes > 1) return SFM_ERR_UNSUPPORTED;  // one thread walks each channel
  if (a->lanes < 0 || a->d_tile < 0 || a->d_tile > kMaxDTile) return SFM_ERR_UNSUPPORTED;
  if (a->chunk < 0 || a->chunk > kMaxChunk || (a->chunk % 8) != 0) return SFM_ERR_UNSUPPORTED;
  if (a->exp2_split < 0 || a->exp2_split > 4) return SFM_ERR_UNSUPPORTED;
  if (a->chans_per_thread < 0 || a->chans_per_thread > 2) return SFM_ERR_UNSUPPORTED;
  const void* acts[] = {a->x, a->dt, a->z, a->Bm, a->Cm, a->y};
  for (const void* p : acts)
    if (p && !aligned16(p)) return SFM_ERR_MISALIGNED;
  if (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) return SFM_ERR_MISALIGNED;
  const long long si = esize_of(a->in_dtype), so = esize_of(a->out_dtype);
  const long long dl = (long long)a->D * a->L;
  const long long xbytes = (long long)a->D * (a->aux_init ? a->L - 2LL * a->B : a->L) * si;
  const long long bcbytes = (long long)a->N * a->L * si, ybytes = dl * so;
  if (overlaps(a->y, ybytes, a->x, xbytes) || overlaps(a->y, ybytes, a->dt, dl * si) ||
      overlaps(a->y, ybytes, a->z, dl * si) || overlaps(a->y, ybytes, a->Bm, bcbytes) ||
      overlaps(a->y, ybytes, a->Cm, bcbytes) || overlaps(a->y, ybytes, cu_seqlens, 4LL * (a->B + 1)))
    return SFM_ERR_INVALID_ARG;
  return SFM_OK;
}

constexpr int kBwdDTile = 64;

// The backward takes a plain scan (input u, no conv, no aux tokens, no swap).
sfm_status validate_bwd_args(const sfm_scan_args* a) {
  const sfm_status st = validate_scan(a, true);
  if (st != SFM_OK) return st;
  if (a->conv_w || a->aux_init || a->swap_out) return SFM_ERR_UNSUPPORTED;
  return SFM_OK;
}

sfm_status validate_grads(const sfm_scan_args* a, const sfm_scan_grads* g) {
  if (!g || g->size != sizeof(sfm_scan_grads)) return SFM_ERR_INVALID_ARG;
  if (!g->dout || !g->du || !g->ddt || !g->dA || !g->dB || !g->dC) return SFM_ERR_INVALID_ARG;
  if (a->z && !g->dz) return SFM_ERR_INVALID_ARG;
  if (!aligned16(g->dout)) return SFM_ERR_MISALIGNED;
  const float* outs[] = {g->du, g->ddt, g->dz, g->dA, g->dDskip, g->ddt_bias, g->dB, g->dC};
  for (const float* o : outs)
    if (o && (reinterpret_cast<uintptr_t>(o) & 3u)) return SFM_ERR_MISALIGNED;
  const long long si = esize_of(a->in_dtype), so = esize_of(a->out_dtype);
  const long long bdl = (long long)a->B * a->D * a->L, bnl = (long long)a->B * a->N * a->L;
  const void* ins[] = {a->x, a->dt, a->z, a->Bm, a->Cm, g->dout, a->A, a->Dskip, a->dt_bias};
  const long long insz[] = {bdl * si, bdl * si, bdl * si, bnl * si, bnl * si, bdl * so,
                            (long long)a->D * a->N * 4, (long long)a->D * 4, (long long)a->D * 4};
  const long long outsz[] = {bdl * 4, bdl * 4, bdl * 4, (long long)a->D * a->N * 4, (long long)a->D * 4,
                             (long long)a->D * 4, bnl * 4, bnl * 4};
  for (int i = 0; i < 8; ++i) {
    for (int j = 0; j < 9; ++j)
      if (overlaps(outs[i], outsz[i], ins[j], insz[j])) return SFM_ERR_INVALID_ARG;
    for (int j = i + 1; j < 8; ++j)
      if (overlaps(outs[i], outsz[i], outs[j], outsz[j])) return SFM_ERR_INVALID_ARG;
  }
  return SFM_OK;
}

BwdParams make_bwd_params(const sfm_scan_args* a, const sfm_scan_grads* g) {
  BwdParams p;
  std::memset(&p, 0, sizeof(p));
  p.u = a->x;
  p.dt = a->dt;
  p.z = a->z;
  p.Bm = a->Bm;
  p.Cm = a->Cm;
  p.dout = g->dout;
  p.A = a->A;
  p.Dskip = a->Dskip;
  p.dt_bias = a->dt_bias;
  p.du = g->du;
  p.ddt = g->ddt;
  p.dz = a->z ? g->dz : nullptr;
  p.dA = g->dA;
  p.dDskip = a->Dskip ? g->dDskip : nullptr;
  p.ddt_bias = a->dt_bias ? g->ddt_bias : nullptr;
  p.dB = g->dB;
  p.dC = g->dC;
  p.B = a->B;
  p.D = a->D;
  p.L = a->L;
  p.N = a->N;
  p.d_tile = kBwdDTile;
  p.ntiles = (a->D + kBwdDTile - 1) / kBwdDTile;
  p.softplus = a->dt_softplus;
  return p;
}

sfm_status validate_mixer_grads(const sfm_scan_args* a, const sfm_mixer_grads* g) {
  if (!g || g->size != sizeof(sfm_mixer_grads)) return SFM_ERR_INVALID_ARG;
  if (!g->dout || !g->dx || !g->ddt || !g->dA || !g->dB || !g->dC) return SFM_ERR_INVALID_ARG;
  if ((a->conv_w && !g->dconv_w) || (a->conv_b && a->conv_w && !g->dconv_b) || (a->z && !g->dz) ||
      (a->Dskip && !g->dDskip) || (a->dt_bias && !g->ddt_bias))
    return SFM_ERR_INVALID_ARG;
  if (!aligned16(g->dout)) return SFM_ERR_MISALIGNED;
  const float* outs[] = {g->dx, g->dconv_w, g->dconv_b, g->ddt, g->dz, g->dA, g->dDskip, g->ddt_bias, g->dB, g->dC};
  for (const float* o : outs)
    if (o && (reinterpret_cast<uintptr_t>(o) & 3u)) return SFM_ERR_MISALIGNED;
  const long long si = esize_of(a->in_dtype), so = esize_of(a->out_dtype);
  const long long bdl = (long long)a->B * a->D * a->L, bnl = (long long)a->B * a->N * a->L;
  const long long bdx = (long long)a->B * a->D * (a->aux_init ? a->L - 2 : a->L);
  const int K = a->conv_w ? a->K : 0;
  const void* ins[] = {a->x, a->dt, a->z, a->Bm, a->Cm, g->dout, a->A, a->Dskip, a->dt_bias, a->conv_w, a->conv_b};
  const long long insz[] = {bdx * si, bdl * si, bdl * si, bnl * si, bnl * si, bdl * so, (long long)a->D * a->N * 4,
                            (long long)a->D * 4, (long long)a->D * 4, (long long)a->D * K * 4, (long long)a->D * 4};
  const long long outsz[] = {bdx * 4, (long long)a->D * K * 4, (long long)a->D * 4, bdl * 4, bdl * 4,
                             (long long)a->D * a->N * 4, (long long)a->D * 4, (long long)a->D * 4, bnl * 4, bnl * 4};
  for (int i = 0; i < 10; ++i) {
    for (int j = 0; j < 11; ++j)
      if (overlaps(outs[i], outsz[i], ins[j], insz[j])) return SFM_ERR_INVALID_ARG;
    for (int j = i + 1; j < 10; ++j)
      if (overlaps(outs[i], outsz[i], outs[j], outsz[j])) return SFM_ERR_INVALID_ARG;
  }
  return SFM_OK;
}

}  // namespace

extern "C" {

const char* sfm_status_string(int status) {
  switch (status) {
    case SFM_OK: return "SFM_OK";
    case SFM_ERR_INVALID_ARG: return "SFM_ERR_INVALID_ARG: invalid argument";
    case SFM_ERR_MISALIGNED: return "SFM_ERR_MISALIGNED: tensor base not 16-byte aligned";
    case SFM_ERR_UNSUPPORTED: return "SFM_ERR_UNSUPPORTED: outside the supported sizes";
    case SFM_ERR_CUDA: return "SFM_ERR_CUDA: CUDA launch error";
    case SFM_ERR_TIMEOUT: return "SFM_ERR_TIMEOUT: a kernel gave up a bounded wait";
    default: return "SFM_ERR_UNKNOWN";
  }
}

int sfm_abi_version(void) { return kAbiVersion; }

const char* sfm_last_cuda_error(void) { return t_last_cuda_error; }

sfm_status sfm_aux_init(const void* x, void* xa, int B, int D, int T, sfm_dtype dtype, sfm_stream_t stream) {
  if (!x || !xa || B < 1 || D < 1 || T < 1 || !dtype_ok(dtype)) return SFM_ERR_INVALID_ARG;
  if (T + 2 > SFM_MAX_L) return SFM_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(xa)) return SFM_ERR_MISALIGNED;
  const int es = esize_of(dtype);
  if (overlaps(x, (long long)B * D * T * es, xa, (long long)B * D * (T + 2) * es)) return SFM_ERR_INVALID_ARG;
  if (fault_injected()) return SFM_ERR_CUDA;
  return cuda_status(launch_aux_init(x, xa, B, D, T, es, stream));
}

sfm_status sfm_aux_swap(void* y, int B, int D, int L, sfm_dtype dtype, sfm_stream_t stream) {
  if (!y || B < 1 || D < 1 || L < 2 || !dtype_ok(dtype)) return SFM_ERR_INVALID_ARG;
  if (L > SFM_MAX_L) return SFM_ERR_UNSUPPORTED;
  if (!aligned16(y)) return SFM_ERR_MISALIGNED;
  if (fault_injected()) return SFM_ERR_CUDA;
  return cuda_status(launch_aux_swap(y, B, D, L, esize_of(dtype), stream));
}

sfm_status sfm_fold_conv1d(const void* x, const float* w, const float* bias, void* u, int B, int D, int L, int K,
                           int pad_left, int B2, int silu, sfm_dtype dtype, sfm_stream_t stream) {
  if (!x || !w || !u || B < 1 || D < 1 || L < 1 || !dtype_ok(dtype)) return SFM_ERR_INVALID_ARG;
  if (K < 1 || K > SFM_MAX_K || pad_left < 0 || pad_left >= K) return SFM_ERR_INVALID_ARG;
  if (B2 < 1 || B % B2 != 0 || (silu & ~1)) return SFM_ERR_INVALID_ARG;
  if (L > SFM_MAX_L) return SFM_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(u)) return SFM_ERR_MISALIGNED;
  const long long bytes = (long long)B * D * L * esize_of(dtype);
  if (overlaps(x, bytes, u, bytes)) return SFM_ERR_INVALID_ARG;
  if (fault_injected()) return SFM_ERR_CUDA;
  return cuda_status(launch_conv1d(x, w, bias, u, B, D, L, K, pad_left, silu, dtype, stream));
}

sfm_status sfm_conv1d_tokens(const void* x, const float* w, const float* bias, void* u, int B, int D, int L, int K,
                             int pad_left, int silu, sfm_dtype dtype, sfm_stream_t stream) {
  if (!x || !w || !u || B < 1 || D < 1 || L < 1 || !dtype_ok(dtype)) return SFM_ERR_INVALID_ARG;
  if (K < 1 || K > SFM_MAX_K || pad_left < 0 || pad_left >= K || (silu & ~1)) return SFM_ERR_INVALID_ARG;
  if (L > SFM_MAX_L || B > 65535) return SFM_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(u)) return SFM_ERR_MISALIGNED;
  const long long bytes = (long long)B * D * L * esize_of(dtype);
  if (overlaps(x, bytes, u, bytes)) return SFM_ERR_INVALID_ARG;
  if (fault_injected()) return SFM_ERR_CUDA;
  return cuda_status(launch_conv1d_tokens(x, w, bias, u, B, D, L, K, pad_left, silu, dtype, stream));
}

sfm_status sfm_choose_variant(int B, int T, int D, int N, sfm_variant* out) {
  if (!out || B < 1 || T < 1 || D < 1 || N < 1) return SFM_ERR_INVALID_ARG;
  *out = choose(B, T, D, N);
  return SFM_OK;
}

sfm_status sfm_choose_b1(int B, int T, int D, int N, int* B1_out) {
  if (!B1_out) return SFM_ERR_INVALID_ARG;
  sfm_variant v;
  sfm_status st = sfm_choose_variant(B, T, D, N, &v);
  if (st != SFM_OK) return st;
  *B1_out = v.B1;
  return SFM_OK;
}

sfm_status sfm_selective_scan_fold(const sfm_scan_args* a, sfm_stream_t stream) {
  sfm_status st = validate_scan(a, false);
  if (st != SFM_OK) return st;
  const int T = a->aux_init ? a->L - 2 : a->L;
  const sfm_variant v = choose(a->B, T, a->D, a->N);
  FwdParams p;
  std::memset(&p, 0, sizeof(p));
  p.x = a->x;
  p.dt = a->dt;
  p.z = a->z;
  p.Bm = a->Bm;
  p.Cm = a->Cm;
  p.A = a->A;
  p.Dskip = a->Dskip;
  p.dt_bias = a->dt_bias;
  p.conv_w = a->conv_w;
  p.conv_b = a->conv_b;
  p.y = a->y;
  p.final_state = a->final_state;
  p.B = a->B;
  p.D = a->D;
  p.L = a->L;
  p.N = a->N;
  p.Tx = a->aux_init ? a->L - 2 : a->L;
  p.x_cs = p.Tx;
  p.io_cs = p.bc_cs = a->L;
  p.x_elems = (long long)a->B * a->D * p.Tx;
  p.io_elems = (long long)a->B * a->D * a->L;
  p.bc_elems = (long long)a->B * a->N * a->L;
  p.K = a->conv_w ? a->K : 1;
  p.pad_left = a->conv_w ? a->pad_left : 0;
  p.B2 = a->B / (a->B1 ? a->B1 : v.B1);
  p.d_tile = a->d_tile ? a->d_tile : v.d_tile;
  p.chunk = a->chunk ? a->chunk : v.chunk;
  p.exp2_fma_pairs = a->exp2_split ? a->exp2_split - 1 : v.exp2_pairs;
  p.cpt = a->chans_per_thread ? a->chans_per_thread : ((a->d_tile || a->chunk) ? 1 : v.chans_per_thread);
  // two channels per thread: the standard mixer at 8 < N <= 16 with an even tile and D
  if (p.cpt == 2 && !(a->conv_w && a->z && a->dt_softplus && a->K == 4 && a->N > 8 && a->N <= 16 &&
                      a->D % 2 == 0 && p.d_tile % 2 == 0))
    p.cpt = 1;
  p.flags = (a->dt_softplus ? kSoftplus : 0) | (a->aux_init ? kAuxInit : 0) |
            (a->swap_out && a->L >= 2 ? kSwapOut : 0) | (a->conv_w ? kConv : 0) | (a->z ? kGate : 0);
  const int si = esize_of(a->in_dtype), so = esize_of(a->out_dtype);
  int NP = 2;
  while (NP < a->N) NP <<= 1;
  p.np = NP;
  if (a->B / p.B2 > kMaxB1) return SFM_ERR_UNSUPPORTED;
  // whole-sample mode: the chunk covers the sample and every slab of every tensor starts
  // on a 16-byte boundary with a size that is a multiple of 16 bytes (bulk-copy rules)
  auto slab_ok = [&](long long per_row_bytes) {
    const long long rem = (long long)(a->D % p.d_tile) * per_row_bytes;
    return ((long long)a->D * per_row_bytes) % 16 == 0 && ((long long)p.d_tile * per_row_bytes) % 16 == 0 &&
           rem % 16 == 0;
  };
  const bool aligned = slab_ok((long long)p.Tx * si) && slab_ok((long long)a->L * si) &&
                       slab_ok((long long)a->L * so) && ((long long)a->N * a->L * si) % 16 == 0;
  p.mode = kModeChunk;
  // an explicit channel tile or chunk without explicit lanes asks for one thread per channel
  p.lanes = a->lanes ? a->lanes : ((a->d_tile || a->chunk) ? 1 : v.lanes);
  // more than kMaxNFused states only fit the lanes mode, which walks the states in pairs
  if (a->N > kMaxNFused) {
    if (a->lanes == 1) return SFM_ERR_UNSUPPORTED;
    if (p.lanes < 2) {
      p.lanes = 4;
      if (!a->d_tile) p.d_tile = 16;
    }
  }
  if (p.lanes > 1) {
    p.mode = kModeLanes;
    if (!a->d_tile) {
      if (p.d_tile * p.lanes > 256) p.d_tile = 256 / p.lanes;
      if (p.d_tile * p.lanes < 32) p.d_tile = 32 / p.lanes;
    }
    if (p.d_tile * p.lanes > 256 || (p.d_tile * p.lanes) % 32 != 0) return SFM_ERR_UNSUPPORTED;
    auto shape = [&]() {
      p.chunk = p.lanes * kLaneTokens;
      p.x_row = fwd_x_row(p.chunk, 4, si);
      p.io_row = fwd_io_row(p.chunk, si);
      p.y_row = fwd_y_row(p.chunk, so);
      p.smem_bytes = fwd_lanes_smem(p, si, so, NP);
    };
    shape();
    // automatic shapes shrink (fewer lanes, then fewer channels) until the smem fits
    while (p.smem_bytes > fwd_max_smem() && !a->lanes && p.lanes > 2) {
      p.lanes /= 2;
      if (!a->d_tile) p.d_tile = (p.d_tile * 2 * p.lanes <= 256) ? p.d_tile * 2 : p.d_tile;
      shape();
    }
    while (p.smem_bytes > fwd_max_smem() && !a->d_tile && p.d_tile * p.lanes > 32) {
      p.d_tile /= 2;
      shape();
    }
    if (p.smem_bytes > fwd_max_smem()) return SFM_ERR_UNSUPPORTED;
  } else if (p.chunk >= a->L && aligned) {
    p.mode = kModeWhole;
    p.smem_bytes = fwd_whole_smem(p, si, so, NP);
    if (p.smem_bytes > kWholeSmemCap) p.mode = kModeChunk;
  }
  if (p.mode == kModeChunk) {
    if (p.chunk > kMaxChunk) p.chunk = kMaxChunk;
    p.x_row = fwd_x_row(p.chunk, 4, si);
    p.io_row = fwd_io_row(p.chunk, si);
    p.y_row = fwd_y_row(p.chunk, so);
    p.smem_bytes = fwd_chunk_smem(p, si, so, NP);
    if (p.smem_bytes > fwd_max_smem()) {
      if (a->chunk || a->d_tile) return SFM_ERR_UNSUPPORTED;  // explicit shape that does not fit
      while (p.smem_bytes > fwd_max_smem() && p.d_tile > 32) {
        p.d_tile /= 2;
        p.smem_bytes = fwd_chunk_smem(p, si, so, NP);
      }
      if (p.smem_bytes > fwd_max_smem()) return SFM_ERR_UNSUPPORTED;
    }
  }
  if (fault_injected()) return SFM_ERR_CUDA;
  return cuda_status(launch_fwd(p, a->in_dtype, a->out_dtype, NP, stream));
}

sfm_status sfm_selective_scan_fold_varlen(const sfm_scan_args* a, const int* cu_seqlens, sfm_stream_t stream) {
  sfm_status st = validate_varlen(a, cu_seqlens);
  if (st != SFM_OK) return st;
  // the launch shape of the look-up table at the mean sample length, in chunked mode
  const int Lmean = (int)std::max(1LL, (long long)a->L / a->B);
  const int Tmean = std::max(1, a->aux_init ? Lmean - 2 : Lmean);
  const sfm_variant v = choose(a->B, Tmean, a->D, a->N);
  FwdParams p;
  std::memset(&p, 0, sizeof(p));
  p.x = a->x;
  p.dt = a->dt;
  p.z = a->z;
  p.Bm = a->Bm;
  p.Cm = a->Cm;
  p.A = a->A;
  p.Dskip = a->Dskip;
  p.dt_bias = a->dt_bias;
  p.conv_w = a->conv_w;
  p.conv_b = a->conv_b;
  p.y = a->y;
  p.final_state = a->final_state;
  p.cu_seqlens = cu_seqlens;
  p.B = a->B;
  p.D = a->D;
  p.L = a->L;
  p.N = a->N;
  p.Tx = a->aux_init ? a->L - 2 * a->B : a->L;
  p.x_cs = p.Tx;
  p.io_cs = p.bc_cs = a->L;
  p.x_elems = (long long)a->D * p.Tx;
  p.io_elems = (long long)a->D * a->L;
  p.bc_elems = (long long)a->N * a->L;
  p.K = a->conv_w ? a->K : 1;
  p.pad_left = a->conv_w ? a->pad_left : 0;
  p.B2 = a->B / (a->B1 ? a->B1 : v.B1);
  const bool lut_chunked = v.lanes == 1;
  p.d_tile = a->d_tile ? a->d_tile : (lut_chunked ? v.d_tile : 64);
  // samples of unequal length: chunks of 32..64 tokens measured best (fewer steps per sample
  // than the fixed layout's short chunks, little waste in each sample's last chunk)
  p.chunk = a->chunk ? a->chunk : (lut_chunked ? std::max(32, std::min(v.chunk, 64)) : 64);
  p.exp2_fma_pairs = a->exp2_split ? a->exp2_split - 1 : v.exp2_pairs;
  p.cpt = a->chans_per_thread ? a->chans_per_thread : ((a->d_tile || a->chunk || !lut_chunked) ? 1 : v.chans_per_thread);
  if (p.cpt == 2 && !(a->conv_w && a->z && a->dt_softplus && a->K == 4 && a->N > 8 && a->N <= 16 &&
                      a->D % 2 == 0 && p.d_tile % 2 == 0))
    p.cpt = 1;
  p.flags = (a->dt_softplus ? kSoftplus : 0) | (a->aux_init ? kAuxInit : 0) | (a->swap_out ? kSwapOut : 0) |
            (a->conv_w ? kConv : 0) | (a->z ? kGate : 0);
  const int si = esize_of(a->in_dtype), so = esize_of(a->out_dtype);
  int NP = 2;
  while (NP < a->N) NP <<= 1;
  p.np = NP;
  if (a->B / p.B2 > kMaxB1) return SFM_ERR_UNSUPPORTED;
  p.mode = kModeChunk;
  p.lanes = 1;
  p.x_row = fwd_x_row(p.chunk, 4, si);
  p.io_row = fwd_io_row(p.chunk, si);
  p.y_row = fwd_y_row(p.chunk, so);
  p.smem_bytes = fwd_chunk_smem(p, si, so, NP);
  while (p.smem_bytes > fwd_max_smem() && !a->d_tile && p.d_tile > 32) {
    p.d_tile /= 2;
    p.smem_bytes = fwd_chunk_smem(p, si, so, NP);
  }
  if (p.smem_bytes > fwd_max_smem()) return SFM_ERR_UNSUPPORTED;
  if (fault_injected()) return SFM_ERR_CUDA;
  return cuda_status(launch_fwd(p, a->in_dtype, a->out_dtype, NP, stream));
}

sfm_status sfm_proj_gemm(const sfm_proj_args* a, sfm_stream_t stream) {
  if (!a || a->size != sizeof(sfm_proj_args) || !a->W || !a->X || !a->out0) return SFM_ERR_INVALID_ARG;
  if (a->M < 1 || a->K < 1 || a->Ntok < 1 || a->L < 1 || a->Ntok % a->L != 0) return SFM_ERR_INVALID_ARG;
  if ((a->token_major & ~1) || !dtype_ok(a->out_dtype)) return SFM_ERR_INVALID_ARG;
  if (a->token_major ? (a->M0 != a->M || a->out1) : (a->M0 < 1 || a->M0 > a->M || ((a->M0 < a->M) != !!a->out1)))
    return SFM_ERR_INVALID_ARG;
  if (a->tile_n != 0 && a->tile_n != 128 && a->tile_n != 256) return SFM_ERR_UNSUPPORTED;
  if (a->schedule < 0 || a->schedule > 2) return SFM_ERR_INVALID_ARG;
  if (a->K % 8 != 0) return SFM_ERR_UNSUPPORTED;  // TMA: the row pitch of W and X is a multiple of 16 bytes
  const void* ptrs[] = {a->W, a->X, a->out0, a->out1};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return SFM_ERR_MISALIGNED;
  const long long os = esize_of(a->out_dtype);
  const long long wb = (long long)a->M * a->K * 2, xb = (long long)a->Ntok * a->K * 2;
  const long long o0 = (long long)a->Ntok * (a->token_major ? a->M : a->M0) * os;
  const long long o1 = (long long)a->Ntok * (a->M - a->M0) * os;
  if (overlaps(a->out0, o0, a->W, wb) || overlaps(a->out0, o0, a->X, xb) || overlaps(a->out1, o1, a->W, wb) ||
      overlaps(a->out1, o1, a->X, xb) || overlaps(a->out0, o0, a->out1, o1))
    return SFM_ERR_INVALID_ARG;
  ProjParams p;
  std::memset(&p, 0, sizeof(p));
  p.W = a->W;
  p.X = a->X;
  p.out0 = a->out0;
  p.out1 = a->out1;
  p.M = a->M;
  p.K = a->K;
  p.Ntok = a->Ntok;
  p.M0 = a->M0;
  p.L = a->L;
  p.token_major = a->token_major;
  p.out_f32 = a->out_dtype == SFM_F32;
  // Short K (the projections): one CTA per tile of 128 channels, several CTAs per SM, so
  // many warps store while others load -- the outputs' coalesced row stores bound these.
  // Long K: the MMAs dominate; one persistent CTA per SM with tiles of 256 channels, its
  // epilogue overlapping the next tile's loads and MMAs.
  const bool long_k = a->K > 640;
  p.bn = a->tile_n ? a->tile_n : (long_k ? 256 : 128);
  p.persistent = a->schedule == 2 || (a->schedule == 0 && long_k);
  if (fault_injected()) return SFM_ERR_CUDA;
  return cuda_status(launch_proj(p, stream));
}

sfm_status sfm_scan_bwd_workspace_size(const sfm_scan_args* a, size_t* bytes) {
  if (!bytes) return SFM_ERR_INVALID_ARG;
  const sfm_status st = validate_bwd_args(a);
  if (st != SFM_OK) return st;
  *bytes = bwd_workspace_bytes(a->B, a->D, a->L, a->N, kBwdDTile);
  return SFM_OK;
}

sfm_status sfm_selective_scan_fold_bwd(const sfm_scan_args* a, const sfm_scan_grads* g, void* ws, size_t wsb,
                                       sfm_stream_t stream) {
  sfm_status st = validate_bwd_args(a);
  if (st != SFM_OK) return st;
  if ((st = validate_grads(a, g)) != SFM_OK) return st;
  if (!ws) return SFM_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return SFM_ERR_MISALIGNED;
  if (wsb < bwd_workspace_bytes(a->B, a->D, a->L, a->N, kBwdDTile)) return SFM_ERR_INVALID_ARG;
  if (fault_injected()) return SFM_ERR_CUDA;
  BwdParams p = make_bwd_params(a, g);
  bwd_carve(p, static_cast<char*>(ws));
  return cuda_status(launch_bwd(p, a->in_dtype, a->out_dtype, stream));
}

sfm_status sfm_mixer_bwd_workspace_size(const sfm_scan_args* a, size_t* bytes) {
  if (!bytes) return SFM_ERR_INVALID_ARG;
  const sfm_status st = validate_scan(a, true);
  if (st != SFM_OK) return st;
  *bytes = mixer_bwd_workspace_bytes(a->B, a->D, a->L, a->N, a->conv_w ? a->K : 1, kBwdDTile);
  return SFM_OK;
}

sfm_status sfm_mixer_bwd(const sfm_scan_args* a, const sfm_mixer_grads* g, void* ws, size_t wsb,
                         sfm_stream_t stream) {
  sfm_status st = validate_scan(a, true);
  if (st != SFM_OK) return st;
  if ((st = validate_mixer_grads(a, g)) != SFM_OK) return st;
  if (!ws) return SFM_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return SFM_ERR_MISALIGNED;
  if (wsb < mixer_bwd_workspace_bytes(a->B, a->D, a->L, a->N, a->conv_w ? a->K : 1, kBwdDTile))
    return SFM_ERR_INVALID_ARG;
  if (fault_injected()) return SFM_ERR_CUDA;
  sfm_scan_grads sg;
  std::memset(&sg, 0, sizeof(sg));
  sg.dout = g->dout;
  sg.ddt = g->ddt;
  sg.dz = g->dz;
  sg.dA = g->dA;
  sg.dDskip = g->dDskip;
  sg.ddt_bias = g->ddt_bias;
  sg.dB = g->dB;
  sg.dC = g->dC;
  BwdParams p = make_bwd_params(a, &sg);
  p.mixer = 1;
  p.swap_dout = a->swap_out && a->L >= 2;
  p.aux = a->aux_init;
  p.conv = a->conv_w != nullptr;
  p.K = p.conv ? a->K : 1;
  p.pad_left = p.conv ? a->pad_left : 0;
  p.Tx = a->aux_init ? a->L - 2 : a->L;
  p.x = a->x;
  p.conv_w = a->conv_w;
  p.conv_b = p.conv ? a->conv_b : nullptr;
  p.dx = g->dx;
  p.dconv_w = g->dconv_w;
  p.dconv_b = p.conv ? g->dconv_b : nullptr;
  mixer_bwd_carve(p, static_cast<char*>(ws));
  return cuda_status(launch_mixer_bwd(p, a->in_dtype, a->out_dtype, stream));
}

sfm_status sfm_selective_scan_fold_bwd_noalloc(const sfm_scan_args* a, const sfm_scan_grads* g,
                                               sfm_stream_t stream) {
  sfm_status st = validate_bwd_args(a);
  if (st != SFM_OK) return st;
  if ((st = validate_grads(a, g)) != SFM_OK) return st;
  if (bwd_workspace_bytes(a->B, a->D, a->L, a->N, kBwdDTile) > (size_t)SFM_NOALLOC_SCRATCH_BYTES)
    return SFM_ERR_UNSUPPORTED;  // larger than the built-in workspace
  if (fault_injected()) return SFM_ERR_CUDA;
  void* ws = nullptr;
  if ((st = cuda_status(noalloc_scratch(&ws))) != SFM_OK) return st;
  BwdParams p = make_bwd_params(a, g);
  bwd_carve(p, static_cast<char*>(ws));
  return cuda_status(launch_bwd(p, a->in_dtype, a->out_dtype, stream));
}

sfm_status sfm_selftest_wait_timeout(int limit_us, sfm_stream_t stream) {
  if (limit_us < 1 || limit_us > 1000000) return SFM_ERR_INVALID_ARG;
  if (fault_injected()) return SFM_ERR_CUDA;
  return cuda_status(launch_wait_selftest(limit_us, stream));
}

sfm_status sfm_get_device_error(sfm_stream_t stream, int clear, int* code) {
  if (!code) return SFM_ERR_INVALID_ARG;
  unsigned v = 0, w = 0;
  sfm_status st = cuda_status(read_device_error(stream, clear, &v));
  if (st != SFM_OK) return st;
  st = cuda_status(read_proj_error(clear, &w));  // the projection kernels' word
  if (st != SFM_OK) return st;
  *code = (int)(v ? v : w);
  return SFM_OK;
}

}  // extern "C"
