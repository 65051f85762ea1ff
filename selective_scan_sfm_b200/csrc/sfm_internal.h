// sfm_internal.h -- launch parameters shared by the host API and the kernels of libsfm.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "sfm.h"

namespace sfm {

enum FwdFlags : int {
  kSoftplus = 1 << 0,  // Delta = softplus(dt + dt_bias)
  kAuxInit = 1 << 1,   // x holds T = L-2 tokens; aux tokens = mean, built on load
  kSwapOut = 1 << 2,   // exchange output tokens 0 and L-1
  kConv = 1 << 3,      // depthwise conv + SiLU on the input
  kGate = 1 << 4,      // multiply by SiLU(z)
};

struct FwdParams {
  const void* x;
  const void* dt;
  const void* z;
  const void* Bm;
  const void* Cm;
  const float* A;
  const float* Dskip;
  const float* dt_bias;
  const float* conv_w;
  const float* conv_b;
  void* y;
  float* final_state;
  int B, D, L, N, Tx;  // Tx = tokens per row of x (L-2 with aux init, else L)
  // Ragged layout (chunked mode only): B samples packed along time, sample s at packed
  // positions [cu_seqlens[s], cu_seqlens[s+1]); L and Tx are then the packed totals.
  // NULL for the fixed [B,D,L] layout.
  const int* cu_seqlens;
  long long x_cs, io_cs, bc_cs;           // elements between channel rows (x; dt, z, y) and state rows (B, C)
  long long x_elems, io_elems, bc_elems;  // elements of x, of each of dt/z/y, of each of B/C
  int K, pad_left;
  int B2;              // samples walked by one CTA (samples per folded row)
  int d_tile;          // channels per CTA (= threads per CTA for one lane per channel)
  int chunk;           // tokens staged per step of the walk
  int flags;
  int mode;            // kModeWhole, kModeChunk or kModeLanes
  int lanes;           // lanes per channel in kModeLanes (chunk = lanes * kLaneTokens)
  int cpt;             // channels per thread in the whole/chunk modes (1 or 2)
  int np;              // N padded to a power of two (at least 2)
  int exp2_fma_pairs;  // state pairs per token whose exp2 runs on the FMA pipe (N = 16 path)
  // shared-memory carve-up (bytes), computed on the host
  int x_row, io_row, y_row, smem_bytes;
};

// Staging modes of the forward kernel: whole-sample slabs by bulk copy, or token chunks.
constexpr int kModeChunk = 0;
constexpr int kModeWhole = 1;
constexpr int kModeLanes = 2;  // P lanes per channel split the tokens (warp-shuffle scan)
constexpr int kLaneTokens = 16;  // tokens per lane per chunk in kModeLanes

// The per-token projection GEMM: P[m, n] = sum_k W[m, k] * X[n, k].
struct ProjParams {
  const void* W;    // [M, K] bf16
  const void* X;    // [Ntok, K] bf16
  void* out0;       // channel-major [B, M0, L] (rows [0, M0)) or token-major [Ntok, M]
  void* out1;       // channel-major [B, M - M0, L] (rows [M0, M)), or NULL
  int M, K, Ntok, M0, L;
  int token_major;  // 1: out0 is [Ntok, M]
  int out_f32;      // 1: fp32 outputs, else bf16
  int bn;           // output channels per CTA tile: 128 or 256
  int persistent;   // 1: one CTA per SM walks its tiles, epilogue overlapped with the next tile
};

struct BwdParams {
  const void* u;
  const void* dt;
  const void* z;
  const void* Bm;
  const void* Cm;
  const void* dout;
  const float* A;
  const float* Dskip;
  const float* dt_bias;
  float *du, *ddt, *dz, *dA, *dDskip, *ddt_bias, *dB, *dC;
  // workspace regions (carved by bwd_carve); hbuf, cB, cC and the tm_* arrays are
  // time-major [B, L, D], so the channels of a warp touch one contiguous run per token
  float *hbuf, *cB, *cC, *partBC, *partA, *partD, *partBias;
  float *tm_u, *tm_dl, *tm_gy, *tm_du, *tm_dd, *tm_y;
  float* hstore;    // [B, L, N, D]: the forward states, for the register-resident kernel
  int B, D, L, N, d_tile, ntiles;
  int softplus;
  // mixer mode (the whole layer): the scan input u = SiLU(conv(xa)) is built from x into
  // u_ws; the output gradient is read through the head<->tail swap when swap_dout
  int mixer, swap_dout, aux, conv, K, pad_left, Tx;
  const void* x;
  const float *conv_w, *conv_b;
  float *u_ws, *dx, *dconv_w, *dconv_b, *dw_part, *db_part;
};

// The dynamic shared-memory limit a kernel has been raised to, per device (the attribute
// belongs to the function on each device).  raise_smem_limit calls cudaFuncSetAttribute
// only when `bytes` exceeds what is recorded for the current device; on a device past the
// table it always calls it.  A race between host threads only repeats the same call.
struct SmemLimit {
  int have[64] = {};  // 0: the default 48 KB
};
template <typename Kern>
inline cudaError_t raise_smem_limit(Kern k, int bytes, SmemLimit& lim) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cached = dev >= 0 && dev < 64;
  if (cached && bytes <= (lim.have[dev] ? lim.have[dev] : 48 * 1024)) return cudaSuccess;
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && cached) lim.have[dev] = bytes;
  return e;
}

// Launchers (defined in the .cu files).  They only enqueue work; they return the
// cudaError_t of the launch.
cudaError_t launch_fwd(const FwdParams& p, sfm_dtype in_dtype, sfm_dtype out_dtype, int NP, cudaStream_t s);
int fwd_whole_smem(const FwdParams& p, int in_size, int out_size, int NP);
int fwd_chunk_smem(const FwdParams& p, int in_size, int out_size, int NP);
int fwd_lanes_smem(const FwdParams& p, int in_size, int out_size, int NP);
int fwd_max_smem();
int fwd_x_row(int chunk, int K, int esize);
int fwd_io_row(int chunk, int esize);
int fwd_y_row(int chunk, int esize);
cudaError_t launch_conv1d_tokens(const void* x, const float* w, const float* bias, void* u, int B, int D, int L,
                                 int K, int pad_left, int silu_on, sfm_dtype dtype, cudaStream_t s);
cudaError_t launch_proj(const ProjParams& p, cudaStream_t s);
cudaError_t launch_wait_selftest(int limit_us, cudaStream_t s);
cudaError_t read_proj_error(int clear, unsigned* value);
cudaError_t read_device_error(cudaStream_t s, int clear, unsigned* value);

cudaError_t launch_bwd(const BwdParams& p, sfm_dtype in_dtype, sfm_dtype dout_dtype, cudaStream_t s);
size_t bwd_workspace_bytes(int B, int D, int L, int N, int d_tile);
void bwd_carve(BwdParams& p, char* ws);
size_t mixer_bwd_workspace_bytes(int B, int D, int L, int N, int K, int d_tile);
void mixer_bwd_carve(BwdParams& p, char* ws);
cudaError_t launch_mixer_bwd(const BwdParams& p, sfm_dtype in_dtype, sfm_dtype dout_dtype, cudaStream_t s);
cudaError_t noalloc_scratch(void** out);  // device address of the built-in workspace

cudaError_t launch_aux_init(const void* x, void* xa, int B, int D, int T, int esize, cudaStream_t s);
cudaError_t launch_aux_swap(void* y, int B, int D, int L, int esize, cudaStream_t s);
cudaError_t launch_conv1d(const void* x, const float* w, const float* bias, void* u, int B, int D, int L, int K,
                          int pad_left, int silu, sfm_dtype dtype, cudaStream_t s);

}  // namespace sfm
