// sfm_misc.cu -- the single steps of the hot path as standalone kernels (sm_100a):
// aux init, aux swap and the boundary-safe depthwise conv1d.  They serve callers that
// run the steps separately and the unfused comparison; the fused forward kernel does
// the same work inside its loads and stores.
//
// Sources: "Seeing Both Ways, Running One Way" (sungsoo.github.io) section 3.2 (aux tokens,
// head<->tail swap) and section 8.1 item 5 (conv that does not cross folded sample
// boundaries); "SF-Mamba：重新思考视觉 Mamba 的信息流与并行效率" (techloop.online), Auxiliary Patch
// Swapping and the convolution-boundary paragraph.
#include "sfm_device.cuh"
#include "sfm_internal.h"

namespace sfm {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One warp per (b,d) row: coalesced read of the T tokens, warp-reduced fp32 mean,
// coalesced write of the T+2 tokens of xa.
template <typename T>
__global__ void aux_init_kernel(const T* __restrict__ x, T* __restrict__ xa, long long rows, int Tn) {
  const int lane = threadIdx.x & 31;
  const long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= rows) return;
  const T* xr = x + r * Tn;
  T* ar = xa + r * (Tn + 2);
  float s = 0.0f;
  for (int t = lane; t < Tn; t += 32) s += to_f(xr[t]);
  s = warp_sum(s);
  const T m = from_f<T>(s / (float)Tn);
  for (int t = lane; t < Tn; t += 32) ar[t + 1] = xr[t];
  if (lane == 0) {
    ar[0] = m;
    ar[Tn + 1] = m;
  }
}

// One thread per row exchanges tokens 0 and L-1.
template <typename T>
__global__ void aux_swap_kernel(T* __restrict__ y, long long rows, int L) {
  const long long r = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= rows) return;
  T* yr = y + r * L;
  const T h = yr[0];
  yr[0] = yr[L - 1];
  yr[L - 1] = h;
}

// One warp per (b,d) row; lane i produces tokens i, i+32, ...  Reads outside [0, L) of
// the row's own sample are zeros: a folded row never sees its neighbour sample.
template <typename T>
__global__ void conv1d_kernel(const T* __restrict__ x, const float* __restrict__ w, const float* __restrict__ bias,
                              T* __restrict__ u, long long rows, int D, int L, int K, int pad_left, int silu_on) {
  const int lane = threadIdx.x & 31;
  const long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int d = (int)(r % D);
  float wk[SFM_MAX_K];
#pragma unroll
  for (int k = 0; k < SFM_MAX_K; ++k) wk[k] = k < K ? w[(size_t)d * K + k] : 0.0f;
  const float b0 = bias ? bias[d] : 0.0f;
  const T* xr = x + r * L;
  T* ur = u + r * L;
  for (int t = lane; t < L; t += 32) {
    float acc = b0;
#pragma unroll
    for (int k = 0; k < SFM_MAX_K; ++k) {
      const int s = t + k - pad_left;
      if (k < K && s >= 0 && s < L) acc = fmaf(wk[k], to_f(xr[s]), acc);
    }
    ur[t] = from_f<T>(silu_on ? silu(acc) : acc);
  }
}

// The same conv written token-major, u[b*L + t, d]: the layout the state projection reads
// (one row of D features per token).  A CTA takes 32 tokens x 64 channels of one sample:
// the x rows it needs (with the taps' halo, zero outside the sample) are staged in shared
// memory by coalesced row reads, and each token's 64 channels leave as one contiguous run.
template <typename T>
__global__ void __launch_bounds__(256) conv1d_tokens_kernel(const T* __restrict__ x, const float* __restrict__ w,
                                                            const float* __restrict__ bias, T* __restrict__ u,
                                                            int D, int L, int K, int pad_left, int silu_on) {
  constexpr int TT = 32, DT = 64, HALO = SFM_MAX_K - 1, ROW = TT + HALO + 1;  // odd row stride: no bank conflicts
  __shared__ float xs[DT][ROW];
  const int t0 = blockIdx.x * TT, d0 = blockIdx.y * DT, b = blockIdx.z;
  const int tid = threadIdx.x;
  for (int e = tid; e < DT * (TT + HALO); e += blockDim.x) {
    const int c = e / (TT + HALO), i = e % (TT + HALO);
    const int d = d0 + c, s = t0 - pad_left + i;
    xs[c][i] = (d < D && s >= 0 && s < L) ? to_f(x[((size_t)b * D + d) * L + s]) : 0.0f;
  }
  __syncthreads();
  for (int e = tid; e < TT * DT; e += blockDim.x) {
    const int i = e / DT, c = e % DT;  // channel fastest: the stores of a token are contiguous
    const int t = t0 + i, d = d0 + c;
    if (t >= L || d >= D) continue;
    float acc = bias ? bias[d] : 0.0f;
    for (int k = 0; k < K; ++k) acc = fmaf(w[(size_t)d * K + k], xs[c][i + k], acc);
    u[((size_t)b * L + t) * D + d] = from_f<T>(silu_on ? silu(acc) : acc);
  }
}

static unsigned blocks_for(long long items, int per_block) { return (unsigned)((items + per_block - 1) / per_block); }

cudaError_t launch_conv1d_tokens(const void* x, const float* w, const float* bias, void* u, int B, int D, int L,
                                 int K, int pad_left, int silu_on, sfm_dtype dtype, cudaStream_t s) {
  dim3 grid((L + 31) / 32, (D + 63) / 64, B);
  if (dtype == SFM_F32)
    conv1d_tokens_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float*>(x), w, bias, static_cast<float*>(u),
                                                     D, L, K, pad_left, silu_on);
  else
    conv1d_tokens_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), w, bias,
                                                             static_cast<__nv_bfloat16*>(u), D, L, K, pad_left,
                                                             silu_on);
  return cudaGetLastError();
}

cudaError_t launch_aux_init(const void* x, void* xa, int B, int D, int T, int esize, cudaStream_t s) {
  const long long rows = (long long)B * D;
  const int threads = 256, per = threads / 32;
  if (esize == 4)
    aux_init_kernel<float><<<blocks_for(rows, per), threads, 0, s>>>(static_cast<const float*>(x),
                                                                      static_cast<float*>(xa), rows, T);
  else
    aux_init_kernel<__nv_bfloat16><<<blocks_for(rows, per), threads, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<__nv_bfloat16*>(xa), rows, T);
  return cudaGetLastError();
}

cudaError_t launch_aux_swap(void* y, int B, int D, int L, int esize, cudaStream_t s) {
  const long long rows = (long long)B * D;
  const int threads = 256;
  if (esize == 4)
    aux_swap_kernel<float><<<blocks_for(rows, threads), threads, 0, s>>>(static_cast<float*>(y), rows, L);
  else
    aux_swap_kernel<__nv_bfloat16><<<blocks_for(rows, threads), threads, 0, s>>>(static_cast<__nv_bfloat16*>(y),
                                                                                  rows, L);
  return cudaGetLastError();
}

cudaError_t launch_conv1d(const void* x, const float* w, const float* bias, void* u, int B, int D, int L, int K,
                          int pad_left, int silu_on, sfm_dtype dtype, cudaStream_t s) {
  const long long rows = (long long)B * D;
  const int threads = 256, per = threads / 32;
  if (dtype == SFM_F32)
    conv1d_kernel<float><<<blocks_for(rows, per), threads, 0, s>>>(static_cast<const float*>(x), w, bias,
                                                                    static_cast<float*>(u), rows, D, L, K,
                                                                    pad_left, silu_on);
  else
    conv1d_kernel<__nv_bfloat16><<<blocks_for(rows, per), threads, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), w, bias, static_cast<__nv_bfloat16*>(u), rows, D, L, K, pad_left,
        silu_on);
  return cudaGetLastError();
}

}  // namespace sfm
