// sfm_device.cuh -- device helpers shared by the libsfm kernels (sm_100a only).
//
// Hardware transcendental instructions are called directly (ex2/lg2/rcp are the MUFU
// unit); the few functions built from them (softplus, SiLU) are written here from
// their mathematical definitions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sfm {

constexpr float kLog2e = 1.4426950408889634f;  // log2(e)
constexpr float kLn2 = 0.6931471805599453f;    // ln(2)

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// SiLU(v) = v * sigmoid(v) = v / (1 + e^-v).  For e^-v = inf the reciprocal is 0.
__device__ __forceinline__ float silu(float v) { return v * rcp(1.0f + ex2(-v * kLog2e)); }

// softplus(v) = log(1 + e^v), and v itself above 20 (same threshold as the usual
// deep-learning definition).  log(1+w) is taken from the Mercator series
// w - w^2/2 + ... - w^6/6 when w = e^v < e^-2.5 (truncation < 5e-8 relative), where
// 1 + w would lose the low bits of w; otherwise from lg2(1 + w).
__device__ __forceinline__ float softplus(float v) {
  const float w = ex2(v * kLog2e);
  const float series =
      w * fmaf(w, fmaf(w, fmaf(w, fmaf(w, fmaf(w, -1.0f / 6.0f, 0.2f), -0.25f), 1.0f / 3.0f), -0.5f), 1.0f);
  const float viaLog = lg2(1.0f + w) * kLn2;
  const float r = v < -2.5f ? series : viaLog;
  return v > 20.0f ? v : r;
}

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte asynchronous global->shared copy (L2 only).  src_bytes < 16 copies that many
// bytes and zero-fills the rest of the granule; src_bytes == 0 copies nothing.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(smem_dst)), "l"(gsrc),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Copies the element range [e0, e0 + cnt) of a tensor whose base is 16-byte aligned and
// whose total size is `tensor_bytes`, into `dst` (16-byte aligned), starting at the
// 16-byte granule that holds element e0.  The element e0 lands at byte
// (e0 * esize) & 15 of dst.  Granules past the tensor end are zero-filled, never read.
// Lanes [lane0, lane0 + nlanes) of the calling group issue the granules.
__device__ __forceinline__ void copy_span_async(char* dst, const char* base, long long e0, int cnt, int esize,
                                                long long tensor_bytes, int lane, int nlanes) {
  if (cnt <= 0) return;
  const long long g = e0 * esize;
  const long long ga = g & ~15LL;
  const int total = (int)(g - ga) + cnt * esize;
  const int granules = (total + 15) >> 4;
  for (int q = lane; q < granules; q += nlanes) {
    const long long off = ga + 16LL * q;
    long long rem = tensor_bytes - off;
    const int bytes = rem >= 16 ? 16 : (rem > 0 ? (int)rem : 0);
    cp_async16(dst + 16 * q, base + (bytes > 0 ? off : ga), bytes);
  }
}

__device__ __forceinline__ int span_head(long long e0, int esize) { return (int)((e0 * esize) & 15); }

}  // namespace sfm
