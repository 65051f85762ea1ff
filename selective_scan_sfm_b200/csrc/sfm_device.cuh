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

__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---- functions on the FMA pipe, to take load off the transcendental unit -------------
// Coefficients: minimax polynomials fitted by the Remez exchange in
// selective_scan_sfm_b200/poly_fit.py (fp32-rounded; the script reports their error).

// 2^x for a pair of values.  Cody-Waite split x = j + f, j = round(x) (by adding and
// subtracting 1.5*2^23), f in [-1/2, 1/2]; 2^f from a degree-5 polynomial (max relative
// error 2.4e-7 in fp32, the accuracy of the hardware ex2.approx); 2^j is added into the
// exponent field.  x is clamped to [-126, 126] so the result stays a normal number (a
// NaN passes through the comparisons and stays NaN).
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  x.x = x.x < -126.0f ? -126.0f : x.x;
  x.y = x.y < -126.0f ? -126.0f : x.y;
  x.x = x.x > 126.0f ? 126.0f : x.x;
  x.y = x.y > 126.0f ? 126.0f : x.y;
  const float2 M = make_float2(12582912.0f, 12582912.0f), mM = make_float2(-12582912.0f, -12582912.0f);
  const float2 t = __fadd2_rn(x, M);
  const float2 j = __fadd2_rn(t, mM);
  const float2 f = __ffma2_rn(j, make_float2(-1.0f, -1.0f), x);
  float2 p = __ffma2_rn(make_float2(1.327647245e-03f, 1.327647245e-03f), f,
                        make_float2(9.675540961e-03f, 9.675540961e-03f));
  p = __ffma2_rn(p, f, make_float2(5.550713092e-02f, 5.550713092e-02f));
  p = __ffma2_rn(p, f, make_float2(2.402212024e-01f, 2.402212024e-01f));
  p = __ffma2_rn(p, f, make_float2(6.931469440e-01f, 6.931469440e-01f));
  p = __ffma2_rn(p, f, make_float2(1.000000119e+00f, 1.000000119e+00f));
  p.x = __int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23));
  p.y = __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23));
  return p;
}

// softplus(v) = max(v, 0) + log(1 + w), w = e^-|v| in (0, 1], with log(1 + w) = w * q(w)
// and q a degree-7 polynomial (max relative error 3.3e-7 in fp32): one transcendental.
__device__ __forceinline__ float softplus_fast(float v) {
  const float w = ex2(-fabsf(v) * kLog2e);
  float q = fmaf(-8.539208211e-03f, w, 4.408963397e-02f);
  q = fmaf(q, w, -1.076817140e-01f);
  q = fmaf(q, w, 1.774524152e-01f);
  q = fmaf(q, w, -2.449546307e-01f);
  q = fmaf(q, w, 3.327547908e-01f);
  q = fmaf(q, w, -4.999740422e-01f);
  q = fmaf(q, w, 9.999998212e-01f);
  return fmaxf(v, 0.0f) + w * q;
}

// SiLU(v) = v * (1 + tanh(v/2)) / 2 with the hardware tanh (relative error about 2^-11):
// one transcendental instead of two.  Used only where the output is rounded to bf16.
__device__ __forceinline__ float silu_fast(float v) {
  const float h = 0.5f * v;
  return fmaf(h, tanh_approx(h), h);
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
  const char* src = base + ga;
  if (ga + 16LL * granules <= tensor_bytes) {  // every granule lies inside the tensor
    for (int q = lane; q < granules; q += nlanes) cp_async16(dst + 16 * q, src + 16 * q, 16);
    return;
  }
  for (int q = lane; q < granules; q += nlanes) {  // the span reaches the tensor's last granule
    const long long rem = tensor_bytes - (ga + 16LL * q);
    const int bytes = rem >= 16 ? 16 : (rem > 0 ? (int)rem : 0);
    cp_async16(dst + 16 * q, bytes > 0 ? src + 16 * q : src, bytes);
  }
}

// Stores the row segment staged at smem `src` (element 0 at byte (e0*esize) & 15 of a
// 16-byte granule, the layout copy_span_async produces) to global elements
// [e0, e0 + cnt) of `base`: 16-byte vector stores where both sides are aligned, element
// stores at the ragged ends.  `skip0` leaves element e0 untouched.
template <typename T>
__device__ __forceinline__ void store_row(T* base, long long e0, const char* src_granule, int cnt, bool skip0) {
  constexpr int es = sizeof(T), per16 = 16 / es;
  const int head = (int)((e0 * es) & 15);
  const T* s = reinterpret_cast<const T*>(src_granule + head);
  T* d = base + e0;
  int i = 0;
  const int lead = head ? min(cnt, (16 - head) / es) : 0;  // elements before the first aligned granule
  for (; i < lead; ++i)
    if (!(skip0 && i == 0)) d[i] = s[i];
  for (; i + per16 <= cnt; i += per16) {
    const int4 v = *reinterpret_cast<const int4*>(s + i);
    if (skip0 && i == 0) {  // only when the row starts aligned: keep element 0 as it is
      for (int k = 1; k < per16; ++k) d[k] = s[k];
    } else {
      *reinterpret_cast<int4*>(d + i) = v;
    }
  }
  for (; i < cnt; ++i)
    if (!(skip0 && i == 0)) d[i] = s[i];
}

__device__ __forceinline__ int span_head(long long e0, int esize) { return (int)((e0 * esize) & 15); }


// ------------------------------------------------------------------ mbarriers with bounded waits

constexpr unsigned long long kWaitNs = 2000000000ull;  // every wait on an mbarrier gives up after 2 s


__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Polls the barrier until the phase with `parity` completes or kWaitNs elapse.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, unsigned parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity))
    if (global_ns() - t0 > kWaitNs) return false;
  return true;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}

// A bounded wait with an explicit limit in nanoseconds (the self-test of the timeout path).
__device__ __forceinline__ bool mbar_wait_for(uint64_t* bar, unsigned parity, unsigned long long limit_ns) {
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    __nanosleep(1000);
    if (global_ns() - t0 > limit_ns) return false;
  }
  return true;
}

// The same bounded wait for threads off the critical path (a whole CTA waiting for its
// accumulator): they sleep between polls so co-resident CTAs keep the issue slots.
__device__ __forceinline__ bool mbar_wait_bounded_sleepy(uint64_t* bar, unsigned parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    __nanosleep(256);
    if (global_ns() - t0 > kWaitNs) return false;
  }
  return true;
}

}  // namespace sfm
