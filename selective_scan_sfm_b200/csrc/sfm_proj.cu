// sfm_proj.cu -- the per-token projections around the scan as tcgen05 GEMMs on B200.
//
// A Mamba mixer feeds its scan through dense per-token linear maps: the input projection
// gives the conv input x and the gate z, the state projection gives the step size (at low
// rank, widened by a second map) and B, C.  Each is
//
//     P[m, n] = sum_k W[m, k] * X[n, k]        (m: output channel, n: token, k: input channel)
//
// with W a [M, K] weight (the nn.Linear layout) and X one row of K features per token.
// The tokens are the MMA's M side (128 per CTA, flattened over the samples) and the
// output channels its N side, so TMEM lane i of a CTA's accumulator is token n0 + i and
// column j is channel c0 + j.  A warp owns 32 TMEM lanes = 32 consecutive tokens; for
// each channel it writes those 32 tokens with one coalesced store into the channel's
// row of the scan's channel-major [B, rows, L] layout (a run that breaks at most where a
// sample ends), straight from registers.
//
//   * operands: bf16 tiles of 64 K-elements (one 128-byte swizzle row) moved by TMA
//     (cp.async.bulk.tensor, no multicast) into a ring of STAGES shared-memory stages,
//     each stage signalled by an mbarrier with its byte count;
//   * math: one thread issues tcgen05.mma.cta_group::1.kind::f16 (bf16 x bf16 -> fp32),
//     M = 128 tokens, N = 128 or 256 channels, K = 16 per instruction, the accumulator
//     in tensor memory (instruction descriptor: fp32 accumulator, bf16 A and B, both
//     K-major, N >> 3 at bits 17-22, M >> 4 at bits 24-28); tcgen05.commit frees a stage
//     when the MMAs reading it are done;
//   * epilogue: eight warps read the accumulator (32x32b loads; warp w its lane quarter
//     w % 4, column half w / 4), round to the output type and store: per channel one
//     warp store (channel-major), or 16-byte vectors of a token's channels (token-major).
//
// Every mbarrier wait is bounded (kWaitNs); a wait that gives up records SFM_ERR_TIMEOUT
// in the device error word, lets the in-flight copies land (bounded again), frees the
// tensor memory and skips the stores.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sfm.h"
#include "sfm_device.cuh"
#include "sfm_internal.h"

namespace sfm {

__device__ unsigned int g_proj_error = 0;

namespace {

constexpr int kBM = 128;     // weight rows (output channels) per CTA = TMEM lanes
constexpr int kBK = 64;      // K elements per stage: one 128-byte swizzled row of bf16
constexpr int kUmmaK = 16;   // K per tcgen05.mma for 16-bit inputs
constexpr int kThreads = 256;   // 8 warps: warp w reads TMEM lane quarter w % 4, column half w / 4

// Shared-memory matrix descriptor of a K-major bf16 tile stored as TMA writes it with
// 128-byte swizzling: rows of 128 bytes, 8-row groups 1024 bytes apart.
//   bits  0-13 start address >> 4      bits 16-29 leading-dimension offset >> 4 (unused
//   for swizzled K-major; 1)            bits 32-45 stride offset >> 4 (1024 B -> 64)
//   bits 46-47 descriptor version (1 on sm_100)    bits 61-63 swizzle mode (2 = 128 B)
__device__ __forceinline__ uint64_t kmajor_sw128_desc(uint32_t smem_addr) {
  return (uint64_t)((smem_addr & 0x3FFFFu) >> 4) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];\n" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane (base + i)'s
// 32 columns.
__device__ __forceinline__ void tmem_ld_32x32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// A CTA computes 128 tokens (the MMA's M side; TMEM lane = token, flattened over the
// samples) by NT output channels (the N side; TMEM column = channel).  Because a warp's 32
// TMEM lanes are 32 consecutive tokens, writing one channel of them is one coalesced warp
// store into that channel's row of the channel-major output: no staging in shared memory.
template <int NT, int STAGES>
struct ProjSmem {
  static constexpr int kStageA = kBM * kBK * 2;  // bytes of one token tile (A)
  static constexpr int kStageB = NT * kBK * 2;   // bytes of one weight tile (B)
  static constexpr int kRing = STAGES * (kStageA + kStageB);
  static constexpr int kBars = (2 * STAGES + 1) * 8 + 16;
  static constexpr int kBytes = 1024 + kRing + kBars;  // + 1024 for the 1024-byte alignment of the ring
};

template <int NT, int STAGES, typename TO>
__global__ void __launch_bounds__(kThreads)
    proj_gemm_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const ProjParams p) {
  using SM = ProjSmem<NT, STAGES>;
  extern __shared__ __align__(16) char smem_raw[];
  char* ring = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + SM::kRing);
  uint64_t* empty = full + STAGES;
  uint64_t* done = empty + STAGES;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(done + 1) + 1;
  auto stage_a = [&](int s) { return ring + s * SM::kStageA; };
  auto stage_b = [&](int s) { return ring + STAGES * SM::kStageA + s * SM::kStageB; };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * kBM;  // first token
  const int c0 = blockIdx.y * NT;   // first output channel
  const int nk = (p.K + kBK - 1) / kBK;

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 0) {  // the accumulator: NT fp32 columns x 128 lanes
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     smem_u32(const_cast<uint32_t*>(tmem_slot))),
                 "r"((uint32_t)NT)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---- producer: one TMA pair per K step into the ring
    int issued = 0;
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % STAGES;
      if (kb >= STAGES && !mbar_wait_bounded(&empty[s], ((kb / STAGES) - 1) & 1)) {
        atomicExch(&g_proj_error, (unsigned)SFM_ERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      if (*abort_flag) break;
      mbar_expect_tx(&full[s], (unsigned)(SM::kStageA + SM::kStageB));
      tma_load_2d(stage_a(s), &tmX, kb * kBK, n0, &full[s]);
      tma_load_2d(stage_b(s), &tmW, kb * kBK, c0, &full[s]);
      issued = kb + 1;
    }
    if (*abort_flag) {  // let the copies still in flight land before the CTA leaves
      for (int kb = issued > STAGES ? issued - STAGES : 0; kb < issued; ++kb)
        mbar_wait_bounded(&full[kb % STAGES], (kb / STAGES) & 1);
    }
  } else if (warp == 1 && lane == 0) {
    // ---- MMA issuer: M = 128 tokens, N = NT channels, K = 16 per instruction
    const uint32_t idesc =
        (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(NT >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % STAGES;
      if (!mbar_wait_bounded(&full[s], (kb / STAGES) & 1)) {
        atomicExch(&g_proj_error, (unsigned)SFM_ERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint64_t da = kmajor_sw128_desc(smem_u32(stage_a(s)));
      const uint64_t db = kmajor_sw128_desc(smem_u32(stage_b(s)));
#pragma unroll
      for (int kk = 0; kk < kBK / kUmmaK; ++kk)  // +32 bytes (2 in descriptor units) per K step
        umma_f16(tmem, da + 2 * kk, db + 2 * kk, idesc, (kb | kk) != 0);
      umma_commit(&empty[s]);  // the stage is free once these MMAs have read it
    }
    umma_commit(done);  // every MMA issued above has completed (also on the abort path)
  }
  __syncwarp();

  // ---- epilogue: TMEM -> registers -> global, no shared memory
  const bool ok = mbar_wait_bounded_sleepy(done, 0);
  if (!ok && tid == 0) {
    atomicExch(&g_proj_error, (unsigned)SFM_ERR_TIMEOUT);
    *abort_flag = 1;
  }
  tc_fence_after();
  __syncthreads();
  if (ok && !*abort_flag) {
    const int q = warp & 3, half = warp >> 2;
    const int n = n0 + q * 32 + lane;  // this thread's token (TMEM lane)
    const bool tok_ok = n < p.Ntok;
    const int b = n / p.L, t = n - b * p.L;
    // element of (this token, channel m): out0[base0 + m * L] (m < M0) or
    // out1[base1 + (m - M0) * L]; token-major: out0[n * M + m]
    const long long base0 = (long long)b * p.M0 * p.L + t;
    const long long base1 = (long long)b * (p.M - p.M0) * p.L + t;
    TO* out0 = static_cast<TO*>(p.out0);
    TO* out1 = static_cast<TO*>(p.out1);
#pragma unroll 1
    for (int cc = half * (NT / 2); cc < (half + 1) * (NT / 2) && c0 + cc < p.M; cc += 32) {
      float v[32];
      tmem_ld_32x32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)cc, v);
      if (!tok_ok) continue;
      const int m = c0 + cc;
      if (p.token_major) {
        TO* dst = out0 + (size_t)n * p.M + m;
        if (m + 32 <= p.M && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
          constexpr int E = 16 / (int)sizeof(TO);
#pragma unroll
          for (int j = 0; j < 32; j += E) {
            uint32_t w[4];
            if constexpr (sizeof(TO) == 2) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const __nv_bfloat162 h = __floats2bfloat162_rn(v[j + 2 * k], v[j + 2 * k + 1]);
                w[k] = *reinterpret_cast<const uint32_t*>(&h);
              }
            } else {
#pragma unroll
              for (int k = 0; k < 4; ++k) w[k] = __float_as_uint(v[j + k]);
            }
            *reinterpret_cast<uint4*>(dst + j) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (m + j < p.M) dst[j] = from_f<TO>(v[j]);
        }
      } else {  // one coalesced warp store per channel: 32 consecutive tokens of its row
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int mj = m + j;
          if (mj < p.M0)
            out0[base0 + (long long)mj * p.L] = from_f<TO>(v[j]);
          else if (mj < p.M)
            out1[base1 + (long long)(mj - p.M0) * p.L] = from_f<TO>(v[j]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"((uint32_t)NT)
                 : "memory");
  }
}

// ------------------------------------------------------------------ persistent form
//
// One CTA per SM walks its tiles (tile t, t + gridDim.x, ...; the channel tile varies
// fastest) with the work split by warp:
//   warp 0  (one thread) TMA producer: keeps a ring of STAGES K-slices full across tiles;
//   warp 1  (one thread) MMA issuer:   accumulates tile i in TMEM buffer i % 2;
//   warps 2-9            epilogue:     drain buffer i % 2 into registers, hand it back to
//                                      the MMA warp, then store while tile i + 1 accumulates.
// Handshakes are mbarriers: full/empty per ring stage (TMA <-> MMA), acc_full/acc_empty per
// accumulator (MMA <-> epilogue).  Every wait is bounded; a wait that gives up records
// SFM_ERR_TIMEOUT, every role leaves its loop, the MMA warp drains its own MMAs and the
// producer its own copies (both bounded), and the tensor memory is freed.
constexpr int kPThreads = 320;

template <int NT, int STAGES>
struct PSmem {
  static constexpr int kStageA = kBM * kBK * 2;
  static constexpr int kStageB = NT * kBK * 2;
  static constexpr int kRing = STAGES * (kStageA + kStageB);
  static constexpr int kBars = (2 * STAGES + 5) * 8 + 16;
  static constexpr int kBytes = 1024 + kRing + kBars;
};

template <int NT, int STAGES, typename TO>
__global__ void __launch_bounds__(kPThreads, 1)
    proj_gemm_persistent(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                         const ProjParams p) {
  using SM = PSmem<NT, STAGES>;
  extern __shared__ __align__(16) char smem_raw[];
  char* ring = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + SM::kRing);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;  // [2]
  uint64_t* acc_empty = acc_full + 2;   // [2]
  uint64_t* drain = acc_empty + 2;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(drain + 1) + 1;
  auto stage_a = [&](int s) { return ring + s * SM::kStageA; };
  auto stage_b = [&](int s) { return ring + STAGES * SM::kStageA + s * SM::kStageB; };
  auto give_up = [&]() {
    atomicExch(&g_proj_error, (unsigned)SFM_ERR_TIMEOUT);
    *abort_flag = 1;
  };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_ct = (p.M + NT - 1) / NT, n_tt = (p.Ntok + kBM - 1) / kBM;
  const int ntiles = n_ct * n_tt;
  const int nk = (p.K + kBK - 1) / kBK;

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 8);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 0) {  // two accumulators of NT fp32 columns x 128 lanes
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     smem_u32(const_cast<uint32_t*>(tmem_slot))),
                 "r"((uint32_t)(2 * NT))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {  // ---- producer
      long long g = 0;
      for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
        const int n0 = (tile / n_ct) * kBM, c0 = (tile % n_ct) * NT;
        for (int kb = 0; kb < nk; ++kb, ++g) {
          const int s = (int)(g % STAGES);
          const long long u = g / STAGES;
          if (u >= 1 && !mbar_wait_bounded(&empty[s], (unsigned)((u - 1) & 1))) {
            give_up();
            break;
          }
          if (*abort_flag) break;
          mbar_expect_tx(&full[s], (unsigned)(SM::kStageA + SM::kStageB));
          tma_load_2d(stage_a(s), &tmX, kb * kBK, n0, &full[s]);
          tma_load_2d(stage_b(s), &tmW, kb * kBK, c0, &full[s]);
        }
      }
      if (*abort_flag)  // let the copies still in flight land before the CTA leaves
        for (long long q = g > STAGES ? g - STAGES : 0; q < g; ++q)
          mbar_wait_bounded(&full[q % STAGES], (unsigned)((q / STAGES) & 1));
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---- MMA issuer
      const uint32_t idesc =
          (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(NT >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
      long long g = 0;
      int li = 0;
      for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x, ++li) {
        const int a = li & 1, use = li >> 1;
        if (use >= 1 && !mbar_wait_bounded(&acc_empty[a], (unsigned)((use - 1) & 1))) {
          give_up();
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(a * NT);
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb, ++g) {
          const int s = (int)(g % STAGES);
          if (!mbar_wait_bounded(&full[s], (unsigned)((g / STAGES) & 1))) {
            give_up();
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t da = kmajor_sw128_desc(smem_u32(stage_a(s)));
          const uint64_t db = kmajor_sw128_desc(smem_u32(stage_b(s)));
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk)
            umma_f16(acc, da + 2 * kk, db + 2 * kk, idesc, (kb | kk) != 0);
          umma_commit(&empty[s]);
        }
        if (!ok) break;
        umma_commit(&acc_full[a]);
      }
      umma_commit(drain);  // every MMA issued above has completed once this arrives
      if (!mbar_wait_bounded(drain, 0)) give_up();
    }
  } else {  // ---- epilogue: warps 2-9; warp w reads TMEM lane quarter w % 4, column half (w - 2) / 4
    const int q = warp & 3, half = (warp - 2) >> 2;
    int li = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++li) {
      const int a = li & 1, use = li >> 1;
      if (!mbar_wait_bounded_sleepy(&acc_full[a], (unsigned)(use & 1))) {
        if (lane == 0) give_up();
        break;
      }
      if (*abort_flag) break;
      tc_fence_after();
      float v[NT / 2];
#pragma unroll
      for (int j = 0; j < NT / 2; j += 32) {
        float w[32];
        tmem_ld_32x32(tmem + (uint32_t)(a * NT) + ((uint32_t)(q * 32) << 16) + (uint32_t)(half * (NT / 2) + j), w);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[j + i] = w[i];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[a]);  // the accumulator may be overwritten now

      const int n0 = (tile / n_ct) * kBM, cbase = (tile % n_ct) * NT + half * (NT / 2);
      const int n = n0 + q * 32 + lane;
      if (n >= p.Ntok) continue;
      const int b = n / p.L, t = n - b * p.L;
      const long long base0 = (long long)b * p.M0 * p.L + t;
      const long long base1 = (long long)b * (p.M - p.M0) * p.L + t;
      TO* out0 = static_cast<TO*>(p.out0);
      TO* out1 = static_cast<TO*>(p.out1);
      if (p.token_major) {
        TO* dst = out0 + (size_t)n * p.M + cbase;
        if (cbase + NT / 2 <= p.M && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
          constexpr int E = 16 / (int)sizeof(TO);
#pragma unroll
          for (int j = 0; j < NT / 2; j += E) {
            uint32_t w[4];
            if constexpr (sizeof(TO) == 2) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const __nv_bfloat162 h = __floats2bfloat162_rn(v[j + 2 * k], v[j + 2 * k + 1]);
                w[k] = *reinterpret_cast<const uint32_t*>(&h);
              }
            } else {
#pragma unroll
              for (int k = 0; k < 4; ++k) w[k] = __float_as_uint(v[j + k]);
            }
            *reinterpret_cast<uint4*>(dst + j) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < NT / 2; ++j)
            if (cbase + j < p.M) dst[j] = from_f<TO>(v[j]);
        }
      } else {  // one coalesced warp store per channel: 32 consecutive tokens of its row
#pragma unroll
        for (int j = 0; j < NT / 2; ++j) {
          const int m = cbase + j;
          if (m < p.M0)
            out0[base0 + (long long)m * p.L] = from_f<TO>(v[j]);
          else if (m < p.M)
            out1[base1 + (long long)(m - p.M0) * p.L] = from_f<TO>(v[j]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"((uint32_t)(2 * NT))
                 : "memory");
  }
}

// ------------------------------------------------------------------ host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

// [rows, K] bf16, K contiguous; tiles of 64 K-elements x box_rows rows, 128-byte swizzle;
// rows and K past the ends read as zeros.
bool make_kmajor_map(CUtensorMap* map, const void* base, long long rows, int K, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
  cuuint32_t estride[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estride,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NT, int STAGES, typename TO>
cudaError_t launch_nt(const ProjParams& p, const CUtensorMap& mx, const CUtensorMap& mw, cudaStream_t s) {
  constexpr int bytes = ProjSmem<NT, STAGES>::kBytes;
  static SmemLimit lim;
  cudaError_t e = raise_smem_limit(proj_gemm_kernel<NT, STAGES, TO>, bytes, lim);
  if (e != cudaSuccess) return e;
  dim3 grid((p.Ntok + kBM - 1) / kBM, (p.M + NT - 1) / NT);
  proj_gemm_kernel<NT, STAGES, TO><<<grid, kThreads, bytes, s>>>(mx, mw, p);
  return cudaGetLastError();
}

template <int NT, int STAGES, typename TO>
cudaError_t launch_persistent(const ProjParams& p, const CUtensorMap& mx, const CUtensorMap& mw, cudaStream_t s) {
  constexpr int bytes = PSmem<NT, STAGES>::kBytes;
  static SmemLimit lim;
  cudaError_t e = raise_smem_limit(proj_gemm_persistent<NT, STAGES, TO>, bytes, lim);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long tiles = (long long)((p.M + NT - 1) / NT) * ((p.Ntok + kBM - 1) / kBM);
  const int grid = (int)(tiles < sms ? tiles : sms);
  proj_gemm_persistent<NT, STAGES, TO><<<grid, kPThreads, bytes, s>>>(mx, mw, p);
  return cudaGetLastError();
}

template <typename TO>
cudaError_t launch_to(const ProjParams& p, cudaStream_t s) {
  CUtensorMap mx, mw;
  const int nt = p.bn <= 128 ? 128 : 256;
  if (!make_kmajor_map(&mx, p.X, p.Ntok, p.K, kBM) || !make_kmajor_map(&mw, p.W, p.M, p.K, nt))
    return cudaErrorInvalidValue;
  if (p.persistent) {
    if (nt == 128) return launch_persistent<128, 6, TO>(p, mx, mw, s);
    return launch_persistent<256, 4, TO>(p, mx, mw, s);
  }
  // K of at most 10 stages: a 2-stage ring, so several CTAs share an SM and one's epilogue
  // overlaps the others' loads and MMAs; longer K: 4 stages
  const bool short_k = p.K <= 10 * kBK;
  if (nt == 128) return short_k ? launch_nt<128, 2, TO>(p, mx, mw, s) : launch_nt<128, 4, TO>(p, mx, mw, s);
  return short_k ? launch_nt<256, 2, TO>(p, mx, mw, s) : launch_nt<256, 4, TO>(p, mx, mw, s);
}

}  // namespace

cudaError_t launch_proj(const ProjParams& p, cudaStream_t s) {
  return p.out_f32 ? launch_to<float>(p, s) : launch_to<__nv_bfloat16>(p, s);
}

// Self-test of the timeout path: one thread waits on an mbarrier that nothing will ever
// arrive on, with a limit of limit_us; when the wait gives up it records SFM_ERR_TIMEOUT
// in the device error word, exactly as the kernels' own waits do, and returns.
__global__ void wait_timeout_selftest_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  if (!mbar_wait_for(&bar, 0, limit_ns)) atomicExch(&g_proj_error, (unsigned)SFM_ERR_TIMEOUT);
}

cudaError_t launch_wait_selftest(int limit_us, cudaStream_t s) {
  wait_timeout_selftest_kernel<<<1, 32, 0, s>>>(1000ull * (unsigned long long)limit_us);
  return cudaGetLastError();
}

cudaError_t read_proj_error(int clear, unsigned* value) {
  cudaError_t e = cudaMemcpyFromSymbol(value, g_proj_error, sizeof(unsigned));
  if (e != cudaSuccess || !clear) return e;
  const unsigned zero = 0;
  return cudaMemcpyToSymbol(g_proj_error, &zero, sizeof(unsigned));
}

}  // namespace sfm
