/*
 * sfm.h -- C ABI of libsfm: the batch-folded Mamba selective scan of SF-Mamba on B200.
 *
 * The operation (per sample b, channel d, within-sample token t = 0..L-1):
 *
 *   xa      = [avg(x), x_1 .. x_T, avg(x)]              stage-entry layer only (aux init)
 *   u_t     = SiLU(conv_b + sum_k conv_w[k] * xa[t + k - pad_left])   zero outside the sample
 *   Delta_t = softplus(dt_t + dt_bias)
 *   Abar_tn = exp(Delta_t * A_n), except Abar = 0 at every sample start (the reset)
 *   h_tn    = Abar_tn * h_(t-1)n + Delta_t * B_tn * u_t
 *   y_t     = (sum_n C_tn * h_tn + Dskip * u_t) * SiLU(z_t)
 *   out     = y with tokens 0 and L-1 exchanged (aux swap), when requested.
 *
 * Passages this follows:
 *   - recurrence h_t = Abar_t h_{t-1} + Bbar_t x_t, y_t = C_t h_t:
 *     "Seeing Both Ways, Running One Way" (sungsoo.github.io), section 3.1;
 *   - aux head/tail tokens initialised to avg(X), swapped head<->tail between layers:
 *     same page, section 3.2 equations; "SF-Mamba：重新思考视觉 Mamba 的信息流与并行效率"
 *     (techloop.online), Auxiliary Patch Swapping;
 *   - folding [B,D,T] -> [B1,D,B2*T], B = B1*B2, with Abar_t = 0 at every sample start:
 *     sungsoo.github.io section 3.3 equations; techloop.online, Batch Folding with
 *     Periodic State Reset;
 *   - a conv that never crosses folded sample boundaries: techloop.online, the
 *     convolution-boundary paragraph; sungsoo.github.io section 8.1 item 5;
 *   - B1 chosen from an offline look-up table: techloop.online, Adaptive B1;
 *     sungsoo.github.io section 8.1 item 6.
 *   The discretisation (Abar = exp(Delta*A), Bbar = Delta*B), the D skip, softplus and
 *   the SiLU(z) gate are the standard Mamba block; the pages do not spell them out.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library never
 *     allocates device memory, never frees it, and never synchronises the stream
 *     (sfm_get_device_error is the one documented exception).
 *   - Layouts are contiguous row-major: x [B,D,T] (aux init) or [B,D,L]; dt, z, y
 *     [B,D,L]; Bm, Cm [B,N,L] (one group shared by all channels); A [D,N];
 *     Dskip, dt_bias, conv_b [D]; conv_w [D,K]; final_state [B,D,N].
 *   - Activation tensors are fp32 or bf16 (sfm_dtype); parameters are always fp32;
 *     the state and every accumulation are fp32 on the device.
 *   - Argument errors are reported synchronously, before anything is launched, and
 *     leave the device untouched. A launch failure returns SFM_ERR_CUDA.
 *   - Work is enqueued on `stream` (NULL = the legacy default stream).
 *   - Setting the environment variable SFM_FAULT_INJECT=launch makes every compute
 *     entry point return SFM_ERR_CUDA after validation without launching (host-side
 *     fault injection for tests; nothing reaches the GPU).
 */
#ifndef SFM_H
#define SFM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Entry points are the only symbols the shared library exports. */
#if defined(__GNUC__)
#define SFM_API __attribute__((visibility("default")))
#else
#define SFM_API
#endif

/* Same type as cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st* sfm_stream_t;

typedef enum {
  SFM_OK = 0,
  SFM_ERR_INVALID_ARG = 1, /* NULL where a tensor is required, bad size or flag     */
  SFM_ERR_MISALIGNED = 2,  /* a tensor base pointer is not 16-byte aligned          */
  SFM_ERR_UNSUPPORTED = 3, /* valid but outside what the kernels cover (N, K, ...)   */
  SFM_ERR_CUDA = 4,        /* the CUDA runtime reported an error at launch           */
  SFM_ERR_TIMEOUT = 5      /* a kernel gave up a bounded wait (device error word)    */
} sfm_status;

typedef enum { SFM_F32 = 0, SFM_BF16 = 1 } sfm_dtype;

/* Largest supported sizes. */
#define SFM_MAX_N 64      /* state size                                     */
#define SFM_MAX_K 4       /* conv width                                     */
#define SFM_MAX_L 16384   /* tokens per sample (aux tokens included)        */

/* Human-readable name of a status code; never NULL. */
SFM_API const char* sfm_status_string(int status);

/* ABI version (bumped on any change of a struct layout or signature). */
SFM_API int sfm_abi_version(void);

/* Name of the CUDA error behind the calling thread's most recent SFM_ERR_CUDA
 * ("none" if there was none); the string is static. */
SFM_API const char* sfm_last_cuda_error(void);

/*
 * Aux init (stage-entry layer): xa[b,d,0] = xa[b,d,T+1] = mean_t x[b,d,t] (fp32 sum),
 * xa[b,d,1..T] = x[b,d,0..T-1].  x [B,D,T] -> xa [B,D,T+2], both `dtype`.
 * Source: techloop.online, Auxiliary Patch Swapping (avg(X) initialisation);
 * sungsoo.github.io section 3.2.  x and xa must not overlap.
 */
SFM_API sfm_status sfm_aux_init(const void* x, void* xa, int B, int D, int T, sfm_dtype dtype,
                        sfm_stream_t stream);

/*
 * Aux swap between consecutive layers, in place: y[b,d,0] <-> y[b,d,L-1].  L >= 2.
 * Source: sungsoo.github.io section 3.2 (next head = this tail, next tail = this head).
 */
SFM_API sfm_status sfm_aux_swap(void* y, int B, int D, int L, sfm_dtype dtype, sfm_stream_t stream);

/*
 * Boundary-safe depthwise conv1d on the folded layout:
 *   u[b,d,t] = act(bias[d] + sum_{k<K} w[d,k] * x[b,d,t+k-pad_left]),
 * with zeros wherever t+k-pad_left falls outside [0,L) of sample b -- a folded row of
 * B2 samples is never read across a sample boundary.  act = SiLU if silu != 0.
 * x, u [B,D,L] (`dtype`, must not overlap); w [D,K] fp32; bias [D] fp32 or NULL.
 * 1 <= K <= SFM_MAX_K, 0 <= pad_left < K; B2 >= 1 must divide B (the result does not
 * depend on B2).  Source: techloop.online convolution-boundary paragraph;
 * sungsoo.github.io section 8.1 item 5.
 */
SFM_API sfm_status sfm_fold_conv1d(const void* x, const float* w, const float* bias, void* u,
                           int B, int D, int L, int K, int pad_left, int B2, int silu,
                           sfm_dtype dtype, sfm_stream_t stream);

/*
 * The conv of sfm_fold_conv1d (same arguments and zero padding per sample) written
 * token-major: u [B*L, D] (row b*L + t holds the D channels of token t of sample b), the
 * layout the state projection (sfm_proj_gemm) reads as X.  x [B,D,L] and u must not
 * overlap.  Same sources as sfm_fold_conv1d.
 */
SFM_API sfm_status sfm_conv1d_tokens(const void* x, const float* w, const float* bias, void* u, int B, int D,
                                     int L, int K, int pad_left, int silu, sfm_dtype dtype, sfm_stream_t stream);

/* Arguments of the fused folded scan.  `size` must be sizeof(sfm_scan_args). */
typedef struct {
  uint32_t size;
  /* activations (in_dtype) */
  const void* x;        /* conv input: [B,D,L-2] if aux_init else [B,D,L]; with
                           conv_w == NULL it is the scan input u itself            */
  const void* dt;       /* [B,D,L] raw Delta before bias/softplus                  */
  const void* z;        /* [B,D,L] gate input, or NULL for no gate                 */
  const void* Bm;       /* [B,N,L]                                                 */
  const void* Cm;       /* [B,N,L]                                                 */
  /* parameters (fp32) */
  const float* A;       /* [D,N]                                                   */
  const float* Dskip;   /* [D] or NULL                                             */
  const float* dt_bias; /* [D] or NULL                                             */
  const float* conv_w;  /* [D,K] or NULL (no conv: x is u)                         */
  const float* conv_b;  /* [D] or NULL                                             */
  /* outputs */
  void* y;              /* [B,D,L] out_dtype; must not overlap any input          */
  float* final_state;   /* [B,D,N] fp32 state after each sample's last token, or NULL */
  /* sizes */
  int B, D, L, N;
  int K, pad_left;      /* conv width and left padding (used when conv_w != NULL)  */
  int B1;               /* folded rows; 0 = choose with sfm_choose_b1; must divide B */
  int reset_period;     /* 0 or L: the state restarts every L folded positions     */
  /* flags */
  int dt_softplus;      /* Delta = softplus(dt + dt_bias) if set, else dt + dt_bias */
  int aux_init;         /* x holds T = L-2 tokens; build the aux tokens on load    */
  int swap_out;         /* exchange output tokens 0 and L-1 on store               */
  sfm_dtype in_dtype, out_dtype; /* (F32,F32), (BF16,BF16) or (BF16,F32)           */
  /* launch shape overrides for sweeps; 0 = automatic */
  int lanes;            /* lanes per channel sequence (1 = one thread walks it)    */
  int d_tile;           /* channels per CTA (at most 128)                          */
  int chunk;            /* tokens staged per step of the walk                      */
  int exp2_split;       /* 1 + state pairs per token whose exp2 runs on the FMA pipe
                           instead of the transcendental unit (N = 16 only)        */
  int chans_per_thread; /* channels one thread walks side by side (1 or 2; 2 needs the
                           standard mixer at 8 < N <= 16, even D and d_tile)      */
} sfm_scan_args;

/*
 * The fused forward of the hot path: [aux init] -> conv + SiLU -> Delta -> folded
 * scan with reset -> D skip -> SiLU(z) gate -> [aux swap], one kernel launch.
 * Samples are grouped into B1 folded rows of B2 = B/B1 samples; each CTA walks the
 * B2 samples of one row for a tile of channels, restarting the state at every
 * sample start.  The result is independent of B1 (the reset makes the samples
 * independent), so B1 only changes the schedule.
 * Requirements: x, dt, z, Bm, Cm, y 16-byte aligned; 1 <= N <= SFM_MAX_N;
 * 1 <= K <= SFM_MAX_K; 3 <= L <= SFM_MAX_L when aux_init (else 1 <= L); y must not
 * alias an input.  One thread per channel (lanes = 1) holds at most 16 states; above
 * that the lanes mode is chosen (an explicit lanes = 1 is SFM_ERR_UNSUPPORTED).
 * Sources: see the header comment.
 */
SFM_API sfm_status sfm_selective_scan_fold(const sfm_scan_args* args, sfm_stream_t stream);

/*
 * Ragged folding: the fused scan of sfm_selective_scan_fold over B samples of DIFFERENT
 * lengths packed along time, with the state reset at every sample start given by an
 * offset array instead of a fixed period.
 *
 *   cu_seqlens  DEVICE int32 [B+1]: sample s covers packed positions
 *               [cu_seqlens[s], cu_seqlens[s+1]) (L_s = their difference tokens, aux
 *               tokens included); normally 0 = cu_seqlens[0] <= ... <= cu_seqlens[B] = L.
 *
 * In `args`: B = number of samples, L = packed length (all samples' tokens), and the
 * layouts are time-contiguous rows of the packed length:
 *   x   [D, L - 2B] with aux_init (sample s at x offset cu_seqlens[s] - 2s, its T_s =
 *       L_s - 2 patch tokens), else [D, L];
 *   dt, z, y [D, L]; Bm, Cm [N, L]; final_state [B, D, N] (state after each sample).
 * Every sample is computed exactly as sfm_selective_scan_fold computes one sample of
 * length L_s: the conv sees zeros outside the sample, the aux tokens are the mean of the
 * sample's own T_s tokens, the swap exchanges the sample's own first and last outputs.
 * B1 (0 = look-up table at the mean length) groups B/B1 consecutive samples per folded
 * row; reset_period must be 0; N <= 16; lanes must be 0 or 1 (one thread walks each
 * channel, chunked staging).  y positions that belong to no sample are not written.
 *
 * The offsets are read on the device, so they are checked there: a sample whose offsets
 * are out of order or outside [0, L] (or, with aux_init, shorter than 3 tokens or not
 * matching x's packing) is skipped -- nothing of it is read or written -- and the
 * device error word (sfm_get_device_error) is set to SFM_ERR_INVALID_ARG.  Everything
 * else is validated on the host as for sfm_selective_scan_fold.
 * Source: the fold with its per-sample reset and boundary-safe conv of
 * techloop.online (Batch Folding with Periodic State Reset; the convolution-boundary
 * paragraph) and sungsoo.github.io section 3.3, with the period replaced by offsets.
 * Inputs of unequal length are the ones the pages point at beyond classification: the
 * windowed detection backbones of the SF-Mamba repository (kd.iw.mk/sony/SF-Mamba, COCO
 * Cascaded Mask-RCNN) and, in sungsoo.github.io's table of follow-up work, cameras or
 * windows folded as one effective batch with their states kept apart.
 */
SFM_API sfm_status sfm_selective_scan_fold_varlen(const sfm_scan_args* args, const int* cu_seqlens,
                                                  sfm_stream_t stream);


/* Gradients produced by the scan backward (all fp32, caller-owned device memory). */
typedef struct {
  uint32_t size;        /* sizeof(sfm_scan_grads)                                 */
  const void* dout;     /* [B,D,L] upstream gradient of y, args->out_dtype        */
  float* du;            /* [B,D,L]                                                */
  float* ddt;           /* [B,D,L]  (through the softplus when dt_softplus)       */
  float* dz;            /* [B,D,L]  or NULL when args->z is NULL                  */
  float* dA;            /* [D,N]    summed over samples and tokens                */
  float* dDskip;        /* [D]      or NULL when args->Dskip is NULL              */
  float* ddt_bias;      /* [D]      or NULL when args->dt_bias is NULL            */
  float* dB;            /* [B,N,L]  summed over channels                          */
  float* dC;            /* [B,N,L]  summed over channels                          */
} sfm_scan_grads;

/*
 * Workspace (bytes) the scan backward needs for `args`; 256-byte aligned device
 * memory of at least this size goes to sfm_selective_scan_fold_bwd.
 */
SFM_API sfm_status sfm_scan_bwd_workspace_size(const sfm_scan_args* args, size_t* bytes);

/*
 * Backward of the scan (from its input u to the gated output): a reverse adjoint
 * sweep g_t = C_t dy_t + Abar_(t+1) g_(t+1) that never crosses a sample start, where
 * the transition factor is the constant 0.  Reductions over channels (dB, dC) and
 * over samples/tokens (dA, dDskip, ddt_bias) are done in a fixed order, so results
 * are bitwise reproducible.  args must describe a scan without conv, aux init or
 * swap (conv_w == NULL, aux_init == 0, swap_out == 0); args->y is not read.
 * Overwrites every gradient buffer given.  Source: the reset reading of
 * sungsoo.github.io section 3.3; the backward itself is not on the pages.
 */
SFM_API sfm_status sfm_selective_scan_fold_bwd(const sfm_scan_args* args, const sfm_scan_grads* grads,
                                       void* workspace, size_t workspace_bytes,
                                       sfm_stream_t stream);

/* Arguments of the per-token projection GEMM.  `size` must be sizeof(sfm_proj_args). */
typedef struct {
  uint32_t size;
  const void* W;     /* [M, K] bf16, K contiguous (the nn.Linear weight layout)            */
  const void* X;     /* [Ntok, K] bf16, K contiguous: one row of K features per token      */
  void* out0;        /* channel-major: rows [0, M0) as [B, M0, L]; token-major: [Ntok, M]  */
  void* out1;        /* channel-major: rows [M0, M) as [B, M - M0, L]; NULL if M0 == M     */
  int M, K, Ntok;    /* Ntok = B * L tokens, sample-major                                   */
  int M0;            /* rows written to out0 (channel-major); must equal M if token-major   */
  int L;             /* tokens per sample                                                   */
  int token_major;   /* 0: channel-major outputs (the scan's layout), 1: token-major out0   */
  sfm_dtype out_dtype; /* BF16 or F32                                                       */
  int tile_n;        /* output channels per CTA tile: 0 = automatic, 128 or 256             */
  int schedule;      /* 0 = automatic, 1 = one CTA per tile, 2 = persistent (one CTA per SM
                        walking its tiles, the epilogue overlapping the next tile's MMAs)   */
} sfm_proj_args;

/*
 * The dense per-token maps around the scan, on the tensor cores:
 *   P[m, n] = sum_k W[m, k] * X[n, k]      (fp32 accumulation, rounded once to out_dtype)
 * written either channel-major -- P[m, b*L + t] at out[b, m, t], the scan's [B, rows, L]
 * layout, so the input projection's x and z (M0 = D, M = 2D) and the state projection's
 * B and C land where sfm_selective_scan_fold reads them -- or token-major [Ntok, M] (the
 * low-rank step-size features that the next map reads as its X).
 * The maps themselves are the Mamba block's input, state and step-size projections; the
 * pages cite Mamba and MambaVision as the block's background (sungsoo.github.io, Sources
 * and Evidence Notes, items 4 and 5) and do not spell them out.
 * Requirements: K a multiple of 8 (16-byte row pitch), 16-byte aligned pointers, Ntok a
 * multiple of L.  Rows or tokens past the ends are never written.  One launch.  A wait
 * that gives up sets SFM_ERR_TIMEOUT in the device error word and skips the stores.
 */
SFM_API sfm_status sfm_proj_gemm(const sfm_proj_args* args, sfm_stream_t stream);

/*
 * The scan backward without any allocation by the caller or the library.
 *
 * This entry point has no counterpart in the paper.  It is
 * sfm_selective_scan_fold_bwd with its workspace taken from a buffer built into the
 * library instead of one the caller passes in.  It is for callers that cannot call
 * cudaMalloc, for example:
 *   - a plug-in inside a host application that owns all device memory through its own
 *     allocator and gives plug-ins no way to request more;
 *   - a deployment that forbids allocation after start-up (a fixed memory budget
 *     decided up front);
 *   - a latency-critical loop where cudaMalloc's implicit device synchronisation is
 *     not acceptable.
 * The caller still passes every input and output tensor; only the workspace is built in.
 *
 * The built-in workspace is a device array of SFM_NOALLOC_SCRATCH_BYTES.  Every GPU that
 * loads this library holds that much memory until the process exits.  Problems whose
 * workspace (sfm_scan_bwd_workspace_size) exceeds it are rejected with
 * SFM_ERR_UNSUPPORTED before anything is launched; use sfm_selective_scan_fold_bwd then.
 *
 * The first call on a device looks up the array's device address on that device
 * (cudaGetSymbolAddress, with the device current); make that first call before any
 * stream capture.  Later calls reuse the address.
 *
 * All calls on a device share the one array, and it keeps the last call's contents:
 * the backward writes every part of the workspace before reading it, so nothing has to
 * start at zero, but two calls that overlap on the GPU (different streams, or
 * different host threads) race on it and give wrong results.  Serialise them.
 *
 * Arguments, requirements and results are exactly those of sfm_selective_scan_fold_bwd.
 * No cudaMalloc, cudaFree or allocating library routine is called.
 */
#define SFM_NOALLOC_SCRATCH_BYTES (64u << 20) /* 64 MiB */
SFM_API sfm_status sfm_selective_scan_fold_bwd_noalloc(const sfm_scan_args* args,
                                                       const sfm_scan_grads* grads,
                                                       sfm_stream_t stream);

/* Gradients of the whole mixer layer (all fp32, caller-owned device memory). */
typedef struct {
  uint32_t size;        /* sizeof(sfm_mixer_grads)                                    */
  const void* dout;     /* [B,D,L] gradient of the layer output y as the forward stored
                           it (after the swap when swap_out), args->out_dtype          */
  float* dx;            /* [B,D,L-2] if aux_init else [B,D,L]: gradient of x          */
  float* dconv_w;       /* [D,K] (required when args->conv_w is given)                */
  float* dconv_b;       /* [D] or NULL when args->conv_b is NULL                      */
  float* ddt;           /* [B,D,L]                                                    */
  float* dz;            /* [B,D,L] or NULL when args->z is NULL                       */
  float* dA;            /* [D,N]                                                      */
  float* dDskip;        /* [D] or NULL when args->Dskip is NULL                       */
  float* ddt_bias;      /* [D] or NULL when args->dt_bias is NULL                     */
  float* dB;            /* [B,N,L]                                                    */
  float* dC;            /* [B,N,L]                                                    */
} sfm_mixer_grads;

/* Workspace (bytes, 256-byte aligned device memory) sfm_mixer_bwd needs for `args`. */
SFM_API sfm_status sfm_mixer_bwd_workspace_size(const sfm_scan_args* args, size_t* bytes);

/*
 * Backward of the whole fused layer of sfm_selective_scan_fold -- aux init, conv +
 * SiLU, Delta, folded scan, D skip, gate and swap -- for the same args (y is not read):
 * the output gradient is read through the swap, the scan input is rebuilt from x, the
 * scan backward runs as in sfm_selective_scan_fold_bwd, then the conv + SiLU backward
 * gives dx (plus the aux mean's share (dxa[0] + dxa[L-1]) / T on every token when
 * aux_init), dconv_w and dconv_b.  Every reduction runs in a fixed order (bitwise
 * reproducible).  Overwrites every gradient buffer given.  Sources: the layer as
 * defined at the top of this header; the backward itself is not on the pages.
 */
SFM_API sfm_status sfm_mixer_bwd(const sfm_scan_args* args, const sfm_mixer_grads* grads, void* workspace,
                                 size_t workspace_bytes, sfm_stream_t stream);

/*
 * Adaptive B1: the number of folded rows for a batch of B samples of T patch tokens,
 * D channels and state size N, from a look-up table built by a B200 sweep.  The
 * result always divides B.  Source: techloop.online, Adaptive B1; sungsoo.github.io
 * section 8.1 item 6.  Pure host function.
 */
SFM_API sfm_status sfm_choose_b1(int B, int T, int D, int N, int* B1_out);

/* The full launch choice behind sfm_choose_b1: folded rows, lanes per channel
 * sequence, channels per CTA, tokens staged per step, state pairs per token whose
 * exp2 runs on the FMA pipe, and channels per thread. */
typedef struct {
  int B1, lanes, d_tile, chunk, exp2_pairs, chans_per_thread;
} sfm_variant;
SFM_API sfm_status sfm_choose_variant(int B, int T, int D, int N, sfm_variant* out);

/*
 * Reads (and, if clear != 0, resets) the device-side error word that kernels set when
 * a bounded wait gives up (SFM_ERR_TIMEOUT, forward or projection kernels) or ragged
 * offsets are invalid (SFM_ERR_INVALID_ARG).  Synchronises `stream` first.  *code = SFM_OK when clean.
 */
SFM_API sfm_status sfm_get_device_error(sfm_stream_t stream, int clear, int* code);

/*
 * Self-test of the bounded-wait path: launches one thread that waits on an mbarrier
 * nothing arrives on, gives up after limit_us microseconds (1 .. 1e6), records
 * SFM_ERR_TIMEOUT in the device error word exactly as the kernels' own waits do, and
 * returns.  Nothing faults or hangs; read the result with sfm_get_device_error.
 */
SFM_API sfm_status sfm_selftest_wait_timeout(int limit_us, sfm_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SFM_H */
