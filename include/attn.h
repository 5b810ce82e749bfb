/*
 * attn.h -- C ABI of libattn: exact scaled-dot-product attention on NVIDIA B200
 * (sm_100a), computed as one fused tiled kernel with online softmax so that the
 * score matrix S and the probability matrix P never reach device memory.
 *
 * The operation (the pages' definition; "FlashAttention 1-4 详解", section 原算法,
 * and "FlashAttention V4 deep-dive" (pnsm.cn), section 1.1):
 *
 *     O = softmax(scale * Q K^T) V,   LSE_i = ln sum_j exp(scale * <q_i, k_j>)
 *
 * row by row for every (sequence, head).  With `causal`, query i sees only keys
 * j <= i ("FlashAttention 1-4 详解", 其他优化 / FlashAttention 2 的工程优化: causal
 * lower triangle); indices are local to each sequence.
 *
 * Conventions shared by every entry point:
 *  - Every tensor pointer is a DEVICE pointer owned by the caller; the library
 *    never frees or retains it.  Calls are asynchronous on `stream`; argument
 *    errors are returned before anything is launched.
 *  - Q, K, V, O are bf16 (attn_fwd_e4m3: Q, K, V are E4M3), contiguous, head
 *    dimension innermost:
 *      dense:  [B, N, H, d]   (row stride H*d elements)
 *      varlen: [T, H, d]      packed, T = cu_seqlens[B]
 *    Their base addresses must be 16-byte aligned.
 *  - LSE is fp32, natural log, scale included:
 *      dense:  [B, H, N]      varlen: [H, T]
 *  - cu_seqlens (varlen only): DEVICE int32[B+1], non-decreasing prefix sums of the
 *    sequence lengths with cu_seqlens[0] = 0; N is then the maximum length.  Q and
 *    K/V of a sequence have the same length.  Pass NULL for a dense batch.
 *    attn_fwd reads cu_seqlens[B] back to the host (a 4-byte copy that
 *    synchronises `stream`); attn_fwd_ex with opts->total_tokens avoids that.
 *    Inconsistent cu_seqlens (cu[0] != 0, a negative length, cu[B] != the token
 *    count) make the kernel write nothing and record ATTN_ERR_INVALID_ARG in the
 *    device error word.
 *  - Supported: d in {64, 128}; scale finite and > 0.  Varlen: B <= 1024 and
 *    N <= 131072.  B == 0 or N == 0 is a no-op.
 *  - The library allocates, lazily and once per device, one small device buffer:
 *    an error word and 64 slots of work counters for the forward kernel's
 *    scheduler.  Each stream that runs forward passes keeps its own slot (launches
 *    on one stream never overlap, and a launch leaves its slot at zero when it
 *    ends); with more than 64 such streams on a device the least recently used
 *    slot passes to the new stream, so forward launches on more than 64 streams
 *    must not all be in flight at once.  A CUDA graph keeps the slot of the stream
 *    it was captured on: replays of it must not overlap forward launches on that
 *    stream or each other.
 *    A kernel whose internal waits exceed their time limit stops, records
 *    ATTN_ERR_TIMEOUT in the error word, and leaves its outputs undefined;
 *    attn_get_device_status() reports and clears it.
 */
#ifndef LIBATTN_ATTN_H
#define LIBATTN_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* The CUDA stream handle type (identical to cudaStream_t / CUstream). */
typedef struct CUstream_st* attn_stream_t;

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or scale     */
  ATTN_ERR_UNSUPPORTED = 2, /* valid but not supported (d, limits, no sm_100) */
  ATTN_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed              */
  ATTN_ERR_TIMEOUT = 4,     /* a kernel's bounded wait expired (device status) */
  ATTN_ERR_WORKSPACE = 5    /* workspace pointer/size too small               */
} attn_status_t;

/*
 * Forward pass.  Writes O (bf16, layout of Q) and LSE (fp32, layout above).
 * Online softmax: "FlashAttention 1-4 详解", FlashAttention 1 / Online Softmax
 * 数学推导, with deferred normalisation (FlashAttention 2 / 减少非矩阵乘运算占比)
 * and the conditional rescale of "FlashAttention V4 deep-dive", section 3.2.
 * The probabilities enter the P V product as bf16.  O is divided by the sum of
 * those bf16 values over key tiles the mask cuts (the causal diagonal, a
 * sequence's last tile) and of the unrounded fp32 values over full tiles, so
 * rows whose keys all lie in cut tiles get exactly the weights applied to V.
 * Sliding-window calls and unmasked d = 64 calls use the fp32 sum throughout.  LSE
 * always uses the fp32 sum.
 * The result does not depend on how the work is scheduled: each output row is
 * produced by one CTA with a fixed key order, so repeated calls are bitwise equal.
 */
ATTN_API attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                       int B, int H, int N, int d, int causal, float scale,
                       const int32_t* cu_seqlens, attn_stream_t stream);

/* Tuning / test knobs for attn_fwd_ex.  Zero-initialise, then set fields.
 *  rescale_threshold: conditional-rescale threshold tau in log2 units; the
 *      running maximum is replaced (and O, l rescaled) only when a new tile's row
 *      maximum exceeds it by more than tau, so P~ <= 2^tau.  < 0 selects the
 *      default (8.0); values above 64 are rejected (ATTN_ERR_INVALID_ARG).
 *  stats: optional DEVICE pointer to two uint64 counters the kernel ADDS to:
 *      [0] rows rescaled, [1] row-tiles processed after each row's first tile.
 *  timeout_ns: limit of every internal wait; 0 selects the default (2 s).
 *  total_tokens: varlen only; if > 0 it must equal cu_seqlens[B] (checked on the
 *      device).  When 0, attn_fwd_ex (like attn_fwd) reads cu_seqlens[B] back
 *      to the host with a 4-byte copy and a stream synchronisation, because the
 *      TMA views of Q/K/V must not extend past the packed tensors.
 *  test_fault: for tests of the failure path only, 0 otherwise.  1 makes every
 *      CTA withhold the copy of its first query tile, so the wait for it expires
 *      after timeout_ns: the kernel records ATTN_ERR_TIMEOUT, drains its other
 *      copies, frees its tensor memory and returns (outputs undefined).
 *  has_window, window_left, window_right: the mask hook.  When has_window is
 *      nonzero, key j is visible to query i (indices local to the sequence) only
 *      if i - window_left <= j <= i + window_right; a negative bound leaves that
 *      side open, and the causal flag still applies on top (it forces
 *      window_right to 0).  Key tiles that no row of a query tile can see are
 *      skipped, not masked.  Every row keeps its own key visible, so no row is
 *      empty.  The pages name FlexAttention's masks as the interface FA4 serves
 *      ("FlashAttention V4 deep-dive", section 5; FA-4 summary [27]) but define
 *      no mask beyond causal: the sliding window (local attention) is this
 *      library's instance of that interface.  The stats counters are not kept
 *      under a window.
 *  exp_poly_per8: how many of every 8 (even, odd) column pairs of a score row are
 *      exponentiated by the FMA-pipe polynomial instead of MUFU ex2
 *      ("FlashAttention V4 deep-dive", section 3.2: software exp on the FMA
 *      units).  0 (the default, all MUFU), 2 or 8; other values are rejected
 *      (ATTN_ERR_INVALID_ARG).  The polynomial has a relative error below 7.5e-5,
 *      under half a bf16 ulp, so the results differ from the MUFU path only by
 *      the rounding of P~.
 *  cta_pair: nonzero runs the forward in clusters of two CTAs on neighbouring SMs
 *      that share each item of 512 query rows ("FlashAttention V4 deep-dive",
 *      section 3.3, 2-CTA MMA; FA-4 summary [13][14]): the pair's leader issues
 *      tcgen05.mma.cta_group::2 products of 256 rows, and each CTA loads its own
 *      query rows and half of every K/V tile (no multicast), halving each SM's
 *      K/V traffic.  bf16 inputs, d = 128, exp_poly_per8 = 0 (else
 *      ATTN_ERR_UNSUPPORTED).  Results equal the single-CTA path's up to the order
 *      of fp32 accumulation inside the products. */
typedef struct {
  float rescale_threshold;
  unsigned long long* stats;
  uint64_t timeout_ns;
  int64_t total_tokens;
  int test_fault;
  int has_window;
  int window_left;
  int window_right;
  int exp_poly_per8;
  int cta_pair;
} attn_fwd_opts_t;

/* attn_fwd with options (opts may be NULL = defaults). */
ATTN_API attn_status_t attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int H, int N, int d, int causal, float scale,
                          const int32_t* cu_seqlens, const attn_fwd_opts_t* opts,
                          attn_stream_t stream);

/*
 * Forward pass with 8-bit inputs ("FlashAttention 1-4 详解", section 其他优化: the
 * forward runs its matrix products on FP8 tensor cores, the backward stays in
 * BF16).  q, k, v: DEVICE E4M3 (1 sign, 4 exponent, 3 mantissa bits, bias 7,
 * largest finite 448, no infinities; the encoding of torch.float8_e4m3fn), one
 * byte per element, same layouts as attn_fwd, 16-byte aligned.  The real inputs
 * are q * q_scale, k * k_scale, v * v_scale (per-tensor scales, finite and > 0).
 * O is bf16 and LSE fp32 exactly as in attn_fwd (LSE of the scaled scores of the
 * real inputs).  S = Q K^T and O += P~ V run on tcgen05.mma kind::f8f6f4; P~
 * (<= 2^tau) is computed with an extra factor 2^floor(8 - tau), so that it fills
 * E4M3's range (at most 256 of the 448 maximum) and small probabilities stay
 * normal numbers, and is rounded to E4M3 (nearest even, saturating) for the PV
 * product, while the row sum l adds the unrounded fp32 values (the factor cancels
 * in O = sum P~ v / l and is taken out of LSE).  d must be 128
 * (ATTN_ERR_UNSUPPORTED otherwise); opts as for attn_fwd_ex, except that
 * exp_poly_per8 must be 0 or 2, rescale_threshold is at most 8, and its default
 * on this path is 4.  Errors as for attn_fwd_ex.
 */
ATTN_API attn_status_t attn_fwd_e4m3(const void* q, const void* k, const void* v, void* o,
                                     float* lse, int B, int H, int N, int d, int causal,
                                     float scale, float q_scale, float k_scale, float v_scale,
                                     const int32_t* cu_seqlens, const attn_fwd_opts_t* opts,
                                     attn_stream_t stream);

/*
 * Backward pass (dQ, dK, dV) from Q, K, V, O, LSE and dO, recomputing P from LSE
 * ("FlashAttention 1-4 详解", 总结 table: 反向传播重计算; "FlashAttention V4
 * deep-dive", section 3.3).  Same layouts as the forward; dq/dk/dv are bf16.
 * Three launches on `stream`: D_i = <dO_i, O_i> into the workspace, a kernel per
 * 128-key tile accumulating dK and dV, and a kernel per 128-query tile
 * accumulating dQ.  No result is accumulated with atomics, so every call is
 * bitwise reproducible run to run; `deterministic` is accepted for interface
 * compatibility and changes nothing.  `workspace` is a caller-owned DEVICE buffer
 * of at least attn_bwd_workspace_size(...) bytes, 256-byte aligned (may be NULL
 * when that size is 0); too small or misaligned: ATTN_ERR_WORKSPACE.  Same limits
 * as the forward (d in {64, 128}); varlen reads cu_seqlens[B] back to the host
 * (attn_bwd_ex with opts->total_tokens avoids that).
 */
ATTN_API attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o,
                       const float* lse, const void* dout, void* dq, void* dk, void* dv,
                       int B, int H, int N, int d, int causal, float scale,
                       const int32_t* cu_seqlens, int deterministic, void* workspace,
                       size_t workspace_bytes, attn_stream_t stream);

/* Options for attn_bwd_ex.  Zero-initialise, then set fields.
 *  has_window, window_left, window_right: the sliding-window mask of the forward
 *      call whose gradients are wanted, with the meaning they have in
 *      attn_fwd_opts_t (the mask hook; the causal flag still applies on top).
 *  timeout_ns: limit of every internal wait; 0 selects the default (2 s).
 *  total_tokens: varlen only; if > 0 it must equal cu_seqlens[B] and the call does
 *      not synchronise `stream`; when 0, cu_seqlens[B] is read back to the host
 *      (a 4-byte copy and a stream synchronisation).  Either way the kernels check
 *      cu_seqlens on the device: cu[0] != 0, cu[B] != the token count, a negative
 *      length or one above N make them record ATTN_ERR_INVALID_ARG in the device
 *      error word, and the sequences concerned are not processed (their gradients
 *      are left unwritten). */
typedef struct {
  int has_window;
  int window_left;
  int window_right;
  uint64_t timeout_ns;
  int64_t total_tokens;
} attn_bwd_opts_t;

/* attn_bwd with options (opts may be NULL = attn_bwd).  Under a window both
 * kernels visit only the tiles the window reaches and mask its edges; the
 * gradients are those of the windowed forward. */
ATTN_API attn_status_t attn_bwd_ex(const void* q, const void* k, const void* v, const void* o,
                                   const float* lse, const void* dout, void* dq, void* dk,
                                   void* dv, int B, int H, int N, int d, int causal, float scale,
                                   const int32_t* cu_seqlens, int deterministic, void* workspace,
                                   size_t workspace_bytes, const attn_bwd_opts_t* opts,
                                   attn_stream_t stream);

/* Workspace bytes attn_bwd needs (total_tokens = B*N dense, cu_seqlens[B] varlen). */
ATTN_API size_t attn_bwd_workspace_size(int B, int H, int N, int d, int total_tokens, int deterministic);

/*
 * Forward pass that allocates nothing, for callers that cannot call cudaMalloc:
 * a framework that has reserved all device memory for its own pool, code that
 * must not trigger the implicit synchronisation an allocation may cause, or code
 * that runs while a stream is being captured.  (The pages have no counterpart:
 * this is an interface of this library.)  The ordinary entry points allocate a
 * 4-byte device status word on a device's first call; here that scratch lives in
 * a static device array of 256 bytes inside the library, which every GPU that
 * loads the library holds until the process exits.  Same operation, layouts,
 * argument checks and limits as attn_fwd, default rescale threshold; the same
 * kernel runs with the same parameters, so O and LSE are bitwise equal to
 * attn_fwd's.
 *  - total_tokens: varlen only, must equal cu_seqlens[B] (there is no device
 *    read-back; the kernel checks it); 0 is an empty packed batch (nothing is
 *    launched, ATTN_OK); ignored for dense batches.
 *  - check: != 0 = synchronise `stream` and return the status the kernel recorded
 *    (ATTN_ERR_TIMEOUT, or ATTN_ERR_INVALID_ARG for bad cu_seqlens).  0 = return
 *    after launching; the kernel's status then stays in the static array, where
 *    attn_get_device_status does NOT see it (that reads the ordinary entry points'
 *    word), until the next call of this entry point clears it: a caller that needs
 *    the status must pass check != 0.
 *  - The first call on a device does its set-up there (looks up the array's
 *    device address); make that first call before any stream capture.
 *  - Every call shares the array: calls whose kernels overlap on the GPU race on
 *    it (their status words and their work counters mix), so such calls must be
 *    ordered, e.g. issued on one stream.
 *  - The forward kernel uses 16 bytes of the array: the status word and the two
 *    counters through which its CTAs claim work items (each call clears all 16
 *    bytes on `stream` before its launch).  A kernel that needed more scratch than
 *    the array holds would be rejected with ATTN_ERR_WORKSPACE.
 */
ATTN_API attn_status_t attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o,
                                        float* lse, int B, int H, int N, int d, int causal,
                                        float scale, const int32_t* cu_seqlens,
                                        int64_t total_tokens, int check, attn_stream_t stream);

/* Synchronises `stream`, then returns and clears the device error word of the
 * current device (ATTN_OK if no kernel recorded an error). */
ATTN_API attn_status_t attn_get_device_status(attn_stream_t stream);

/* Static string for a status code. */
ATTN_API const char* attn_status_string(attn_status_t s);

/* Message describing the last non-OK status returned on the calling thread. */
ATTN_API const char* attn_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* LIBATTN_ATTN_H */
