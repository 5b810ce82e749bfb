// attn_fwd_sm100.h -- internal launch interface of the forward kernel (not part of
// the public C ABI; see include/attn.h for that).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace attn {

// The mask hook: which (query, key) pairs are visible.  Each kind is a
// compile-time functor of the kernel (attn_fwd_sm100.cu, struct MaskFn).
enum MaskKind : int {
  kMaskNone = 0,    // every key of the sequence
  kMaskCausal = 1,  // key <= query
  kMaskWindow = 2,  // query - wl <= key <= query + wr
};

struct FwdParams {
  __nv_bfloat16* o;      // [T, H, D] bf16 (dense T = B*N)
  float* lse;            // dense [B, H, N]; varlen [H, total]
  const int* cu_seqlens; // device int32[B+1] or null (dense)
  int B, H, N;
  int T;                 // items of the longest sequence: ceil(N / 256) (CTA pairs: / 512)
  int total;             // packed tokens (dense: B*N)
  float scale_log2;      // scale * log2(e)
  float tau;             // conditional-rescale threshold, log2 units
  int* err;              // device error word
  unsigned* work;        // [0] list positions claimed, [1] CTAs finished; zero at launch,
                         // returned to zero by the launch's last CTA
  unsigned long long* stats;  // optional [rescaled rows, row-tiles]
  uint64_t timeout_ns;   // limit of every internal wait
  int test_fault;        // 1: withhold the first Q copy (failure-path tests only)
  int wl, wr;            // kMaskWindow bounds, both >= 0 (an open side holds a large value)
  float o_scale;         // E4M3 path: V's per-tensor scale, applied with 1/l
  float p_shift;         // E4M3 path: P~ carries a factor 2^p_shift (an integer) so
                         // it spans E4M3's normal range; l carries it too
  int stage_off;         // > 0: byte offset (from the 1024-aligned shared-memory base) of
                         // the O staging buffers (4 KB per softmax warp) that TMA stores
                         // write back from; 0: O rows are stored directly
};

struct FwdLaunch {
  // 3-D maps {D, H, total} with 128-byte swizzle; box {64, 1, 128} for bf16 and
  // {128, 1, 128} for E4M3 (one 128-byte row either way); tm_k2: K with box
  // {64, 1, 64} (the K halves of CTA pairs; unused otherwise); tm_o: O (bf16) with
  // box {64, 1, 32} (one softmax warp's 32 rows, 64 head dims)
  CUtensorMap tm_q, tm_k, tm_v, tm_k2, tm_o;
  FwdParams p;
  int grid;
  int smem;
  int pair;  // launch in clusters of two CTAs (tcgen05.mma.cta_group::2); grid even
};

// T: items of the longest sequence (256 query rows each; CTA pairs: 512).
int fwd_smem_bytes(int D, int B, int T, int varlen, int fp8, int pair);
// Offset of the O staging buffers for that launch (0: they do not fit beside the
// kernel's other shared memory) and their size.
int fwd_stage_offset(int D, int B, int T, int varlen, int fp8, int pair);
constexpr int kFwdStageBytes = 8 * 4096;
// Clusters of two CTAs of the pair kernel that fit on the device at once (0: none).
int fwd_pair_max_clusters(int smem);
// poly: exponentials per 8 column pairs on the FMA-pipe polynomial (0, 2 or 8).
// fp8: E4M3 inputs (D = 128, poly = 0 only).
cudaError_t launch_fwd(const FwdLaunch& a, int D, MaskKind mask, int poly, int fp8, cudaStream_t st);

}  // namespace attn
