// attn_bwd_sm100.h -- internal launch interface of the backward kernels (the
// public C ABI is include/attn.h).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace attn {

struct BwdParams {
  const float* lse;        // forward LSE (natural log): dense [B,H,N], varlen [H,total]
  float* dpre;             // workspace D_i = <dO_i, O_i>, same layout as lse
  __nv_bfloat16* dq;       // [total, H, D]
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  const int* cu_seqlens;   // device int32[B+1] or null (dense)
  int B, H, N;
  int total;               // packed tokens (dense: B*N)
  int ntiles;              // ceil(N / 128)
  float scale;             // softmax scale
  float scale_log2;        // scale * log2(e)
  int* err;                // device error word
  uint64_t timeout_ns;
  int wl, wr;              // sliding window (mask kind 2): key j visible to query i iff
                           // i - wl <= j <= i + wr; both >= 0, an open side holds N
};

struct BwdLaunch {
  CUtensorMap tm_q, tm_k, tm_v, tm_do;  // 3-D maps {D, H, total}, box {64, 1, 128}
  BwdParams p;
  int grid;  // B * ntiles * H CTAs for each main kernel
};

// mask: 0 none, 1 causal, 2 sliding window (the forward's MaskKind values).
cudaError_t launch_bwd(const BwdLaunch& a, const void* o, const void* dout, int D, int mask,
                       cudaStream_t st);

}  // namespace attn
