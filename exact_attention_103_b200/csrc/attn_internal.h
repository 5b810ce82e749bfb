// attn_internal.h -- host-side pieces shared by the entry points of attn_api.cu and
// attn_noalloc.cu (not part of the public C ABI; see include/attn.h for that).
// Nothing declared here allocates device memory.
#pragma once
#include <cstdint>

#include "../../include/attn.h"
#include "attn_fwd_sm100.h"

namespace attn_internal {

// Per-tensor scales of the E4M3 entry point (real value = stored value * scale).
struct E4m3Scales {
  float q, k, v;
};

// The arguments of one forward call, as every forward entry point receives them.
struct FwdCall {
  const void *q, *k, *v;
  void* o;
  float* lse;
  int B, H, N, d, causal;
  float scale;
  const int32_t* cu_seqlens;
  const attn_fwd_opts_t* opts;  // may be null (defaults)
  const E4m3Scales* f8;         // null: bf16 inputs
};

// What validation of a forward call decides before any device work.
struct FwdPlan {
  bool noop;  // B == 0 or N == 0: nothing to launch
  float tau;
  uint64_t timeout;
  unsigned long long* stats;
  int test_fault, poly;
  attn::MaskKind mask;
  int win_l, win_r;
  int pair;  // clusters of two CTAs (opts->cta_pair)
  int64_t T, items_bound, dense_tokens;  // T: items of the longest sequence (256 or 512 rows)
};

// Checks every argument of a forward call on the host; touches no device state.
attn_status_t plan_fwd(const FwdCall& c, FwdPlan* pl);
// Builds the launch of a planned forward call over `total` packed tokens (dense:
// B*N) on a device with `sms` SMs, the kernel recording errors in `err` and
// claiming work items through the two zeroed words at `work` (device addresses);
// pair_clusters: clusters of the CTA-pair kernel that fit at once (pair launches).
attn_status_t fill_fwd_launch(const FwdCall& c, const FwdPlan& pl, int64_t total, int sms, int pair_clusters,
                              int* err, unsigned* work, attn::FwdLaunch* a);
attn_status_t launch_planned_fwd(const FwdCall& c, const FwdPlan& pl, const attn::FwdLaunch& a,
                                 attn_stream_t stream);
// Looks up the driver's tensor-map encoder once per process.
attn_status_t load_tensor_map_encoder();
// Records `message` as the calling thread's last error and returns `s`.
attn_status_t report(attn_status_t s, const char* message);

}  // namespace attn_internal
