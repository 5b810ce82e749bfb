// attn_noalloc.cu -- attn_fwd_noalloc: the forward pass for callers that cannot
// allocate device memory.
//
// The ordinary entry points allocate, once per device, the 4-byte device status
// word the kernel records wait timeouts and bad cu_seqlens in (cudaMalloc on the
// first call).  Some callers cannot do that: a framework that has reserved the
// whole device memory for its own pool (a stray cudaMalloc fails or fragments it),
// code that must not trigger the implicit device synchronisation a cudaMalloc may
// cause, or code that runs where allocation is forbidden while a stream is being
// captured.  This entry point keeps that scratch in a file-scope static device
// array instead, and calls no cudaMalloc, cudaFree or other allocating routine.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "../../include/attn.h"
#include "attn_fwd_sm100.h"
#include "attn_internal.h"

namespace {

// Scratch of the allocation-free forward: the kernel's status word at word 0 and
// its scheduler's two claim counters at words 2 and 3.  Every GPU that loads the
// library holds these bytes until the process exits.
constexpr size_t kScratchBytes = 256;
static __device__ __align__(256) int g_noalloc_scratch[kScratchBytes / sizeof(int)];
constexpr size_t kFwdScratchNeeded = 4 * sizeof(int);  // status word, pad, claim counters

constexpr int kMaxDevices = 64;
struct NoAllocDevice {
  bool ready = false;
  int* scratch = nullptr;  // device address of g_noalloc_scratch on this device
  int sms = 0;
};
std::mutex g_mu;
NoAllocDevice g_dev[kMaxDevices];

// Once per device, with that device current: check it is an sm_100 part, look up
// the device address of the static scratch array (the host-side name is only a
// stand-in, not a device address).
attn_status_t setup_device(NoAllocDevice** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return attn_internal::report(ATTN_ERR_CUDA, "attn_fwd_noalloc: no usable current device");
  std::lock_guard<std::mutex> lk(g_mu);
  NoAllocDevice& d = g_dev[dev];
  if (!d.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return attn_internal::report(ATTN_ERR_CUDA, "attn_fwd_noalloc: device attribute query failed");
    if (major != 10 || minor != 0)
      return attn_internal::report(ATTN_ERR_UNSUPPORTED, "attn_fwd_noalloc needs an sm_100 GPU (B200)");
    int* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr), g_noalloc_scratch);
    if (e != cudaSuccess || ptr == nullptr)
      return attn_internal::report(ATTN_ERR_CUDA, "attn_fwd_noalloc: cudaGetSymbolAddress of the scratch failed");
    d.scratch = ptr;
    d.sms = sms;
    d.ready = true;
  }
  *out = &d;
  return ATTN_OK;
}

}  // namespace

extern "C" attn_status_t attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o,
                                          float* lse, int B, int H, int N, int d, int causal,
                                          float scale, const int32_t* cu_seqlens,
                                          int64_t total_tokens, int check, attn_stream_t stream) {
  using attn_internal::report;
  // Same argument checks and launch construction as attn_fwd (shared helpers),
  // so both entry points launch the same kernel with the same parameters.
  const attn_internal::FwdCall c{q, k, v, o, lse, B, H, N, d, causal, scale, cu_seqlens, nullptr, nullptr};
  attn_internal::FwdPlan pl;
  attn_status_t st = attn_internal::plan_fwd(c, &pl);
  if (st != ATTN_OK || pl.noop) return st;
  int64_t total = pl.dense_tokens;
  if (cu_seqlens) {
    // No device-to-host read of cu_seqlens[B] here: the caller states the count.
    if (total_tokens < 0 || total_tokens > pl.dense_tokens)
      return report(ATTN_ERR_INVALID_ARG, "varlen needs total_tokens = cu_seqlens[B] in [0, B*N]");
    if (total_tokens == 0) return ATTN_OK;  // an empty packed batch, as in attn_fwd
    total = total_tokens;
  }
  if (kFwdScratchNeeded > kScratchBytes)
    return report(ATTN_ERR_WORKSPACE, "the forward kernel needs more scratch than the static array holds");

  NoAllocDevice* dev = nullptr;
  st = setup_device(&dev);
  if (st != ATTN_OK) return st;
  attn::FwdLaunch a;
  st = attn_internal::fill_fwd_launch(c, pl, total, dev->sms, 0, dev->scratch,
                                      reinterpret_cast<unsigned*>(dev->scratch + 2), &a);
  if (st != ATTN_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

  // The status word and the claim counters must start at zero; the array keeps the
  // previous call's values otherwise.
  cudaError_t e = cudaMemsetAsync(dev->scratch, 0, kFwdScratchNeeded, cs);
  if (e != cudaSuccess) return report(ATTN_ERR_CUDA, "attn_fwd_noalloc: clearing the status word failed");
  st = attn_internal::launch_planned_fwd(c, pl, a, stream);
  if (st != ATTN_OK || !check) return st;
  int word = 0;
  e = cudaStreamSynchronize(cs);
  if (e == cudaSuccess) e = cudaMemcpy(&word, dev->scratch, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return report(ATTN_ERR_CUDA, cudaGetErrorString(e));
  if (word != 0) {
    const attn_status_t code = static_cast<attn_status_t>(word & 0xff);
    return report(code, code == ATTN_ERR_TIMEOUT ? "a kernel wait exceeded its time limit"
                                                 : "the kernel rejected cu_seqlens");
  }
  return ATTN_OK;
}
