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

namespace attn_internal {
attn_status_t load_tensor_map_encoder();
bool make_tensor_map(CUtensorMap* m, const void* ptr, int64_t total, int H, int d);
attn_status_t report(attn_status_t s, const char* message);
}  // namespace attn_internal

namespace {

// Scratch of the allocation-free forward: the kernel's status word lives at word 0.
// Every GPU that loads the library holds these bytes until the process exits.
constexpr size_t kScratchBytes = 256;
static __device__ __align__(256) int g_noalloc_scratch[kScratchBytes / sizeof(int)];
constexpr size_t kFwdScratchNeeded = sizeof(int);  // the status word

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
// stand-in, not a device address), and load the tensor-map encoder.
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
    const attn_status_t st = attn_internal::load_tensor_map_encoder();
    if (st != ATTN_OK) return st;
    d.scratch = ptr;
    d.sms = sms;
    d.ready = true;
  }
  *out = &d;
  return ATTN_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" attn_status_t attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o,
                                          float* lse, int B, int H, int N, int d, int causal,
                                          float scale, const int32_t* cu_seqlens,
                                          int64_t total_tokens, int check, attn_stream_t stream) {
  using attn_internal::report;
  if (B < 0 || H <= 0 || N < 0) return report(ATTN_ERR_INVALID_ARG, "B, H or N out of range");
  if (d != 64 && d != 128) return report(ATTN_ERR_UNSUPPORTED, "head dim must be 64 or 128");
  if (!(std::isfinite(scale) && scale > 0.f)) return report(ATTN_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (B == 0 || N == 0) return ATTN_OK;
  if (!q || !k || !v || !o || !lse) return report(ATTN_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return report(ATTN_ERR_INVALID_ARG, "q/k/v/o must be 16-byte aligned and lse 4-byte aligned");
  const bool varlen = cu_seqlens != nullptr;
  if (varlen && (B > 1024 || N > 131072))
    return report(ATTN_ERR_UNSUPPORTED, "varlen supports B <= 1024 and N <= 131072");
  if (varlen && !aligned(cu_seqlens, 4)) return report(ATTN_ERR_INVALID_ARG, "cu_seqlens misaligned");
  const int64_t T256 = (static_cast<int64_t>(N) + 255) / 256;
  const int64_t items_bound = static_cast<int64_t>(B) * T256 * H;
  const int64_t dense_tokens = static_cast<int64_t>(B) * N;
  if (items_bound > INT32_MAX / 2 || dense_tokens > INT32_MAX)
    return report(ATTN_ERR_UNSUPPORTED, "problem too large for 32-bit tile indexing");
  int64_t total = dense_tokens;
  if (varlen) {
    // No device-to-host read of cu_seqlens[B] here: the caller states the count.
    if (total_tokens <= 0 || total_tokens > dense_tokens)
      return report(ATTN_ERR_INVALID_ARG, "varlen needs total_tokens = cu_seqlens[B] in [1, B*N]");
    total = total_tokens;
  }
  if (kFwdScratchNeeded > kScratchBytes)
    return report(ATTN_ERR_WORKSPACE, "the forward kernel needs more scratch than the static array holds");

  NoAllocDevice* dev = nullptr;
  const attn_status_t st = setup_device(&dev);
  if (st != ATTN_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

  attn::FwdLaunch a;
  std::memset(&a, 0, sizeof(a));
  if (!attn_internal::make_tensor_map(&a.tm_q, q, total, H, d) ||
      !attn_internal::make_tensor_map(&a.tm_k, k, total, H, d) ||
      !attn_internal::make_tensor_map(&a.tm_v, v, total, H, d))
    return report(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled rejected the Q/K/V views");
  a.p.o = static_cast<__nv_bfloat16*>(o);
  a.p.lse = lse;
  a.p.cu_seqlens = cu_seqlens;
  a.p.B = B;
  a.p.H = H;
  a.p.N = N;
  a.p.T = static_cast<int>(T256);
  a.p.total = static_cast<int>(total);
  a.p.scale_log2 = scale * 1.4426950408889634f;
  a.p.tau = 8.0f;
  a.p.err = dev->scratch;
  a.p.stats = nullptr;
  a.p.timeout_ns = 2000000000ull;
  a.p.test_fault = 0;
  const int64_t useful = (!varlen && !causal) ? 2 * items_bound : items_bound;
  a.grid = static_cast<int>(useful < dev->sms ? useful : dev->sms);
  a.p.o_scale = 1.f;
  a.smem = attn::fwd_smem_bytes(d, B, static_cast<int>(T256), varlen ? 1 : 0, 0);

  // The status word must start at zero; it keeps the previous call's value otherwise.
  cudaError_t e = cudaMemsetAsync(dev->scratch, 0, kFwdScratchNeeded, cs);
  if (e != cudaSuccess) return report(ATTN_ERR_CUDA, "attn_fwd_noalloc: clearing the status word failed");
  e = attn::launch_fwd(a, d, causal ? attn::kMaskCausal : attn::kMaskNone, 0, 0, cs);
  if (e != cudaSuccess) return report(ATTN_ERR_CUDA, cudaGetErrorString(e));
  if (!check) return ATTN_OK;
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
