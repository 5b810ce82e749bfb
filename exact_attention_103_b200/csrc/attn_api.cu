// attn_api.cu -- the C ABI of libattn (declared in include/attn.h): argument
// validation, TMA descriptor construction, per-device state, and launch.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/attn.h"
#include "attn_fwd_sm100.h"
#include "attn_bwd_sm100.h"
#include "attn_internal.h"

namespace {

thread_local char g_last_error[512] = "";

attn_status_t fail(attn_status_t s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
attn_status_t fail(attn_status_t s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

attn_status_t cuda_fail(cudaError_t e, const char* what) {
  return fail(ATTN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

constexpr int kMaxDevices = 64;

// Claim counters of the forward kernel's dynamic scheduler, two words per slot,
// zero between launches (a launch's last CTA returns its slot to zero).  Two
// launches that run at the same time must not share a slot; launches on one
// stream never do, so each stream keeps its own slot: streams get slots in order
// of first use, and beyond kWorkSlots streams the least recently used slot passes
// to the new stream.
constexpr int kWorkSlots = 64;

struct DeviceState {
  bool ready = false;
  int sms = 0;
  int pair_clusters = -1;  // clusters of the pair kernel that fit at once (-1: not asked yet)
  int* err = nullptr;        // device error word
  unsigned* work = nullptr;  // kWorkSlots claim-counter slots (same allocation)
  cudaStream_t slot_stream[kWorkSlots] = {};
  uint64_t slot_use[kWorkSlots] = {};  // 0 = free, else the tick of the last use
  uint64_t tick = 0;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
EncodeTiledFn g_encode = nullptr;

// Lazily prepares the current device: checks for sm_100, allocates the error word.
attn_status_t device_state(DeviceState** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(ATTN_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& st = g_dev[dev];
  if (!st.ready) {
    cudaDeviceProp prop;
    e = cudaGetDeviceProperties(&prop, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
    if (prop.major != 10 || prop.minor != 0)
      return fail(ATTN_ERR_UNSUPPORTED, "libattn needs an sm_100 GPU (B200); device %d is sm_%d%d",
                  dev, prop.major, prop.minor);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
      if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
        return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    // One allocation: the error word, then (256 bytes in) the claim counters.
    const size_t bytes = 256 + kWorkSlots * 2 * sizeof(unsigned);
    void* mem = nullptr;
    e = cudaMalloc(&mem, bytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(error word and claim counters)");
    e = cudaMemset(mem, 0, bytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(error word and claim counters)");
    st.err = static_cast<int*>(mem);
    st.work = reinterpret_cast<unsigned*>(static_cast<char*>(mem) + 256);
    st.sms = prop.multiProcessorCount;
    st.ready = true;
  }
  *out = &st;
  return ATTN_OK;
}

// The claim-counter slot of `stream` on this device (see kWorkSlots).
unsigned* work_slot(DeviceState* dev, cudaStream_t stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  int pick = 0;
  for (int i = 0; i < kWorkSlots; ++i) {
    if (dev->slot_use[i] != 0 && dev->slot_stream[i] == stream) {
      pick = i;
      break;
    }
    if (dev->slot_use[i] < dev->slot_use[pick]) pick = i;  // a free slot, else the oldest
  }
  dev->slot_stream[pick] = stream;
  dev->slot_use[pick] = ++dev->tick;
  return dev->work + 2 * pick;
}

// A 3-D view {d, H, total} of a token-major [total, H, d] tensor of esz-byte
// elements (2: bf16, 1: E4M3 moved as bytes); box = one 128-byte-wide chunk of
// 128 rows, 128-byte swizzle.
bool make_map_esz(CUtensorMap* m, const void* ptr, int64_t total, int H, int d, int esz) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(total)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * esz,
                                 static_cast<cuuint64_t>(H) * d * esz};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / esz), 1, 128};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(m, esz == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                              3, const_cast<void*>(ptr), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_map(CUtensorMap* m, const void* ptr, int64_t total, int H, int d) {
  return make_map_esz(m, ptr, total, H, d, 2);
}

// The bf16 view {d, H, total} with 64-row boxes (the K halves of a CTA pair).
bool make_map_rows64(CUtensorMap* m, const void* ptr, int64_t total, int H, int d) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(total)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(H) * d * 2};
  const cuuint32_t box[3] = {64, 1, 64};
  const cuuint32_t estr[3] = {1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The bf16 output O as {d, H, total} with box {64, 1, 32} (one softmax warp's 32
// rows, 64 head dims; 128-byte swizzle): the TMA stores of the forward's epilogue.
bool make_map_o(CUtensorMap* m, void* ptr, int64_t total, int H, int d) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(total)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(H) * d * 2};
  const cuuint32_t box[3] = {64, 1, 32};
  const cuuint32_t estr[3] = {1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, ptr, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;
constexpr float kDefaultTau = 8.0f;
// E4M3 path: a lower threshold leaves room to scale P~ up by 2^floor(8 - tau), so
// small probabilities stay normal E4M3 numbers instead of flushing to subnormals.
constexpr float kDefaultTauE4m3 = 4.0f;
constexpr int kMaxVarlenB = 1024;
constexpr int kMaxVarlenN = 131072;

// The mask of a call: a window bound of N - 1 or more hides nothing on that side,
// so a window collapses to the causal or the unmasked kernel where it can; open
// sides hold N.  Causal forces the right bound to 0.
attn_status_t select_mask(int N, int causal, int has_window, int wl, int wr, attn::MaskKind* mask,
                          int* win_l, int* win_r) {
  *mask = causal ? attn::kMaskCausal : attn::kMaskNone;
  *win_l = *win_r = 0;
  if (!has_window) return ATTN_OK;
  if (N >= (1 << 30)) return fail(ATTN_ERR_UNSUPPORTED, "sliding window needs N < 2^30");
  *win_l = (wl < 0 || wl > N) ? N : wl;
  *win_r = causal ? 0 : ((wr < 0 || wr > N) ? N : wr);
  const bool left_open = *win_l >= N - 1, right_open = *win_r >= N - 1;
  if (left_open && right_open) *mask = attn::kMaskNone;
  else if (left_open && *win_r == 0) *mask = attn::kMaskCausal;
  else *mask = attn::kMaskWindow;
  return ATTN_OK;
}

}  // namespace

namespace attn_internal {

// Device preparation and the TMA view builder, for the diagnostic entry point.
attn_status_t prepare_selftest(int** err, bool (**mk)(CUtensorMap*, const void*, int64_t, int, int)) {
  DeviceState* dev = nullptr;
  const attn_status_t st = device_state(&dev);
  if (st != ATTN_OK) return st;
  *err = dev->err;
  *mk = make_map;
  return ATTN_OK;
}

attn_status_t load_tensor_map_encoder() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode) return ATTN_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
    return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  return ATTN_OK;
}

attn_status_t report(attn_status_t s, const char* message) { return fail(s, "%s", message); }

bool make_tensor_map_e4m3(CUtensorMap* m, const void* ptr, int64_t total, int H, int d) {
  return make_map_esz(m, ptr, total, H, d, 1);
}

attn_status_t plan_fwd(const FwdCall& c, FwdPlan* pl) {
  const int B = c.B, H = c.H, N = c.N, d = c.d;
  const attn_internal::E4m3Scales* f8 = c.f8;
  std::memset(pl, 0, sizeof(*pl));
  if (B < 0 || H <= 0 || N < 0) return fail(ATTN_ERR_INVALID_ARG, "B=%d H=%d N=%d", B, H, N);
  if (f8 && d != 128) return fail(ATTN_ERR_UNSUPPORTED, "E4M3 path: head dim %d (supported: 128)", d);
  if (d != 64 && d != 128) return fail(ATTN_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
  if (!(std::isfinite(c.scale) && c.scale > 0.f))
    return fail(ATTN_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (f8 && !(std::isfinite(f8->q) && f8->q > 0.f && std::isfinite(f8->k) && f8->k > 0.f &&
              std::isfinite(f8->v) && f8->v > 0.f))
    return fail(ATTN_ERR_INVALID_ARG, "E4M3 scales must be finite and > 0");
  if (B == 0 || N == 0) {
    pl->noop = true;
    return ATTN_OK;
  }
  if (!c.q || !c.k || !c.v || !c.o || !c.lse) return fail(ATTN_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned(c.q, 16) || !aligned(c.k, 16) || !aligned(c.v, 16) || !aligned(c.o, 16) ||
      !aligned(c.lse, 4))
    return fail(ATTN_ERR_INVALID_ARG, "q/k/v/o must be 16-byte aligned and lse 4-byte aligned");
  const bool varlen = c.cu_seqlens != nullptr;
  if (varlen && (B > kMaxVarlenB || N > kMaxVarlenN))
    return fail(ATTN_ERR_UNSUPPORTED, "varlen supports B <= %d and N <= %d", kMaxVarlenB, kMaxVarlenN);
  const int pair = (c.opts && c.opts->cta_pair) ? 1 : 0;
  pl->pair = pair;
  pl->T = (static_cast<int64_t>(N) + (pair ? 511 : 255)) / (pair ? 512 : 256);
  pl->items_bound = static_cast<int64_t>(B) * pl->T * H;
  pl->dense_tokens = static_cast<int64_t>(B) * N;
  if (pl->items_bound > INT32_MAX / 2 || pl->dense_tokens * H > INT64_MAX / 256 ||
      pl->dense_tokens > INT32_MAX)
    return fail(ATTN_ERR_UNSUPPORTED, "problem too large for 32-bit tile indexing");
  if (varlen && !aligned(c.cu_seqlens, 4)) return fail(ATTN_ERR_INVALID_ARG, "cu_seqlens misaligned");
  pl->tau = f8 ? kDefaultTauE4m3 : kDefaultTau;
  pl->timeout = kDefaultTimeoutNs;
  int has_window = 0, wl = -1, wr = -1;
  if (const attn_fwd_opts_t* opts = c.opts) {
    if (opts->test_fault != 0 && opts->test_fault != 1)
      return fail(ATTN_ERR_INVALID_ARG, "test_fault must be 0 or 1");
    pl->test_fault = opts->test_fault;
    if (opts->rescale_threshold >= 0.f) pl->tau = opts->rescale_threshold;
    if (!(pl->tau <= 64.f)) return fail(ATTN_ERR_INVALID_ARG, "rescale_threshold must be <= 64");
    if (opts->timeout_ns) pl->timeout = opts->timeout_ns;
    pl->stats = opts->stats;
    if (pl->stats && !aligned(pl->stats, 8)) return fail(ATTN_ERR_INVALID_ARG, "stats misaligned");
    pl->poly = opts->exp_poly_per8;
    if (pl->poly != 0 && pl->poly != 2 && pl->poly != 8)
      return fail(ATTN_ERR_INVALID_ARG, "exp_poly_per8 must be 0, 2 or 8");
    if (f8 && pl->poly != 0 && pl->poly != 2)
      return fail(ATTN_ERR_UNSUPPORTED, "E4M3 path: exp_poly_per8 must be 0 or 2");
    if (f8 && !(pl->tau <= 8.f))
      return fail(ATTN_ERR_INVALID_ARG, "E4M3 path: rescale_threshold must be <= 8 (P~ <= 256 < 448)");
    if (opts->has_window) {
      has_window = 1;
      wl = opts->window_left;
      wr = opts->window_right;
    }
    if (opts->cta_pair && (f8 || d != 128 || pl->poly != 0))
      return fail(ATTN_ERR_UNSUPPORTED, "cta_pair: bf16 inputs, d = 128 and exp_poly_per8 = 0 only");
  }
  const attn_status_t st = select_mask(N, c.causal, has_window, wl, wr, &pl->mask, &pl->win_l, &pl->win_r);
  if (st != ATTN_OK) return st;
  if (pl->mask == attn::kMaskWindow) pl->stats = nullptr;  // counters are not kept under a window
  return ATTN_OK;
}

attn_status_t fill_fwd_launch(const FwdCall& c, const FwdPlan& pl, int64_t total, int sms, int pair_clusters,
                              int* err, unsigned* work, attn::FwdLaunch* a) {
  const attn_status_t st = load_tensor_map_encoder();
  if (st != ATTN_OK) return st;
  std::memset(a, 0, sizeof(*a));
  const attn_internal::E4m3Scales* f8 = c.f8;
  const int esz = f8 ? 1 : 2;
  if (!make_map_esz(&a->tm_q, c.q, total, c.H, c.d, esz) || !make_map_esz(&a->tm_k, c.k, total, c.H, c.d, esz) ||
      !make_map_esz(&a->tm_v, c.v, total, c.H, c.d, esz) ||
      (pl.pair && !make_map_rows64(&a->tm_k2, c.k, total, c.H, c.d)) ||
      !make_map_o(&a->tm_o, c.o, total, c.H, c.d))
    return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled rejected the Q/K/V/O views");
  a->pair = pl.pair;
  const bool varlen = c.cu_seqlens != nullptr;
  a->p.o = static_cast<__nv_bfloat16*>(c.o);
  a->p.lse = c.lse;
  a->p.cu_seqlens = c.cu_seqlens;
  a->p.B = c.B;
  a->p.H = c.H;
  a->p.N = c.N;
  a->p.T = static_cast<int>(pl.T);
  a->p.total = static_cast<int>(total);
  // The E4M3 scales of Q and K fold into the score scale; V's into 1/l.  One
  // rounding to fp32, from a double product.
  a->p.scale_log2 = static_cast<float>(static_cast<double>(c.scale) * 1.4426950408889634 *
                                       (f8 ? static_cast<double>(f8->q) * f8->k : 1.0));
  a->p.o_scale = f8 ? f8->v : 1.f;
  a->p.p_shift = f8 ? std::floor(8.f - pl.tau) : 0.f;
  a->p.tau = pl.tau;
  a->p.err = err;
  a->p.work = work;
  a->p.stats = pl.stats;
  a->p.timeout_ns = pl.timeout;
  a->p.test_fault = pl.test_fault;
  a->p.wl = pl.win_l;
  a->p.wr = pl.win_r;
  // Dense unmasked launches may split their last wave into half items (see the
  // kernel), so up to twice as many CTAs can be useful there.
  a->smem = attn::fwd_smem_bytes(c.d, c.B, static_cast<int>(pl.T), varlen ? 1 : 0, f8 ? 1 : 0, pl.pair);
  // O leaves through shared-memory staging and TMA stores where the staging
  // buffers fit beside the rest (not beside the work tables of very many sequences).
  a->p.stage_off = attn::fwd_stage_offset(c.d, c.B, static_cast<int>(pl.T), varlen ? 1 : 0, f8 ? 1 : 0, pl.pair);
  if (a->p.stage_off != 0) a->smem = 1024 + a->p.stage_off + attn::kFwdStageBytes;
  if (pl.pair) {
    // Two CTAs per item; as many clusters as fit at once (SMs left over in a GPC
    // of odd SM count cannot hold a cluster).
    const int64_t fit = pair_clusters > 0 ? pair_clusters : sms / 2;
    const int64_t clusters = pl.items_bound < fit ? pl.items_bound : fit;
    a->grid = static_cast<int>(2 * clusters);
  } else {
    const int64_t useful = (!varlen && pl.mask == attn::kMaskNone) ? 2 * pl.items_bound : pl.items_bound;
    a->grid = static_cast<int>(useful < sms ? useful : sms);
  }
  return ATTN_OK;
}

attn_status_t launch_planned_fwd(const FwdCall& c, const FwdPlan& pl, const attn::FwdLaunch& a,
                                 attn_stream_t stream) {
  const cudaError_t e = attn::launch_fwd(a, c.d, pl.mask, pl.poly, c.f8 ? 1 : 0,
                                         reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "forward kernel launch");
  return ATTN_OK;
}

}  // namespace attn_internal

namespace {

attn_status_t fwd_impl(const attn_internal::FwdCall& c, int64_t total_hint, attn_stream_t stream) {
  attn_internal::FwdPlan pl;
  attn_status_t st = attn_internal::plan_fwd(c, &pl);
  if (st != ATTN_OK || pl.noop) return st;
  DeviceState* dev = nullptr;
  st = device_state(&dev);
  if (st != ATTN_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  int64_t total = pl.dense_tokens;
  if (c.cu_seqlens) {
    if (total_hint >= 0) {
      total = total_hint;
    } else {
      // The TMA views need the packed token count; read cu_seqlens[B] (4 bytes).
      int32_t t = 0;
      cudaError_t e = cudaMemcpyAsync(&t, c.cu_seqlens + c.B, sizeof(int32_t), cudaMemcpyDeviceToHost, cs);
      if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
      if (e != cudaSuccess) return cuda_fail(e, "reading cu_seqlens[B]");
      total = t;
    }
    if (total < 0 || total > pl.dense_tokens)
      return fail(ATTN_ERR_INVALID_ARG, "packed token count %lld outside [0, B*N]", (long long)total);
    if (total == 0) return ATTN_OK;
  }
  attn::FwdLaunch a;
  unsigned* work = work_slot(dev, cs);
  if (pl.pair && dev->pair_clusters < 0) {
    std::lock_guard<std::mutex> lk(g_mu);
    dev->pair_clusters = attn::fwd_pair_max_clusters(
        attn::fwd_smem_bytes(128, c.B, static_cast<int>(pl.T), c.cu_seqlens ? 1 : 0, 0, 1));
  }
  st = attn_internal::fill_fwd_launch(c, pl, total, dev->sms, dev->pair_clusters, dev->err, work, &a);
  if (st != ATTN_OK) return st;
  return attn_internal::launch_planned_fwd(c, pl, a, stream);
}

}  // namespace

extern "C" {

attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                       int H, int N, int d, int causal, float scale, const int32_t* cu_seqlens,
                       attn_stream_t stream) {
  const attn_internal::FwdCall c{q, k, v, o, lse, B, H, N, d, causal, scale, cu_seqlens, nullptr, nullptr};
  return fwd_impl(c, -1, stream);
}

attn_status_t attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                          int H, int N, int d, int causal, float scale, const int32_t* cu_seqlens,
                          const attn_fwd_opts_t* opts, attn_stream_t stream) {
  const int64_t hint = (opts && opts->total_tokens > 0) ? opts->total_tokens : -1;
  const attn_internal::FwdCall c{q, k, v, o, lse, B, H, N, d, causal, scale, cu_seqlens, opts, nullptr};
  return fwd_impl(c, hint, stream);
}

attn_status_t attn_fwd_e4m3(const void* q, const void* k, const void* v, void* o, float* lse,
                            int B, int H, int N, int d, int causal, float scale, float q_scale,
                            float k_scale, float v_scale, const int32_t* cu_seqlens,
                            const attn_fwd_opts_t* opts, attn_stream_t stream) {
  const int64_t hint = (opts && opts->total_tokens > 0) ? opts->total_tokens : -1;
  const attn_internal::E4m3Scales f8{q_scale, k_scale, v_scale};
  const attn_internal::FwdCall c{q, k, v, o, lse, B, H, N, d, causal, scale, cu_seqlens, opts, &f8};
  return fwd_impl(c, hint, stream);
}

}  // extern "C"

namespace {
attn_status_t bwd_impl(const void* q, const void* k, const void* v, const void* o,
                       const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                       int H, int N, int d, int causal, float scale, const int32_t* cu_seqlens,
                       int deterministic, void* workspace, size_t workspace_bytes,
                       const attn_bwd_opts_t* opts, attn_stream_t stream) {
  (void)deterministic;  // every call is deterministic: no atomic accumulation
  if (B < 0 || H <= 0 || N < 0) return fail(ATTN_ERR_INVALID_ARG, "B=%d H=%d N=%d", B, H, N);
  if (d != 64 && d != 128) return fail(ATTN_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
  if (!(std::isfinite(scale) && scale > 0.f)) return fail(ATTN_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (B == 0 || N == 0) return ATTN_OK;
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv)
    return fail(ATTN_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dout, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 4))
    return fail(ATTN_ERR_INVALID_ARG, "tensors must be 16-byte aligned (lse 4-byte)");
  const bool varlen = cu_seqlens != nullptr;
  if (varlen && (B > kMaxVarlenB || N > kMaxVarlenN))
    return fail(ATTN_ERR_UNSUPPORTED, "varlen supports B <= %d and N <= %d", kMaxVarlenB, kMaxVarlenN);
  const int64_t ntiles = (static_cast<int64_t>(N) + 127) / 128;
  const int64_t grid = static_cast<int64_t>(B) * ntiles * H;
  const int64_t dense_tokens = static_cast<int64_t>(B) * N;
  if (grid > INT32_MAX / 2 || dense_tokens > INT32_MAX)
    return fail(ATTN_ERR_UNSUPPORTED, "problem too large for 32-bit tile indexing");
  attn::MaskKind mask;
  int win_l, win_r;
  attn_status_t st = select_mask(N, causal, opts ? opts->has_window : 0, opts ? opts->window_left : -1,
                                 opts ? opts->window_right : -1, &mask, &win_l, &win_r);
  if (st != ATTN_OK) return st;
  DeviceState* dev = nullptr;
  st = device_state(&dev);
  if (st != ATTN_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  int64_t total = dense_tokens;
  if (varlen) {
    if (opts && opts->total_tokens > 0) {
      total = opts->total_tokens;  // checked against cu_seqlens[B] on the device
    } else {
      int32_t t = 0;
      cudaError_t e = cudaMemcpyAsync(&t, cu_seqlens + B, sizeof(int32_t), cudaMemcpyDeviceToHost, cs);
      if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
      if (e != cudaSuccess) return cuda_fail(e, "reading cu_seqlens[B]");
      total = t;
    }
    if (total < 0 || total > dense_tokens)
      return fail(ATTN_ERR_INVALID_ARG, "packed token count %lld outside [0, B*N]", (long long)total);
    if (total == 0) return ATTN_OK;
  }
  const size_t need = attn_bwd_workspace_size(B, H, N, d, static_cast<int>(total), deterministic);
  if (workspace_bytes < need || (need > 0 && (!workspace || !aligned(workspace, 256))))
    return fail(ATTN_ERR_WORKSPACE, "workspace of %zu bytes (256-byte aligned) needed", need);
  attn::BwdLaunch a;
  std::memset(&a, 0, sizeof(a));
  if (!make_map(&a.tm_q, q, total, H, d) || !make_map(&a.tm_k, k, total, H, d) ||
      !make_map(&a.tm_v, v, total, H, d) || !make_map(&a.tm_do, dout, total, H, d))
    return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled rejected the Q/K/V/dO views");
  a.p.lse = lse;
  a.p.dpre = static_cast<float*>(workspace);
  a.p.dq = static_cast<__nv_bfloat16*>(dq);
  a.p.dk = static_cast<__nv_bfloat16*>(dk);
  a.p.dv = static_cast<__nv_bfloat16*>(dv);
  a.p.cu_seqlens = cu_seqlens;
  a.p.B = B;
  a.p.H = H;
  a.p.N = N;
  a.p.total = static_cast<int>(total);
  a.p.ntiles = static_cast<int>(ntiles);
  a.p.scale = scale;
  a.p.scale_log2 = scale * 1.4426950408889634f;
  a.p.err = dev->err;
  a.p.timeout_ns = (opts && opts->timeout_ns) ? opts->timeout_ns : kDefaultTimeoutNs;
  a.p.wl = win_l;
  a.p.wr = win_r;
  a.grid = static_cast<int>(grid);
  const cudaError_t e = attn::launch_bwd(a, o, dout, d, static_cast<int>(mask), cs);
  if (e != cudaSuccess) return cuda_fail(e, "backward kernel launch");
  return ATTN_OK;
}
}  // namespace

extern "C" {

attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o,
                       const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                       int H, int N, int d, int causal, float scale, const int32_t* cu_seqlens,
                       int deterministic, void* workspace, size_t workspace_bytes,
                       attn_stream_t stream) {
  return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, causal, scale, cu_seqlens,
                  deterministic, workspace, workspace_bytes, nullptr, stream);
}

attn_status_t attn_bwd_ex(const void* q, const void* k, const void* v, const void* o,
                          const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                          int H, int N, int d, int causal, float scale, const int32_t* cu_seqlens,
                          int deterministic, void* workspace, size_t workspace_bytes,
                          const attn_bwd_opts_t* opts, attn_stream_t stream) {
  return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, causal, scale, cu_seqlens,
                  deterministic, workspace, workspace_bytes, opts, stream);
}

size_t attn_bwd_workspace_size(int B, int H, int N, int d, int total_tokens, int deterministic) {
  (void)N;
  (void)d;
  (void)deterministic;
  if (B <= 0 || H <= 0 || total_tokens <= 0) return 0;
  const size_t bytes = static_cast<size_t>(total_tokens) * static_cast<size_t>(H) * sizeof(float);
  return (bytes + 255) / 256 * 256;
}

attn_status_t attn_get_device_status(attn_stream_t stream) {
  DeviceState* dev = nullptr;
  attn_status_t st = device_state(&dev);
  if (st != ATTN_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(cs);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int word = 0;
  e = cudaMemcpy(&word, dev->err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  if (word == 0) return ATTN_OK;
  e = cudaMemset(dev->err, 0, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
  const int code = word & 0xff, site = word >> 8;
  return fail(static_cast<attn_status_t>(code), "device error %d recorded at site %d", code, site);
}

const char* attn_status_string(attn_status_t s) {
  switch (s) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG";
    case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
    case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT";
    case ATTN_ERR_WORKSPACE: return "ATTN_ERR_WORKSPACE";
  }
  return "unknown attn_status_t";
}

const char* attn_last_error(void) { return g_last_error; }

}  // extern "C"
