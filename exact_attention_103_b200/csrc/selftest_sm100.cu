// selftest_sm100.cu -- one-tile check of the forward kernel's tensor-core building
// blocks (see include/attn_selftest.h).  Uses exactly the descriptors, tensor-map
// format and TMEM moves of attn_fwd_sm100.cu, in a plain sequential order.
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/attn_selftest.h"
#include "sm100_ptx.cuh"
#include "softmax_math.cuh"

namespace attn {
namespace {

// The forward kernel's FMA-pipe exponential over an input array: y_poly from the
// packed two-lane form (the one the kernel runs), y_scalar from the scalar form,
// y_ref from CUDA's exp2f.
__global__ void exp2_selftest_kernel(const float* __restrict__ x, float* y_poly, float* y_scalar,
                                     float* y_ref, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  float a = x[i], e = (i + 1 < n) ? x[i + 1] : 0.f;
  float pa = a, pe = e;
  exp2_poly_x2(pa, pe);
  y_poly[i] = pa;
  y_scalar[i] = exp2_poly(a);
  y_ref[i] = exp2f(a);
  if (i + 1 < n) {
    y_poly[i + 1] = pe;
    y_scalar[i + 1] = exp2_poly(e);
    y_ref[i + 1] = exp2f(e);
  }
}

// F8: E4M3 inputs (kind::f8f6f4, K = 32 per instruction) and P = e4m3(S).
template <int D, bool F8>
__global__ void __launch_bounds__(128, 1)
    selftest_kernel(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb,
                    const __grid_constant__ CUtensorMap tv, float* s_out, float* o_out, int* err) {
  constexpr int ESZ = F8 ? 1 : 2;               // bytes per element
  constexpr int TILE = 128 * D * ESZ, CHUNK = 128 * 128;
  constexpr int KSTEP = 32 / ESZ;               // elements per MMA K step (32 bytes)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t bar_tma = sb + 3 * TILE, bar_mma = bar_tma + 8;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + 3 * TILE + 16);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(bar_tma, 1);
    mbar_init(bar_mma, 1);
    misc[1] = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(sb + 3 * TILE + 16, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  WaitCtl wc;
  wc.abort = reinterpret_cast<volatile uint32_t*>(misc + 1);
  wc.err = err;
  wc.limit_ns = 1000000000ull;
  const uint64_t pol = l2_policy_evict_first();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar_tma, 3 * TILE);
    for (int c = 0; c < TILE / CHUNK; ++c) {
      tma_load_3d(sb + 0 * TILE + c * CHUNK, &ta, bar_tma, c * (128 / ESZ), 0, 0, pol);
      tma_load_3d(sb + 1 * TILE + c * CHUNK, &tb, bar_tma, c * (128 / ESZ), 0, 0, pol);
      tma_load_3d(sb + 2 * TILE + c * CHUNK, &tv, bar_tma, c * (128 / ESZ), 0, 0, pol);
    }
  }
  bool ok = __all_sync(0xffffffffu, mbar_wait(bar_tma, 0, wc, 4 | (1 << 8)));
  const uint32_t tS = tmem, tO = tmem + 256;
  if (ok && threadIdx.x == 0) {
    tc_fence_after();
    for (int kk = 0; kk < D / KSTEP; ++kk) {
      const uint32_t off = (kk >> 2) * CHUNK + (kk & 3) * 32;
      const uint64_t da = sdesc_sw128(sb + off, 16, 1024), db = sdesc_sw128(sb + TILE + off, 16, 1024);
      if constexpr (F8)
        mma_ss_f8(tS, da, db, idesc_e4m3_f32(128, 128, 0, 0), kk > 0 ? 1u : 0u);
      else
        mma_ss(tS, da, db, idesc_bf16_f32(128, 128, 0, 0), kk > 0 ? 1u : 0u);
    }
    tc_commit(bar_mma);
  }
  if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_mma, 0, wc, 4 | (2 << 8)));
  const int r = warp * 32 + lane;
  const uint32_t lane_bits = static_cast<uint32_t>(warp * 32) << 16;
  if (ok) {
    tc_fence_after();
    uint32_t sv[128];
    tmem_ld_x128(tS + lane_bits, sv);
    for (int c = 0; c < 128; ++c) s_out[r * 128 + c] = __uint_as_float(sv[c]);
    if constexpr (F8) {
      uint32_t pk[32];
      for (int c = 0; c < 32; ++c)
        pk[c] = pack_e4m3x2(__uint_as_float(sv[4 * c]), __uint_as_float(sv[4 * c + 1])) |
                (pack_e4m3x2(__uint_as_float(sv[4 * c + 2]), __uint_as_float(sv[4 * c + 3])) << 16);
      tmem_st_x32(tS + lane_bits, pk);
    } else {
      uint32_t pk[64];
      for (int c = 0; c < 64; ++c) pk[c] = pack_bf16x2(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1]));
      tmem_st_x64(tS + lane_bits, pk);
    }
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (ok && threadIdx.x == 0) {
    // One K step covers KSTEP keys = 32 bytes of a P row = 8 TMEM columns, and
    // KSTEP rows of V (128 bytes each).
    for (int kk = 0; kk < 128 / KSTEP; ++kk) {
      const uint64_t dv = sdesc_sw128(sb + 2 * TILE + kk * KSTEP * 128, CHUNK, 1024);
      if constexpr (F8)
        mma_ts_f8(tO, tS + kk * 8, dv, idesc_e4m3_f32(128, D, 0, 1), kk > 0 ? 1u : 0u);
      else
        mma_ts(tO, tS + kk * 8, dv, idesc_bf16_f32(128, D, 0, 1), kk > 0 ? 1u : 0u);
    }
    tc_commit(bar_mma);
  }
  if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_mma, 1, wc, 4 | (3 << 8)));
  if (ok) {
    tc_fence_after();
    for (int c = 0; c < D / 32; ++c) {
      uint32_t ov[32];
      tmem_ld_x32(tO + lane_bits + 32 * c, ov);
      for (int i = 0; i < 32; ++i) o_out[r * D + 32 * c + i] = __uint_as_float(ov[i]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace
}  // namespace attn

// Shared with attn_api.cu (defined there).
namespace attn_internal {
attn_status_t prepare_selftest(int** err, bool (**mk)(CUtensorMap*, const void*, int64_t, int, int));
bool make_tensor_map_e4m3(CUtensorMap* m, const void* ptr, int64_t total, int H, int d);
}

extern "C" attn_status_t attn_selftest_umma(const void* a, const void* b, const void* v,
                                            float* s_out, float* o_out, int d,
                                            attn_stream_t stream) {
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (!a || !b || !v || !s_out || !o_out) return ATTN_ERR_INVALID_ARG;
  int* err = nullptr;
  bool (*mk)(CUtensorMap*, const void*, int64_t, int, int) = nullptr;
  attn_status_t st = attn_internal::prepare_selftest(&err, &mk);
  if (st != ATTN_OK) return st;
  alignas(64) CUtensorMap ta, tb, tv;
  if (!mk(&ta, a, 128, 1, d) || !mk(&tb, b, 128, 1, d) || !mk(&tv, v, 128, 1, d))
    return ATTN_ERR_INVALID_ARG;
  const int smem = 1024 + 3 * 128 * d * 2 + 64;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (d == 128) {
    e = cudaFuncSetAttribute(attn::selftest_kernel<128, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) attn::selftest_kernel<128, false><<<1, 128, smem, cs>>>(ta, tb, tv, s_out, o_out, err);
  } else {
    e = cudaFuncSetAttribute(attn::selftest_kernel<64, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) attn::selftest_kernel<64, false><<<1, 128, smem, cs>>>(ta, tb, tv, s_out, o_out, err);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

extern "C" attn_status_t attn_selftest_umma_e4m3(const void* a, const void* b, const void* v,
                                                 float* s_out, float* o_out, attn_stream_t stream) {
  if (!a || !b || !v || !s_out || !o_out) return ATTN_ERR_INVALID_ARG;
  int* err = nullptr;
  bool (*mk)(CUtensorMap*, const void*, int64_t, int, int) = nullptr;
  attn_status_t st = attn_internal::prepare_selftest(&err, &mk);
  if (st != ATTN_OK) return st;
  alignas(64) CUtensorMap ta, tb, tv;
  if (!attn_internal::make_tensor_map_e4m3(&ta, a, 128, 1, 128) ||
      !attn_internal::make_tensor_map_e4m3(&tb, b, 128, 1, 128) ||
      !attn_internal::make_tensor_map_e4m3(&tv, v, 128, 1, 128))
    return ATTN_ERR_INVALID_ARG;
  const int smem = 1024 + 3 * 128 * 128 + 64;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaFuncSetAttribute(attn::selftest_kernel<128, true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) attn::selftest_kernel<128, true><<<1, 128, smem, cs>>>(ta, tb, tv, s_out, o_out, err);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

extern "C" attn_status_t attn_selftest_exp2(const float* x, float* y_poly, float* y_scalar,
                                            float* y_ref, int n, attn_stream_t stream) {
  if (n < 0) return ATTN_ERR_INVALID_ARG;
  if (n == 0) return ATTN_OK;
  if (!x || !y_poly || !y_scalar || !y_ref) return ATTN_ERR_INVALID_ARG;
  const int threads = 256;
  const int pairs = (n + 1) / 2;
  attn::exp2_selftest_kernel<<<(pairs + threads - 1) / threads, threads, 0,
                               reinterpret_cast<cudaStream_t>(stream)>>>(x, y_poly, y_scalar, y_ref, n);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}
