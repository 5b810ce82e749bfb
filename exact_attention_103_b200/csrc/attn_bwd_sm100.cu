// attn_bwd_sm100.cu -- backward pass of exact attention for B200 (sm_100a).
//
// The pages say only that the backward recomputes P instead of storing it
// ("FlashAttention 1-4 详解", 总结 table, 反向传播重计算; "FlashAttention V4
// deep-dive" section 3.3: P and other intermediates kept in TMEM).  With
// P_ij = exp(scale*<q_i,k_j> - LSE_i), D_i = <dO_i, O_i>, dP = dO V^T and
// dS = P o (dP - D) (the textbook backward), three kernels run in order:
//   bwd_pre_kernel   D_i for every (row, head)                (fp32, workspace)
//   bwd_dkdv_kernel  one CTA per 128-key tile: loops over query tiles i and
//                    accumulates dV += P^T dO_i and dK += scale dS^T Q_i in TMEM
//   bwd_dq_kernel    one CTA per 128-query tile: loops over key tiles j and
//                    accumulates dQ += scale dS K_j in TMEM
// Computing dQ in its own kernel recomputes S and dP once more but needs no
// atomic accumulation, so every result is bitwise reproducible run to run.
//
// Both main kernels: warps 0-7 elementwise work (warp w owns TMEM lanes
// 32(w%4)..+31, one row per thread, and columns 64*(w/4)..+63 of each 128-column
// tile), warp 8 TMA producer, warp 9 TMEM owner and MMA issuer (whole warp, one
// elected lane issues).  The MMA warps issue their products in a software-
// pipelined order so the next tile's exponentials overlap the current tile's
// products (dK/dV: dV(n), S^T(n+1), dK(n), dP^T(n+1); dQ: dQ(j), dP(j+1), S(j+2)
// with S double-buffered).  Streamed tiles sit in single-tile ring slots, each
// released as soon as its last product has read it (dK/dV: dO after dV, Q after
// dK; dQ: V after dP, K after dQ), so the next copies start early.
//
// In the dK/dV kernel the per-query LSE and D vary along the TMEM columns, the
// same for every thread of a warp.  Rather than broadcast them across lanes, the
// kernel lets the tensor core subtract them: S^T and dP^T get one more K-step of
// 16 in which A is a constant tile of ones and B holds -LSE/scale (resp. -D) of
// each query, split into three bf16 terms (hi + mid + lo, exact to ~2^-24 of the
// value), so TMEM receives S^T - LSE/scale and dP^T - D directly.  Queries past
// the sequence end get -inf (P = 0).
//
// MASK selects the visibility rule of the forward's mask hook: none, causal, or
// the sliding window (only the tiles the window reaches are visited).  Every wait
// is bounded as in the forward kernel.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "attn_bwd_sm100.h"
#include "sm100_ptx.cuh"
#include "softmax_math.cuh"

namespace attn {

namespace {

constexpr int kThreads = 320;
constexpr int kTile = 128;  // rows of every tile (keys or queries)
constexpr float kLog2e = 1.4426950408889634f;

__host__ __device__ constexpr int timeout_code(int site) { return 4 | (site << 8); }
enum BwdSite { kSiteKv = 32, kSiteStageFull, kSiteStageEmpty, kSiteS, kSiteP, kSiteDs, kSiteAcc,
               kSiteDrain, kSiteBadLen };

// Shared memory of the dK/dV kernel (offsets from a 1024-aligned base): resident
// K_j (A0) and V_j (A1); ONES, the A operand of the extra K-step; two Q slots and
// two dO slots, each a tile followed by its 128 x 16 extra-step operand (XTRA).
template <int D>
struct DkdvLayout {
  static constexpr int TILE = kTile * D * 2;
  static constexpr int CHUNK = kTile * 128;  // 128 rows x 64 columns, 128-byte swizzle
  static constexpr int XTRA = kTile * 32;    // 128 rows x 16 bf16, no swizzle
  static constexpr int SLOT = TILE + XTRA;
  static constexpr int NSLOT = 2;            // per operand (Q, dO)
  static constexpr int A0_OFF = 0;
  static constexpr int A1_OFF = TILE;
  static constexpr int ONES_OFF = 2 * TILE;
  static constexpr int Q_OFF = ONES_OFF + XTRA;
  static constexpr int DO_OFF = Q_OFF + NSLOT * SLOT;
  static constexpr int BAR_OFF = DO_OFF + NSLOT * SLOT;
  // B_S0 / B_S1: query columns 0-63 / 64-127 of S^T in TMEM region A; B_DP: dP^T in
  // region B; B_P0 / B_P1: P^T of those columns written back by the four warps that
  // own them; B_DS: dS^T written back by all eight.
  static constexpr int B_RES = 0, B_QFULL = 1, B_QEMPTY = 3, B_OFULL = 5, B_OEMPTY = 7, B_S0 = 9,
                       B_S1 = 10, B_DP = 11, B_P0 = 12, B_P1 = 13, B_DS = 14, B_ACC = 15, B_DRAIN = 16,
                       NBARS = 17;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int SMEM = MISC_OFF + 64;
  // TMEM columns: region A (S^T, then packed P^T), region B (dP^T, then packed
  // dS^T), the dV and dK accumulators.
  static constexpr int TM_A = 0, TM_B = 128, TM_DV = 256, TM_DK = 256 + D;
  static_assert(Q_OFF % 1024 == 0 && SLOT % 1024 == 0, "swizzled tiles stay 1024-aligned");
  static_assert(1024 + SMEM <= 232448, "fits in shared memory");
};

// Shared memory of the dQ kernel: resident Q_i (A0) and dO_i (A1); three K slots
// and two V slots.
template <int D>
struct DqLayout {
  static constexpr int TILE = kTile * D * 2;
  static constexpr int CHUNK = kTile * 128;
  static constexpr int NK = 3, NV = 2;
  static constexpr int A0_OFF = 0;
  static constexpr int A1_OFF = TILE;
  static constexpr int K_OFF = 2 * TILE;
  static constexpr int V_OFF = K_OFF + NK * TILE;
  static constexpr int BAR_OFF = V_OFF + NV * TILE;
  // B_S / B_S1: S in TMEM region A / A'; B_DP: dP in region B; B_DS: dS written back.
  static constexpr int B_RES = 0, B_KFULL = 1, B_KEMPTY = 4, B_VFULL = 7, B_VEMPTY = 9, B_S = 11,
                       B_S1 = 12, B_DP = 13, B_DS = 14, B_ACC = 15, B_DRAIN = 16, NBARS = 17;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int SMEM = MISC_OFF + 64;
  // TMEM columns: region A (S), region B (dP, then packed dS), the dQ accumulator,
  // region A' (the second score buffer).
  static constexpr int TM_A = 0, TM_B = 128, TM_DQ = 256, TM_A2 = 256 + D;
  static_assert(TM_A2 + kTile <= 512, "A' fits in TMEM");
  static_assert(1024 + SMEM <= 232448, "fits in shared memory");
};

// Shared-memory matrix descriptor of a K-major operand without swizzling: core
// matrices of 8 rows x 16 bytes stored contiguously (128 bytes), lbo bytes between
// core matrices adjacent along K, sbo bytes between 8-row groups.
__device__ __forceinline__ uint64_t sdesc_kmajor_plain(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;  // descriptor version of this architecture; layout type 0 = no swizzle
  return d;
}
// Byte offset of row r's first core-matrix row in a 128 x 16 operand of that layout
// (lbo = 128, sbo = 256).
__device__ __forceinline__ uint32_t xtra_row_off(int r) { return (r & 7) * 16 + (r >> 3) * 256; }


// -x as three bf16 terms whose sum is -x to ~2^-24 relative (x = +inf: -inf, 0, 0),
// packed as the first four bf16 of an extra-step row: {t0, t1, t2, 0}.
__device__ __forceinline__ uint2 neg_split3(float x) {
  if (isinf(x)) return make_uint2(pack_bf16x2(-INFINITY, 0.f), 0u);
  const float y = -x;
  const float t0 = __bfloat162float(__float2bfloat16_rn(y));
  const float r1 = y - t0;
  const float t1 = __bfloat162float(__float2bfloat16_rn(r1));
  const float t2 = r1 - t1;
  return make_uint2(pack_bf16x2(t0, t1), pack_bf16x2(t2, 0.f));
}

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Pairs of exponentials (of every 8) computed on the FMA pipe by exp2_poly_x2
// instead of MUFU ex2 (the exponential split of the forward kernel).
#ifndef ATTN_BWD_POLY8
#define ATTN_BWD_POLY8 0
#endif
constexpr int kBwdPoly8 = ATTN_BWD_POLY8;
static_assert(kBwdPoly8 >= 0 && kBwdPoly8 <= 8, "pairs per 8");

// y <- 2^y for 64 log2-domain arguments, two at a time.  MUFU ex2 gives 0 for
// y = -inf; the polynomial clamps at 2^-125 (used only where such rows are masked
// or never stored).
__device__ __forceinline__ void exp2_cols(float (&y)[64]) {
#pragma unroll
  for (int c = 0; c < 64; c += 2) {
    if (((c >> 1) & 7) >= 8 - kBwdPoly8) {
      exp2_poly_x2(y[c], y[c + 1]);
    } else {
      y[c] = fast_exp2(y[c]);
      y[c + 1] = fast_exp2(y[c + 1]);
    }
  }
}

__device__ __forceinline__ int64_t vec_index(const BwdParams& p, int b, int h, int seq_start,
                                             int row) {
  return p.cu_seqlens == nullptr ? (static_cast<int64_t>(b) * p.H + h) * p.N + row
                                 : static_cast<int64_t>(h) * p.total + seq_start + row;
}

// Packed bf16 columns of a thread's 64-column half live in the first 32 TMEM
// columns of that half (so the two halves never write into each other's scores);
// the K-step kk of an MMA that reads them as its A operand starts here:
__device__ __forceinline__ uint32_t packed_col(int kk) { return (kk < 4) ? kk * 8 : 64 + (kk - 4) * 8; }

// Block -> (sequence, head, tile).  Blocks are dealt in groups of kBwdGroup
// (sequence, head) pairs, longest-first inside each group (for the key-tile kernel
// (causal) small tile indices have the most query tiles; for the query-tile
// kernel large indices have the most key tiles).  The CTAs running at any time
// then belong to a few heads, whose streamed tiles (4 MB per head at N = 8192,
// d = 128) stay in L2 while every CTA of the group reads them.
#ifndef ATTN_BWD_GROUP
#define ATTN_BWD_GROUP 8
#endif
constexpr int kBwdGroup = ATTN_BWD_GROUP;
struct BwdItem {
  int b, h, tile, seq_start, L;
};
// False when the CTA has no work.  Varlen: a sequence whose bounds fall outside
// [0, total) or whose length exceeds ntiles * 128 is not processed (its CTAs write
// nothing) and ATTN_ERR_INVALID_ARG is recorded in the device error word, as is
// cu[0] != 0 or cu[B] != total; so a malformed cu_seqlens never makes a store
// leave the packed tensors.
__device__ __forceinline__ bool decode_block(const BwdParams& p, bool key_tiles, bool causal,
                                             BwdItem& it) {
  const int nbh = p.B * p.H;
  const int idx = static_cast<int>(blockIdx.x);
  const int G = nbh < kBwdGroup ? nbh : kBwdGroup;
  const int grp = idx / (G * p.ntiles);
  const int gsize = min(G, nbh - grp * G);  // the last group may be smaller
  const int rem = idx - grp * G * p.ntiles;
  const int rank = rem / gsize, bh = grp * G + (rem - rank * gsize);
  it.b = bh / p.H;
  it.h = bh - it.b * p.H;
  it.tile = (causal && !key_tiles) ? p.ntiles - 1 - rank : rank;
  if (p.cu_seqlens == nullptr) {
    it.seq_start = it.b * p.N;
    it.L = p.N;
  } else {
    const int c0 = __ldg(p.cu_seqlens + it.b), c1 = __ldg(p.cu_seqlens + it.b + 1);
    const bool bad = c0 < 0 || c1 < c0 || c1 > p.total ||
                     static_cast<int64_t>(c1 - c0) > static_cast<int64_t>(p.ntiles) * kTile;
    const bool bad_ends = idx == 0 && (__ldg(p.cu_seqlens) != 0 || __ldg(p.cu_seqlens + p.B) != p.total);
    if (bad || bad_ends) {
      if (threadIdx.x == 0 && p.err) atomicCAS(p.err, 0, 1 | (kSiteBadLen << 8));
      if (bad) return false;
    }
    it.seq_start = c0;
    it.L = c1 - c0;
  }
  return it.tile * kTile < it.L;
}

__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
  return true;
}

// Stores a thread's half row (D/2 columns) of a TMEM accumulator as bf16, times mul.
template <int D>
__device__ __forceinline__ void store_half_row(uint32_t t_acc, __nv_bfloat16* dst, float mul,
                                               bool store) {
#pragma unroll
  for (int c = 0; c < D / 64; ++c) {
    uint32_t v[32];
    tmem_ld_x32(t_acc + 32 * c, v);
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      w[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * mul, __uint_as_float(v[2 * i + 1]) * mul);
    if (store) {
      uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
      for (int i = 0; i < 4; ++i) d4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
    }
  }
}

// Shared set-up of both main kernels: barriers (counts from `counts`, NB of them),
// TMEM (512 columns), abort flag.  Returns the TMEM base address.
template <int NB>
__device__ __forceinline__ uint32_t bwd_setup(uint8_t* smem, uint32_t sb, int bar_off, int misc_off,
                                              int warp, const uint8_t (&counts)[NB]) {
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + misc_off);
  if (threadIdx.x == 0) {
    for (int i = 0; i < NB; ++i) mbar_init(sb + bar_off + 8 * i, counts[i]);
    misc[1] = 0u;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(sb + misc_off, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  return misc[0];
}

// Arrive once per warp after this thread's TMEM stores are complete.
__device__ __forceinline__ void warp_release(uint32_t bar, int lane) {
  tmem_st_wait();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}

// ---------------------------------------------------------------------- D_i
// D_i = <dO_i, O_i> for every (token, head) row: HBM-bound (two bf16 rows read per
// float written).  A row is read by D/8 lanes with 16-byte loads and reduced by
// shuffles within those lanes; the grid strides over rows.
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                      const __nv_bfloat16* __restrict__ dout, BwdParams p) {
  constexpr int LPR = D / 8;        // lanes per row
  constexpr int RPW = 32 / LPR;     // rows per warp and step
  const int lane = threadIdx.x & 31;
  const int sub = lane % LPR;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t units = static_cast<int64_t>(p.total) * p.H;
  // The loop bound is uniform across the warp (every lane joins the shuffles).
  for (int64_t base = (static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5)) * RPW;
       base < units; base += warps * RPW) {
    const int64_t u = base + lane / LPR;
    const bool valid = u < units;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    const uint4 a = valid ? __ldg(reinterpret_cast<const uint4*>(o + u * D) + sub) : zero;
    const uint4 g = valid ? __ldg(reinterpret_cast<const uint4*>(dout + u * D) + sub) : zero;
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, gw[4] = {g.x, g.y, g.z, g.w};
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 af = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&aw[i]));
      const float2 gf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gw[i]));
      acc = fmaf(af.x, gf.x, acc);
      acc = fmaf(af.y, gf.y, acc);
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (valid && sub == 0) {
      const int64_t tok = u / p.H;
      const int h = static_cast<int>(u - tok * p.H);
      int64_t idx;
      if (p.cu_seqlens == nullptr) {
        const int b = static_cast<int>(tok / p.N);
        idx = (static_cast<int64_t>(b) * p.H + h) * p.N + (tok - static_cast<int64_t>(b) * p.N);
      } else {
        idx = static_cast<int64_t>(h) * p.total + tok;
      }
      p.dpre[idx] = acc;
    }
  }
}

// ------------------------------------------------------------------ dK, dV
// CTA: key tile j of (b, h).  Resident: K_j (A0), V_j (A1).  Streamed: Q_i, dO_i.
// Per query tile i (extra K-step: see the file comment):
//   S'^T = K_j Q_i^T - LSE_i/scale (TMEM A), dP'^T = V_j dO_i^T - D_i (TMEM B);
//   P^T = exp2(scale*log2e * S'^T) (causal: zero where query < key) -> A;
//   dV += P^T dO_i;  dS^T = P^T o dP'^T -> B;  dK += dS^T Q_i.
// MASK: 0 none, 1 causal, 2 sliding window (see BwdParams::wl, wr).
template <int D, int MASK>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const BwdParams p) {
  using Lay = DkdvLayout<D>;
  // The dQ kernel that follows reads nothing this kernel writes: let it be
  // scheduled onto SMs as they free up in this grid's last wave.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  BwdItem it;
  constexpr bool CAUSAL = MASK == 1;
  if (!decode_block(p, true, CAUSAL, it)) return;  // uniform for the CTA
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + Lay::BAR_OFF + 8 * i; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // The extra-step operands: ONES = {1, 1, 1, 0, ...} in every row; the slots'
  // operands are zero beyond their first four columns (the producer writes only
  // those).
  {
    uint4* z = reinterpret_cast<uint4*>(smem + Lay::ONES_OFF);
    const uint32_t one2 = pack_bf16x2(1.f, 1.f), one0 = pack_bf16x2(1.f, 0.f);
    for (int u = threadIdx.x; u < Lay::XTRA / 16; u += kThreads) {
      // 16-byte unit u: core-matrix row (u & 7) of row group (u >> 4); units with
      // bit 3 set hold K columns 8..15
      z[u] = ((u >> 3) & 1) ? make_uint4(0u, 0u, 0u, 0u) : make_uint4(one2, one0, 0u, 0u);
    }
    for (int s2 = 0; s2 < 2 * Lay::NSLOT; ++s2) {
      uint4* x = reinterpret_cast<uint4*>(smem + Lay::Q_OFF + s2 * Lay::SLOT + Lay::TILE);
      for (int u = threadIdx.x; u < Lay::XTRA / 16; u += kThreads) x[u] = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
  }
  const uint8_t counts[Lay::NBARS] = {1, 2, 2, 1, 1, 2, 2, 1, 1, 1, 1, 1, 4, 4, 8, 1, 1};
  const uint32_t tmem = bwd_setup<Lay::NBARS>(smem, sb, Lay::BAR_OFF, Lay::MISC_OFF, warp, counts);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Lay::MISC_OFF);
  WaitCtl wc;
  wc.abort = reinterpret_cast<volatile uint32_t*>(misc + 1);
  wc.err = p.err;
  wc.limit_ns = p.timeout_ns;

  const int j = it.tile;
  const int ntiles = ceil_div(it.L, kTile);
  // Query tiles that see some key of this tile: causal from the diagonal on; a
  // window from key - wr to key + wl.
  int i_first = CAUSAL ? j : 0, i_end = ntiles;
  if (MASK == 2) {
    i_first = max(j * kTile - p.wr, 0) / kTile;
    i_end = min(ntiles, (j * kTile + kTile - 1 + p.wl) / kTile + 1);
  }
  const int nq = i_end - i_first;
  auto q_slot = [&](int n) -> uint32_t { return sb + Lay::Q_OFF + (n & 1) * Lay::SLOT; };
  auto o_slot = [&](int n) -> uint32_t { return sb + Lay::DO_OFF + (n & 1) * Lay::SLOT; };

  if (warp < 8) {
    // ---------------------------------------------------- elementwise work
    const int hf = warp >> 2, wq = warp & 3;
    const int r = wq * 32 + lane;  // key row within the tile
    const int key = j * kTile + r;
    const uint32_t lane_bits = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tA = tmem + lane_bits + Lay::TM_A + 64 * hf;
    const uint32_t tB = tmem + lane_bits + Lay::TM_B + 64 * hf;
    const float sl = p.scale_log2;
    uint32_t s_phase = 0, dp_phase = 0;
    bool ok = true;
    for (int n = 0; n < nq && ok; ++n) {
      const int i = i_first + n;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_S0 + hf), s_phase, wc, timeout_code(kSiteS)));
      if (!ok) break;
      s_phase ^= 1u;
      tc_fence_after();
      uint32_t sv[64];
      tmem_ld_x64(tA, sv);
      // P^T for this thread's 64 query columns (causal diagonal tile: a query
      // sees the key only if query >= key).  Window: query q = qb + c sees this
      // key iff key - wr <= q <= key + wl.
      int lim = (CAUSAL && i == j) ? r - 64 * hf : -1;  // columns < lim are masked
      int lim_hi = 64;                                   // columns > lim_hi are masked
      if (MASK == 2) {
        const int qb = i * kTile + 64 * hf;
        lim = key - p.wr - qb;
        lim_hi = key + p.wl - qb;
      }
      float pv[64];
#pragma unroll
      for (int c = 0; c < 64; c += 2)
        fmul2_bc(pv[c], pv[c + 1], __uint_as_float(sv[c]), __uint_as_float(sv[c + 1]), sl);
      exp2_cols(pv);
      // Only the diagonal tile (causal) and the window's edge tiles mask columns.
      if (__any_sync(0xffffffffu, lim > 0 || (MASK == 2 && lim_hi < 63))) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c < lim || (MASK == 2 && c > lim_hi)) pv[c] = 0.f;
      }
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) pk[c] = pack_bf16x2(pv[2 * c], pv[2 * c + 1]);
      tmem_st_x32(tA, pk);
      warp_release(bar(Lay::B_P0 + hf), lane);
      ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_DP), dp_phase, wc, timeout_code(kSiteS)));
      if (!ok) break;
      dp_phase ^= 1u;
      tc_fence_after();
      // dS^T = P^T o (dP^T - D) (the subtraction done by the tensor core).
      {
        uint32_t dv[64];
        tmem_ld_x64(tB, dv);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          float d0, d1;
          ffma2_vb(d0, d1, __uint_as_float(dv[2 * c]), __uint_as_float(dv[2 * c + 1]), pv[2 * c],
                   pv[2 * c + 1], 0.f);
          pk[c] = pack_bf16x2(d0, d1);
        }
      }
      tmem_st_x32(tB, pk);
      warp_release(bar(Lay::B_DS), lane);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_ACC), 0, wc, timeout_code(kSiteAcc)));
    if (ok) {
      tc_fence_after();
      const bool store = key < it.L;
      const int64_t row = (static_cast<int64_t>(it.seq_start + key) * p.H + it.h) * D + (D / 2) * hf;
      const uint32_t t_dv = tmem + lane_bits + Lay::TM_DV + (D / 2) * hf;
      const uint32_t t_dk = tmem + lane_bits + Lay::TM_DK + (D / 2) * hf;
      store_half_row<D>(t_dv, p.dv + row, 1.f, store);
      store_half_row<D>(t_dk, p.dk + row, p.scale, store);
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ producer
    const uint64_t pol_res = l2_policy_evict_first();
    const uint64_t pol_ring = l2_policy_evict_last();
    if (elect_one()) {
      mbar_arrive_expect_tx(bar(Lay::B_RES), 2 * Lay::TILE);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(sb + Lay::A0_OFF + c * Lay::CHUNK, &tm_k, bar(Lay::B_RES), c * 64, it.h,
                    it.seq_start + j * kTile, pol_res);
        tma_load_3d(sb + Lay::A1_OFF + c * Lay::CHUNK, &tm_v, bar(Lay::B_RES), c * 64, it.h,
                    it.seq_start + j * kTile, pol_res);
      }
    }
    __syncwarp();
    const float l_to_s = kLog2e / p.scale_log2;  // LSE -> the same units as K Q^T (1/scale)
    bool ok = true;
    for (int n = 0; n < nq && ok; ++n) {
      const int i = i_first + n;
      // The extra-step rows of this query tile: lane l writes rows 4l..4l+3 (read
      // into registers before the slots are free, so the latency overlaps the waits).
      uint2 xl[4], xd[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int qrow = i * kTile + 4 * lane + u;
        const bool in = qrow < it.L;
        const int64_t vi = vec_index(p, it.b, it.h, it.seq_start, in ? qrow : 0);
        xl[u] = neg_split3(in ? __ldg(p.lse + vi) * l_to_s : INFINITY);
        xd[u] = neg_split3(in ? __ldg(p.dpre + vi) : 0.f);
      }
      // Each slot's barrier counts two arrivals: the copies' (with their bytes)
      // and the warp's, after it has written the extra-step rows.
      auto fill = [&](uint32_t slot, uint32_t full, const CUtensorMap* tm, const uint2 (&x)[4]) {
        if (elect_one()) {
          mbar_arrive_expect_tx(full, Lay::TILE);
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(slot + c * Lay::CHUNK, tm, full, c * 64, it.h, it.seq_start + i * kTile, pol_ring);
        }
        uint8_t* xs = smem + (slot - sb) + Lay::TILE;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          *reinterpret_cast<uint2*>(xs + xtra_row_off(4 * lane + u)) = x[u];
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(full);
      };
      const int sl2 = n & 1;
      if (n >= Lay::NSLOT) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_QEMPTY + sl2), ((n >> 1) - 1) & 1u, wc,
                                               timeout_code(kSiteStageEmpty)));
        if (!ok) break;
      }
      fill(q_slot(n), bar(Lay::B_QFULL + sl2), &tm_q, xl);
      if (n >= Lay::NSLOT) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_OEMPTY + sl2), ((n >> 1) - 1) & 1u, wc,
                                               timeout_code(kSiteStageEmpty)));
        if (!ok) break;
      }
      fill(o_slot(n), bar(Lay::B_OFULL + sl2), &tm_do, xd);
    }
    // Drain: copies still in flight must land before the CTA exits.
    drain_wait(bar(Lay::B_RES), 0u, kDrainLimitNs);
    for (int n = (nq > Lay::NSLOT ? nq - Lay::NSLOT : 0); n < nq; ++n) {
      drain_wait(bar(Lay::B_QFULL + (n & 1)), (n >> 1) & 1u, kDrainLimitNs);
      drain_wait(bar(Lay::B_OFULL + (n & 1)), (n >> 1) & 1u, kDrainLimitNs);
    }
  } else {
    // ---------------------------------------------------------------- MMA
    // Each product's K-steps are issued back to back by one elected lane, with
    // descriptors built once and advanced by compile-time offsets.
    constexpr uint32_t idesc_s = idesc_bf16_f32(kTile, kTile, 0, 0);
    constexpr uint32_t idesc_h = idesc_bf16_f32(kTile, kTile / 2, 0, 0);
    constexpr uint32_t idesc_acc = idesc_bf16_f32(kTile, D, 0, 1);
    const uint32_t tA = tmem + Lay::TM_A, tB = tmem + Lay::TM_B;
    const uint32_t tdV = tmem + Lay::TM_DV, tdK = tmem + Lay::TM_DK;
    const uint64_t ones = sdesc_kmajor_plain(sb + Lay::ONES_OFF, 128, 256);
    const uint64_t dK0 = sdesc_sw128(sb + Lay::A0_OFF, 16, 1024), dV0 = sdesc_sw128(sb + Lay::A1_OFF, 16, 1024);
    bool ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_RES), 0, wc, timeout_code(kSiteKv)));
    uint32_t p_phase = 0, ds_phase = 0;
    auto wait_full = [&](int b0, int n) -> bool {
      const bool r = __all_sync(0xffffffffu, mbar_wait(bar(b0 + (n & 1)), (n >> 1) & 1u, wc,
                                                       timeout_code(kSiteStageFull)));
      if (r) tc_fence_after();
      return r;
    };
    // t = A (K_j or V_j, K-major) times the streamed tile's transpose (K-major), plus
    // the extra step, into TMEM region t; commit to `done`.
    auto issue_score = [&](uint32_t t, uint64_t a0, uint32_t slot, uint32_t done) {
      if (elect_one()) {
        const uint64_t b0 = sdesc_sw128(slot, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * Lay::CHUNK + (kk & 3) * 32;
          mma_ss(t, desc_add(a0, off), desc_add(b0, off), idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_ss(t, ones, sdesc_kmajor_plain(slot + Lay::TILE, 128, 256), idesc_s, 1u);
        tc_commit(done);
      }
      __syncwarp();
    };
    // S^T for query columns 64h..64h+63 only (N = 64): rows 64h.. of the Q slot and
    // of its extra-step operand, into TMEM columns 64h..; commit to B_S0 + h.
    auto issue_st_half = [&](int h, uint32_t slot) {
      if (elect_one()) {
        const uint64_t b0 = sdesc_sw128(slot + h * 64 * 128, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * Lay::CHUNK + (kk & 3) * 32;
          mma_ss(tA + 64 * h, desc_add(dK0, off), desc_add(b0, off), idesc_h, kk > 0 ? 1u : 0u);
        }
        mma_ss(tA + 64 * h, ones, sdesc_kmajor_plain(slot + Lay::TILE + h * 8 * 256, 128, 256), idesc_h, 1u);
        tc_commit(bar(Lay::B_S0 + h));
      }
      __syncwarp();
    };
    // dV += the P^T columns of half h (K steps 4h..4h+3) times dO (MN-major).
    auto issue_dv_half = [&](int h, uint32_t slot, bool first) {
      if (elect_one()) {
        const uint64_t b0 = sdesc_sw128(slot, Lay::CHUNK, 1024);
#pragma unroll
        for (int kk = 4 * h; kk < 4 * h + 4; ++kk)
          mma_ts(tdV, tA + packed_col(kk), desc_add(b0, kk * 2048), idesc_acc, (!first || kk > 0) ? 1u : 0u);
      }
      __syncwarp();
    };
    // acc += (packed bf16 from TMEM region ta) times the streamed tile (MN-major);
    // commit to `done` (the tile's slot is then free).
    auto issue_acc = [&](uint32_t acc, uint32_t ta, uint32_t slot, bool first, uint32_t done) {
      if (elect_one()) {
        const uint64_t b0 = sdesc_sw128(slot, Lay::CHUNK, 1024);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          mma_ts(acc, ta + packed_col(kk), desc_add(b0, kk * 2048), idesc_acc, (!first || kk > 0) ? 1u : 0u);
        tc_commit(done);
      }
      __syncwarp();
    };
    // Software pipeline over query tiles: per tile n the tensor pipe runs
    //   dV(n), S^T(n+1), dK(n), dP^T(n+1)
    // so the elementwise work on tile n+1 (exponentials) overlaps dK(n) and
    // dP^T(n+1), and dS of tile n overlaps dV(n) and S^T(n+1).  dV and S^T are
    // issued in two halves of 64 query columns, each half as soon as the four warps
    // that own those columns release them, so half the exponentials of tile n+1
    // start while the other half of S^T(n+1) is still being computed.  Region A is
    // rewritten by S^T(n+1) only after dV(n) has read P^T(n) (one issuing thread:
    // in order), region B by dP^T(n+1) only after dK(n) has read dS^T(n).  dO(n)'s
    // slot is released after dV(n), Q(n)'s after dK(n).
    if (ok && nq > 0) {
      ok = wait_full(Lay::B_QFULL, 0);
      if (ok) {
        issue_st_half(0, q_slot(0));
        issue_st_half(1, q_slot(0));
      }
      if (ok) ok = wait_full(Lay::B_OFULL, 0);
      if (ok) issue_score(tB, dV0, o_slot(0), bar(Lay::B_DP));
    }
    for (int n = 0; n < nq && ok; ++n) {
      const int sl2 = n & 1;
      // dV += P^T dO (A = P^T from TMEM, B = dO MN-major), half by half.
#pragma unroll
      for (int h = 0; h < 2 && ok; ++h) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_P0 + h), p_phase, wc, timeout_code(kSiteP)));
        if (!ok) break;
        tc_fence_after();
        issue_dv_half(h, o_slot(n), n == 0);
      }
      if (!ok) break;
      p_phase ^= 1u;
      if (elect_one()) tc_commit(bar(Lay::B_OEMPTY + sl2));
      __syncwarp();
      if (n + 1 < nq) {
        ok = wait_full(Lay::B_QFULL, n + 1);
        if (!ok) break;
        issue_st_half(0, q_slot(n + 1));
        issue_st_half(1, q_slot(n + 1));
      }
      // dK += dS^T Q (A = dS^T from TMEM, B = Q MN-major); scale applied at the end.
      ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_DS), ds_phase, wc, timeout_code(kSiteDs)));
      if (!ok) break;
      ds_phase ^= 1u;
      tc_fence_after();
      issue_acc(tdK, tB, q_slot(n), n == 0, bar(Lay::B_QEMPTY + sl2));
      if (n + 1 < nq) {
        ok = wait_full(Lay::B_OFULL, n + 1);
        if (!ok) break;
        issue_score(tB, dV0, o_slot(n + 1), bar(Lay::B_DP));
      }
    }
    if (elect_one()) {
      if (ok) tc_commit(bar(Lay::B_ACC));
      tc_commit(bar(Lay::B_DRAIN));
    }
    __syncwarp();
    if (!__all_sync(0xffffffffu, drain_wait(bar(Lay::B_DRAIN), 0u, kDrainLimitNs)) && lane == 0 && p.err)
      atomicCAS(p.err, 0, timeout_code(kSiteDrain));
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, 512);
}

// ----------------------------------------------------------------------- dQ
// CTA: query tile i of (b, h).  Resident: Q_i (A0), dO_i (A1).  Streamed: K_j, V_j.
// Per key tile j:  S = Q_i K_j^T (TMEM A or A'), dP = dO_i V_j^T (TMEM B);
//   P = exp2(scale*log2e*S - LSE2_row) (causal: zero where key > query);
//   dS = P o (dP - D_row) -> B;  dQ += dS K_j.  dQ is scaled at the end.
template <int D, int MASK>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const BwdParams p) {
  using Lay = DqLayout<D>;
  BwdItem it;
  constexpr bool CAUSAL = MASK == 1;
  if (!decode_block(p, false, CAUSAL, it)) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    return;
  }  // uniform for the CTA
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + Lay::BAR_OFF + 8 * i; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint8_t counts[Lay::NBARS] = {1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 8, 1, 1};
  const uint32_t tmem = bwd_setup<Lay::NBARS>(smem, sb, Lay::BAR_OFF, Lay::MISC_OFF, warp, counts);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Lay::MISC_OFF);
  WaitCtl wc;
  wc.abort = reinterpret_cast<volatile uint32_t*>(misc + 1);
  wc.err = p.err;
  wc.limit_ns = p.timeout_ns;

  const int i = it.tile;
  const int ntiles = ceil_div(it.L, kTile);
  // Key tiles [j_first, j_first + nk) holding a key some row of this tile sees.
  int j_first = 0, j_end = CAUSAL ? (i + 1 < ntiles ? i + 1 : ntiles) : ntiles;
  if (MASK == 2) {
    j_first = max(i * kTile - p.wl, 0) / kTile;
    j_end = min(ntiles, ceil_div(i * kTile + kTile + p.wr, kTile));
  }
  const int nk = j_end - j_first;
  auto k_slot = [&](int j) -> uint32_t { return sb + Lay::K_OFF + (j % Lay::NK) * Lay::TILE; };
  auto v_slot = [&](int j) -> uint32_t { return sb + Lay::V_OFF + (j % Lay::NV) * Lay::TILE; };
  if (warp < 8) {
    const int hf = warp >> 2, wq = warp & 3;
    const int r = wq * 32 + lane;
    const int q_row = i * kTile + r;
    const uint32_t lane_bits = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tA0 = tmem + lane_bits + Lay::TM_A + 64 * hf;
    const uint32_t tA1 = tmem + lane_bits + Lay::TM_A2 + 64 * hf;
    const uint32_t tB = tmem + lane_bits + Lay::TM_B + 64 * hf;
    const float sl = p.scale_log2;
    const bool in = q_row < it.L;
    const int64_t vi = vec_index(p, it.b, it.h, it.seq_start, in ? q_row : 0);
    const float lse2 = in ? __ldg(p.lse + vi) * kLog2e : INFINITY;
    const float dd = in ? __ldg(p.dpre + vi) : 0.f;
    uint32_t dp_phase = 0;
    bool ok = true;
    for (int j = 0; j < nk && ok; ++j) {
      // S of key tile j is in region A (j even) or A' (j odd); each buffer's
      // barrier completes once per two tiles.
      const int sb2 = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(sb2 ? Lay::B_S1 : Lay::B_S), (j >> 1) & 1u, wc,
                                             timeout_code(kSiteS)));
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[64];
      tmem_ld_x64(sb2 ? tA1 : tA0, sv);
      // keys visible to this row: key < L, (causal) key <= q_row, (window)
      // q_row - wl <= key <= q_row + wr
      const int kb = (j_first + j) * kTile + 64 * hf;
      int lim = it.L - kb, lim_lo = 0;
      if (CAUSAL && q_row - kb + 1 < lim) lim = q_row - kb + 1;
      if (MASK == 2) {
        lim = min(lim, q_row + p.wr + 1 - kb);
        lim_lo = q_row - p.wl - kb;
      }
      float pv[64];
#pragma unroll
      for (int c = 0; c < 64; c += 2)
        ffma2_bc(pv[c], pv[c + 1], __uint_as_float(sv[c]), __uint_as_float(sv[c + 1]), sl, -lse2);
      exp2_cols(pv);
      if (__any_sync(0xffffffffu, lim < 64 || (MASK == 2 && lim_lo > 0))) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (!(c < lim && (MASK != 2 || c >= lim_lo))) pv[c] = 0.f;
      }
      ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_DP), dp_phase, wc, timeout_code(kSiteS)));
      if (!ok) break;
      dp_phase ^= 1u;
      tc_fence_after();
      uint32_t pk[32];
      {
        uint32_t dv[64];
        tmem_ld_x64(tB, dv);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          float d0, d1;
          fsub2_bc(d0, d1, __uint_as_float(dv[2 * c]), __uint_as_float(dv[2 * c + 1]), dd);
          ffma2_vb(d0, d1, d0, d1, pv[2 * c], pv[2 * c + 1], 0.f);
          pk[c] = pack_bf16x2(d0, d1);
        }
      }
      tmem_st_x32(tB, pk);
      warp_release(bar(Lay::B_DS), lane);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_ACC), 0, wc, timeout_code(kSiteAcc)));
    if (ok) {
      tc_fence_after();
      const int64_t row = (static_cast<int64_t>(it.seq_start + q_row) * p.H + it.h) * D + (D / 2) * hf;
      store_half_row<D>(tmem + lane_bits + Lay::TM_DQ + (D / 2) * hf, p.dq + row, p.scale, in);
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ producer
    const uint64_t pol_res = l2_policy_evict_first();
    const uint64_t pol_ring = l2_policy_evict_last();
    if (elect_one()) {
      mbar_arrive_expect_tx(bar(Lay::B_RES), 2 * Lay::TILE);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(sb + Lay::A0_OFF + c * Lay::CHUNK, &tm_q, bar(Lay::B_RES), c * 64, it.h,
                    it.seq_start + i * kTile, pol_res);
        tma_load_3d(sb + Lay::A1_OFF + c * Lay::CHUNK, &tm_do, bar(Lay::B_RES), c * 64, it.h,
                    it.seq_start + i * kTile, pol_res);
      }
    }
    __syncwarp();
    auto load = [&](uint32_t slot, uint32_t full, const CUtensorMap* tm, int j) {
      if (elect_one()) {
        mbar_arrive_expect_tx(full, Lay::TILE);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(slot + c * Lay::CHUNK, tm, full, c * 64, it.h, it.seq_start + (j_first + j) * kTile,
                      pol_ring);
      }
      __syncwarp();
    };
    bool ok = true;
    for (int j = 0; j < nk && ok; ++j) {
      const int ks = j % Lay::NK, vs = j % Lay::NV;
      if (j >= Lay::NK) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_KEMPTY + ks), ((j / Lay::NK) - 1) & 1u, wc,
                                               timeout_code(kSiteStageEmpty)));
        if (!ok) break;
      }
      load(k_slot(j), bar(Lay::B_KFULL + ks), &tm_k, j);
      if (j >= Lay::NV) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_VEMPTY + vs), ((j / Lay::NV) - 1) & 1u, wc,
                                               timeout_code(kSiteStageEmpty)));
        if (!ok) break;
      }
      load(v_slot(j), bar(Lay::B_VFULL + vs), &tm_v, j);
    }
    drain_wait(bar(Lay::B_RES), 0u, kDrainLimitNs);
    for (int j = (nk > Lay::NK ? nk - Lay::NK : 0); j < nk; ++j)
      drain_wait(bar(Lay::B_KFULL + j % Lay::NK), (j / Lay::NK) & 1u, kDrainLimitNs);
    for (int j = (nk > Lay::NV ? nk - Lay::NV : 0); j < nk; ++j)
      drain_wait(bar(Lay::B_VFULL + j % Lay::NV), (j / Lay::NV) & 1u, kDrainLimitNs);
  } else {
    // ---------------------------------------------------------------- MMA
    constexpr uint32_t idesc_s = idesc_bf16_f32(kTile, kTile, 0, 0);
    constexpr uint32_t idesc_acc = idesc_bf16_f32(kTile, D, 0, 1);
    const uint32_t tB = tmem + Lay::TM_B, tdQ = tmem + Lay::TM_DQ;
    const uint64_t dQ0 = sdesc_sw128(sb + Lay::A0_OFF, 16, 1024), dO0 = sdesc_sw128(sb + Lay::A1_OFF, 16, 1024);
    bool ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_RES), 0, wc, timeout_code(kSiteKv)));
    uint32_t ds_phase = 0;
    auto wait_k = [&](int j) -> bool {
      const bool r = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_KFULL + j % Lay::NK), (j / Lay::NK) & 1u,
                                                       wc, timeout_code(kSiteStageFull)));
      if (r) tc_fence_after();
      return r;
    };
    auto wait_v = [&](int j) -> bool {
      const bool r = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_VFULL + j % Lay::NV), (j / Lay::NV) & 1u,
                                                       wc, timeout_code(kSiteStageFull)));
      if (r) tc_fence_after();
      return r;
    };
    // t = A (Q_i or dO_i) times the streamed tile's transpose, both K-major, issued
    // back to back by one elected lane; commit to `done` (and `done2`, if given).
    auto issue_score = [&](uint32_t t, uint64_t a0, uint32_t slot, uint32_t done, uint32_t done2) {
      if (elect_one()) {
        const uint64_t b0 = sdesc_sw128(slot, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * Lay::CHUNK + (kk & 3) * 32;
          mma_ss(t, desc_add(a0, off), desc_add(b0, off), idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(done);
        if (done2 != 0u) tc_commit(done2);
      }
      __syncwarp();
    };
    // S = Q K_j^T into region A (j even) or A' (j odd).
    auto issue_s = [&](int j) {
      issue_score(tmem + ((j & 1) ? Lay::TM_A2 : Lay::TM_A), dQ0, k_slot(j), bar((j & 1) ? Lay::B_S1 : Lay::B_S),
                  0u);
    };
    // dP = dO V_j^T into region B, with its own commit; V_j's slot is then free.
    auto issue_dp = [&](int j) {
      issue_score(tB, dO0, v_slot(j), bar(Lay::B_DP), bar(Lay::B_VEMPTY + j % Lay::NV));
    };
    // Per key tile j the tensor pipe runs dQ(j), dP(j+1), S(j+2): S(j+1) is
    // already in the other score buffer, so the exponentials of tile j+1 start as
    // soon as dS(j) is released.  The elementwise warps read S(j) and dP(j) before
    // releasing dS(j), and one thread issues every MMA in order, so dP(j+1)
    // overwrites region B only after dQ(j) has read dS(j), and S(j+2) reuses S(j)'s
    // buffer only after that release.  K_j's slot is released after dQ(j).
    if (ok && nk > 0) {
      ok = wait_k(0);
      if (ok) issue_s(0);
      if (ok) ok = wait_v(0);
      if (ok) issue_dp(0);
      if (ok && nk > 1) {
        ok = wait_k(1);
        if (ok) issue_s(1);
      }
    }
    for (int j = 0; j < nk && ok; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_DS), ds_phase, wc, timeout_code(kSiteDs)));
      if (!ok) break;
      ds_phase ^= 1u;
      tc_fence_after();
      // dQ += dS K (A = dS from TMEM, B = K MN-major).
      if (elect_one()) {
        const uint64_t b0 = sdesc_sw128(k_slot(j), Lay::CHUNK, 1024);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          mma_ts(tdQ, tB + packed_col(kk), desc_add(b0, kk * 2048), idesc_acc, (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar(Lay::B_KEMPTY + j % Lay::NK));
      }
      __syncwarp();
      if (j + 1 < nk) {
        ok = wait_v(j + 1);
        if (!ok) break;
        issue_dp(j + 1);
      }
      if (j + 2 < nk) {
        ok = wait_k(j + 2);
        if (!ok) break;
        issue_s(j + 2);
      }
    }
    if (elect_one()) {
      if (ok) tc_commit(bar(Lay::B_ACC));
      tc_commit(bar(Lay::B_DRAIN));
    }
    __syncwarp();
    if (!__all_sync(0xffffffffu, drain_wait(bar(Lay::B_DRAIN), 0u, kDrainLimitNs)) && lane == 0 && p.err)
      atomicCAS(p.err, 0, timeout_code(kSiteDrain));
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, 512);
  // Launched to overlap the dK/dV kernel's tail: finish only after that grid has
  // (its results are then visible to whatever the stream runs next).
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <int D, int MASK>
cudaError_t launch_main(const BwdLaunch& a, cudaStream_t st) {
  const int smem1 = 1024 + DkdvLayout<D>::SMEM;
  const int smem2 = 1024 + DqLayout<D>::SMEM;
  auto k1 = bwd_dkdv_kernel<D, MASK>;
  auto k2 = bwd_dq_kernel<D, MASK>;
  cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, smem1);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2);
  if (e != cudaSuccess) return e;
  k1<<<a.grid, kThreads, smem1, st>>>(a.tm_q, a.tm_k, a.tm_v, a.tm_do, a.p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = a.grid;
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem2;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k2, a.tm_q, a.tm_k, a.tm_v, a.tm_do, a.p);
}

}  // namespace

cudaError_t launch_bwd(const BwdLaunch& a, const void* o, const void* dout, int D, int mask,
                       cudaStream_t st) {
  const int64_t units = static_cast<int64_t>(a.p.total) * a.p.H;
  const int rows_per_block = 256 / (D / 8);  // 256 threads, D/8 lanes per row
  int64_t blocks = (units + rows_per_block - 1) / rows_per_block;
  if (blocks > 148 * 8) blocks = 148 * 8;  // 8 blocks of 256 threads per SM, grid-stride beyond
  if (blocks < 1) blocks = 1;
  if (D == 128)
    bwd_pre_kernel<128><<<static_cast<int>(blocks), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(o),
                                                                  static_cast<const __nv_bfloat16*>(dout), a.p);
  else
    bwd_pre_kernel<64><<<static_cast<int>(blocks), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(o),
                                                                 static_cast<const __nv_bfloat16*>(dout), a.p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (D == 128) {
    if (mask == 2) return launch_main<128, 2>(a, st);
    return mask == 1 ? launch_main<128, 1>(a, st) : launch_main<128, 0>(a, st);
  }
  if (mask == 2) return launch_main<64, 2>(a, st);
  return mask == 1 ? launch_main<64, 1>(a, st) : launch_main<64, 0>(a, st);
}

}  // namespace attn
