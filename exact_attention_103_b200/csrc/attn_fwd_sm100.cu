// attn_fwd_sm100.cu -- fused exact-attention forward kernel for B200 (sm_100a).
//
// One persistent CTA per SM walks a static list of work items.  A work item is
// (sequence b, head h, query tile-pair t): 256 query rows split into two 128-row
// sub-tiles that share every K/V tile, so the tensor core alternates between the
// two sub-tiles while the other one's softmax runs ("FlashAttention V4 deep-dive"
// (pnsm.cn), section 3.1, two Q tiles in ping-pong).
//
// Warp roles (384 threads; warps 0-7 run with 192 registers, warps 8-11 with 120,
// moved by setmaxnreg after the set-up):
//   warps 0-3   softmax + epilogue of sub-tile 0 (one query row per thread)
//   warps 4-7   softmax + epilogue of sub-tile 1
//   warp  8     TMA producer: Q pair, then K_j / V_j tiles into an smem ring
//   warp  9     TMEM owner and tcgen05.mma issuer (whole warp; one elected lane
//               issues each instruction)
//   warps 10-11 no role: they complete warpgroup 2, whose registers go to 0-7
//
// Per sub-tile s and key tile j ("FlashAttention 1-4 详解", FlashAttention 1 /
// Online Softmax 数学推导; FlashAttention 2 / 减少非矩阵乘运算占比):
//   S_s = Q_s K_j^T                    tcgen05.mma, A and B from smem, fp32 in TMEM
//   m   = rowmax(scale*S) (log2 units) the row's own thread, from TMEM
//   conditional rescale: only when m exceeds the reference maximum by > tau
//       ("FlashAttention V4 deep-dive", section 3.2; "FlashAttention 1-4 详解",
//        FlashAttention 4 / 三项核心技术 (2)): O_s, l scaled by 2^(m_ref - m)
//   P~  = 2^(scale*S*log2e - m_ref)    MUFU ex2, or for POLY of every 8 column pairs
//       the FMA-pipe polynomial ("FlashAttention V4 deep-dive", section 3.2);
//       l += sum P~ (fp32, before rounding) -- the LSE's sum; the sum O is divided
//       by takes the same fp32 P~ on a full tile and, on a tile the mask cuts,
//       the bf16 P~ that the PV product uses (read back from TMEM; bf16 causal
//       kernels and d = 128 unmasked ones)
//   P~ -> bf16 (E4M3 on the 8-bit path), written back over S_s in TMEM in two
//       halves of 64 keys, each released to the MMA warp as soon as it is stored
//   O_s += P~ V_j                      tcgen05.mma, A = P~ from TMEM, B = V from smem,
//                                      issued per half of P~
// after the last key tile: O = O_s / (that second sum) -> bf16 -> global;
// LSE = ln2*(m_ref + log2 l).
// The mask hook (MaskFn below) decides which key tiles an item visits and which
// keys of a tile are hidden: causal items skip key tiles above the diagonal
// ("FlashAttention 1-4 详解", 其他优化 / FlashAttention 2 的工程优化) and mask the
// diagonal tile; sliding-window items skip tiles outside the window and mask its
// edges; packed variable-length batches mask keys past the sequence end.
//
// Scheduling ("FlashAttention V4 deep-dive", section 3.4 dynamic tile scheduling;
// FlashAttention-4 summary (reportify.cn) item [14], the new tile scheduler): a
// dynamic scheduler.  Items form one list; each CTA's producer warp claims the
// next list position from a device counter when it is ready for a new item and
// hands it to the CTA's other roles through a two-entry shared-memory queue, so
// CTAs that finish early take more work.  The list keeps the items of one
// (sequence, head) together (its K/V tiles stay in L2 while the CTAs that claimed
// its items stream them), longest sequences first, and puts its last groups in
// longest-item-first order so the final claims are the short items.
//
// TMEM columns: S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D, 256+2D).
// Every wait is bounded (see sm100_ptx.cuh); on expiry the CTA stops, drains
// its in-flight copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "attn_fwd_sm100.h"
#include "sm100_ptx.cuh"
#include "softmax_math.cuh"

namespace attn {

namespace {

constexpr int kThreads = 384;
constexpr int kBM = 128;  // query rows per sub-tile
constexpr int kBN = 128;  // keys per key tile
constexpr float kLn2 = 0.693147180559945309f;
// P~ of a key tile is handed to the PV product in this many parts of 128/kPSplit keys.
// Measured on B200 (same-box A/B): 2 is fastest; against 1, dense +6% and causal +1%;
// 4 costs 8% (four release round trips per tile outweigh the earlier start).
#ifndef ATTN_P_SPLIT
#define ATTN_P_SPLIT 2
#endif
constexpr int kPSplit = ATTN_P_SPLIT;
#ifndef ATTN_EARLY_PAIRS
#define ATTN_EARLY_PAIRS 8
#endif
constexpr int kEarlyPairs = ATTN_EARLY_PAIRS;
static_assert(kPSplit == 1 || kPSplit == 2 || kPSplit == 4, "P~ split");

// Error codes recorded in the device error word: 4 (= ATTN_ERR_TIMEOUT) in the
// low byte, the waiting site above it.
__host__ __device__ constexpr int timeout_code(int site) { return 4 | (site << 8); }
enum WaitSite {
  kSiteQEmpty = 1, kSiteKvEmpty, kSiteQFull, kSiteKvFull, kSitePFull, kSiteSFull, kSiteOFull,
  kSiteDrain, kSiteBadLen, kSiteItemFull, kSiteItemEmpty
};

// PAIR: a CTA pair runs tcgen05.mma.cta_group::2 (M = 256 rows per product, 128 in
// each CTA); each CTA keeps its own 128 query rows per sub-tile and half of every
// K/V tile (keys 64r..64r+63 of K, head-dim columns 64r..64r+63 of V for rank r),
// so a ring slot is half a tile.
template <int D, bool F8, bool PAIR = false>
struct Layout {
  static constexpr int ESZ = F8 ? 1 : 2;              // bytes per element (E4M3 / bf16)
  static constexpr int TILE = kBM * D * ESZ;          // bytes of one 128 x D tile
  static constexpr int CHUNK = kBM * 128;             // one 128-byte-wide swizzle chunk
  static constexpr int NCHUNK = TILE / CHUNK;
  static constexpr int KSTEP = 32 / ESZ;              // elements per MMA K step (32 bytes)
  static constexpr int SLOT = PAIR ? TILE / 2 : TILE; // bytes of one K/V ring slot
  static constexpr int NSTAGE = (SLOT <= 16384) ? 8 : 4;  // K/V ring slots
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = 2 * TILE;
  static constexpr int BAR_OFF = KV_OFF + NSTAGE * SLOT;
  // barrier indices
  // B_PFULL + kPSplit*s + h: part h of P~ of sub-tile s is in TMEM
  static constexpr int B_QFULL = 0, B_QEMPTY = 1, B_SFULL = 2, B_PFULL = 4,
                       B_OFULL = 4 + 2 * kPSplit, B_DRAIN = B_OFULL + 2, B_ITEMF = B_DRAIN + 1,
                       B_ITEME = B_ITEMF + 2, B_KVFULL = B_ITEME + 2, B_KVEMPTY = B_KVFULL + NSTAGE;
  static constexpr int NBARS = B_KVEMPTY + NSTAGE;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int TABLE_OFF = MISC_OFF + 64;
  static constexpr int TM_S0 = 0, TM_S1 = 128, TM_O0 = 256, TM_O1 = 256 + D;
};

// A work item: query rows [row_base, row_base + 2 * SUB) of one (sequence, head) as
// two sub-tiles of SUB rows (SUB = 128; a CTA pair: 256, 128 per CTA), or only the
// first sub-tile when `two` is false.
struct Item {
  int b, h, seq_start, L, row_base;
  bool two;
};

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// The work list, decoded identically by every role.  Groups are (sequence, head)
// pairs, sequences in list order (dense: b = 0..B-1; varlen: by tile-pair count,
// descending, stable), heads inside; group g has T_g items (256-row tile pairs).
//   bulk: groups [0, gtail), each group's items consecutive, t = T_g - 1 down to 0;
//   tail: groups [gtail, groups), t-major: for t from the largest T_g down to 0,
//         every tail group with T_g > t (the tail groups are sorted by T_g, so they
//         are a prefix of the tail).
// The tail holds the last groups covering at least two items per CTA, so the
// claims that end the launch are the shortest items.  Dense non-causal launches
// whose last wave would leave CTAs idle split their last `split` items into two
// 128-row half items each.
struct Sched {
  const int* cu;      // device cu_seqlens or null (dense)
  int B, H, T;        // T: tile pairs of the longest sequence
  int N;
  const int* order;   // varlen: sorted position -> sequence
  const int* gstart;  // varlen: first item of sorted sequence i (items of earlier sequences)
  const int* tstart;  // varlen tail: first tail item of level t (levels t' > t first)
  int pairs;          // 256-row items before any split
  int split;          // dense non-causal: the last `split` items become 2*split half items
  int count;          // number of list positions
  int nbulk;          // items in the bulk
  int gtail;          // first tail group
  int ishift;         // log2 of the query rows of an item (8: 256 rows; a CTA pair: 9)

  __device__ __forceinline__ int seq_T(int i, int& b, int& start, int& L) const {
    if (cu == nullptr) {
      b = i;
      start = i * N;
      L = N;
      return T;
    }
    b = order[i];
    start = __ldg(cu + b);
    L = __ldg(cu + b + 1) - start;
    return (L + (1 << ishift) - 1) >> ishift;
  }

  // SPLIT: the launch may hold half items (dense non-causal only).
  template <bool SPLIT>
  __device__ __forceinline__ Item decode(int idx) const {
    Item it;
    int sub = -1;  // >= 0: a half item made of sub-tile `sub` of its pair
    if (SPLIT && idx >= pairs - split) {
      const int u = idx - (pairs - split);
      idx = pairs - split + (u >> 1);
      sub = u & 1;
    }
    int g, t;  // group and tile pair
    if (idx < nbulk) {
      if (cu == nullptr) {
        g = idx / T;
        t = T - 1 - (idx - g * T);
      } else {
        int lo = 0, hi = B - 1;  // last sorted sequence with gstart <= idx
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (gstart[mid] <= idx) lo = mid; else hi = mid - 1;
        }
        int b, st, L;
        const int Ti = seq_T(lo, b, st, L);
        const int r = idx - gstart[lo];
        const int hh = r / Ti;
        g = lo * H + hh;
        t = Ti - 1 - (r - hh * Ti);
      }
    } else {
      const int u = idx - nbulk;
      if (cu == nullptr) {
        const int k = B * H - gtail;  // tail groups, all with T items
        const int lev = u / k;
        t = T - 1 - lev;
        g = gtail + (u - lev * k);
      } else {
        int lo = 0, hi = T - 1;  // smallest t with tstart[t] <= u
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (tstart[mid] <= u) hi = mid; else lo = mid + 1;
        }
        t = lo;
        g = gtail + (u - tstart[lo]);
      }
    }
    const int i = g / H;
    it.h = g - i * H;
    seq_T(i, it.b, it.seq_start, it.L);
    it.row_base = (t << ishift) + ((SPLIT && sub > 0) ? kBM : 0);
    it.two = !SPLIT || sub < 0;
    return it;
  }
};


// The mask hook, one compile-time functor per MaskKind.  For query rows of a
// sequence of length L:
//   tiles()   the key tiles [lo, hi) holding a key visible to some row of
//             [row0, row0 + nrows); the tiles outside are skipped, not loaded;
//   partial() whether key tile kb (its first key) may hide a key from some row of
//             the 128 rows [row0, row0 + 128);
//   cols()    the visible columns [c_lo, c_hi) of that tile for query row q.
// Causal is the lower triangle of "FlashAttention 1-4 详解", 其他优化 (tiles above
// the diagonal skipped).  The window is this library's instance of the
// FlexAttention mask interface ("FlashAttention V4 deep-dive", section 5):
// q - wl <= key <= q + wr.  A new mask is a new MaskKind with these three members.
template <int MASK>
struct MaskFn {
  int wl, wr;  // kMaskWindow only; both >= 0 and below 2^30
  __device__ __forceinline__ void tiles(int row0, int nrows, int L, int& lo, int& hi) const {
    const int all = ceil_div(L, kBN);
    lo = 0;
    hi = all;
    if (MASK == kMaskCausal) {
      hi = min((row0 + nrows - 1) / kBN + 1, all);  // up to and including the last row's diagonal tile
    } else if (MASK == kMaskWindow) {
      lo = max(row0 - wl, 0) / kBN;
      hi = ceil_div(min(row0 + nrows + wr, L), kBN);
    }
  }
  __device__ __forceinline__ bool partial(int kb, int row0, int L) const {
    if (kb + kBN > L) return true;
    if (MASK == kMaskCausal) return kb + kBN - 1 > row0;
    if (MASK == kMaskWindow) return kb < row0 + kBM - 1 - wl || kb + kBN - 1 > row0 + wr;
    return false;
  }
  __device__ __forceinline__ void cols(int q, int kb, int L, int& c_lo, int& c_hi) const {
    c_lo = 0;
    c_hi = L - kb;
    if (MASK == kMaskCausal) c_hi = min(c_hi, q - kb + 1);
    if (MASK == kMaskWindow) {
      c_lo = q - wl - kb;
      c_hi = min(c_hi, q + wr + 1 - kb);
    }
  }
};

// Key tiles [lo, hi) that sub-tile s (SUB rows) of an item processes (empty when
// its rows are all past L, or for the missing second sub-tile of a half item).
template <int MASK, int SUB = kBM>
__device__ __forceinline__ void kv_range(const Item& it, int s, const MaskFn<MASK>& mk, int& lo,
                                         int& hi) {
  lo = hi = 0;
  if (s == 1 && !it.two) return;
  const int row0 = it.row_base + s * SUB;
  if (row0 >= it.L) return;
  mk.tiles(row0, SUB, it.L, lo, hi);
}

// Key tiles of the whole item: the union of its sub-tiles' ranges (sub-tile 0 is
// never empty and its range starts no later than sub-tile 1's).
template <int MASK, int SUB = kBM>
__device__ __forceinline__ void item_range(const Item& it, const MaskFn<MASK>& mk, int& lo, int& n) {
  int lo0, hi0, lo1, hi1;
  kv_range<MASK, SUB>(it, 0, mk, lo0, hi0);
  kv_range<MASK, SUB>(it, 1, mk, lo1, hi1);
  lo = lo0;
  n = (hi1 > hi0 ? hi1 : hi0) - lo0;
}

// Inclusive warp scan (sum) of one value per lane.
__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// Varlen table layout in shared memory (ints):
//   order[B] | gstart[B+1] | off[T+1] | cnt[T+1] | tstart[T]
__host__ __device__ constexpr int varlen_table_ints(int B, int T) { return 2 * B + 3 * T + 3; }

// Builds the varlen list tables (one warp): sequences sorted by item count (items of
// 2^ishift query rows; descending, stable counting sort), the items before each
// sorted sequence, and
// the tail of the list (the last groups holding at least `tail_items` items, see
// Sched).  Writes gtail and nbulk; returns the number of items, or -1 if cu[0] !=
// 0, cu[B] != total, or some length is negative or exceeds T items.
__device__ int build_varlen_tables(const int* cu, int B, int H, int T, int total, int tail_items,
                                   int ishift, int* tab, int lane, int* gtail_out, int* nbulk_out) {
  auto items_of = [&](int L) { return (L + (1 << ishift) - 1) >> ishift; };
  int* order = tab;
  int* gstart = order + B;
  int* off = gstart + B + 1;
  int* cnt = off + T + 1;
  int* tstart = cnt + T + 1;
  for (int i = lane; i <= T; i += 32) off[i] = 0;
  __syncwarp();
  int bad = (lane == 0 && (__ldg(cu) != 0 || __ldg(cu + B) != total)) ? 1 : 0;
  for (int b = lane; b < B; b += 32) {
    const int L = __ldg(cu + b + 1) - __ldg(cu + b);
    const int nt = L < 0 ? 0 : items_of(L);
    if (L < 0 || nt > T) { bad = 1; continue; }
    atomicAdd(&off[nt], 1);
  }
  bad = __any_sync(0xffffffffu, bad);
  __syncwarp();
  if (bad) return -1;
  // off[n] = #{b : nt_b > n}: exclusive suffix scan of the histogram from n = T down.
  int carry = 0;
  for (int base = 0; base <= T; base += 32) {
    const int n = T - (base + lane);
    const int v = n >= 0 ? off[n] : 0;
    const int incl = warp_incl_scan(v, lane);
    __syncwarp();
    if (n >= 0) off[n] = carry + incl - v;
    carry += __shfl_sync(0xffffffffu, incl, 31);
    __syncwarp();
  }
  for (int t = lane; t <= T; t += 32) cnt[t] = off[t];
  __syncwarp();
  // Stable placement of sequences by tile-pair count, descending.
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int base = 0; base < B; base += 32) {
    const int b = base + lane;
    int key = -1;
    if (b < B) key = items_of(__ldg(cu + b + 1) - __ldg(cu + b));
    const uint32_t same = __match_any_sync(0xffffffffu, key);
    const int rank = __popc(same & lt_mask);
    if (b < B) order[off[key] + rank] = b;
    __syncwarp();
    if (b < B && lane == __ffs(same) - 1) off[key] += __popc(same);
    __syncwarp();
  }
  // gstart[i] = H * sum_{i' < i} nt(order[i']): exclusive prefix scan.
  carry = 0;
  for (int base = 0; base < B; base += 32) {
    const int i = base + lane;
    int v = 0;
    if (i < B) {
      const int b = order[i];
      v = H * items_of(__ldg(cu + b + 1) - __ldg(cu + b));
    }
    const int incl = warp_incl_scan(v, lane);
    if (i < B) gstart[i] = carry + incl - v;
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  const int items = carry;
  if (lane == 0) gstart[B] = items;
  __syncwarp();
  // The tail: the last groups (sorted sequence i0 from head h0 on, then every later
  // sequence) that hold at least tail_items items; everything when there are fewer.
  int i0 = 0, h0 = 0;
  if (items > tail_items) {
    int lo = 0, hi = B - 1;  // last sorted sequence with gstart <= items - tail_items
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (gstart[mid] <= items - tail_items) lo = mid; else hi = mid - 1;
    }
    i0 = lo;
    const int Ti = (gstart[i0 + 1] - gstart[i0]) / H;  // >= 1: empty sequences sort last
    const int rest = items - gstart[i0 + 1];
    h0 = H - ceil_div(tail_items - rest, Ti);
    if (h0 < 0) h0 = 0;
  }
  const int Ti0 = (gstart[i0 + 1] - gstart[i0]) / H;
  // n(t) = tail groups with more than t tile pairs; tstart[t] = sum_{t' > t} n(t').
  carry = 0;
  for (int base = 0; base < T; base += 32) {
    const int t = T - 1 - (base + lane);
    int v = 0;
    if (t >= 0) {
      const int later = cnt[t] - (i0 + 1);  // sorted sequences after i0 with nt > t
      v = H * (later > 0 ? later : 0) + (Ti0 > t ? H - h0 : 0);
    }
    const int incl = warp_incl_scan(v, lane);
    if (t >= 0) tstart[t] = carry + incl - v;
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  __syncwarp();
  *gtail_out = i0 * H + h0;
  *nbulk_out = gstart[i0] + h0 * Ti0;
  return items;
}

// Bounded wait that ignores the abort flag (used to drain before exit).
__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
  return true;
}

// POLY: of every 8 consecutive (even, odd) column pairs of a score row, this many
// are exponentiated on the FMA pipe by exp2_poly; the rest use MUFU ex2.
// F8: Q, K, V are E4M3 with per-tensor scales (S = Q K^T and O += P~ V with
// tcgen05.mma kind::f8f6f4, P~ rounded to E4M3; "FlashAttention 1-4 详解", 其他优化:
// FP8 tensor cores for the forward's matrix products).
// PAIR: the launch runs in clusters of two CTAs that share every item ("FlashAttention
// V4 deep-dive", section 3.3: 2-CTA MMA; FA-4 summary items [13][14]).  An item is
// 512 query rows, two sub-tiles of 256 rows with 128 in each CTA.  The leader (rank
// 0) claims items and issues every tcgen05.mma.cta_group::2 (M = 256) for both CTAs;
// each CTA loads its own query rows and half of each K/V tile (K by keys, V by
// head-dim columns) from this GPU's memory, with no multicast, so a CTA moves and
// stores half the K/V bytes of the single-CTA kernel; the softmax warps of both CTAs
// work on their own rows and release P~ to the leader.  tm_k2 views K with 64-row
// boxes (the K halves); it is unused otherwise.
template <int D, int MASK, int POLY, bool F8, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_k2,
               const __grid_constant__ CUtensorMap tm_o, const FwdParams p) {
  using Lay = Layout<D, F8, PAIR>;
  static_assert(!F8 || D == 128, "E4M3 path: one 128-byte row per head");
  static_assert(!PAIR || (D == 128 && !F8), "CTA pairs: bf16, d = 128");
  constexpr int NS = Lay::NSTAGE;
  constexpr bool SPLIT = MASK == kMaskNone && !PAIR;  // the launch may hold half items
  constexpr int SUB = PAIR ? 2 * kBM : kBM;            // query rows of a sub-tile (pair-wide)
  static_assert(POLY >= 0 && POLY <= 8, "pairs per 8");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sb + Lay::BAR_OFF + 8 * i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Lay::MISC_OFF);
  // misc[0] TMEM base, misc[1] abort flag, misc[2] items in the list, misc[3] first
  // tail group, misc[4] bulk items, misc[8 + e] list position in queue entry e
  volatile int* queue = reinterpret_cast<volatile int*>(misc + 8);
  int* tab = reinterpret_cast<int*>(smem + Lay::TABLE_OFF);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;  // 0: the pair's leader (or a lone CTA)
  const bool leader = rank == 0;
  // CTAs (pairs) that claim items; the list's tail holds two items per claimer.
  const int claimers = PAIR ? static_cast<int>(gridDim.x) / 2 : static_cast<int>(gridDim.x);
  const int tail_items = 2 * claimers;
  // The leader's copy of a barrier, as a shared::cluster address (pair mode).
  auto lbar = [&](int i) -> uint32_t { return PAIR ? mapa_shared(bar(i), 0) : bar(i); };

  if (threadIdx.x == 0) {
    mbar_init(bar(Lay::B_QFULL), 1);
    mbar_init(bar(Lay::B_QEMPTY), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(Lay::B_SFULL + s), 1);
      // the 4 softmax warps of the sub-tile (of both CTAs of a pair) release P~
      for (int h = 0; h < kPSplit; ++h) mbar_init(bar(Lay::B_PFULL + kPSplit * s + h), PAIR ? 8 : 4);
      mbar_init(bar(Lay::B_OFULL + s), 1);
      mbar_init(bar(Lay::B_ITEMF + s), 1);  // the producer publishes a claimed position
      // read by the MMA warp and the 8 softmax warps (a pair: and the follower's
      // producer and 8 softmax warps)
      mbar_init(bar(Lay::B_ITEME + s), PAIR ? 18 : 9);
    }
    mbar_init(bar(Lay::B_DRAIN), 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(bar(Lay::B_KVFULL + i), 1);
      mbar_init(bar(Lay::B_KVEMPTY + i), 1);
    }
    misc[1] = 0u;
    fence_barrier_init();
  }
  if (warp == 9) {
    if constexpr (PAIR) {
      tmem_alloc_pair(sb + Lay::MISC_OFF, 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(sb + Lay::MISC_OFF, 512);
      tmem_relinquish();
    }
  }
  if (warp == 8) {
    int count, gtail, nbulk;
    if (p.cu_seqlens == nullptr) {
      const int groups = p.B * p.H;
      int k = ceil_div(tail_items, p.T);
      if (k > groups) k = groups;
      count = groups * p.T;
      gtail = groups - k;
      nbulk = gtail * p.T;
    } else {
      count = build_varlen_tables(p.cu_seqlens, p.B, p.H, p.T, p.total, tail_items, PAIR ? 9 : 8, tab,
                                  lane, &gtail, &nbulk);
      if (count < 0) {
        count = gtail = nbulk = 0;
        if (lane == 0 && p.err) atomicCAS(p.err, 0, 1 | (kSiteBadLen << 8));
      }
    }
    if (lane == 0) {
      misc[2] = static_cast<uint32_t>(count);
      misc[3] = static_cast<uint32_t>(gtail);
      misc[4] = static_cast<uint32_t>(nbulk);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if constexpr (PAIR) {  // both CTAs' barriers exist before either arrives on the other's
    cluster_arrive();
    cluster_wait();
  }

  const uint32_t tmem = misc[0];
  Sched sch;
  sch.cu = p.cu_seqlens;
  sch.B = p.B; sch.H = p.H; sch.N = p.N; sch.T = p.T;
  sch.order = tab;
  sch.gstart = tab + p.B;
  sch.tstart = tab + 2 * p.B + 2 * p.T + 3;
  sch.pairs = static_cast<int>(misc[2]);
  sch.gtail = static_cast<int>(misc[3]);
  sch.nbulk = static_cast<int>(misc[4]);
  sch.ishift = PAIR ? 9 : 8;
  // Dense non-causal items all cost the same: when the last wave would leave
  // CTAs idle, its items are split into 128-row half items so it spreads over
  // more SMs (a half item runs without a ping-pong partner, but the wave is
  // shorter).  Causal and varlen lists end with their shortest items.
  sch.split = 0;
  if (SPLIT && p.cu_seqlens == nullptr) {
    const int rem = sch.pairs % claimers;
    if (rem > 0 && 2 * rem <= claimers) sch.split = rem;
  }
  sch.count = sch.pairs + sch.split;
  WaitCtl wc;
  wc.abort = reinterpret_cast<volatile uint32_t*>(misc + 1);
  wc.err = p.err;
  wc.limit_ns = p.timeout_ns;
  MaskFn<MASK> mk;
  mk.wl = p.wl;
  mk.wr = p.wr;
  // Consumer roles (the MMA warp, the softmax warps): the k-th list position this
  // CTA claimed, from the queue (one arrival per warp frees the entry); -1 ends
  // the list, and so does an expired wait.
  // In a pair every entry is published to both CTAs and freed on the leader.
  auto take_item = [&](int k) -> int {
    const int e = k & 1;
    if (!__all_sync(0xffffffffu, mbar_wait<PAIR>(bar(Lay::B_ITEMF + e), (k >> 1) & 1, wc,
                                                 timeout_code(kSiteItemFull))))
      return -1;
    const int idx = queue[e];
    __syncwarp();
    if (lane == 0) {
      if (PAIR && !leader) mbar_arrive_remote(lbar(Lay::B_ITEME + e));
      else mbar_arrive(bar(Lay::B_ITEME + e));
    }
    return idx;
  };

  // Registers move from warpgroup 2 (producer, MMA issuer, two idle warps) to the
  // two softmax warpgroups.  The launch gives every thread 168 (three warps share
  // each SM sub-partition); 4 x 32 x (168 - 120) = 6144 are released and
  // 8 x 32 x (192 - 168) = 6144 taken, so the increase always finds its registers.
  // Each warpgroup changes its budget at one instruction at the head of its
  // branch, so the code after it is compiled for the new budget.
  if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 192;\n" ::: "memory");
    // ------------------------------------------------------------ softmax
    // Sub-tile s = warp / 4; warp w owns TMEM lanes 32(w%4)..+31: one query row per
    // thread, all 128 key columns of each tile.
    const int s = warp >> 2, wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_bits = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t t_s = tmem + lane_bits + (s ? Lay::TM_S1 : Lay::TM_S0);
    const uint32_t t_o = tmem + lane_bits + (s ? Lay::TM_O1 : Lay::TM_O0);
    const float sl = p.scale_log2;
    uint32_t s_phase = 0, o_phase = 0;
    uint32_t n_rescale = 0, n_rowtiles = 0;  // this thread's row: < 2^32 tiles per launch
    for (int k = 0;; ++k) {
      const int idx = take_item(k);
      if (idx < 0) break;
      const Item it = sch.template decode<SPLIT>(idx);
      const int b = it.b, h = it.h, seq_start = it.seq_start, L = it.L;
      int jlo, jhi;  // the sub-tile's key tiles (of both CTAs of a pair)
      kv_range<MASK, SUB>(it, s, mk, jlo, jhi);
      if (jhi <= jlo) continue;
      const int row0 = it.row_base + s * SUB + static_cast<int>(rank) * kBM;  // this CTA's rows
      const int q_row = row0 + r;
      float m_ref = -INFINITY, l = 0.f, lr = 0.f;  // lr: the row sum O is divided by
      bool ok = true;
      for (int j = jlo; j < jhi; ++j) {
        ok = mbar_wait(bar(Lay::B_SFULL + s), s_phase, wc, timeout_code(kSiteSFull));
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        s_phase ^= 1u;
        tc_fence_after();
        // The score row in two halves: the second half's load is in flight while
        // the first half's maximum is taken.
        uint32_t sa[64], sz[64];
        tmem_ld_x64(t_s, sa);
        tmem_ld_x64_async(t_s + 64, sz);
        const int kb = j * kBN;
        const bool part = mk.partial(kb, row0, L);
        int c_lo = 0, c_hi = kBN;  // keys [kb + c_lo, kb + c_hi) are visible to this row
        if (part) {
          mk.cols(q_row, kb, L, c_lo, c_hi);
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c < c_lo || c >= c_hi) sa[c] = __float_as_uint(-INFINITY);
        }
        // Row maximum: four independent 3-input max chains, then a small tree.
        float m4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          m4[i] = fmax3(__uint_as_float(sa[i]), __uint_as_float(sa[i + 4]), __uint_as_float(sa[i + 8]));
#pragma unroll
        for (int c = 12; c < 60; c += 8)
#pragma unroll
          for (int i = 0; i < 4; ++i)
            m4[i] = fmax3(m4[i], __uint_as_float(sa[c + i]), __uint_as_float(sa[c + 4 + i]));
#pragma unroll
        for (int i = 0; i < 4; ++i) m4[i] = fmaxf(m4[i], __uint_as_float(sa[60 + i]));
        tmem_wait_ld_x64(sz);
        if (part) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c + 64 < c_lo || c + 64 >= c_hi) sz[c] = __float_as_uint(-INFINITY);
        }
#pragma unroll
        for (int c = 0; c < 64; c += 8)
#pragma unroll
          for (int i = 0; i < 4; ++i)
            m4[i] = fmax3(m4[i], __uint_as_float(sz[c + i]), __uint_as_float(sz[c + 4 + i]));
        const float m_tile = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]) * sl;
        bool need = false;
        float alpha = 1.f;
        // A window can hide every key of a tile from a row (m_tile = -inf): the
        // row's reference is then set by its first tile with a visible key.
        if (MASK == kMaskWindow ? m_ref == -INFINITY : j == jlo) {
          m_ref = m_tile;
        } else {
          ++n_rowtiles;
          if (m_tile - m_ref > p.tau) {
            need = true;
            alpha = fast_exp2(m_ref - m_tile);
            m_ref = m_tile;
            l *= alpha;
            lr *= alpha;
            ++n_rescale;
          }
        }
        // P~ = 2^(s*scale*log2e - m_ref): one packed FMA per column pair for the
        // arguments, MUFU ex2 or (for POLY of every 8 pairs) the packed FMA-pipe
        // polynomial for the exponentials, packed partial row sums, packing.  In
        // kPSplit parts: each is stored and released to the MMA warp (the PV K steps
        // over its keys) while the next is computed.
        float nm = (MASK == kMaskWindow && m_ref == -INFINITY) ? 0.f : -m_ref;
        if constexpr (F8) nm += p.p_shift;  // P~ * 2^p_shift <= 256 stays in E4M3's range
        float ls[4] = {0.f, 0.f, 0.f, 0.f};
        // On a tile the mask cuts for this sub-tile, the sum O is divided by is
        // taken over the bf16 P~ the PV product uses, read back from TMEM after
        // the stores (every score and P~ register is dead by then).  Not in the
        // sliding-window kernels nor the unmasked d = 64 ones: there the read-back
        // costs the softmax loop its registers, and their rows keep the fp32 sum.
        constexpr bool RSUM = !F8 && MASK != kMaskWindow && !(D == 64 && MASK == kMaskNone);
        auto rounded_sum = [&]() -> float {
          tmem_st_wait();
          uint32_t pr[64];
          tmem_ld_x64(t_s, pr);
          float q0 = 0.f, q1 = 0.f;
#pragma unroll
          for (int i = 0; i < 64; ++i)
            fadd2_acc(q0, q1, __uint_as_float(pr[i] << 16), __uint_as_float(pr[i] & 0xffff0000u));
          return q0 + q1;
        };
        if constexpr (!F8 && kPSplit == 2 && kEarlyPairs > 0) {
          // bf16, two parts: the first pairs of the second part are computed before
          // waiting for the first part's TMEM store, so that wait returns at once.
          auto pair_bf16 = [&](int c) -> uint32_t {  // column pair c (keys 2c, 2c+1)
            const uint32_t x0 = c < 32 ? sa[2 * c] : sz[2 * c - 64];
            const uint32_t x1 = c < 32 ? sa[2 * c + 1] : sz[2 * c - 63];
            float a, e;
            ffma2_bc(a, e, __uint_as_float(x0), __uint_as_float(x1), sl, nm);
            if ((c & 7) >= 8 - POLY) {
              exp2_poly_x2(a, e);
            } else {
              a = fast_exp2(a);
              e = fast_exp2(e);
            }
            if (c & 1) fadd2_acc(ls[2], ls[3], a, e);
            else fadd2_acc(ls[0], ls[1], a, e);
            return pack_bf16x2(a, e);
          };
          auto release = [&](int half) {
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              if (PAIR && !leader) mbar_arrive_remote(lbar(Lay::B_PFULL + kPSplit * s + half));
              else mbar_arrive(bar(Lay::B_PFULL + kPSplit * s + half));
            }
          };
          uint32_t pk0[32], pk1[32];
#pragma unroll
          for (int cc = 0; cc < 32; ++cc) pk0[cc] = pair_bf16(cc);
          tmem_st_x32(t_s, pk0);
          if (__any_sync(0xffffffffu, need)) {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t ov[32];
              tmem_ld_x32(t_o + 32 * c, ov);
#pragma unroll
              for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
              tmem_st_x32(t_o + 32 * c, ov);
            }
          }
#pragma unroll
          for (int cc = 0; cc < kEarlyPairs; ++cc) pk1[cc] = pair_bf16(32 + cc);
          release(0);
#pragma unroll
          for (int cc = kEarlyPairs; cc < 32; ++cc) pk1[cc] = pair_bf16(32 + cc);
          tmem_st_x32(t_s + 32, pk1);
          const float lq = (RSUM && part) ? rounded_sum() : 0.f;
          release(1);
          const float lt = (ls[0] + ls[1]) + (ls[2] + ls[3]);
          l += lt;
          lr += (RSUM && part) ? lq : lt;
          continue;
        }
        float lq_gen = 0.f;
#pragma unroll
        for (int half = 0; half < kPSplit; ++half) {
          constexpr int PAIRS = 64 / kPSplit;  // column pairs per part
          uint32_t pk[F8 ? PAIRS / 2 : PAIRS];
#pragma unroll
          for (int cc = 0; cc < PAIRS; ++cc) {
            const int c = PAIRS * half + cc;  // column pair (keys 2c, 2c+1)
            const uint32_t x0 = c < 32 ? sa[2 * c] : sz[2 * c - 64];
            const uint32_t x1 = c < 32 ? sa[2 * c + 1] : sz[2 * c - 63];
            float a, e;
            ffma2_bc(a, e, __uint_as_float(x0), __uint_as_float(x1), sl, nm);
            if ((c & 7) >= 8 - POLY) {
              exp2_poly_x2(a, e);
            } else {
              a = fast_exp2(a);
              e = fast_exp2(e);
            }
            if (c & 1) fadd2_acc(ls[2], ls[3], a, e);
            else fadd2_acc(ls[0], ls[1], a, e);
            if constexpr (F8) {
              const uint32_t h = pack_e4m3x2(a, e);  // bytes 2(c&1), +1 of word c/2
              if (cc & 1) pk[cc >> 1] |= h << 16; else pk[cc >> 1] = h;
            } else {
              pk[cc] = pack_bf16x2(a, e);
            }
          }
          if constexpr (F8) {
            if constexpr (PAIRS == 64) tmem_st_x32(t_s, pk);
            else if constexpr (PAIRS == 32) tmem_st_x16(t_s + 16 * half, pk);
            else tmem_st_x8(t_s + 8 * half, pk);
          } else {
            if constexpr (PAIRS == 64) tmem_st_x64(t_s, pk);
            else if constexpr (PAIRS == 32) tmem_st_x32(t_s + 32 * half, pk);
            else tmem_st_x16(t_s + 16 * half, pk);
          }
          // O_s is stable here (the commit that signalled S(s, j) also covers
          // PV(s, j-1)); the rare rescale must land before PV(s, j) starts, i.e.
          // before the first half is released.
          if (half == 0 && __any_sync(0xffffffffu, need)) {
            if constexpr (kPSplit <= 2) {
#pragma unroll
              for (int c = 0; c < D / 32; ++c) {
                uint32_t ov[32];
                tmem_ld_x32(t_o + 32 * c, ov);
#pragma unroll
                for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                tmem_st_x32(t_o + 32 * c, ov);
              }
            } else {  // most of the score row is still live: small chunks
#pragma unroll 1
              for (int c = 0; c < D / 8; ++c) {
                uint32_t ov[8];
                tmem_ld_x8(t_o + 8 * c, ov);
#pragma unroll
                for (int i = 0; i < 8; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                tmem_st_x8(t_o + 8 * c, ov);
              }
            }
          }
          if constexpr (RSUM) {
            if (half == kPSplit - 1 && part) lq_gen = rounded_sum();
          }
          tmem_st_wait();
          // One arrival per warp: every lane's TMEM stores are complete (wait::st)
          // and fenced before the warp converges; lane 0 then releases them.
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (PAIR && !leader) mbar_arrive_remote(lbar(Lay::B_PFULL + kPSplit * s + half));
            else mbar_arrive(bar(Lay::B_PFULL + kPSplit * s + half));
          }
        }
        const float lt = (ls[0] + ls[1]) + (ls[2] + ls[3]);
        l += lt;
        lr += (RSUM && part) ? lq_gen : lt;
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      ok = mbar_wait(bar(Lay::B_OFULL + s), o_phase, wc, timeout_code(kSiteOFull));
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      o_phase ^= 1u;
      tc_fence_after();
      float inv = 1.f / lr;
      if constexpr (F8) inv *= p.o_scale;  // V's per-tensor scale
      const bool store = q_row < L;
      __nv_bfloat16* dst =
          p.o + (static_cast<int64_t>(seq_start + q_row) * p.H + h) * static_cast<int64_t>(D);
      // The whole O row in one TMEM load (the score registers are free by now).
      uint32_t ov[D];
      if constexpr (D == 128) tmem_ld_x128(t_o, ov);
      else tmem_ld_x64(t_o, ov);
      // Asynchronous write-back: when all 32 rows of this warp lie inside the
      // sequence, the warp writes them, 64 head dims at a time, into its staging
      // buffer (the 128-byte-swizzled layout of a {64, 1, 32} box) and one lane
      // hands each half to a TMA store; the warp goes on without waiting for the
      // global writes.  Warps whose rows cross the sequence end store directly.
      const bool staged = p.stage_off != 0 && __all_sync(0xffffffffu, store);
      uint8_t* stg = smem + p.stage_off + warp * 4096;
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float x0, x1;
          fmul2_bc(x0, x1, __uint_as_float(ov[8 * c + 2 * i]), __uint_as_float(ov[8 * c + 2 * i + 1]), inv);
          w[i] = pack_bf16x2(x0, x1);
        }
        if (staged) {
          if ((c & 7) == 0) {
            // the previous store from this buffer has finished reading it
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
          }
          *reinterpret_cast<uint4*>(stg + lane * 128 + (((c & 7) ^ (lane & 7)) << 4)) =
              make_uint4(w[0], w[1], w[2], w[3]);
          if ((c & 7) == 7) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(&tm_o, smem_u32(stg), (c >> 3) * 64, h, seq_start + row0 + wq * 32);
              bulk_commit_group();
            }
          }
        } else if (store) {
          reinterpret_cast<uint4*>(dst)[c] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      if (store) {
        float lse2 = m_ref + __log2f(l);
        if constexpr (F8) lse2 -= p.p_shift;
        const float lse = lse2 * kLn2;
        int64_t li;
        if (p.cu_seqlens == nullptr)
          li = (static_cast<int64_t>(b) * p.H + h) * p.N + q_row;
        else
          li = static_cast<int64_t>(h) * p.total + seq_start + q_row;
        p.lse[li] = lse;
      }
    }
    // Every TMA store of this warp has completed before the CTA exits.
    if (lane == 0) bulk_wait_all();
    __syncwarp();
    if (p.stats) {
      atomicAdd(p.stats, static_cast<unsigned long long>(n_rescale));
      atomicAdd(p.stats + 1, static_cast<unsigned long long>(n_rowtiles));
    }
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 120;\n" ::: "memory");
    if (warp == 8) {
      // ----------------------------------------------------------- producer
      // Whole warp walks the loop and waits; one elected lane issues the copies.
      if (elect_one()) {
        tma_prefetch_map(&tm_q);
        tma_prefetch_map(PAIR ? &tm_k2 : &tm_k);
        tma_prefetch_map(&tm_v);
      }
      __syncwarp();
      const uint64_t pol_kv = l2_policy_evict_last();
      const uint64_t pol_q = l2_policy_evict_first();
      uint32_t n_ld = 0, qe_phase = 0;
      int n_items = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        // Claim the next list position once its queue entry is free, and publish it
        // (to both CTAs of a pair; the follower's producer takes it like the other roles).
        const int e = k & 1;
        int idx = -1;
        if (PAIR && !leader) {
          idx = take_item(k);
        } else {
          if (k >= 2) {
            ok = __all_sync(0xffffffffu, mbar_wait<PAIR>(bar(Lay::B_ITEME + e), ((k >> 1) - 1) & 1, wc,
                                                         timeout_code(kSiteItemEmpty)));
            if (!ok) break;
          }
          if (lane == 0) {
            const unsigned c = atomicAdd(p.work, 1u);
            if (c < static_cast<unsigned>(sch.count)) idx = static_cast<int>(c);
            queue[e] = idx;
            mbar_arrive(bar(Lay::B_ITEMF + e));
            if constexpr (PAIR) {
              const uint32_t qaddr = sb + Lay::MISC_OFF + 4 * (8 + e);
              st_shared_remote_u32(mapa_shared(qaddr, 1), static_cast<uint32_t>(idx));
              mbar_arrive_remote(mapa_shared(bar(Lay::B_ITEMF + e), 1));  // release: orders the store
            }
          }
          idx = __shfl_sync(0xffffffffu, idx, 0);
        }
        if (idx < 0) break;
        const Item it = sch.template decode<SPLIT>(idx);
        const int h = it.h, seq_start = it.seq_start;
        int jlo, nkv;
        item_range<MASK, SUB>(it, mk, jlo, nkv);
        if (k > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_QEMPTY), qe_phase, wc, timeout_code(kSiteQEmpty)));
          if (!ok) break;
          qe_phase ^= 1u;
        }
        // Failure-path test: the first query tile's copy is never issued, so its
        // consumers' waits run out.
        const bool withhold = p.test_fault == 1 && k == 0;
        if (!withhold && elect_one()) {
          // Each CTA loads its own query rows; the leader counts the pair's bytes.
          if (leader) mbar_arrive_expect_tx(bar(Lay::B_QFULL), (PAIR ? 4 : 2) * Lay::TILE);
#pragma unroll
          for (int s = 0; s < 2; ++s) {
            const int qr = seq_start + it.row_base + s * SUB + static_cast<int>(rank) * kBM;
#pragma unroll
            for (int c = 0; c < Lay::NCHUNK; ++c) {
              const uint32_t dst = sb + Lay::Q_OFF + s * Lay::TILE + c * Lay::CHUNK;
              if constexpr (PAIR) tma_load_3d_pair(dst, &tm_q, lbar(Lay::B_QFULL), c * 64, h, qr, pol_q);
              else tma_load_3d(dst, &tm_q, bar(Lay::B_QFULL), c * (128 / Lay::ESZ), h, qr, pol_q);
            }
          }
        }
        __syncwarp();
        if (!withhold) ++n_items;
        for (int j = 0; j < nkv && ok; ++j) {
          const int key0 = seq_start + (jlo + j) * kBN;
#pragma unroll
          for (int which = 0; which < 2; ++which) {
            const uint32_t slot = n_ld % NS;
            if (n_ld >= static_cast<uint32_t>(NS)) {
              ok = __all_sync(0xffffffffu, mbar_wait(bar(Lay::B_KVEMPTY + slot), ((n_ld / NS) - 1) & 1u,
                                                     wc, timeout_code(kSiteKvEmpty)));
              if (!ok) break;
            }
            if (elect_one()) {
              const uint32_t dst = sb + Lay::KV_OFF + slot * Lay::SLOT;
              if constexpr (PAIR) {
                // K: keys 64*rank..+63 (two 64-row boxes, one per 64 head-dim columns);
                // V: all 128 keys, head-dim columns 64*rank..+63 (one box).
                if (leader) mbar_arrive_expect_tx(bar(Lay::B_KVFULL + slot), 2 * Lay::SLOT);
                if (which == 0) {
#pragma unroll
                  for (int c = 0; c < 2; ++c)
                    tma_load_3d_pair(dst + c * (Lay::SLOT / 2), &tm_k2, lbar(Lay::B_KVFULL + slot), c * 64, h,
                                     key0 + static_cast<int>(rank) * 64, pol_kv);
                } else {
                  tma_load_3d_pair(dst, &tm_v, lbar(Lay::B_KVFULL + slot), static_cast<int>(rank) * 64, h,
                                   key0, pol_kv);
                }
              } else {
                mbar_arrive_expect_tx(bar(Lay::B_KVFULL + slot), Lay::TILE);
#pragma unroll
                for (int c = 0; c < Lay::NCHUNK; ++c)
                  tma_load_3d(dst + c * Lay::CHUNK, which ? &tm_v : &tm_k, bar(Lay::B_KVFULL + slot),
                              c * (128 / Lay::ESZ), h, key0, pol_kv);
              }
            }
            __syncwarp();
            ++n_ld;
          }
        }
      }
      // Drain: every issued copy must have landed before the CTA may exit (a pair's
      // copies all complete on the leader's barriers; the leader drains them, and
      // the pair waits for each other before exiting).
      if (leader) {
        const uint32_t first = n_ld > static_cast<uint32_t>(NS) ? n_ld - NS : 0u;
        for (uint32_t n = first; n < n_ld; ++n)
          drain_wait(bar(Lay::B_KVFULL + n % NS), (n / NS) & 1u, kDrainLimitNs);
        if (n_items > 0) drain_wait(bar(Lay::B_QFULL), (n_items - 1) & 1u, kDrainLimitNs);
      }
    } else if (warp == 9 && leader) {
      // ---------------------------------------------------------------- MMA
      // (a pair's follower has no MMA role: the leader issues the pair's products)
      // The whole warp walks the loop and waits; one elected lane issues each MMA
      // and commit.  Issue order per key tile j (ping-pong of the two sub-tiles):
      //   PV(0, j-1), S(0, j), PV(1, j-1), S(1, j)
      // each only where tile j (j-1) lies in that sub-tile's key range.
      // S(s, j) overwrites P(s, j-1) in TMEM, which PV(s, j-1) read just before; the
      // tensor pipe executes one thread's MMAs in issue order.
      constexpr int M = PAIR ? 2 * kBM : kBM;  // rows of one product (a pair: 128 in each CTA)
      constexpr uint32_t idesc_s = F8 ? idesc_e4m3_f32(M, kBN, 0, 0) : idesc_bf16_f32(M, kBN, 0, 0);
      constexpr uint32_t idesc_o = F8 ? idesc_e4m3_f32(M, D, 0, 1) : idesc_bf16_f32(M, D, 0, 1);
      // Commit to this CTA's barrier, or to the barrier at the same offset in both
      // CTAs of a pair.
      auto commit = [&](int i) {
        if constexpr (PAIR) tc_commit_pair(bar(i), 0x3);
        else tc_commit(bar(i));
      };
      const uint32_t tS0 = tmem + Lay::TM_S0, tS1 = tmem + Lay::TM_S1;
      const uint32_t tO0 = tmem + Lay::TM_O0, tO1 = tmem + Lay::TM_O1;
      uint32_t n_ld = 0, q_phase = 0, p_phase0 = 0, p_phase1 = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int idx = take_item(k);
        if (idx < 0) break;
        const Item it = sch.template decode<SPLIT>(idx);
        int jlo, nkv, lo0, hi0, lo1, hi1;
        item_range<MASK, SUB>(it, mk, jlo, nkv);
        kv_range<MASK, SUB>(it, 0, mk, lo0, hi0);
        kv_range<MASK, SUB>(it, 1, mk, lo1, hi1);
        ok = __all_sync(0xffffffffu, mbar_wait<PAIR>(bar(Lay::B_QFULL), q_phase, wc, timeout_code(kSiteQFull)));
        if (!ok) break;
        q_phase ^= 1u;
        tc_fence_after();
        for (int jj = 0; jj <= nkv && ok; ++jj) {
          const int j = jlo + jj;              // key tile
          const uint32_t nK = n_ld + 2u * jj;  // load sequence number of K_j
          const uint32_t nV = nK - 1u;        // ... and of V_{j-1}
          const uint32_t slotK = nK % NS, slotV = nV % NS;
          if (jj < nkv)
            ok = __all_sync(0xffffffffu, mbar_wait<PAIR>(bar(Lay::B_KVFULL + slotK), (nK / NS) & 1u, wc,
                                                         timeout_code(kSiteKvFull)));
          if (ok && jj > 0)
            ok = __all_sync(0xffffffffu, mbar_wait<PAIR>(bar(Lay::B_KVFULL + slotV), (nV / NS) & 1u, wc,
                                                         timeout_code(kSiteKvFull)));
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int s = 0; s < 2; ++s) {
            const uint32_t tS = s ? tS1 : tS0, tO = s ? tO1 : tO0;
            const int los = s ? lo1 : lo0, his = s ? hi1 : hi0;
            if (ok && jj > 0 && j - 1 >= los && j - 1 < his) {
              uint32_t& ph = s ? p_phase1 : p_phase0;
              const uint32_t vbase = sb + Lay::KV_OFF + slotV * Lay::SLOT;
              constexpr int NK = kBN / Lay::KSTEP;  // PV K steps per key tile
              // Each part of P~ is multiplied as soon as the softmax warps release it.
              // One K step: KSTEP keys = 32 bytes of a P~ row (8 TMEM columns) and
              // KSTEP rows of V (128 bytes each).
              static_assert(NK % kPSplit == 0, "K steps per part");
#pragma unroll
              for (int half = 0; half < kPSplit && ok; ++half) {
                ok = __all_sync(0xffffffffu, mbar_wait<PAIR>(bar(Lay::B_PFULL + kPSplit * s + half), ph, wc,
                                                             timeout_code(kSitePFull)));
                if (!ok) break;
                tc_fence_after();
                // The part's K steps are issued back to back by one elected lane.
                if (elect_one()) {
                  // V (a pair: this CTA's 64 head-dim columns of it) is MN-major.
                  const uint64_t dv0 = sdesc_sw128(vbase, Lay::CHUNK, 1024);
#pragma unroll
                  for (int kk = half * NK / kPSplit; kk < (half + 1) * NK / kPSplit; ++kk) {
                    const uint64_t dv = desc_add(dv0, kk * Lay::KSTEP * 128);
                    const uint32_t acc = (j - 1 > los || kk > 0) ? 1u : 0u;
                    if constexpr (PAIR) mma_ts_pair(tO, tS + kk * 8, dv, idesc_o, acc);
                    else if constexpr (F8) mma_ts_f8(tO, tS + kk * 8, dv, idesc_o, acc);
                    else mma_ts(tO, tS + kk * 8, dv, idesc_o, acc);
                  }
                }
                __syncwarp();
              }
              if (ok) {
                ph ^= 1u;
                if (j == his) {
                  if (elect_one()) commit(Lay::B_OFULL + s);
                  __syncwarp();
                }
              }
            }
            if (ok && j >= los && j < his) {
              const uint32_t qbase = sb + Lay::Q_OFF + s * Lay::TILE;
              const uint32_t kbase = sb + Lay::KV_OFF + slotK * Lay::SLOT;
              // K's rows (a pair: this CTA's 64 keys) in 128-byte chunks of head dims.
              constexpr int KCHUNK = PAIR ? Lay::SLOT / 2 : Lay::CHUNK;
              if (elect_one()) {
                const uint64_t da0 = sdesc_sw128(qbase, 16, 1024);
                const uint64_t db0 = sdesc_sw128(kbase, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < D / Lay::KSTEP; ++kk) {
                  const uint64_t da = desc_add(da0, (kk >> 2) * Lay::CHUNK + (kk & 3) * 32);
                  const uint64_t db = desc_add(db0, (kk >> 2) * KCHUNK + (kk & 3) * 32);
                  if constexpr (PAIR) mma_ss_pair(tS, da, db, idesc_s, kk > 0 ? 1u : 0u);
                  else if constexpr (F8) mma_ss_f8(tS, da, db, idesc_s, kk > 0 ? 1u : 0u);
                  else mma_ss(tS, da, db, idesc_s, kk > 0 ? 1u : 0u);
                }
                commit(Lay::B_SFULL + s);
              }
              __syncwarp();
            }
          }
          if (!ok) break;
          if (elect_one()) {
            if (jj < nkv) commit(Lay::B_KVEMPTY + slotK);
            if (jj > 0) commit(Lay::B_KVEMPTY + slotV);
            // The query tiles are free after the item's last S product (an item
            // without key tiles -- an empty half item -- frees them at once).
            if (jj == (nkv > 0 ? nkv - 1 : 0)) commit(Lay::B_QEMPTY);
          }
          __syncwarp();
        }
        n_ld += 2u * nkv;
      }
      // Drain: every MMA issued by this warp completes before TMEM is freed.
      if (elect_one()) {
        if constexpr (PAIR) tc_commit_pair(bar(Lay::B_DRAIN), 0x1);
        else tc_commit(bar(Lay::B_DRAIN));
      }
      __syncwarp();
      if (!__all_sync(0xffffffffu, drain_wait(bar(Lay::B_DRAIN), 0u, kDrainLimitNs)) && lane == 0 && p.err)
        atomicCAS(p.err, 0, timeout_code(kSiteDrain));
    }
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) {  // neither CTA of a pair leaves while the other may still use its memory
    cluster_arrive();
    cluster_wait();
  }
  tc_fence_after();
  if (warp == 9) {
    if constexpr (PAIR) tmem_dealloc_pair(tmem, 512);
    else tmem_dealloc(tmem, 512);
  }
  // The last CTA to finish returns the claim counter to zero for the next launch
  // that uses it: every CTA's producer has made its last claim before its CTA
  // counts itself finished here.
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.work + 1, 1u) == gridDim.x - 1) {
      atomicExch(p.work, 0u);
      atomicExch(p.work + 1, 0u);
    }
  }
}

template <int D, bool F8, bool PAIR = false>
constexpr int smem_bytes_fixed() { return 1024 + Layout<D, F8, PAIR>::TABLE_OFF; }

}  // namespace

int fwd_smem_bytes(int D, int B, int T, int varlen, int fp8, int pair) {
  const int fixed = pair ? smem_bytes_fixed<128, false, true>()
                         : fp8 ? smem_bytes_fixed<128, true>()
                               : (D == 128 ? smem_bytes_fixed<128, false>() : smem_bytes_fixed<64, false>());
  return fixed + (varlen ? varlen_table_ints(B, T) * 4 : 0);
}

int fwd_stage_offset(int D, int B, int T, int varlen, int fp8, int pair) {
  const int end = fwd_smem_bytes(D, B, T, varlen, fp8, pair) - 1024;  // from the aligned base
  const int off = (end + 1023) & ~1023;
  return (1024 + off + kFwdStageBytes <= 232448) ? off : 0;
}

template <int D, int MASK, int POLY, bool F8 = false, bool PAIR = false>
static cudaError_t launch_t(const FwdLaunch& a, cudaStream_t st) {
  auto kern = fwd_kernel<D, MASK, POLY, F8, PAIR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, a.smem);
  if (e != cudaSuccess) return e;
  if constexpr (PAIR) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = a.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, a.tm_q, a.tm_k, a.tm_v, a.tm_k2, a.tm_o, a.p);
    if (e != cudaSuccess) return e;
  } else {
    kern<<<a.grid, kThreads, a.smem, st>>>(a.tm_q, a.tm_k, a.tm_v, a.tm_k2, a.tm_o, a.p);
  }
  return cudaGetLastError();
}

template <int D, int MASK>
static cudaError_t launch_p(const FwdLaunch& a, int poly, cudaStream_t st) {
  if (poly == 2) return launch_t<D, MASK, 2>(a, st);
  if (poly == 8) return launch_t<D, MASK, 8>(a, st);
  return launch_t<D, MASK, 0>(a, st);
}

template <int D>
static cudaError_t launch_m(const FwdLaunch& a, MaskKind mask, int poly, cudaStream_t st) {
  if (mask == kMaskCausal) return launch_p<D, kMaskCausal>(a, poly, st);
  if (mask == kMaskWindow) return launch_p<D, kMaskWindow>(a, poly, st);
  return launch_p<D, kMaskNone>(a, poly, st);
}

cudaError_t launch_fwd(const FwdLaunch& a, int D, MaskKind mask, int poly, int fp8, cudaStream_t st) {
  if (a.pair) {  // CTA pairs: bf16, d = 128, exponentials on MUFU
    if (mask == kMaskCausal) return launch_t<128, kMaskCausal, 0, false, true>(a, st);
    if (mask == kMaskWindow) return launch_t<128, kMaskWindow, 0, false, true>(a, st);
    return launch_t<128, kMaskNone, 0, false, true>(a, st);
  }
  if (fp8) {  // E4M3: d = 128; exponentials all on MUFU or 2 of every 8 pairs on the FMA pipe
    if (poly == 2) {
      if (mask == kMaskCausal) return launch_t<128, kMaskCausal, 2, true>(a, st);
      if (mask == kMaskWindow) return launch_t<128, kMaskWindow, 2, true>(a, st);
      return launch_t<128, kMaskNone, 2, true>(a, st);
    }
    if (mask == kMaskCausal) return launch_t<128, kMaskCausal, 0, true>(a, st);
    if (mask == kMaskWindow) return launch_t<128, kMaskWindow, 0, true>(a, st);
    return launch_t<128, kMaskNone, 0, true>(a, st);
  }
  return D == 128 ? launch_m<128>(a, mask, poly, st) : launch_m<64>(a, mask, poly, st);
}

int fwd_pair_max_clusters(int smem) {
  // Clusters of two CTAs of this kernel (causal, MUFU exponentials) that fit at once.
  auto kern = fwd_kernel<128, kMaskCausal, 0, false, true>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) return 0;
  return n;
}

}  // namespace attn
