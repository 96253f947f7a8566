// Two-branch block selection ([RBS-en] "The Fix: A Radius-Adaptive Rescue
// Branch"; [RBS-id] "Dual-Branch Selection"):
//   s_c(i, j) = qbar_i . c_j
//   s_r(i, j) = s_c(i, j) + |qbar_i| * r_j * beta_j
// each branch keeps its own top ceil(rho * n_i) of the n_i visible key
// blocks (ties to the lower index), the kept sets are OR-ed with the forced
// blocks, and the rows are compacted into CSR lists.
//
// Kernels:
//   select_rows_kernel  persistent: CTA c walks the work items (query block
//                       i, group of R q heads of one KV head, batch) c,
//                       c + grid, ... in longest-row-first order.  Warps 8-9
//                       pool the NEXT item's query block (mean of its BQ
//                       queries per head) out of a TMA-fed ring of 8-row
//                       chunks while warps 0-7 work on the current item:
//                       centroid tiles of 512 blocks x 16 dims are staged
//                       through shared memory (16-byte chunks swizzled so
//                       both the stores and the row reads are conflict-free),
//                       every thread forms the fp32 dot products of two
//                       blocks with all R pooled queries, and then warp
//                       w < R finds both branches' exact top-k of its row
//                       (a pruned search over order-preserving keys, with a
//                       full 32-step bitwise search as the fallback), breaks
//                       ties by block index with warp ballots, and emits one
//                       32-bit mask word per 32 blocks.
//   group_counts_kernel (KV_GROUP lists) one warp per (batch, KV head, query
//                       block) counts the union of its q heads' masks.
//   scan_tiles_kernel   exclusive scan of the sums of 256 rows' counts (the
//                       selection kernels add each row's count to its tile's
//                       sum as they write it).
//   compact_lists_kernel one warp per list row: its row pointer (tile prefix +
//                       the tile's earlier counts), and its mask words (OR-ed over
//                       the q heads of a KV_GROUP row) into ascending block
//                       indices and per-entry branch flags.
#pragma once

#include "common.cuh"

namespace rbs {

struct SelectArgs {
  const float* C;      // [B, Hkv, nkb, 128]
  const float* rad;    // [B, Hkv, nkb]
  const float* beta;   // [B, Hkv, nkb]
  int B, Hq, Hkv, nqb, nkb, R, nwords;
  int items;           // B * nqb * (Hq / R)
  int Lq;              // query tokens; the last query block holds Lq - (nqb - 1) BQ of them
  int seq_inner;       // 1 when Q's token stride is smaller than its head stride
  int q_block_offset, causal, force_diag, force_sink;
  float rho_c, rho_r;
  int threshold_mode;    // 0 = top-k fraction, 1 = within delta of the row maximum
  float delta_c, delta_r;
  uint32_t* mask_c;  // [rows, nwords]
  uint32_t* mask_r;  // [rows, nwords]
  int* counts;       // [rows]
  // [ceil(rows / kScanTile)] sums of the counts of kScanTile consecutive rows
  // (zero on entry, added to as rows finish), or null when another kernel
  // forms the list rows' counts
  int* tile_sums;
};

constexpr int kScanTile = 256;  // rows per partial sum of the row-pointer scan

constexpr int kSelComputeThreads = 256;  // warps 0-7: scores and top-k
constexpr int kSelPoolThreads = 64;      // warps 8-9: pooling of the next item
constexpr int kSelThreads = kSelComputeThreads + kSelPoolThreads;
constexpr int kSelMaxR = 8;
constexpr int kStageJ = 512;   // key blocks per staged centroid tile (two per compute thread)
constexpr int kStageD = 16;    // dims per staged tile: 64-byte rows of four 16-byte chunks
constexpr int kPoolRows = 8;   // query rows per TMA chunk
constexpr int kPoolStages = 2;
constexpr int kPoolChunkBytes = kPoolRows * kSelMaxR * 128 * 2;  // the largest chunk (R = 8)
constexpr int kTopkCap = 128;  // candidates per branch in the pruned top-k (four per lane)

// Dynamic shared memory of select_rows_kernel, in bytes from a 128-byte
// aligned base: the chunk ring, the centroid staging tile (reused as top-k
// scratch), two buffers of pooled queries [128][8], then r*beta [npad] and
// the centroid-branch scores [8][npad].
constexpr int kSelOffCs = kPoolStages * kPoolChunkBytes;
constexpr int kSelOffQs = kSelOffCs + kStageJ * kStageD * 4;
constexpr int kSelOffRb = kSelOffQs + 2 * 128 * kSelMaxR * 4;
__host__ __device__ constexpr size_t sel_smem_bytes(int npad) {
  return static_cast<size_t>(kSelOffRb) + static_cast<size_t>(1 + kSelMaxR) * npad * 4;
}
// top-k scratch of one warp: candidate keys and blocks of both branches,
// then both branches' mask words
__host__ __device__ constexpr int sel_topk_scratch_words(int nwords) { return 4 * kTopkCap + 2 * nwords; }
static_assert(kSelComputeThreads / 32 * sel_topk_scratch_words(RBS_MAX_KV_BLOCKS / 32) * 4 <= kStageJ * kStageD * 4,
              "top-k scratch must fit in the staging tile");

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The float whose order_key is k (order_key is a bijection).
__device__ __forceinline__ float key_to_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

__device__ __forceinline__ int keep_count(float rho, int n) {
  // k = ceil(rho * n) within [1, n]; rho is the float32 parameter widened to
  // double, and the 1e-4 slack absorbs its float32 representation error.
  int k = static_cast<int>(ceil(static_cast<double>(rho) * n - 1e-4));
  return k < 1 ? 1 : (k > n ? n : k);
}

// Warp sums of two small counts (each total below 2^16) in one reduction:
// the first in the low 16 bits, the second in the high 16 bits.
__device__ __forceinline__ void sum2(int x, int y, int& sx, int& sy) {
  const uint32_t s = __reduce_add_sync(0xffffffffu, static_cast<uint32_t>(x) | (static_cast<uint32_t>(y) << 16));
  sx = static_cast<int>(s & 0xFFFFu);
  sy = static_cast<int>(s >> 16);
}

// Exact top-k of the warp's keys for two branches at once (key 0 = not a
// candidate; k <= #candidates).  The k-th largest key T is built bit by bit
// from the top (the largest T with at least k keys >= T); keys above T are
// kept, and of the keys equal to T the ones with the lowest block index.
// Returns, per lane, the mask words this lane owns (word t is owned by lane
// t % 32) with bit `lane` of word t set iff block 32t + lane is kept.
template <int KPL>
__device__ __forceinline__ void warp_topk2(const uint32_t (&kc)[KPL], const uint32_t (&kr)[KPL], int k_c, int k_r,
                                           int lane, uint32_t (&own_c)[(KPL + 31) / 32],
                                           uint32_t (&own_r)[(KPL + 31) / 32]) {
  uint32_t Tc = 0, Tr = 0;
#pragma unroll 1
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cc = Tc | (1u << bit), cr = Tr | (1u << bit);
    int nc2[2] = {0, 0}, nr2[2] = {0, 0};  // two partial counts per branch (shorter add chains)
#pragma unroll
    for (int t = 0; t < KPL; ++t) {
      nc2[t & 1] += kc[t] >= cc ? 1 : 0;
      nr2[t & 1] += kr[t] >= cr ? 1 : 0;
    }
    int nc, nr;
    sum2(nc2[0] + nc2[1], nr2[0] + nr2[1], nc, nr);
    if (nc >= k_c) Tc = cc;
    if (nr >= k_r) Tr = cr;
  }
  int gc = 0, gr = 0;
#pragma unroll
  for (int t = 0; t < KPL; ++t) {
    gc += kc[t] > Tc ? 1 : 0;
    gr += kr[t] > Tr ? 1 : 0;
  }
  int above_c, above_r;
  sum2(gc, gr, above_c, above_r);
  const int need_c = k_c - above_c, need_r = k_r - above_r;  // ties at T to keep, lowest index first
  const uint32_t lt_mask = (1u << lane) - 1u;
  int base_c = 0, base_r = 0;
#pragma unroll
  for (int t = 0; t < (KPL + 31) / 32; ++t) own_c[t] = own_r[t] = 0;
#pragma unroll
  for (int t = 0; t < KPL; ++t) {
    const bool tie_c = kc[t] == Tc, tie_r = kr[t] == Tr;
    const uint32_t bc = __ballot_sync(0xffffffffu, tie_c), br = __ballot_sync(0xffffffffu, tie_r);
    const bool sel_c = kc[t] > Tc || (tie_c && base_c + __popc(bc & lt_mask) < need_c);
    const bool sel_r = kr[t] > Tr || (tie_r && base_r + __popc(br & lt_mask) < need_r);
    const uint32_t wc = __ballot_sync(0xffffffffu, sel_c), wr = __ballot_sync(0xffffffffu, sel_r);
    if (lane == (t & 31)) {
      own_c[t >> 5] = wc;
      own_r[t >> 5] = wr;
    }
    base_c += __popc(bc);
    base_r += __popc(br);
  }
}

// For a search value known to lie in [lo, hi] (lo <= hi): start = the bits
// above the highest bit where lo and hi differ (shared by every value in the
// range), top = that bit (-1 when lo == hi, nothing left to search).
__device__ __forceinline__ void common_prefix(uint32_t lo, uint32_t hi, uint32_t& start, int& top) {
  const int p = __clz(lo ^ hi);  // leading bits shared by lo and hi (32 when equal)
  start = p == 32 ? lo : (p == 0 ? 0u : lo & ~(0xffffffffu >> p));
  top = 31 - p;
}

// Insert x into the descending list (t0 >= t1 >= t2 >= t3).
__device__ __forceinline__ void top4_insert(uint32_t& t0, uint32_t& t1, uint32_t& t2, uint32_t& t3, uint32_t x) {
  const uint32_t y0 = min(t0, x);
  t0 = max(t0, x);
  const uint32_t y1 = min(t1, y0);
  t1 = max(t1, y0);
  const uint32_t y2 = min(t2, y1);
  t2 = max(t2, y1);
  t3 = max(t3, y2);
}

// Bitonic sort across the warp, descending, of the 32 E values x[e] at
// positions p = lane + 32 e, for two sequences (x and y) at once.  Position p
// ends up holding the (p + 1)-th largest value.  Warp-uniform.
template <int E>
__device__ __forceinline__ void warp_sort_desc2(uint32_t (&x)[E], uint32_t (&y)[E], int lane) {
#pragma unroll
  for (int k = 2; k <= 32 * E; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j >= 32) {
        // partner p + 32: element e + 1 of the same lane (only k = 64 here,
        // a descending block: the lower position keeps the larger value)
#pragma unroll
        for (int e = 0; e + 1 < E; e += 2) {
          const uint32_t hx = max(x[e], x[e + 1]), lx = min(x[e], x[e + 1]);
          const uint32_t hy = max(y[e], y[e + 1]), ly = min(y[e], y[e + 1]);
          x[e] = hx;
          x[e + 1] = lx;
          y[e] = hy;
          y[e + 1] = ly;
        }
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int p = lane + 32 * e;
          // in a descending block (bit k of p clear) the lower position of
          // the pair keeps the larger value, in an ascending block the smaller
          const bool keep_max = ((p & j) == 0) == ((p & k) == 0);
          const uint32_t px = __shfl_xor_sync(0xffffffffu, x[e], j);
          const uint32_t py = __shfl_xor_sync(0xffffffffu, y[e], j);
          x[e] = keep_max ? max(x[e], px) : min(x[e], px);
          y[e] = keep_max ? max(y[e], py) : min(y[e], py);
        }
      }
    }
  }
}

// The k-th largest (1 <= k <= 32 E) of the values sorted by warp_sort_desc2.
template <int E>
__device__ __forceinline__ uint32_t sorted_kth(const uint32_t (&x)[E], int k) {
  const int p = k - 1;
  uint32_t v = x[0];
#pragma unroll
  for (int e = 1; e < E; ++e)
    if ((p >> 5) == e) v = x[e];
  return __shfl_sync(0xffffffffu, v, p & 31);
}

// Both branches' selection from lower bounds Lc <= T_c and Lr <= T_r of
// their k-th largest keys (T), each reached by at least k keys and above
// key 0 (so no absent slot qualifies).  Every key >= L is a candidate; when
// at most kTopkCap keys of each branch are, they are compacted in ascending
// block order into shared memory and T is found among them: by sorting them
// across the warp when there are at most 64, else by a bitwise search (the
// largest T with at least k candidates >= T).  The keys above T are kept and
// of the ties at T the lowest block indices, and the kept blocks are OR-ed
// into words[0, nwords) (cleared first).  Returns false, having written
// nothing the caller uses, when a branch has more than kTopkCap candidates.
// Slots from nt on hold only absent keys.  Warp-uniform.
template <typename KeyC, typename KeyR>
__device__ __forceinline__ bool topk2_from_bounds(KeyC key_c, KeyR key_r, uint32_t Lc, uint32_t Lr, int k_c, int k_r,
                                                  int nt, int lane, int nwords, uint32_t* scratch,
                                                  uint32_t* words_c, uint32_t* words_r) {
  uint32_t* ck_c = scratch;  // candidate keys and blocks of each branch
  int* ci_c = reinterpret_cast<int*>(scratch + kTopkCap);
  uint32_t* ck_r = scratch + 2 * kTopkCap;
  int* ci_r = reinterpret_cast<int*>(scratch + 3 * kTopkCap);
  const uint32_t lt_mask = (1u << lane) - 1u;
  int base_c = 0, base_r = 0;
#pragma unroll 4
  for (int t = 0; t < nt; ++t) {
    const uint32_t uc = key_c(t), ur = key_r(t);
    const bool cand_c = uc >= Lc, cand_r = ur >= Lr;
    const uint32_t bc = __ballot_sync(0xffffffffu, cand_c), br = __ballot_sync(0xffffffffu, cand_r);
    const int pc = base_c + __popc(bc & lt_mask), pr = base_r + __popc(br & lt_mask);
    if (cand_c && pc < kTopkCap) {
      ck_c[pc] = uc;
      ci_c[pc] = 32 * t + lane;
    }
    if (cand_r && pr < kTopkCap) {
      ck_r[pr] = ur;
      ci_r[pr] = 32 * t + lane;
    }
    base_c += __popc(bc);
    base_r += __popc(br);
  }
  if (base_c > kTopkCap || base_r > kTopkCap) return false;
  __syncwarp();
  // candidate position p = lane + 32 s holds slot s of this lane (0 = none)
  const int cmax = max(base_c, base_r);
  const int ns = (cmax + 31) >> 5;  // slots holding a candidate of either branch
  uint32_t a[4], bk[4];
  int ia[4], ib[4];
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const int p = lane + 32 * s;
    a[s] = p < base_c ? ck_c[p] : 0u;
    ia[s] = p < base_c ? ci_c[p] : 0;
    bk[s] = p < base_r ? ck_r[p] : 0u;
    ib[s] = p < base_r ? ci_r[p] : 0;
  }
  uint32_t Tc, Tr;
  if (cmax <= 32) {
    uint32_t x[1] = {a[0]}, y[1] = {bk[0]};
    warp_sort_desc2<1>(x, y, lane);
    Tc = sorted_kth<1>(x, k_c);
    Tr = sorted_kth<1>(y, k_r);
  } else if (cmax <= 64) {
    uint32_t x[2] = {a[0], a[1]}, y[2] = {bk[0], bk[1]};
    warp_sort_desc2<2>(x, y, lane);
    Tc = sorted_kth<2>(x, k_c);
    Tr = sorted_kth<2>(y, k_r);
  } else {
    // T lies between L (at least k candidates reach it) and the largest
    // candidate: it carries their common leading bits
    int tpc, tpr;
    common_prefix(Lc, __reduce_max_sync(0xffffffffu, max(max(a[0], a[1]), max(a[2], a[3]))), Tc, tpc);
    common_prefix(Lr, __reduce_max_sync(0xffffffffu, max(max(bk[0], bk[1]), max(bk[2], bk[3]))), Tr, tpr);
#pragma unroll 1
    for (int bit = max(tpc, tpr); bit >= 0; --bit) {
      const uint32_t xc = Tc | (1u << bit), xr = Tr | (1u << bit);
      int nc, nr;
      sum2((a[0] >= xc) + (a[1] >= xc) + (a[2] >= xc) + (a[3] >= xc),
           (bk[0] >= xr) + (bk[1] >= xr) + (bk[2] >= xr) + (bk[3] >= xr), nc, nr);
      if (bit <= tpc && nc >= k_c) Tc = xc;
      if (bit <= tpr && nr >= k_r) Tr = xr;
    }
  }
  int above_c, above_r;
  sum2((a[0] > Tc) + (a[1] > Tc) + (a[2] > Tc) + (a[3] > Tc), (bk[0] > Tr) + (bk[1] > Tr) + (bk[2] > Tr) + (bk[3] > Tr),
       above_c, above_r);
  const int need_c = k_c - above_c, need_r = k_r - above_r;
  for (int w = lane; w < nwords; w += 32) words_c[w] = words_r[w] = 0u;
  __syncwarp();
  // positions ascend with the block index, so a tie's rank is the number of
  // ties at lower positions
  int rank_c = 0, rank_r = 0;
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    if (s >= ns) break;
    const bool tc = a[s] == Tc, tr = bk[s] == Tr;
    const uint32_t bc = __ballot_sync(0xffffffffu, tc), br = __ballot_sync(0xffffffffu, tr);
    const bool sc = a[s] > Tc || (tc && rank_c + __popc(bc & lt_mask) < need_c);
    const bool sr = bk[s] > Tr || (tr && rank_r + __popc(br & lt_mask) < need_r);
    if (sc) atomicOr(&words_c[ia[s] >> 5], 1u << (ia[s] & 31));
    if (sr) atomicOr(&words_r[ib[s] >> 5], 1u << (ib[s] & 31));
    rank_c += __popc(bc);
    rank_r += __popc(br);
  }
  __syncwarp();
  return true;
}

// Exact top-k of both branches, for k <= 64, from a sorted subset (key(t) =
// this lane's key in slot t, block 32 t + lane, 0 for an absent slot).  Each
// lane keeps its E largest keys per branch (E = 1 when k <= 32, else 2); the
// subset's k-th largest key L (found by sorting the 32 E keys across the
// warp) is at most the row's k-th largest, and at least k keys reach it.
// The subset holds at least k present keys (min(n, 32 E) >= k), so L > 0
// unless the row's keys are themselves 0 (one NaN pattern), which is left to
// the caller's other searches like an overflow.  Returns false when k > 64,
// L = 0, or a branch has more than kTopkCap candidates.  Warp-uniform.
template <int KP, typename KeyC, typename KeyR>
__device__ __forceinline__ bool warp_topk2_sorted(KeyC key_c, KeyR key_r, int k_c, int k_r, int n, int lane,
                                                  int nwords, uint32_t* scratch, uint32_t* words_c,
                                                  uint32_t* words_r) {
  if (k_c > 64 || k_r > 64) return false;
  const int nt = min(KP, (n + 31) >> 5);  // slots holding a visible block
  uint32_t Lc, Lr;
  if (max(k_c, k_r) <= 32) {
    uint32_t x[1] = {0u}, y[1] = {0u};
#pragma unroll 4
    for (int t = 0; t < nt; ++t) {
      x[0] = max(x[0], key_c(t));
      y[0] = max(y[0], key_r(t));
    }
    warp_sort_desc2<1>(x, y, lane);
    Lc = sorted_kth<1>(x, k_c);
    Lr = sorted_kth<1>(y, k_r);
  } else {
    uint32_t x[2] = {0u, 0u}, y[2] = {0u, 0u};
#pragma unroll 4
    for (int t = 0; t < nt; ++t) {
      const uint32_t uc = key_c(t), ur = key_r(t);
      x[1] = max(x[1], min(x[0], uc));
      x[0] = max(x[0], uc);
      y[1] = max(y[1], min(y[0], ur));
      y[0] = max(y[0], ur);
    }
    warp_sort_desc2<2>(x, y, lane);
    Lc = sorted_kth<2>(x, k_c);
    Lr = sorted_kth<2>(y, k_r);
  }
  if (Lc == 0u || Lr == 0u) return false;
  return topk2_from_bounds(key_c, key_r, Lc, Lr, k_c, k_r, nt, lane, nwords, scratch, words_c, words_r);
}

// Exact top-k of both branches by pruning, for k <= 64 (key(t) = this
// lane's key in slot t, block 32 t + lane, 0 for an absent slot).  Each lane
// keeps its four largest keys per branch; that subset of the row holds at
// least k present keys (all of them when n <= 128, 128 otherwise), so its
// k-th largest key, rounded down to 24 bits (L), is at most the row's k-th
// largest key T, and every key >= T is a candidate (key >= L); the rest is
// topk2_from_bounds.  Returns false when k > 64 or a branch has more than
// kTopkCap candidates (many near-equal keys); the caller then runs the full
// search.  Both branches advance together so their reduction chains overlap.
// Slots from ceil(n / 32) on hold only absent keys (blocks >= n): they can
// neither enter a lane's top four nor become candidates, so both passes stop
// before them.  Warp-uniform.
template <int KP, typename KeyC, typename KeyR>
__device__ __noinline__ bool warp_topk2_pruned(KeyC key_c, KeyR key_r, int k_c, int k_r, int n, int lane,
                                                  int nwords, uint32_t* scratch, uint32_t* words_c,
                                                  uint32_t* words_r) {
  if (k_c > 64 || k_r > 64) return false;
  const int nt = min(KP, (n + 31) >> 5);  // slots holding a visible block
  uint32_t c0 = 0, c1 = 0, c2 = 0, c3 = 0, r0 = 0, r1 = 0, r2 = 0, r3 = 0;
#pragma unroll 4
  for (int t = 0; t < nt; ++t) {
    top4_insert(c0, c1, c2, c3, key_c(t));
    top4_insert(r0, r1, r2, r3, key_r(t));
  }
  // L lies between the subset's smallest lane second-largest key (each lane
  // has two keys at least that large: 64 >= k of them), rounded down to 8
  // bits, and the subset's largest key, so it carries their common leading
  // bits and the search starts below them.
  uint32_t Lc, Lr;
  int topc, topr;
  common_prefix(__reduce_min_sync(0xffffffffu, c1) & ~255u, __reduce_max_sync(0xffffffffu, c0), Lc, topc);
  common_prefix(__reduce_min_sync(0xffffffffu, r1) & ~255u, __reduce_max_sync(0xffffffffu, r0), Lr, topr);
#pragma unroll 1
  for (int bit = max(topc, topr); bit >= 8; --bit) {
    const uint32_t xc = Lc | (1u << bit), xr = Lr | (1u << bit);
    int nc, nr;
    sum2((c0 >= xc) + (c1 >= xc) + (c2 >= xc) + (c3 >= xc), (r0 >= xr) + (r1 >= xr) + (r2 >= xr) + (r3 >= xr), nc,
         nr);
    if (bit <= topc && nc >= k_c) Lc = xc;
    if (bit <= topr && nr >= k_r) Lr = xr;
  }
  // Every float's key but one NaN pattern is >= 256, so L > 0 and no absent
  // slot (key 0) becomes a candidate.
  return topk2_from_bounds(key_c, key_r, Lc, Lr, k_c, k_r, nt, lane, nwords, scratch, words_c, words_r);
}

// The row's mask words (and forced blocks) -> the mask arrays and the row's
// union count.  Warp-wide.
__device__ __forceinline__ void emit_row(const SelectArgs& a, const uint32_t* words_c, const uint32_t* words_r,
                                         int64_t row, int lane, int gi) {
  int cnt = 0;
  for (int t = lane; t < a.nwords; t += 32) {
    const uint32_t wc = words_c[t], wr = words_r[t];
    uint32_t f = 0;
    if (a.force_diag && gi < a.nkb && (gi >> 5) == t) f |= 1u << (gi & 31);
    if (a.force_sink && t == 0) f |= 1u;
    cnt += __popc(wc | wr | f);
    a.mask_c[row * a.nwords + t] = wc;
    a.mask_r[row * a.nwords + t] = wr;
  }
  cnt = __reduce_add_sync(0xffffffffu, cnt);
  if (lane == 0) {
    a.counts[row] = cnt;
    if (a.tile_sums != nullptr) atomicAdd(a.tile_sums + row / kScanTile, cnt);
  }
}

// The full 32-step bitwise search of both branches (the last fallback: k > 64
// or many equal keys), into the mask words.  Warp-wide.
template <int KP, typename KC, typename KR>
__device__ __noinline__ void select_row_full(KC key_c, KR key_r, int k_c, int k_r, int lane, int nwords,
                                             uint32_t* words_c, uint32_t* words_r) {
  uint32_t kc[KP], kr[KP];
#pragma unroll
  for (int t = 0; t < KP; ++t) {
    kc[t] = key_c(t);
    kr[t] = key_r(t);
  }
  constexpr int NO = (KP + 31) / 32;
  uint32_t own_c[NO], own_r[NO];
  warp_topk2<KP>(kc, kr, k_c, k_r, lane, own_c, own_r);
  for (int w = lane; w < nwords; w += 32) {
    const bool mine = w < KP;  // word w is owned by lane w % 32 as own[w / 32]
    words_c[w] = mine ? own_c[(w >> 5) < NO ? (w >> 5) : 0] : 0u;
    words_r[w] = mine ? own_r[(w >> 5) < NO ? (w >> 5) : 0] : 0u;
  }
  __syncwarp();
}

// Both branches' top-k (TOPK_FRACTION) of one list row from order-preserving
// keys: key_c(t), key_r(t) = the keys of block 32t + lane (0 past the n
// visible blocks); KP slots per lane, mask words covering nwords <=
// (KPMAX + 31) / 32 * 32 words.  Warp-wide.
template <int KP, int KPMAX, typename KC, typename KR>
__device__ __forceinline__ void select_row_keys(const SelectArgs& a, KC key_c, KR key_r, int64_t row, int lane,
                                                int gi, int n, uint32_t* scratch) {
  uint32_t* words_c = scratch + 4 * kTopkCap;
  uint32_t* words_r = words_c + a.nwords;
  const int k_c = keep_count(a.rho_c, n), k_r = keep_count(a.rho_r, n);
  // the fallbacks (rare) are separate functions, out of the hot path's code
  const bool done =
      warp_topk2_sorted<KP>(key_c, key_r, k_c, k_r, n, lane, a.nwords, scratch, words_c, words_r) ||
      warp_topk2_pruned<KP>(key_c, key_r, k_c, k_r, n, lane, a.nwords, scratch, words_c, words_r);
  if (!done) select_row_full<KP>(key_c, key_r, k_c, k_r, lane, a.nwords, words_c, words_r);
  emit_row(a, words_c, words_r, row, lane, gi);
}

// Both branches' selection of one list row (warp-wide) -> mask words and the
// row's union count.  score_c(j), score_r(j) give the branches' scores of the
// visible block j < n; the top-k runs on KP key slots per lane.
template <int KP, int KPMAX, typename SC, typename SR>
__device__ __forceinline__ void select_row(const SelectArgs& a, SC score_c, SR score_r, int64_t row, int lane,
                                           int gi, int n, uint32_t* scratch) {
  if (a.threshold_mode == 1) {
    // Each branch keeps every visible block scoring at least its row maximum
    // minus delta; the threshold is formed in fp32 from the maximum score.
    uint32_t* words_c = scratch + 4 * kTopkCap;
    uint32_t* words_r = words_c + a.nwords;
    float mc = -INFINITY, mr = -INFINITY;
    for (int j = lane; j < n; j += 32) {
      mc = fmaxf(mc, score_c(j));
      mr = fmaxf(mr, score_r(j));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, o));
      mr = fmaxf(mr, __shfl_xor_sync(0xffffffffu, mr, o));
    }
    const uint32_t tc = order_key(mc - a.delta_c), tr = order_key(mr - a.delta_r);
    for (int w = lane; w < a.nwords; w += 32) {
      uint32_t wc = 0, wr = 0;
      for (int bit = 0; bit < 32; ++bit) {
        const int j = 32 * w + bit;
        if (j < n) {
          if (order_key(score_c(j)) >= tc) wc |= 1u << bit;
          if (order_key(score_r(j)) >= tr) wr |= 1u << bit;
        }
      }
      words_c[w] = wc;
      words_r[w] = wr;
    }
    __syncwarp();
    emit_row(a, words_c, words_r, row, lane, gi);
    return;
  }
  auto key_c = [&](int t) -> uint32_t {
    const int j = 32 * t + lane;
    return j < n ? order_key(score_c(j)) : 0u;
  };
  auto key_r = [&](int t) -> uint32_t {
    const int j = 32 * t + lane;
    return j < n ? order_key(score_r(j)) : 0u;
  };
  select_row_keys<KP, KPMAX>(a, key_c, key_r, row, lane, gi, n, scratch);
}

// The mean-pooled scores of row `warp` of the CTA's item:
//   s_c(j) = sc[warp][j], s_r(j) = s_c(j) + |qbar| r_j beta_j.
template <int KP, int KPMAX>
__device__ __forceinline__ void select_topk_row(const SelectArgs& a, const float* sc, const float* rb, float qnv,
                                                int warp, int lane, int hq0, int b, int i, int gi, int n, int npad,
                                                uint32_t* scratch) {
  const int64_t row = (static_cast<int64_t>(b) * a.Hq + hq0 + warp) * a.nqb + i;
  const float* srow = sc + warp * npad;
  select_row<KP, KPMAX>(
      a, [&](int j) { return srow[j]; }, [&](int j) { return fmaf(qnv, rb[j], srow[j]); }, row, lane, gi, n,
      scratch);
}

// Work item w -> (batch, query block, first q head): longest rows first.
__device__ __forceinline__ void sel_item(const SelectArgs& a, int w, int& b, int& i, int& hq0) {
  const int nh = a.Hq / a.R;
  const int per_i = a.B * nh;
  i = a.nqb - 1 - w / per_i;
  const int rem = w % per_i;
  b = rem / nh;
  hq0 = (rem % nh) * a.R;
}

// Dot products of one 16-dim slice of the staged tile with the pooled
// queries: NP head pairs, the thread's block jA and, when TWO, jB = jA + 256.
template <int NP, bool TWO>
__device__ __forceinline__ void score_slice(const float* cs, const float* qd, int jA, float2 (&accA)[4],
                                            float2 (&accB)[4]) {
  const int jB = jA + 256;
  const float* rowA = cs + jA * kStageD;
  const float* rowB = cs + jB * kStageD;
  const int swA = (jA >> 1) & 3, swB = (jB >> 1) & 3;
#pragma unroll
  for (int dq = 0; dq < kStageD / 4; ++dq) {
    const float4 cA = *reinterpret_cast<const float4*>(rowA + 4 * (dq ^ swA));
    float4 cB = make_float4(0.f, 0.f, 0.f, 0.f);
    if (TWO) cB = *reinterpret_cast<const float4*>(rowB + 4 * (dq ^ swB));
    const float ca[4] = {cA.x, cA.y, cA.z, cA.w}, cb[4] = {cB.x, cB.y, cB.z, cB.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float* q = qd + (4 * dq + e) * kSelMaxR;
      const float4 q0 = *reinterpret_cast<const float4*>(q);
      const float2 xa = make_float2(ca[e], ca[e]), xb = make_float2(cb[e], cb[e]);
      accA[0] = ffma2(make_float2(q0.x, q0.y), xa, accA[0]);
      accA[1] = ffma2(make_float2(q0.z, q0.w), xa, accA[1]);
      if (TWO) {
        accB[0] = ffma2(make_float2(q0.x, q0.y), xb, accB[0]);
        accB[1] = ffma2(make_float2(q0.z, q0.w), xb, accB[1]);
      }
      if (NP > 2) {
        const float4 q1 = *reinterpret_cast<const float4*>(q + 4);
        accA[2] = ffma2(make_float2(q1.x, q1.y), xa, accA[2]);
        accA[3] = ffma2(make_float2(q1.z, q1.w), xa, accA[3]);
        if (TWO) {
          accB[2] = ffma2(make_float2(q1.x, q1.y), xb, accB[2]);
          accB[3] = ffma2(make_float2(q1.z, q1.w), xb, accB[3]);
        }
      }
    }
  }
}

template <int KPL, int BQ>
__global__ void __launch_bounds__(kSelThreads, KPL <= 32 ? 2 : 1)
    select_rows_kernel(const __grid_constant__ CUtensorMap qmap, SelectArgs a) {
  extern __shared__ __align__(128) uint8_t sel_smem[];
  __shared__ __align__(8) uint64_t full_bar[kPoolStages];
  __shared__ float qn_s[2][kSelMaxR];
  __shared__ int abort_flag;
  uint8_t* qring = sel_smem;
  float* cs = reinterpret_cast<float*>(sel_smem + kSelOffCs);
  float* qs_all = reinterpret_cast<float*>(sel_smem + kSelOffQs);  // [2][128 dims][8 heads]
  const int npad = (a.nkb + 31) & ~31;
  float* rb = reinterpret_cast<float*>(sel_smem + kSelOffRb);  // [npad]  r_j * beta_j
  float* sc = rb + npad;                                        // [8][npad] centroid-branch scores

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int R = a.R;
  const int G = a.Hq / a.Hkv;
  const int nitems = a.items > static_cast<int>(blockIdx.x)
                         ? (a.items - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                         : 0;
  constexpr int kChunks = BQ / kPoolRows;

  if (tid == 0) {
    for (int s = 0; s < kPoolStages; ++s) mbar_init(smem_u32(&full_bar[s]), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  for (int o = tid; o < 2 * 128 * kSelMaxR; o += kSelThreads) qs_all[o] = 0.f;  // heads >= R stay 0
  __syncthreads();

  if (warp >= kSelComputeThreads / 32) {
    // ===== pooling warps: item k's query block, while item k - 1 is scored.
    // Chunk g = k * kChunks + c holds rows c * 8 .. c * 8 + 7 of item k's
    // query block for its R heads, d 0-63 then d 64-127, in stage g % 2.
    const int ptid = tid - kSelComputeThreads;
    const int h = ptid >> 3, dq = ptid & 7;  // head, 16-dim group of this thread
    const int total = nitems * kChunks;
    const uint32_t chunk_bytes = static_cast<uint32_t>(kPoolRows * R * 128 * 2);
    int issued = 0;
    auto issue = [&](int g) {
      const int k = g / kChunks, c = g % kChunks;
      int b, i, hq0;
      sel_item(a, static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x), b, i, hq0);
      const int s = g % kPoolStages;
      const uint32_t bar = smem_u32(&full_bar[s]);
      const uint32_t dst = smem_u32(qring + s * kPoolChunkBytes);
      const int row0 = i * BQ + c * kPoolRows;
      const int c1 = a.seq_inner ? row0 : hq0, c2 = a.seq_inner ? hq0 : row0;
      mbar_arrive_expect_tx(bar, chunk_bytes);
      tma_load_4d(dst, &qmap, bar, 0, c1, c2, b);
      tma_load_4d(dst + chunk_bytes / 2, &qmap, bar, 64, c1, c2, b);
      issued = g + 1;
    };
    if (ptid == 0) {
      tma_prefetch_desc(&qmap);
      for (int g = 0; g < kPoolStages && g < total; ++g) issue(g);
    }
    // element offset of this thread's 16 dims of row r: [half][row][head][64]
    // for token-major Q, [half][head][row][64] for head-major Q.  Threads of
    // the upper half read their two 16-byte pieces in the other order, so a
    // quarter warp covers all banks.
    const int hoff = (dq >> 2) * (kPoolRows * R * 64) + (a.seq_inner ? h * kPoolRows * 64 : h * 64) + (dq & 3) * 16;
    const int rstride = a.seq_inner ? 64 : R * 64;
    const int p0 = (dq >> 2) * 8, p1 = 8 - p0;  // element offsets of the two pieces, in reading order
    for (int k = 0; k < nitems; ++k) {
      float acc[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) acc[e] = 0.f;
      for (int c = 0; c < kChunks; ++c) {
        const int g = k * kChunks + c, s = g % kPoolStages;
        const bool ok = mbar_wait(smem_u32(&full_bar[s]), static_cast<uint32_t>((g / kPoolStages) & 1), &abort_flag);
        if (ok && h < R) {
          const __nv_bfloat16* chunk = reinterpret_cast<const __nv_bfloat16*>(qring + s * kPoolChunkBytes) + hoff;
#pragma unroll
          for (int r = 0; r < kPoolRows; ++r) {
            const uint4 v0 = *reinterpret_cast<const uint4*>(chunk + r * rstride + p0);
            const uint4 v1 = *reinterpret_cast<const uint4*>(chunk + r * rstride + p1);
            const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              acc[2 * q] += bf16lo(w[q]);
              acc[2 * q + 1] += bf16hi(w[q]);
            }
          }
        }
        named_bar_sync(2, kSelPoolThreads);  // stage s is free
        if (ptid == 0 && g + kPoolStages < total && !abort_flag) issue(g + kPoolStages);
      }
      float* qs = qs_all + (k & 1) * 128 * kSelMaxR;
      int ib, ii, ih;
      sel_item(a, static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x), ib, ii, ih);
      const int nq = min(BQ, a.Lq - ii * BQ);  // rows past Lq were loaded as zeros
      const float inv_n = nq == BQ ? 1.0f / BQ : 1.0f / nq;
      float s2 = 0.f;
      if (h < R) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          // acc[e] is dim 16 dq + e of the first piece read, then the second
          const int d = 16 * dq + (e < 8 ? p0 : p1) + (e & 7);
          const float m = acc[e] * inv_n;
          qs[d * kSelMaxR + h] = m;
          s2 = fmaf(m, m, s2);
        }
      }
#pragma unroll
      for (int o = 4; o >= 1; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);  // the 8 threads of head h
      if (dq == 0 && h < R) qn_s[k & 1][h] = sqrtf(s2);
      __syncthreads();  // item k pooled; item k - 1 scored
    }
    __syncthreads();  // the last item scored
    if (ptid == 0 && abort_flag) {
      // after a timeout, wait (bounded) for the chunks still in flight
      for (int g = issued - kPoolStages; g < issued; ++g)
        if (g >= 0) mbar_drain(smem_u32(&full_bar[g % kPoolStages]), static_cast<uint32_t>((g / kPoolStages) & 1));
    }
    return;
  }

  // ===== scoring and top-k warps
  __syncthreads();  // item 0 pooled
  constexpr int kSlices = 128 / kStageD;
  constexpr int kLoads = kStageJ * kStageD / 4 / kSelComputeThreads;  // float4 per thread per stage
  for (int k = 0; k < nitems; ++k) {
    int b, i, hq0;
    sel_item(a, static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x), b, i, hq0);
    const int kvh = hq0 / G;
    const int gi = i + a.q_block_offset;
    const int n = a.causal ? min(a.nkb, gi + 1) : a.nkb;
    const int64_t kv_off = static_cast<int64_t>(b * a.Hkv + kvh) * a.nkb;
    const float* qs = qs_all + (k & 1) * 128 * kSelMaxR;
    for (int j = tid; j < n; j += kSelComputeThreads) rb[j] = a.rad[kv_off + j] * a.beta[kv_off + j];

    // ---- s_c for j < n: tile of 512 blocks x 16 dims per stage; thread t
    // owns blocks j0 + t and j0 + t + 256.  Stage st + 1's global loads are
    // in flight while stage st is used.
    const float* Cb = a.C + kv_off * 128;
    const int nstages = ((n + kStageJ - 1) / kStageJ) * kSlices;
    float4 pre[kLoads];
    auto load_stage = [&](int st) {
      const int j0 = (st / kSlices) * kStageJ, d0 = (st % kSlices) * kStageD;
      const int jn = min(kStageJ, n - j0);
#pragma unroll
      for (int u = 0; u < kLoads; ++u) {
        const int idx = tid + kSelComputeThreads * u;
        const int jl = idx >> 2, q4 = idx & 3;
        pre[u] = jl < jn ? *reinterpret_cast<const float4*>(Cb + static_cast<int64_t>(j0 + jl) * 128 + d0 + 4 * q4)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    };
    float2 accA[4], accB[4];
    load_stage(0);
    for (int st = 0; st < nstages; ++st) {
      const int j0 = (st / kSlices) * kStageJ, d0 = (st % kSlices) * kStageD;
      const int jn = min(kStageJ, n - j0);
      if (d0 == 0) {
#pragma unroll
        for (int p = 0; p < 4; ++p) accA[p] = accB[p] = make_float2(0.f, 0.f);
      }
      named_bar_sync(1, kSelComputeThreads);  // the previous stage is consumed
#pragma unroll
      for (int u = 0; u < kLoads; ++u) {
        const int idx = tid + kSelComputeThreads * u;
        const int jl = idx >> 2, q4 = idx & 3;
        *reinterpret_cast<float4*>(cs + jl * kStageD + 4 * (q4 ^ ((jl >> 1) & 3))) = pre[u];
      }
      named_bar_sync(1, kSelComputeThreads);  // this stage is visible
      if (st + 1 < nstages) load_stage(st + 1);
      const float* qd = qs + d0 * kSelMaxR;
      if (tid < jn) {
        if (jn > 256) {
          if (R > 4) score_slice<4, true>(cs, qd, tid, accA, accB);
          else score_slice<2, true>(cs, qd, tid, accA, accB);
        } else {
          if (R > 4) score_slice<4, false>(cs, qd, tid, accA, accB);
          else score_slice<2, false>(cs, qd, tid, accA, accB);
        }
      }
      if (d0 + kStageD == 128) {
#pragma unroll
        for (int hh = 0; hh < kSelMaxR; ++hh) {
          if (hh < R) {
            const float va = (hh & 1) ? accA[hh >> 1].y : accA[hh >> 1].x;
            const float vb = (hh & 1) ? accB[hh >> 1].y : accB[hh >> 1].x;
            if (tid < jn) sc[hh * npad + j0 + tid] = va;
            if (tid + 256 < jn) sc[hh * npad + j0 + tid + 256] = vb;
          }
        }
      }
    }
    named_bar_sync(1, kSelComputeThreads);  // scores complete; the staging tile is free

    // ---- per-branch top-k (both branches together), one warp per row, with
    // as few key slots per lane as this row needs
    if (warp < R) {
      uint32_t* scratch = reinterpret_cast<uint32_t*>(cs) + warp * sel_topk_scratch_words(a.nwords);
      const float qnv = qn_s[k & 1][warp];
      if (KPL > 2 && n <= 64) select_topk_row<2, KPL>(a, sc, rb, qnv, warp, lane, hq0, b, i, gi, n, npad, scratch);
      else if (KPL > 8 && n <= 256) select_topk_row<8, KPL>(a, sc, rb, qnv, warp, lane, hq0, b, i, gi, n, npad, scratch);
      else if (KPL > 16 && n <= 512) select_topk_row<16, KPL>(a, sc, rb, qnv, warp, lane, hq0, b, i, gi, n, npad, scratch);
      else if (KPL > 32 && n <= 1024) select_topk_row<32, KPL>(a, sc, rb, qnv, warp, lane, hq0, b, i, gi, n, npad, scratch);
      else if (KPL > 64 && n <= 2048) select_topk_row<64, KPL>(a, sc, rb, qnv, warp, lane, hq0, b, i, gi, n, npad, scratch);
      else select_topk_row<KPL, KPL>(a, sc, rb, qnv, warp, lane, hq0, b, i, gi, n, npad, scratch);
    }
    __syncthreads();  // item k done; item k + 1 pooled
  }
}

// Exclusive scan of the tile sums (one CTA of 1024 threads; each thread owns
// a contiguous run of tiles) into tile_prefix, and the total into
// row_ptr[rows].  The row pointers themselves are formed by the compaction.
__global__ void __launch_bounds__(1024) scan_tiles_kernel(const int* __restrict__ tile_sums, int ntiles,
                                                          int* __restrict__ tile_prefix, int* __restrict__ row_ptr,
                                                          int rows, int64_t capacity) {
  __shared__ long long wsum[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (ntiles + 1023) / 1024;
  const int s0 = min(ntiles, tid * per), s1 = min(ntiles, s0 + per);
  long long local = 0;
  for (int t = s0; t < s1; ++t) local += tile_sums[t];
  long long incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const long long w = wsum[lane];
    long long wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long x = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += x;
    }
    wsum[lane] = wi - w;
  }
  __syncthreads();
  long long run = wsum[warp] + incl - local;
  for (int t = s0; t < s1; ++t) {
    tile_prefix[t] = static_cast<int>(run);
    run += tile_sums[t];
  }
  if (tid == 1023) {
    row_ptr[rows] = static_cast<int>(run);
    if (run > capacity || run > 0x7fffffffll) raise_error(RBS_DEVERR_ROW_PTR);
  }
}

struct CompactArgs {
  const uint32_t* mask_c;  // [B * Hq * nqb, nwords], one row per q head
  const uint32_t* mask_r;
  int32_t* col_idx;
  uint8_t* flags;
  int64_t capacity;
  int rows, nqb, nkb, nwords, q_block_offset, force_diag, force_sink;
  int Hq, Hl, glist;  // list row (b, hl, i) = union of q heads hl * glist .. + glist - 1
};

// Forced-block bits of mask word t of a row whose global query block is gi.
__device__ __forceinline__ uint32_t forced_word(int t, int gi, int nkb, int force_diag, int force_sink) {
  uint32_t f = 0;
  if (force_diag && gi < nkb && (gi >> 5) == t) f |= 1u << (gi & 31);
  if (force_sink && t == 0) f |= 1u;
  return f;
}

// Mask word t of list row (b, hl, i): the OR over the row's q heads.
__device__ __forceinline__ void list_row_word(const CompactArgs& a, int b, int hl, int i, int t, uint32_t& c,
                                              uint32_t& r) {
  if (a.glist == 1) {  // one list per q head: the list row is the mask row
    const int64_t m = ((static_cast<int64_t>(b) * a.Hq + hl) * a.nqb + i) * a.nwords + t;
    c = a.mask_c[m];
    r = a.mask_r[m];
    return;
  }
  c = r = 0;
  for (int hh = 0; hh < a.glist; ++hh) {
    const int64_t m = ((static_cast<int64_t>(b) * a.Hq + hl * a.glist + hh) * a.nqb + i) * a.nwords + t;
    c |= a.mask_c[m];
    r |= a.mask_r[m];
  }
}

// KV_GROUP lists: the entry count of every list row (b, g, i).
__global__ void __launch_bounds__(256) group_counts_kernel(CompactArgs a, int* __restrict__ counts,
                                                           int* __restrict__ tile_sums) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= a.rows) return;
  const int i = row % a.nqb, bh = row / a.nqb;
  const int b = bh / a.Hl, hl = bh % a.Hl;
  const int gi = i + a.q_block_offset;
  int cnt = 0;
  for (int t = lane; t < a.nwords; t += 32) {
    uint32_t c, r;
    list_row_word(a, b, hl, i, t, c, r);
    cnt += __popc(c | r | forced_word(t, gi, a.nkb, a.force_diag, a.force_sink));
  }
  cnt = __reduce_add_sync(0xffffffffu, cnt);
  if (lane == 0) {
    counts[row] = cnt;
    atomicAdd(tile_sums + row / kScanTile, cnt);
  }
}

// One warp per list row: its row pointer (the tile's prefix plus the counts
// of the tile's earlier rows) and its entries.
__global__ void __launch_bounds__(256) compact_lists_kernel(CompactArgs a, const int* __restrict__ counts,
                                                            const int* __restrict__ tile_prefix,
                                                            int* __restrict__ row_ptr) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= a.rows) return;
  const int i = row % a.nqb, bh = row / a.nqb;
  const int b = bh / a.Hl, hl = bh % a.Hl;
  const int gi = i + a.q_block_offset;
  // the row's first mask words are loaded together with its extent
  uint32_t c0 = 0, r0 = 0;
  if (lane < a.nwords) list_row_word(a, b, hl, i, lane, c0, r0);
  const int t0 = row - row % kScanTile;
  int before = 0;  // counts of rows t0 .. row - 1
#pragma unroll
  for (int u = 0; u < kScanTile / 32; ++u) {
    const int r = t0 + u * 32 + lane;
    before += r < row ? counts[r] : 0;
  }
  before = __reduce_add_sync(0xffffffffu, before);
  const long long beg64 = static_cast<long long>(tile_prefix[row / kScanTile]) + before;
  const long long end64 = beg64 + counts[row];
  if (end64 > a.capacity || end64 > 0x7fffffffll) {
    if (lane == 0) raise_error(RBS_DEVERR_ROW_PTR);
    return;
  }
  const int beg = static_cast<int>(beg64), end = static_cast<int>(end64);
  if (lane == 0) row_ptr[row] = beg;
  int run = beg;
  for (int w0 = 0; w0 < a.nwords; w0 += 32) {
    const int t = w0 + lane;
    uint32_t c = 0, r = 0, f = 0;
    if (t < a.nwords) {
      if (w0 == 0) {
        c = c0;
        r = r0;
      } else {
        list_row_word(a, b, hl, i, t, c, r);
      }
      f = forced_word(t, gi, a.nkb, a.force_diag, a.force_sink);
    }
    uint32_t u = c | r | f;
    const int cnt = __popc(u);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int pos = run + incl - cnt;
    while (u) {
      const int bit = __ffs(u) - 1;
      u &= u - 1;
      if (pos < end) {
        a.col_idx[pos] = 32 * t + bit;
        if (a.flags != nullptr)
          a.flags[pos] = static_cast<uint8_t>(((c >> bit) & 1u) | (((r >> bit) & 1u) << 1) | (((f >> bit) & 1u) << 2));
      }
      ++pos;
    }
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0 && run != end) raise_error(RBS_DEVERR_ROW_PTR);
}

}  // namespace rbs
