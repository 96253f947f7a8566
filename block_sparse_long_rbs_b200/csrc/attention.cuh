// Block-sparse prefill attention on the 5th-generation tensor core.
// ([RBS-en] "The Fix": exact softmax attention over the selected key blocks,
// compatible with standard multi-head / grouped-query attention;
// [QUILT] Abstract: query tiles that select the same key blocks share their
// loads; [BA] 2.4 Block fine-tune: the Block-attention token mask.)
//
// Work item = a PAIR of list rows (a row is one (batch, q head, query block):
// a 128-row query tile against the row's listed key blocks).  The rows of a
// pair are consecutive in a work order that keeps one KV head's rows together
// and, within it, starts with the last query blocks (the longest causal rows):
// normally two q heads of one KV head at the same query block.  Persistent
// CTAs take pairs round-robin.
//
// Two query tiles per CTA ("slots" 0 and 1), each with its own S and O in
// TMEM, so the tensor core works on one slot's tile while the softmax warps
// of the other slot work on theirs (ping-pong).  The two rows' key-block
// lists are walked as ONE merged stream in ascending block order: a block
// both rows list (same batch and KV head) is loaded once and feeds both
// slots' S = Q K^T and O += P V products; a block only one row lists feeds
// that slot alone.  Every role walks the same merged stream, so they agree
// on the order without exchanging it.
//
// Roles (384 threads):
//   warps 0-3  softmax of slot 0, warps 4-7 softmax of slot 1: one thread per
//              query row (TMEM lane), all BK columns of S.  Per tile: load S,
//              apply the masks (causal diagonal, keys past Lk, the token-level
//              segment bound, dead tiles), take the row max, lazily update
//              the running max m (O rescaled in TMEM only when it grows by
//              more than 2^8; the final normalisation uses the same m, so the
//              result is exact), form P = exp2(S*c - m) (3 of every 8 element
//              pairs on the FMA pipe, see exp2_fma2, the rest on the SFU),
//              write P as packed bf16 pairs over the first BK/2 columns of the
//              slot's S.  A tile of a rescue-only block whose contribution is
//              weighted by w has log2(w) added to its scaled scores.  At the
//              end of a row: O / l -> bf16, and the LSE.
//   warp 8     Q and K producer, warp 9 V producer (one thread each): TMA
//              loads of the slots' Q tiles and of the merged stream's K / V
//              tiles, gathered by block index (4-D tensor maps over
//              [B, L, H, 128], 128B swizzle, no multicast) into 2-deep rings.
//   warp 10    TMEM allocator and S issuer, warp 11 PV issuer (each warp runs
//              its loop; one elected lane issues):
//                S_s  = Q_s K_u^T    A = Q_s (smem), B = K_u (smem)
//                O_s += P_s V_u      A = P_s (TMEM), B = V_u (MN-major smem)
//              for each slot s that step u of the merged stream feeds.  S_s
//              of a slot's next tile overwrites its P, so the S issuer waits
//              for that slot's previous PV; otherwise the two issuers run
//              independently.  A ring stage is refilled when the issuer that
//              read it commits the stage's "empty" barrier.
// TMEM columns: S_0 [0, 128), S_1 [128, 256), O_0 [256, 384), O_1 [384, 512).
//
// Every mbarrier wait is bounded (a.wait_ns); on a timeout all roles unwind,
// in-flight TMA loads and MMAs are drained (bounded), TMEM is freed, and the
// device error word records RBS_DEVERR_TIMEOUT.  No named barriers are used
// after set-up, so an aborting warp can never strand another.
#pragma once

#include "common.cuh"

namespace rbs {

struct AttnArgs {
  CUtensorMap tmQ, tmK, tmV;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  int64_t capacity;
  __nv_bfloat16* O;
  int64_t ob, os, oh;
  float* lse;
  int B, Hq, Hkv, nqb, nkb, Lq;
  int k_tail;  // keys in the last key block (BK unless Lk is not a block multiple)
  int q_block_off, causal, num_rows;  // num_rows: B * Hq * nqb list rows to compute
  int group_lists;  // 1: list row (b, KV head, i) serves every q head of the KV head
  // rescue blocks weighted by w: entries whose flags are exactly "rescue
  // branch only" get log2(w) added to their logits (in log2 units); flags is
  // null when every block has weight 1
  const uint8_t* flags;
  float rescue_bias;
  float scale_log2;
  uint64_t wait_ns;  // time limit of every pipeline wait
  int stall_after;   // testing only: the K producer stops after this many tiles (< 0: never)
  // Block-attention token mask ([BA] 2.4): a query at key position p <
  // seg_final sees only keys at or after the start of its passage (the last
  // seg_start <= p); seg_n == 0 disables it
  int seg_n, seg_final;
  int seg_start[RBS_MAX_SEGMENTS];
};

constexpr int kAttnThreads = 384;
constexpr int kNS = 2;  // K and V ring depth
// Registers per thread after set-up.  The block is launched with 168 per
// thread (384 x 168 = 64512); the producer / issuer warpgroup gives part of
// its share to the two softmax warpgroups, which hold up to 96 values of a
// row of S each: 128 x 120 + 256 x 192 = 64512.  The host refuses to launch
// a build whose register count per thread makes the block's total smaller
// than that sum (the softmax warpgroups' increase would never be granted).
constexpr uint32_t kRegsLaunch = 168, kRegsIO = 120, kRegsSoftmax = 192;
constexpr uint32_t kRegsSplitTotal = 128 * kRegsIO + 256 * kRegsSoftmax;
static_assert(kRegsSplitTotal <= kAttnThreads * kRegsLaunch, "register split");

// Software base-2 exponential of two values at once, on the FMA pipe:
// Cody-Waite range reduction 2^x = 2^n * 2^f, n = rint(x) (via the 1.5*2^23
// shifter), f = x - n in [-1/2, 1/2], then p(f) = 1 + c1 f + c2 f^2 + c3 f^3,
// a degree-3 fit by the Remez exchange algorithm for minimum relative error
// (max 4.315e-4; csrc/exp2_poly_fit.py derives the coefficients).  The
// exponent n is added to p's exponent field.  Inputs are clamped at -127, where
// the result is +0 (p(0) = 1 exactly); inputs above 127 are not expected
// (the running max keeps them at or below 8).  Below -126 the sum leaves the
// normal range and the result is only within 2^-126 of 2^x (absolute).
constexpr float kExp2C1 = 0.6957668f;
constexpr float kExp2C2 = 0.24203052f;
constexpr float kExp2C3 = 0.04169875f;

__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  x.x = fmaxf(x.x, -127.f);
  x.y = fmaxf(x.y, -127.f);
  const float2 t = fadd2(x, make_float2(12582912.f, 12582912.f));
  const float2 n = fadd2(t, make_float2(-12582912.f, -12582912.f));
  const float2 f = ffma2(n, make_float2(-1.f, -1.f), x);
  float2 p = ffma2(make_float2(kExp2C3, kExp2C3), f, make_float2(kExp2C2, kExp2C2));
  p = ffma2(p, f, make_float2(kExp2C1, kExp2C1));
  p = ffma2(p, f, make_float2(1.f, 1.f));
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

// The software exponential over an array, for the library's tests: y[i] =
// exp2_fma2(x[i]), two elements per thread.
__global__ void __launch_bounds__(256) exp2_test_kernel(const float* __restrict__ x, float* __restrict__ y,
                                                        int64_t n) {
  const int64_t i = 2 * (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float x1 = i + 1 < n ? x[i + 1] : 0.f;
  const float2 r = exp2_fma2(make_float2(x[i], x1));
  y[i] = r.x;
  if (i + 1 < n) y[i + 1] = r.y;
}

template <int N>
struct integral_c {
  static constexpr int value = N;
};

// Softmax helpers on one 32-column chunk of a thread's row of S.
// Columns c0 + e outside [lo, hi] become -inf.
__device__ __forceinline__ void mask_chunk(uint32_t (&w)[32], int c0, int lo, int hi) {
#pragma unroll
  for (int e = 0; e < 32; ++e)
    if (c0 + e < lo || c0 + e > hi) w[e] = __float_as_uint(-INFINITY);
}

__device__ __forceinline__ float max_chunk(const uint32_t (&w)[32]) {
  float m0 = __uint_as_float(w[0]);
#pragma unroll
  for (int e = 1; e < 31; e += 2) m0 = fmax3(m0, __uint_as_float(w[e]), __uint_as_float(w[e + 1]));
  return fmaxf(m0, __uint_as_float(w[31]));
}

// P = exp2(s * c + nm) of the chunk's 16 column pairs -> packed bf16 pairs in
// out[OFF .. OFF + 15] (out may be w itself: pair k is written after it and
// every earlier pair were read); the values are added into acc.  Pairs 1, 4
// and 6 of every 8 use the FMA-pipe exponential, the rest the SFU.
template <int OFF>
__device__ __forceinline__ void exp_pack_chunk(const uint32_t (&w)[32], uint32_t (&out)[32], float2 c2, float2 nm2,
                                               float2 (&acc)[4]) {
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float2 arg = ffma2(make_float2(__uint_as_float(w[2 * k]), __uint_as_float(w[2 * k + 1])), c2, nm2);
    const int pi = k & 7;
    const float2 p = (pi == 1 || pi == 4 || pi == 6) ? exp2_fma2(arg) : make_float2(ptx_exp2(arg.x), ptx_exp2(arg.y));
    acc[k & 3] = fadd2(acc[k & 3], p);
    out[OFF + k] = pack_bf16x2(p.x, p.y);
  }
}

template <int BK>
struct AttnSmem {
  static constexpr int kQBytes = 128 * 128 * 2;  // one Q tile: 128 rows x 128 dims (two 64-dim halves)
  static constexpr int kKVBytes = BK * 128 * 2;  // BK rows x 128 dims (two halves)
  static constexpr int kQ = 0;                   // Q tiles of slot 0 and slot 1
  static constexpr int kK = kQ + 2 * kQBytes;
  static constexpr int kV = kK + kNS * kKVBytes;
  static constexpr int kSeg = kV + kNS * kKVBytes;  // int [RBS_MAX_SEGMENTS] passage starts
  static constexpr int kBar = kSeg + RBS_MAX_SEGMENTS * 4;
  static constexpr int kBarBytes = 256;
  static constexpr int kTotal = kBar + kBarBytes;
  static constexpr int kAlloc = kTotal + 1024;  // slack to align the base to 1024
  static constexpr uint32_t kTmemCols = 512;
  __host__ __device__ static constexpr uint32_t col_s(int slot) { return slot * 128; }
  // P of keys 16 kk .. 16 kk + 15 (8 packed columns) within a slot's S
  // columns: the keys of each half of the tile sit at the start of that
  // half's S columns (BK = 128: keys 0-63 in columns 0-31, keys 64-127 in
  // columns 64-95), so the S product of one key half never overwrites the
  // other half's P
  static constexpr int kStepsHalf = BK / 32;  // 16-key MMA steps per key half
  __host__ __device__ static constexpr uint32_t col_p(int kk) {
    return (kk / kStepsHalf) * (BK / 2) + (kk % kStepsHalf) * 8;
  }
  __host__ __device__ static constexpr uint32_t col_o(int slot) { return 256 + slot * 128; }
};

// barrier slots (8 bytes each)
enum : int {
  kBarQFull = 0,                  // + slot: the slot's Q tile landed (one phase per row)
  kBarQEmpty = kBarQFull + 2,     // + slot: the row's last S completed
  kBarSFull = kBarQEmpty + 2,     // + slot: S ready (one phase per tile of the slot)
  kBarPFull = kBarSFull + 2,      // + slot: P written (4 warps arrive)
  kBarPVaDone = kBarPFull + 2,    // + slot: the PV product of the tile's first key half completed
  kBarPVbDone = kBarPVaDone + 2,  // + slot: the whole PV product completed
  kBarOFull = kBarPVbDone + 2,    // + slot: the row's last PV completed
  kBarOEmpty = kBarOFull + 2,     // + slot: the epilogue read O (4 warps arrive)
  kBarKFull = kBarOEmpty + 2,     // + stage
  kBarKEmpty = kBarKFull + kNS,   // + stage: the step's S products completed
  kBarVFull = kBarKEmpty + kNS,   // + stage
  kBarVEmpty = kBarVFull + kNS,   // + stage: the step's PV products completed
  kBarDrain = kBarVEmpty + kNS,   // the MMA issuer's last products
  kNumBars = kBarDrain + 1
};
static_assert(kNumBars * 8 + 16 <= 256, "barrier area");

// Work order index w -> (batch, q head, query block) and its list row: batch
// entry, then KV head, then query block from the last (the longest causal
// rows first), then the G q heads sharing that KV head.  The CTAs working at
// the same time therefore read the K/V tiles of one KV head, which fit in L2
// (64 MiB for 131072 tokens), instead of every head's.
__device__ __forceinline__ void decode_work(const AttnArgs& a, int w, int& b, int& h, int& i, int& row) {
  const int G = a.Hq / a.Hkv;
  const int per_b = a.Hq * a.nqb, per_kvh = G * a.nqb;
  b = w / per_b;
  const int rem = w % per_b;
  const int kvh = rem / per_kvh, r2 = rem % per_kvh;
  i = a.nqb - 1 - r2 / G;
  h = kvh * G + r2 % G;
  row = (a.group_lists ? b * a.Hkv + kvh : b * a.Hq + h) * a.nqb + i;
}

// Row extent with validation (identical in every role): -1 for a corrupt row.
__device__ __forceinline__ int row_extent(const AttnArgs& a, int row, int& beg) {
  beg = __ldg(a.row_ptr + row);
  const int end = __ldg(a.row_ptr + row + 1);
  if (beg < 0 || end < beg || end > a.capacity) return -1;
  return end - beg;
}

struct Slot {
  int b, h, i, kvh, beg, n;  // n <= 0: nothing to compute in the main loop
};

struct Pair {
  int p;  // pair index; rows 2p (slot 0) and 2p + 1 (slot 1) of the work order
  Slot s[2];
};

__device__ __forceinline__ Slot load_slot(const AttnArgs& a, int w) {
  Slot s;
  s.b = s.h = s.i = s.kvh = s.beg = 0;
  s.n = 0;
  if (w < a.num_rows) {
    int row;
    decode_work(a, w, s.b, s.h, s.i, row);
    s.kvh = s.h / (a.Hq / a.Hkv);
    s.n = row_extent(a, row, s.beg);
  }
  return s;
}

__device__ __forceinline__ int num_pairs(const AttnArgs& a) { return (a.num_rows + 1) >> 1; }

// The first pair at or after p in this CTA's round-robin order with work.
__device__ __forceinline__ Pair next_pair(const AttnArgs& a, int p) {
  Pair x;
  for (; p < num_pairs(a); p += gridDim.x) {
    x.s[0] = load_slot(a, 2 * p);
    x.s[1] = load_slot(a, 2 * p + 1);
    if (x.s[0].n > 0 || x.s[1].n > 0) break;
  }
  x.p = p;
  return x;
}

// The pair's two lists as one stream.  A block that both rows list next
// (same batch and KV head) is one step feeding both slots.  Otherwise the
// row that has consumed fewer entries goes next, so single-row steps
// alternate between the slots (the tensor core then always has the other
// slot's work while one slot's softmax runs); with equal counts the smaller
// block index goes first, so lists that advance together meet on their
// shared blocks.
struct Merge {
  int n0, n1, beg0, beg1;
  int p0, p1;  // entries of each row consumed
  int j0, j1;  // each row's next entry
  bool share;

  __device__ __forceinline__ void init(const AttnArgs& a, const Pair& x) {
    n0 = max(x.s[0].n, 0);
    n1 = max(x.s[1].n, 0);
    beg0 = x.s[0].beg;
    beg1 = x.s[1].beg;
    p0 = p1 = 0;
    j0 = n0 > 0 ? __ldg(a.col_idx + beg0) : 0;
    j1 = n1 > 0 ? __ldg(a.col_idx + beg1) : 0;
    share = n0 > 0 && n1 > 0 && x.s[0].b == x.s[1].b && x.s[0].kvh == x.s[1].kvh;
  }
  __device__ __forceinline__ bool done() const { return p0 >= n0 && p1 >= n1; }
  // The next step: the slots it feeds (bit s) and its key block.
  __device__ __forceinline__ int step(const AttnArgs& a, int& j) {
    const bool h0 = p0 < n0, h1 = p1 < n1;
    int mask;
    if (h0 && h1) {
      if (share && j0 == j1) mask = 3;
      else if (p0 != p1) mask = p0 < p1 ? 1 : 2;  // the row that is behind: the slots alternate
      else mask = j0 <= j1 ? 1 : 2;
    } else {
      mask = h0 ? 1 : 2;
    }
    j = (mask & 1) ? j0 : j1;
    if (mask & 1) {
      ++p0;
      if (p0 < n0) j0 = __ldg(a.col_idx + beg0 + p0);
    }
    if (mask & 2) {
      ++p1;
      if (p1 < n1) j1 = __ldg(a.col_idx + beg1 + p1);
    }
    return mask;
  }
};

// First key position query position p may see under the segment mask.
__device__ __forceinline__ int segment_key_start(const int* seg, int n, int final_start, int p) {
  if (n <= 0 || p >= final_start) return 0;
  int lo = 0, hi = n - 1;  // the last passage whose start <= p
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (seg[mid] <= p) lo = mid; else hi = mid - 1;
  }
  return seg[lo];
}

template <int BQ, int BK>
__global__ void __launch_bounds__(kAttnThreads, 1) bsa_prefill_kernel(const __grid_constant__ AttnArgs a) {
  using L = AttnSmem<BK>;
  constexpr int kWGWarps = 4;  // barriers a softmax warpgroup completes count one arrival per warp
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + L::kQ;
  const uint32_t sK = sbase + L::kK;
  const uint32_t sV = sbase + L::kV;
  int* seg = reinterpret_cast<int*>(smem + L::kSeg);
  const uint32_t bars = sbase + L::kBar;
  auto bar = [&](int k) -> uint32_t { return bars + 8u * k; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kBar + kNumBars * 8 + 4);
  const uint64_t limit = a.wait_ns;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBarQFull + s), 1);
      mbar_init(bar(kBarQEmpty + s), 1);
      mbar_init(bar(kBarSFull + s), 1);
      mbar_init(bar(kBarPFull + s), kWGWarps);
      mbar_init(bar(kBarPVaDone + s), 1);
      mbar_init(bar(kBarPVbDone + s), 1);
      mbar_init(bar(kBarOFull + s), 1);
      mbar_init(bar(kBarOEmpty + s), kWGWarps);
    }
    for (int s = 0; s < kNS; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarVEmpty + s), 1);
    }
    mbar_init(bar(kBarDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int k = tid; k < a.seg_n; k += kAttnThreads) seg[k] = a.seg_start[k];
  if (BQ < 128) {
    // rows BQ..127 of the Q tiles are never loaded: make them zeros once
    uint4* q4 = reinterpret_cast<uint4*>(smem + L::kQ);
    for (int k = tid; k < 2 * L::kQBytes / 16; k += kAttnThreads) q4[k] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();  // order these writes before the TMA loads into the same tiles
  }
  if (warp == 10) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
  regs_dec<kRegsIO>();  // the whole warpgroup (warps 8-11), before it splits into roles
  if (warp == 8 || warp == 9) {
    // ------------------------------------------------------------ Q+K / V producers
    if (lane == 0) {
      const bool isK = warp == 8;
      const CUtensorMap* map = isK ? &a.tmK : &a.tmV;
      const uint32_t ring = isK ? sK : sV;
      const int full0 = isK ? kBarKFull : kBarVFull;
      const int empty0 = isK ? kBarKEmpty : kBarVEmpty;
      tma_prefetch_desc(map);
      if (isK) tma_prefetch_desc(&a.tmQ);
      uint32_t nf = 0, nq[2] = {0, 0};  // ring fills, Q fills per slot
      bool ok = true;
      for (Pair x = next_pair(a, blockIdx.x); x.p < num_pairs(a) && ok; x = next_pair(a, x.p + gridDim.x)) {
        if (isK) {
#pragma unroll
          for (int s = 0; s < 2; ++s) {
            if (!ok || x.s[s].n <= 0) continue;
            // the slot's previous row must be done with its Q tile (its last
            // S completed); the next phase of that barrier needs this load
            if (nq[s] > 0 && !mbar_wait(bar(kBarQEmpty + s), (nq[s] - 1) & 1, abort_flag, limit)) { ok = false; break; }
            const uint32_t dst = sQ + s * L::kQBytes;
            mbar_arrive_expect_tx(bar(kBarQFull + s), BQ * 256);
            tma_load_4d(dst, &a.tmQ, bar(kBarQFull + s), 0, x.s[s].h, x.s[s].i * BQ, x.s[s].b);
            tma_load_4d(dst + 128 * 128, &a.tmQ, bar(kBarQFull + s), 64, x.s[s].h, x.s[s].i * BQ, x.s[s].b);
            ++nq[s];
          }
          if (!ok) break;
        }
        Merge m;
        m.init(a, x);
        while (!m.done()) {
          if (isK && a.stall_after >= 0 && static_cast<int>(nf) >= a.stall_after) { ok = false; break; }
          int j;
          const int mask = m.step(a, j);
          const bool from0 = mask & 1;  // the K/V head and batch of the slot(s) the step feeds
          const int src_kvh = from0 ? x.s[0].kvh : x.s[1].kvh, src_b = from0 ? x.s[0].b : x.s[1].b;
          if (j < 0 || j >= a.nkb) j = 0;  // the softmax masks such a tile and reports it
          const int st = nf % kNS;
          // the stage's previous step, nf - kNS, must be consumed; the next
          // phase of its empty barrier needs this load, so the parity is
          // unambiguous
          if (nf >= kNS && !mbar_wait(bar(empty0 + st), ((nf / kNS) - 1) & 1, abort_flag, limit)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(full0 + st), BK * 256);
          tma_load_4d(ring + st * L::kKVBytes, map, bar(full0 + st), 0, src_kvh, j * BK, src_b);
          tma_load_4d(ring + st * L::kKVBytes + BK * 128, map, bar(full0 + st), 64, src_kvh, j * BK, src_b);
          ++nf;
        }
      }
      // drain: every load issued must land before the CTA exits.  Stage s was
      // filled at fill numbers s, s + depth, ...; its last fill completes
      // phase (uses - 1).
      for (uint32_t s = 0; s < kNS; ++s)
        if (s < nf) mbar_drain(bar(full0 + s), ((nf - s + kNS - 1) / kNS - 1) & 1, limit);
      if (isK)
        for (int s = 0; s < 2; ++s)
          if (nq[s] > 0) mbar_drain(bar(kBarQFull + s), (nq[s] - 1) & 1, limit);
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------ MMA issuer
    // (the whole warp runs the loop; one elected lane issues each tcgen05
    // instruction).  Order: for each step of the merged stream and each slot
    // it feeds, first the slot's previous tile's PV product, then the slot's
    // S for this step.  With the slots alternating, the tensor core runs
    //   PV_0(t-1)  S_0(t)  PV_1(t-1)  S_1(t)  PV_0(t)  S_0(t+1) ...
    // so each slot's softmax overlaps the other slot's two products.  S and
    // PV are each issued as two key halves; the S of one half waits only for
    // the PV half that read the same TMEM columns, which completes while the
    // other PV half runs.
    constexpr uint32_t idS = idesc_bf16_f32(128, BK / 2, 0, 0);
    constexpr uint32_t idPV = idesc_bf16_f32(128, 128, 0, 1);
    // Descriptors are built once; a buffer or k-step only adds its
    // start-address offset (16-byte units) to the low field (addresses stay
    // below 256 KB: no carry out of the 14-bit field).
    const uint64_t qdesc0 = smem_desc(sQ, 16, 1024, kLayoutSW128);
    const uint64_t kdesc0 = smem_desc(sK, 16, 1024, kLayoutSW128);
    const uint64_t vdesc0 = smem_desc(sV, BK * 128, 1024, kLayoutSW128);
    constexpr uint32_t kQUnits = L::kQBytes >> 4, kStageUnits = L::kKVBytes >> 4;
    constexpr uint32_t kQHalf = (128 * 128) >> 4, kKHalf = (BK * 128) >> 4;
    constexpr uint32_t kKRowsHalf = ((BK / 2) * 128) >> 4;  // the second half of the key rows
    auto wait = [&](int k, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar(k), parity, abort_flag, limit));
    };
    struct PendingPV {
      bool v, first, last;
      uint32_t step;
    };
    PendingPV pv0{false, false, false, 0}, pv1{false, false, false, 0};
    uint32_t ts[2] = {0, 0};  // S products issued per slot (over all rows)
    uint32_t tp[2] = {0, 0};  // PV products issued per slot
    uint32_t rs[2] = {0, 0};  // rows of each slot whose last S was issued (Q tiles used)
    uint32_t ro[2] = {0, 0};  // rows of each slot whose first PV was issued (O used)
    // The pending PV product of slot S.  Its V stage is released once the
    // step's last PV is issued (the other slot may still owe one for the
    // same step).
    auto issue_pv = [&](auto S_) -> bool {
      constexpr int s = decltype(S_)::value;
      PendingPV& p = s == 0 ? pv0 : pv1;
      const PendingPV& o = s == 0 ? pv1 : pv0;
      const uint32_t st = p.step % kNS;
      if (!wait(kBarVFull + st, (p.step / kNS) & 1)) return false;
      if (!wait(kBarPFull + s, tp[s] & 1)) return false;
      // the first PV of a row overwrites O: the previous row's epilogue must
      // have read it
      if (p.first && ro[s] > 0 && !wait(kBarOEmpty + s, (ro[s] - 1) & 1)) return false;
      tc_fence_after();
      const uint64_t vd = vdesc0 + st * kStageUnits;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int k = 0; k < L::kStepsHalf; ++k) {
          const int kk = h * L::kStepsHalf + k;
          umma_ts_warp(tmem + L::col_o(s), tmem + L::col_s(s) + L::col_p(kk), vd + kk * (2048 >> 4), idPV,
                       (p.first && kk == 0) ? 0u : 1u);
        }
        umma_commit_warp(bar((h == 0 ? kBarPVaDone : kBarPVbDone) + s));
      }
      if (p.last) umma_commit_warp(bar(kBarOFull + s));
      if (!(o.v && o.step == p.step)) umma_commit_warp(bar(kBarVEmpty + st));
      if (p.first) ++ro[s];
      ++tp[s];
      p.v = false;
      return true;
    };
    // S of slot S for the step in K stage st.
    auto issue_s = [&](auto S_, uint32_t st, bool first, bool last) -> bool {
      constexpr int s = decltype(S_)::value;
      if (first && !wait(kBarQFull + s, rs[s] & 1)) return false;
      const uint64_t qd = qdesc0 + s * kQUnits;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // S of key half h overwrites that half's P of the slot's previous
        // tile: its PV half must be complete.  That barrier's next phase
        // needs this S, so the parity is exact.
        if (ts[s] > 0 && !wait((h == 0 ? kBarPVaDone : kBarPVbDone) + s, (ts[s] - 1) & 1)) return false;
        tc_fence_after();
        const uint64_t kd = kdesc0 + st * kStageUnits + h * kKRowsHalf;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t offq = (kk >> 2) * kQHalf + (kk & 3) * 2, offk = (kk >> 2) * kKHalf + (kk & 3) * 2;
          umma_ss_warp(tmem + L::col_s(s) + h * (BK / 2), qd + offq, kd + offk, idS, kk > 0 ? 1u : 0u);
        }
      }
      umma_commit_warp(bar(kBarSFull + s));
      if (last) {
        umma_commit_warp(bar(kBarQEmpty + s));
        ++rs[s];
      }
      ++ts[s];
      return true;
    };
    using I0 = integral_c<0>;
    using I1 = integral_c<1>;
    uint32_t g = 0;  // merged steps
    bool ok = true;
    for (Pair x = next_pair(a, blockIdx.x); x.p < num_pairs(a) && ok; x = next_pair(a, x.p + gridDim.x)) {
      Merge m;
      m.init(a, x);
      int tr0 = 0, tr1 = 0;  // tiles of the current row of each slot
      while (ok && !m.done()) {
        int j;
        const int mask = m.step(a, j);
        const uint32_t st = g % kNS;
        // A product still pending from kNS steps back holds the V stage this
        // step's V load needs: issue it first (the older one first).
        const bool old0 = pv0.v && pv0.step + kNS <= g, old1 = pv1.v && pv1.step + kNS <= g;
        if (old0 && old1 && pv1.step < pv0.step) {
          ok = issue_pv(I1{}) && issue_pv(I0{});
        } else {
          if (old0) ok = issue_pv(I0{});
          if (ok && old1) ok = issue_pv(I1{});
        }
        if (!ok || !wait(kBarKFull + st, (g / kNS) & 1)) { ok = false; break; }
        if (mask & 1) {
          if (pv0.v && !issue_pv(I0{})) { ok = false; break; }
          const bool first = tr0 == 0, last = tr0 + 1 == x.s[0].n;
          if (!issue_s(I0{}, st, first, last)) { ok = false; break; }
          pv0 = PendingPV{true, first, last, g};
          ++tr0;
        }
        if (mask & 2) {
          if (pv1.v && !issue_pv(I1{})) { ok = false; break; }
          const bool first = tr1 == 0, last = tr1 + 1 == x.s[1].n;
          if (!issue_s(I1{}, st, first, last)) { ok = false; break; }
          pv1 = PendingPV{true, first, last, g};
          ++tr1;
        }
        umma_commit_warp(bar(kBarKEmpty + st));
        ++g;
      }
    }
    // the last products, the older first
    if (ok && pv0.v && pv1.v && pv1.step < pv0.step) ok = issue_pv(I1{});
    if (ok && pv0.v) ok = issue_pv(I0{});
    if (ok && pv1.v) ok = issue_pv(I1{});
    // drain the outstanding tensor-core work before TMEM is freed
    umma_commit_warp(bar(kBarDrain));
    mbar_drain(bar(kBarDrain), 0, limit);
  }
  } else {
    // ------------------------------------------------------------ softmax (warps 0-7)
    regs_inc<kRegsSoftmax>();  // each softmax warpgroup as a whole
    const int slot = warp >> 2, quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row within the tile == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float c = a.scale_log2;
    auto warp_arrive = [&](int k) {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(k));
    };

    // Rows with no (or a corrupt) list: zeros and LSE = -inf, no pipeline
    // work.  Each of the 256 softmax threads checks one of this CTA's rows
    // (pair p, slot e & 1) per pass; a warp then clears the empty rows it
    // found together.
    for (int base = 0; blockIdx.x + static_cast<int64_t>(gridDim.x) * (base >> 1) < num_pairs(a); base += 256) {
      const int e = base + tid;
      const int64_t w = 2 * (blockIdx.x + static_cast<int64_t>(gridDim.x) * (e >> 1)) + (e & 1);
      int b = 0, h = 0, i = 0, n = 1;
      if (w < a.num_rows) {
        int row, beg;
        decode_work(a, static_cast<int>(w), b, h, i, row);
        n = row_extent(a, row, beg);
        if (n < 0) raise_error(RBS_DEVERR_ROW_PTR);
      }
      for (uint32_t emp = __ballot_sync(0xffffffffu, n <= 0); emp != 0; emp &= emp - 1) {
        const int src = __ffs(emp) - 1;
        const int eb = __shfl_sync(0xffffffffu, b, src), eh = __shfl_sync(0xffffffffu, h, src);
        const int ei = __shfl_sync(0xffffffffu, i, src);
        for (int k = lane; k < BQ * 16; k += 32) {
          const int64_t qrow = static_cast<int64_t>(ei) * BQ + (k >> 4);
          if (qrow < a.Lq)
            reinterpret_cast<uint4*>(a.O + eb * a.ob + qrow * a.os + eh * a.oh)[k & 15] = make_uint4(0, 0, 0, 0);
        }
        if (a.lse != nullptr)
          for (int k = lane; k < BQ; k += 32)
            if (static_cast<int64_t>(ei) * BQ + k < a.Lq)
              a.lse[(static_cast<int64_t>(eb) * a.Hq + eh) * a.Lq + static_cast<int64_t>(ei) * BQ + k] = -INFINITY;
      }
    }

    uint32_t g = 0, item = 0;  // tiles and rows of this slot
    bool ok = true;
    for (Pair px = next_pair(a, blockIdx.x); px.p < num_pairs(a) && ok; px = next_pair(a, px.p + gridDim.x)) {
      const Slot x = slot ? px.s[1] : px.s[0];
      if (x.n <= 0) continue;
      const int n = x.n;
      const int gi = x.i + a.q_block_off;
      // the segment mask's first visible key of this thread's query
      const int key_lo = segment_key_start(seg, a.seg_n, a.seg_final, gi * BK + r);
      float m_used = -INFINITY;  // running max, in log2 units (score * c)
      float2 l2 = make_float2(0.f, 0.f);  // row sum (two partial sums)
      int j_next = __ldg(a.col_idx + x.beg);
      int f_next = a.flags != nullptr ? __ldg(a.flags + x.beg) : 0;
      for (int t = 0; t < n; ++t, ++g) {
        const int j = j_next;
        // log2 weight of this tile: log2(w) for a rescue-only block, else 0
        const float bias = (f_next & 7) == 2 ? a.rescue_bias : 0.f;
        if (t + 1 < n) {
          j_next = __ldg(a.col_idx + x.beg + t + 1);
          if (a.flags != nullptr) f_next = __ldg(a.flags + x.beg + t + 1);
        }
        if (!__all_sync(0xffffffffu, mbar_wait(bar(kBarSFull + slot), g & 1, abort_flag, limit))) { ok = false; break; }
        tc_fence_after();
        const bool bad = j < 0 || j >= a.nkb;
        const bool dead = bad || (a.causal && j > gi);
        const bool diag = a.causal && j == gi;
        const bool tail = j == a.nkb - 1 && a.k_tail < BK;  // keys past Lk were loaded as zeros
        const int lo_col = key_lo - j * BK;                  // columns below are before the passage start
        if (dead && r == 0) raise_error(bad ? RBS_DEVERR_BLOCK_INDEX : RBS_DEVERR_NONCAUSAL);
        // column e of the tile is kept when lo_c <= e <= hi_c
        const bool need_mask = __any_sync(0xffffffffu, dead || diag || tail || lo_col > 0);
        const int lo_c = lo_col;
        int hi_c = dead ? -1 : BK - 1;
        if (diag) hi_c = min(hi_c, r);
        if (tail) hi_c = min(hi_c, a.k_tail - 1);
        const uint32_t sc = lane_base + L::col_s(slot);
        const float2 c2 = make_float2(c, c);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        float factor = 1.f;
        bool rescale = false;
        // The running max after this tile (a lazy update), from the tile's
        // row maximum mx; P is formed against m_exp.
        auto update_max = [&](float mx) -> float {
          const float m_new = fmaxf(m_used, fmaf(mx, c, bias));
          if (t == 0) {
            m_used = m_new;
          } else if (m_new - m_used > 8.f) {
            factor = ptx_exp2(m_used - m_new);
            m_used = m_new;
            rescale = true;
          }
          return m_used == -INFINITY ? 0.f : m_used;
        };
        if constexpr (BK == 128) {
          // Keys 64-127 stay in registers from the max pass to the
          // exponentials; keys 0-63 are read twice (32 columns at a time), so
          // a thread never holds more than 96 values of S.  P of keys 64-127
          // goes to columns 64-95, of keys 0-63 to columns 0-31.
          uint32_t vh[2][32], vc[32];
          tmem_ld32(sc + 64, vh[0]);
          tmem_ld32(sc + 96, vh[1]);
          tmem_ld32(sc, vc);
          tmem_wait_ld();
          if (need_mask) {
            mask_chunk(vh[0], 64, lo_c, hi_c);
            mask_chunk(vh[1], 96, lo_c, hi_c);
            mask_chunk(vc, 0, lo_c, hi_c);
          }
          float mx = fmaxf(fmaxf(max_chunk(vh[0]), max_chunk(vh[1])), max_chunk(vc));
          tmem_ld32(sc + 32, vc);
          tmem_wait_ld();
          if (need_mask) mask_chunk(vc, 32, lo_c, hi_c);
          mx = fmaxf(mx, max_chunk(vc));
          const float m_exp = update_max(mx);
          const float2 nm2 = make_float2(bias - m_exp, bias - m_exp);
          exp_pack_chunk<0>(vh[0], vh[0], c2, nm2, acc);
          exp_pack_chunk<16>(vh[1], vh[0], c2, nm2, acc);
          tmem_st32(sc + 64, vh[0]);
          exp_pack_chunk<16>(vc, vh[1], c2, nm2, acc);  // keys 32-63
          tmem_ld32(sc, vc);                              // keys 0-31 again
          tmem_wait_ld();
          if (need_mask) mask_chunk(vc, 0, lo_c, hi_c);
          exp_pack_chunk<0>(vc, vh[1], c2, nm2, acc);
          tmem_st32(sc, vh[1]);
        } else {
          uint32_t v[2][32];
          tmem_ld32(sc, v[0]);
          tmem_ld32(sc + 32, v[1]);
          tmem_wait_ld();
          if (need_mask) {
            mask_chunk(v[0], 0, lo_c, hi_c);
            mask_chunk(v[1], 32, lo_c, hi_c);
          }
          const float m_exp = update_max(fmaxf(max_chunk(v[0]), max_chunk(v[1])));
          const float2 nm2 = make_float2(bias - m_exp, bias - m_exp);
          exp_pack_chunk<0>(v[0], v[0], c2, nm2, acc);   // keys 0-31 -> columns 0-15
          exp_pack_chunk<0>(v[1], v[1], c2, nm2, acc);   // keys 32-63 -> columns 32-47
          tmem_st16(sc, &v[0][0]);
          tmem_st16(sc + 32, &v[1][0]);
        }
        l2.x *= factor;
        l2.y *= factor;
        l2 = fadd2(l2, fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3])));
        if (__any_sync(0xffffffffu, rescale)) {
          // O is scaled after P is formed, so the wait below overlaps the
          // exponentials.  O must hold every earlier tile's product first;
          // the next phase of that barrier needs this tile's P.
          if (!__all_sync(0xffffffffu, mbar_wait(bar(kBarPVbDone + slot), (g - 1) & 1, abort_flag, limit))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t o[32];
            tmem_ld32(lane_base + L::col_o(slot) + 32 * q, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
            tmem_st32(lane_base + L::col_o(slot) + 32 * q, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        warp_arrive(kBarPFull + slot);
      }
      if (!ok) break;

      // ---- epilogue: O / l -> bf16, LSE
      const float lt = l2.x + l2.y;
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(kBarOFull + slot), item & 1, abort_flag, limit))) { ok = false; break; }
      tc_fence_after();
      const int64_t qrow = static_cast<int64_t>(x.i) * BQ + r;
      uint4* dst = reinterpret_cast<uint4*>(a.O + x.b * a.ob + qrow * a.os + x.h * a.oh);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t o[32];
        tmem_ld32(lane_base + L::col_o(slot) + 32 * q, o);
        tmem_wait_ld();
        if (r < BQ && qrow < a.Lq) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            dst[4 * q + k] = make_uint4(
                pack_bf16x2(__uint_as_float(o[8 * k]) * inv, __uint_as_float(o[8 * k + 1]) * inv),
                pack_bf16x2(__uint_as_float(o[8 * k + 2]) * inv, __uint_as_float(o[8 * k + 3]) * inv),
                pack_bf16x2(__uint_as_float(o[8 * k + 4]) * inv, __uint_as_float(o[8 * k + 5]) * inv),
                pack_bf16x2(__uint_as_float(o[8 * k + 6]) * inv, __uint_as_float(o[8 * k + 7]) * inv));
        }
      }
      if (a.lse != nullptr && r < BQ && qrow < a.Lq) {
        a.lse[(static_cast<int64_t>(x.b) * a.Hq + x.h) * a.Lq + qrow] =
            lt > 0.f ? (m_used + __log2f(lt)) * 0.69314718055994530942f : -INFINITY;
      }
      tc_fence_before();
      warp_arrive(kBarOEmpty + slot);
      ++item;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 10) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace rbs
