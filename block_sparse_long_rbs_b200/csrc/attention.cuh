// Block-sparse prefill attention on the 5th-generation tensor core.
// ([RBS-en] "The Fix": exact softmax attention over the selected key blocks,
// compatible with standard multi-head / grouped-query attention; [BA] 2.4
// Block fine-tune: the Block-attention token mask.)
//
// Work item = one list row (batch b, q head h, query block i): a 128-row
// query tile (BQ valid rows) against the row's listed key blocks, in list
// order.  Persistent CTAs take non-empty work items round-robin in an order
// that keeps one KV head's rows together and, within it, starts with the last
// query blocks (the longest causal rows).
//
// One softmax pipeline with two S buffers in TMEM.  While the softmax warps
// work on tile t, the tensor core computes S for tile t+1 and accumulates
// P_{t-1} V_{t-1}, so the tensor core and the softmax overlap without either
// waiting on the other's latency.
//
// Each key tile is split into two column halves, and each half has its own
// softmax state: running max m_h, row sum l_h and accumulator
// O_h = sum over tiles of P_h V_h (the P and V rows of that half's keys).
// The two halves are merged exactly once per row, in the epilogue:
//   O = (O_0 2^(m_0-m) + O_1 2^(m_1-m)) / (l_0 2^(m_0-m) + l_1 2^(m_1-m)),
// so the two warps that share a query row never wait for each other inside
// the key loop.
//
// Roles (384 threads):
//   warps 0-7  softmax: warp w owns query rows 32(w%4) .. 32(w%4)+31 (its
//              TMEM lane quarter) and column half h = w/4 of every key tile.
//              Pass 1 reads its half row of S into registers and takes its
//              maximum; the running max is lazily updated (O_h rescaled in
//              TMEM only when it grows by more than 2^8; the final
//              normalisation uses the same max, so the result is exact).
//              A tile of a rescue-only block whose contribution is weighted
//              by w has log2(w) added to its scaled scores (max and
//              exponentials alike), which weights its softmax mass by w.
//              Pass 2 forms P = exp2(S*c - m_h) from the registers (3 of every
//              8 element pairs on the FMA pipe, see exp2_fma2, the rest on the
//              SFU) and writes it as packed bf16 pairs over the first quarter
//              of its own S columns.  In the epilogue the two warps of a
//              quarter exchange (m_h, l_h) and each writes 64 of the 128
//              output dims from both accumulators.
//   warp 8     Q and K producer, warp 9 V producer (one thread each): TMA
//              loads of the Q tile (double-buffered) and of the K_j / V_j
//              tiles gathered by block index (4-D tensor maps over
//              [B, L, H, 128], 128B swizzle, no multicast) into 2-deep K and
//              V rings; list indices fetched one tile ahead.
//   warp 10    TMEM allocator and S issuer, warp 11 PV issuer (each warp runs
//              its loop; one elected lane issues):
//                S_g   = Q K_g^T      into S buffer g%2  A = Q (smem), B = K_g (smem)
//                O_h  += P_g,h V_g,h  for h = 0, 1       A = P (TMEM), B = V_g (MN-major smem)
//              over the CTA's tiles g = 0, 1, 2, ... of all its rows in
//              sequence.  S_{g+2} overwrites P_g, so the S issuer waits for
//              PV_g to complete; otherwise the two issuers run independently,
//              so each one's waits and commits overlap the other's MMAs.
//              The K and V producers refill a ring stage when the S (PV)
//              barrier of the tile that used it completes.
// TMEM columns: S buffers [0, BK), [128, 128+BK); O_0 [256, 384), O_1 [384, 512).
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
  int q_block_off, causal, num_rows;  // num_rows: work items, B * Hq * nqb
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

template <int BK>
struct AttnSmem {
  static constexpr int kQBytes = 128 * 128 * 2;  // one Q tile: 128 rows x 128 dims (two 64-dim halves)
  static constexpr int kKVBytes = BK * 128 * 2;  // BK rows x 128 dims (two halves)
  static constexpr int kQ = 0;                   // two Q buffers
  static constexpr int kK = kQ + 2 * kQBytes;
  static constexpr int kV = kK + kNS * kKVBytes;
  static constexpr int kX = kV + kNS * kKVBytes;  // float [2 exchange parity][2 halves][(m, l)][128 rows]
  static constexpr int kSeg = kX + 2 * 2 * 2 * 128 * 4;  // int [RBS_MAX_SEGMENTS] passage starts
  static constexpr int kBar = kSeg + RBS_MAX_SEGMENTS * 4;
  static constexpr int kBarBytes = 256;
  static constexpr int kTotal = kBar + kBarBytes;
  static constexpr int kAlloc = kTotal + 1024;  // slack to align the base to 1024
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kSBufs = 2;
  __host__ __device__ static constexpr uint32_t col_s(int buf) { return buf * 128; }
  __host__ __device__ static constexpr uint32_t col_o(int half) { return 256 + half * 128; }
};

// barrier slots (8 bytes each)
enum : int {
  kBarQFull = 0,                 // + buffer (2)
  kBarQEmpty = kBarQFull + 2,    // + buffer (2)
  kBarKFull = kBarQEmpty + 2,    // + stage
  kBarVFull = kBarKFull + kNS,   // + stage
  kBarSFull = kBarVFull + kNS,   // + S buffer (2)
  kBarPFull = kBarSFull + 2,     // + S buffer (2)
  kBarPVDone = kBarPFull + 2,    // + tile index mod 4: one phase per fourth PV
  kBarOFull = kBarPVDone + 4,    // one phase per row
  kBarOEmpty = kBarOFull + 1,    // one phase per row
  kBarX = kBarOEmpty + 1,        // + lane quarter (4): the two warps' exchanges
  kBarDrain = kBarX + 4,         // + issuer (2)
  kNumBars = kBarDrain + 2
};
static_assert(kNumBars * 8 + 16 <= 256, "barrier area");

// Work order: batch entry, then KV head, then query block from the last (the
// longest causal rows first), then the G q heads sharing that KV head.  The
// CTAs working at the same time therefore read the K/V tiles of one KV head,
// which fit in L2 (64 MiB for 131072 tokens), instead of every head's.
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

struct Work {
  int w, b, h, i, row, beg, n;
};

// The first non-empty work item at or after w in this CTA's round-robin order.
__device__ __forceinline__ Work next_work(const AttnArgs& a, int w) {
  Work x;
  for (; w < a.num_rows; w += gridDim.x) {
    decode_work(a, w, x.b, x.h, x.i, x.row);
    x.n = row_extent(a, x.row, x.beg);
    if (x.n > 0) break;
  }
  x.w = w;
  return x;
}

template <int BQ, int BK>
__global__ void __launch_bounds__(kAttnThreads, 1) bsa_prefill_kernel(const __grid_constant__ AttnArgs a) {
  using L = AttnSmem<BK>;
  constexpr int kSoftmaxWarps = 8;  // barriers the softmax warps complete count one arrival per warp
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + L::kQ;
  const uint32_t sK = sbase + L::kK;
  const uint32_t sV = sbase + L::kV;
  float* xch = reinterpret_cast<float*>(smem + L::kX);
  const uint32_t bars = sbase + L::kBar;
  auto bar = [&](int k) -> uint32_t { return bars + 8u * k; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kBar + kNumBars * 8 + 4);
  int* seg = reinterpret_cast<int*>(smem + L::kSeg);
  const uint64_t limit = a.wait_ns;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBarQFull + s), 1);
      mbar_init(bar(kBarQEmpty + s), 1);
    }
    for (int s = 0; s < kNS; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarVFull + s), 1);
    }
    for (int s = 0; s < L::kSBufs; ++s) {
      mbar_init(bar(kBarSFull + s), 1);
      mbar_init(bar(kBarPFull + s), kSoftmaxWarps);
    }
    for (int s = 0; s < 4; ++s) mbar_init(bar(kBarPVDone + s), 1);
    mbar_init(bar(kBarOFull), 1);
    mbar_init(bar(kBarOEmpty), kSoftmaxWarps);
    for (int q = 0; q < 4; ++q) mbar_init(bar(kBarX + q), 2);
    mbar_init(bar(kBarDrain + 0), 1);
    mbar_init(bar(kBarDrain + 1), 1);
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

  if (warp == 8 || warp == 9) {
    // ------------------------------------------------------------ Q+K / V producers
    if (lane == 0) {
      const bool isK = warp == 8;
      const CUtensorMap* map = isK ? &a.tmK : &a.tmV;
      const uint32_t ring = isK ? sK : sV;
      const int full0 = isK ? kBarKFull : kBarVFull;
      tma_prefetch_desc(map);
      if (isK) tma_prefetch_desc(&a.tmQ);
      // Q tiles are read once; the K / V tiles of a KV head are read by
      // every row of its q heads and should stay in L2 meanwhile
      const uint64_t pol_q = l2_policy_evict_first(), pol_kv = l2_policy_evict_last();
      uint32_t nf = 0, nq = 0;  // ring fills, Q fills issued
      bool ok = true;
      for (Work x = next_work(a, blockIdx.x); x.w < a.num_rows && ok; x = next_work(a, x.w + gridDim.x)) {
        int j_next = __ldg(a.col_idx + x.beg);
        if (isK) {
          const int qb = nq & 1;
          if (nq >= 2 && !mbar_wait(bar(kBarQEmpty + qb), ((nq >> 1) - 1) & 1, abort_flag, limit)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(kBarQFull + qb), BQ * 256);
          tma_load_4d_hint(sQ + qb * L::kQBytes, &a.tmQ, bar(kBarQFull + qb), 0, x.h, x.i * BQ, x.b, pol_q);
          tma_load_4d_hint(sQ + qb * L::kQBytes + 128 * 128, &a.tmQ, bar(kBarQFull + qb), 64, x.h, x.i * BQ, x.b,
                           pol_q);
          ++nq;
        }
        const int kvh = x.h / (a.Hq / a.Hkv);
        for (int t = 0; t < x.n; ++t) {
          if (isK && a.stall_after >= 0 && static_cast<int>(nf) >= a.stall_after) { ok = false; break; }
          int j = j_next;
          if (t + 1 < x.n) j_next = __ldg(a.col_idx + x.beg + t + 1);
          if (j < 0 || j >= a.nkb) j = 0;
          const int s = nf % kNS;
          // the stage's previous tile, nf - kNS, must be consumed: its S (for
          // K) or PV (for V) is complete.  Neither barrier can move past that
          // phase before this load lands, so the parity is unambiguous.
          if (nf >= kNS) {
            const uint32_t prev = nf - kNS;
            const bool done = isK ? mbar_wait(bar(kBarSFull + prev % L::kSBufs), (prev / L::kSBufs) & 1, abort_flag, limit)
                                  : mbar_wait(bar(kBarPVDone + (prev & 3)), (prev >> 2) & 1, abort_flag, limit);
            if (!done) { ok = false; break; }
          }
          mbar_arrive_expect_tx(bar(full0 + s), BK * 256);
          tma_load_4d_hint(ring + s * L::kKVBytes, map, bar(full0 + s), 0, kvh, j * BK, x.b, pol_kv);
          tma_load_4d_hint(ring + s * L::kKVBytes + BK * 128, map, bar(full0 + s), 64, kvh, j * BK, x.b, pol_kv);
          ++nf;
        }
      }
      // drain: every load issued must land before the CTA exits.  Buffer s
      // was filled at fill numbers s, s + depth, ...; its last fill completes
      // phase (uses - 1).
      for (uint32_t s = 0; s < kNS; ++s)
        if (s < nf) mbar_drain(bar(full0 + s), ((nf - s + kNS - 1) / kNS - 1) & 1, limit);
      if (isK)
        for (uint32_t s = 0; s < 2; ++s)
          if (s < nq) mbar_drain(bar(kBarQFull + s), ((nq - s + 1) / 2 - 1) & 1, limit);
    }
  } else if (warp == 10 || warp == 11) {
    // ------------------------------------------------------------ S issuer / PV issuer
    {  // the whole warp runs the loop; one elected lane issues each tcgen05 instruction
      const bool isS = warp == 10;
      constexpr uint32_t idS = idesc_bf16_f32(128, BK, 0, 0);
      constexpr uint32_t idPV = idesc_bf16_f32(128, 128, 0, 1);
      // Descriptors are built once; a buffer or k-step only adds its
      // start-address offset (16-byte units) to the low field (addresses
      // stay below 256 KB: no carry out of the 14-bit field).
      const uint64_t qdesc0 = smem_desc(sQ, 16, 1024, kLayoutSW128);
      const uint64_t kdesc0 = smem_desc(sK, 16, 1024, kLayoutSW128);
      const uint64_t vdesc0 = smem_desc(sV, BK * 128, 1024, kLayoutSW128);
      constexpr uint32_t kQUnits = L::kQBytes >> 4, kStageUnits = L::kKVBytes >> 4;
      constexpr uint32_t kQHalf = (128 * 128) >> 4, kKHalf = (BK * 128) >> 4;
      constexpr int kStepsHalf = BK / 32;  // K16 steps per half of a key tile
      auto wait = [&](int k, uint32_t parity) { return __all_sync(0xffffffffu, mbar_wait(bar(k), parity, abort_flag, limit)); };
      // Each issuer walks the CTA's (row, tile) sequence: g counts tiles over
      // all rows, it rows.
      Work x = next_work(a, blockIdx.x);
      int t = 0;
      uint32_t g = 0, it = 0;
      bool ok = true;
      for (; ok && x.w < a.num_rows; ++g) {
        const int b = g % L::kSBufs, s = g % kNS;
        if (isS) {
          const int qb = it & 1;
          if (t == 0 && !wait(kBarQFull + qb, (it >> 1) & 1)) break;
          if (!wait(kBarKFull + s, (g / kNS) & 1)) break;
          // S_g overwrites P_{g-2}: PV_{g-2} must be complete.  The next phase
          // of that barrier is PV_{g+2}, which needs S_{g+2}: not yet issued.
          if (g >= L::kSBufs && !wait(kBarPVDone + ((g - 2) & 3), ((g - 2) >> 2) & 1)) break;
          tc_fence_after();
          const uint64_t qd = qdesc0 + qb * kQUnits, kd = kdesc0 + s * kStageUnits;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t offq = (kk >> 2) * kQHalf + (kk & 3) * 2, offk = (kk >> 2) * kKHalf + (kk & 3) * 2;
            umma_ss_warp(tmem + L::col_s(b), qd + offq, kd + offk, idS, kk > 0 ? 1u : 0u);
          }
          umma_commit_warp(bar(kBarSFull + b));
          if (t == x.n - 1) umma_commit_warp(bar(kBarQEmpty + qb));
        } else {
          if (!wait(kBarPFull + b, (g / L::kSBufs) & 1)) break;
          if (!wait(kBarVFull + s, (g / kNS) & 1)) break;
          if (t == 0 && it > 0 && !wait(kBarOEmpty, (it - 1) & 1)) break;
          tc_fence_after();
          const uint64_t vd = vdesc0 + s * kStageUnits;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // key half h = kk / kStepsHalf: its P sits at the start of that
            // half's S columns and accumulates into O_h
            const int h = kk / kStepsHalf;
            const uint32_t pcol = L::col_s(b) + h * (BK / 2) + (kk % kStepsHalf) * 8;
            umma_ts_warp(tmem + L::col_o(h), tmem + pcol, vd + kk * (2048 >> 4), idPV,
                         (t == 0 && kk % kStepsHalf == 0) ? 0u : 1u);
          }
          umma_commit_warp(bar(kBarPVDone + (g & 3)));
          if (t == x.n - 1) umma_commit_warp(bar(kBarOFull));
        }
        if (++t == x.n) {
          x = next_work(a, x.w + gridDim.x);
          t = 0;
          ++it;
        }
      }
      // drain this issuer's outstanding tensor-core work before TMEM is freed
      umma_commit_warp(bar(kBarDrain + (isS ? 0 : 1)));
      mbar_drain(bar(kBarDrain + (isS ? 0 : 1)), 0, limit);
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0-7)
    constexpr int kHalf = BK / 2;  // S columns per warp
    const int quarter = warp & 3, hf = warp >> 2;
    const int r = quarter * 32 + lane;  // query row within the tile == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float c = a.scale_log2;
    auto warp_arrive = [&](int k) {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(k));
    };
    // exchange (m, l) of each row with the other warp of this lane quarter
    uint32_t nx = 0;
    auto exchange = [&](float m, float l, float& mo, float& lo) -> bool {
      float* xb = xch + (nx & 1) * 512;  // [2 halves][(m, l)][128 rows]
      xb[hf * 256 + r] = m;
      xb[hf * 256 + 128 + r] = l;
      warp_arrive(kBarX + quarter);
      if (!__all_sync(0xffffffffu, mbar_wait(bar(kBarX + quarter), nx & 1, abort_flag, limit))) return false;
      mo = xb[(hf ^ 1) * 256 + r];
      lo = xb[(hf ^ 1) * 256 + 128 + r];
      ++nx;
      return true;
    };

    // rows with no (or a corrupt) list: zeros and LSE = -inf, no pipeline
    // work.  Each softmax thread checks one of this CTA's rows per pass; a
    // warp then clears the empty rows it found together.
    for (int base = 0; blockIdx.x + static_cast<int64_t>(gridDim.x) * base < a.num_rows; base += 256) {
      const int64_t w = blockIdx.x + static_cast<int64_t>(gridDim.x) * (base + tid);
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

    uint32_t g = 0, item = 0;  // tiles and rows processed by this CTA
    bool ok = true;
    for (Work x = next_work(a, blockIdx.x); x.w < a.num_rows && ok; x = next_work(a, x.w + gridDim.x)) {
      const int n = x.n;
      const int gi = x.i + a.q_block_off;
      // the segment mask's first visible key of this thread's query
      const int key_lo = segment_key_start(seg, a.seg_n, a.seg_final, gi * BK + r);
      float m_used = -INFINITY;  // this half's running max, in log2 units (score * c)
      float2 l2 = make_float2(0.f, 0.f);  // this half's row sum
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
        const int b = g % L::kSBufs;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(kBarSFull + b), (g / L::kSBufs) & 1, abort_flag, limit))) { ok = false; break; }
        tc_fence_after();
        const bool bad = j < 0 || j >= a.nkb;
        const bool dead = bad || (a.causal && j > gi);
        const bool diag = a.causal && j == gi;
        const bool tail = j == a.nkb - 1 && a.k_tail < BK;  // keys past Lk were loaded as zeros
        if (dead && r == 0 && hf == 0) raise_error(bad ? RBS_DEVERR_BLOCK_INDEX : RBS_DEVERR_NONCAUSAL);
        // pass 1: this warp's half row of S into registers, masked; its maximum
        const uint32_t scol = L::col_s(b) + hf * kHalf;
        uint32_t v[kHalf / 32][32];
#pragma unroll
        for (int q = 0; q < kHalf / 32; ++q) tmem_ld32(lane_base + scol + 32 * q, v[q]);
        tmem_wait_ld();
        const int lo_col = key_lo - j * BK;  // tile columns below are before the query's passage start
        if (dead || diag || tail || lo_col > hf * kHalf) {
          // tile column hf * kHalf + 32 q + e is masked when it is above the
          // diagonal, past the last key, before the query's passage start,
          // or always (a dead tile)
#pragma unroll
          for (int q = 0; q < kHalf / 32; ++q) {
            const int col0 = hf * kHalf + 32 * q;
            int lim = dead ? -1 : BK;
            if (diag) lim = min(lim, r - col0);
            if (tail) lim = min(lim, a.k_tail - 1 - col0);
            const int lo = lo_col - col0;
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (e > lim || e < lo) v[q][e] = __float_as_uint(-INFINITY);
          }
        }
        float mx = -INFINITY;
#pragma unroll
        for (int q = 0; q < kHalf / 32; ++q) {
          float m0 = __uint_as_float(v[q][0]);
#pragma unroll
          for (int e = 1; e < 31; e += 2) m0 = fmax3(m0, __uint_as_float(v[q][e]), __uint_as_float(v[q][e + 1]));
          mx = fmax3(mx, m0, __uint_as_float(v[q][31]));
        }
        const float m_new = fmaxf(m_used, fmaf(mx, c, bias));
        float factor = 1.f;
        bool rescale = false;
        if (t == 0) {
          m_used = m_new;
        } else if (m_new - m_used > 8.f) {
          factor = ptx_exp2(m_used - m_new);
          m_used = m_new;
          rescale = true;
        }
        const float m_exp = m_used == -INFINITY ? 0.f : m_used;
        l2.x *= factor;
        l2.y *= factor;
        // pass 2: P = exp2(s*c - m) from the registers, written as packed bf16
        // pairs over the first kHalf/2 of this warp's S columns (already read)
        const float2 c2 = make_float2(c, c), nm2 = make_float2(bias - m_exp, bias - m_exp);
        float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        uint32_t pw[kHalf / 2];
#pragma unroll
        for (int e = 0; e < kHalf; e += 2) {
          const float2 sv = make_float2(__uint_as_float(v[e >> 5][e & 31]), __uint_as_float(v[e >> 5][(e & 31) + 1]));
          const float2 arg = ffma2(sv, c2, nm2);
          const int pi = (e >> 1) & 7;  // pairs 1, 4 and 6 of every 8 on the FMA pipe
          const float2 p = (pi == 1 || pi == 4 || pi == 6) ? exp2_fma2(arg)
                                                             : make_float2(ptx_exp2(arg.x), ptx_exp2(arg.y));
          acc[(e >> 1) & 1] = fadd2(acc[(e >> 1) & 1], p);
          pw[e >> 1] = pack_bf16x2(p.x, p.y);
        }
        if constexpr (kHalf == 64) {
          tmem_st32(lane_base + scol, pw);
        } else {
          tmem_st16(lane_base + scol, pw);
        }
        l2 = fadd2(l2, fadd2(acc[0], acc[1]));
        if (__any_sync(0xffffffffu, rescale)) {
          // O is scaled after P is formed, so the wait below overlaps the
          // exponentials.  O must hold every earlier tile's product first.
          // The next phase of PV_{g-1}'s barrier is PV_{g+3}, which cannot
          // start before this tile's P is complete.
          if (!__all_sync(0xffffffffu, mbar_wait(bar(kBarPVDone + ((g - 1) & 3)), ((g - 1) >> 2) & 1, abort_flag, limit))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t o[32];
            tmem_ld32(lane_base + L::col_o(hf) + 32 * q, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
            tmem_st32(lane_base + L::col_o(hf) + 32 * q, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        warp_arrive(kBarPFull + b);
      }
      if (!ok) break;

      // ---- epilogue: merge the halves, O / l -> bf16 (this warp: dims
      // [64 hf, 64 hf + 64) of both accumulators), LSE
      const float lh = l2.x + l2.y;
      float mo, lo;
      if (!exchange(m_used, lh, mo, lo)) { ok = false; break; }
      const float m0 = hf == 0 ? m_used : mo, l0 = hf == 0 ? lh : lo;
      const float m1 = hf == 0 ? mo : m_used, l1 = hf == 0 ? lo : lh;
      const float m = fmaxf(m0, m1);
      const float w0 = l0 > 0.f ? ptx_exp2(m0 - m) : 0.f;
      const float w1 = l1 > 0.f ? ptx_exp2(m1 - m) : 0.f;
      const float lt = l0 * w0 + l1 * w1;
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      const float s0 = w0 * inv, s1 = w1 * inv;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(kBarOFull), item & 1, abort_flag, limit))) { ok = false; break; }
      tc_fence_after();
      const int64_t qrow = static_cast<int64_t>(x.i) * BQ + r;
      uint4* dst = reinterpret_cast<uint4*>(a.O + x.b * a.ob + qrow * a.os + x.h * a.oh) + 8 * hf;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint32_t va[32], vb[32];
        tmem_ld32(lane_base + L::col_o(0) + 64 * hf + 32 * q, va);
        tmem_ld32(lane_base + L::col_o(1) + 64 * hf + 32 * q, vb);
        tmem_wait_ld();
        float o[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = fmaf(__uint_as_float(vb[e]), s1, __uint_as_float(va[e]) * s0);
        if (r < BQ && qrow < a.Lq) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            // streaming (evict-first) stores: the output is not read again
            // here, and the K / V tiles it would otherwise push out of L2
            // are (as are the next kernel's inputs)
            __stcs(dst + 4 * q + k, make_uint4(pack_bf16x2(o[8 * k], o[8 * k + 1]),
                                               pack_bf16x2(o[8 * k + 2], o[8 * k + 3]),
                                               pack_bf16x2(o[8 * k + 4], o[8 * k + 5]),
                                               pack_bf16x2(o[8 * k + 6], o[8 * k + 7])));
        }
      }
      if (hf == 0 && a.lse != nullptr && r < BQ && qrow < a.Lq) {
        a.lse[(static_cast<int64_t>(x.b) * a.Hq + x.h) * a.Lq + qrow] =
            lt > 0.f ? (m + __log2f(lt)) * 0.69314718055994530942f : -INFINITY;
      }
      tc_fence_before();
      warp_arrive(kBarOEmpty);
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
