// Block-sparse prefill attention on the 5th-generation tensor core.
// ([RBS-en] "The Fix": exact softmax attention over the selected key blocks,
// compatible with standard multi-head / grouped-query attention.)
//
// Work item = one list row (batch b, q head h, query block i): a 128-row
// query tile (BQ valid rows) against the row's listed key blocks, in list
// order.  Persistent CTAs take non-empty work items round-robin in an order
// that starts with the last query blocks (the longest causal rows).
//
// Two softmax streams.  The row's key tiles alternate between stream A
// (tiles 0, 2, 4, ...) and stream B (tiles 1, 3, 5, ...).  Each stream keeps
// its own S tile (P is written back over it), its own O accumulator and its
// own running max and sum, and the two partial results are merged exactly in
// the epilogue:  O = (O_A 2^(m_A-m) + O_B 2^(m_B-m)) / (l_A 2^(m_A-m) + l_B 2^(m_B-m)).
// While one stream's softmax runs, the tensor core works on the other's
// tiles, so neither waits for the other.
//
// Roles (352 threads):
//   warps 0-3  softmax of stream A, warps 4-7 softmax of stream B: thread r
//              owns query row r (TMEM lane r) of its stream's tiles.  Pass 1
//              reads the S row from TMEM for the row maximum; the running max
//              is lazily updated (O rescaled in TMEM only when it grows by
//              more than 2^8; the final normalisation uses the same max, so
//              the result is exact); pass 2 re-reads S and writes
//              P = exp2(S*c - m) as packed bf16 pairs over the S columns
//              (3 of every 8 element pairs on the FMA pipe, see exp2_fma2,
//              the rest on the SFU).  In the epilogue warpgroup g merges and
//              writes dims [64g, 64g+64) of every output row.
//   warp 8     Q and K producer, warp 9 V producer (one thread each): TMA
//              loads of the Q tile (double-buffered) and of the K_j / V_j
//              tiles gathered by block index (4-D tensor maps over
//              [B, L, H, 128], 128B swizzle, no multicast) into 2-deep K and
//              V rings; list indices fetched one tile ahead.
//   warp 10    TMEM allocator and MMA issuer (one thread):
//                S_t  = Q K_t^T  into stream (t&1)'s S   A = Q (smem), B = K_t (smem)
//                O   += P_t V_t  into stream (t&1)'s O   A = P (TMEM), B = V_t (MN-major smem)
//              issue order S_0, S_1, PV_0, S_2, PV_1, S_3, ...; S_{t+2} is
//              issued after PV_t, which reads P_t from the same columns (the
//              tensor core executes one thread's MMAs in order).
// TMEM columns: S_A [0, BK), O_A [128, 256), S_B [256, 256+BK), O_B [384, 512).
//
// Every mbarrier wait is bounded; on a timeout all roles unwind, in-flight
// TMA loads and MMAs are drained (bounded), TMEM is freed, and the device
// error word records RBS_DEVERR_TIMEOUT.  No named barriers are used after
// set-up, so an aborting warp can never strand another.
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
  int q_block_off, causal, num_rows;
  float scale_log2;
};

constexpr int kAttnThreads = 352;
constexpr int kNS = 2;  // K and V ring depth

// Software base-2 exponential of two values at once, on the FMA pipe:
// Cody-Waite range reduction 2^x = 2^n * 2^f, n = rint(x) (via the 1.5*2^23
// shifter), f = x - n in [-1/2, 1/2], then p(f) = 1 + c1 f + c2 f^2 + c3 f^3,
// a degree-3 fit by the Remez exchange algorithm for minimum relative error
// (max 4.3e-4; csrc/exp2_poly_fit.py derives the coefficients).  The
// exponent n is added to p's exponent field.  Inputs are clamped at -127, where
// the result is +0 (p(0) = 1 exactly); inputs above 127 are not expected
// (the running max keeps them at or below 8).
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

template <int BK>
struct AttnSmem {
  static constexpr int kQBytes = 128 * 128 * 2;  // one Q tile: 128 rows x 128 dims (two 64-dim halves)
  static constexpr int kKVBytes = BK * 128 * 2;  // BK rows x 128 dims (two halves)
  static constexpr int kQ = 0;                   // two Q buffers
  static constexpr int kK = kQ + 2 * kQBytes;
  static constexpr int kV = kK + kNS * kKVBytes;
  static constexpr int kX = kV + kNS * kKVBytes;  // float [2 item parity][2 streams][2 (m, l)][128 rows]
  static constexpr int kBar = kX + 2 * 2 * 2 * 128 * 4;
  static constexpr int kBarBytes = 256;
  static constexpr int kTotal = kBar + kBarBytes;
  static constexpr int kAlloc = kTotal + 1024;  // slack to align the base to 1024
  static constexpr uint32_t kTmemCols = 512;
  __host__ __device__ static constexpr uint32_t col_s(int st) { return st * 256; }
  __host__ __device__ static constexpr uint32_t col_o(int st) { return st * 256 + 128; }
};

// barrier slots (8 bytes each)
enum : int {
  kBarQFull = 0,                 // + buffer (2)
  kBarQEmpty = kBarQFull + 2,    // + buffer (2)
  kBarKFull = kBarQEmpty + 2,    // + stage
  kBarKEmpty = kBarKFull + kNS,  // + stage
  kBarVFull = kBarKEmpty + kNS,  // + stage
  kBarVEmpty = kBarVFull + kNS,  // + stage
  kBarSFull = kBarVEmpty + kNS,  // + stream
  kBarPFull = kBarSFull + 2,     // + stream
  kBarOFull = kBarPFull + 2,     // + stream
  kBarOEmpty = kBarOFull + 2,    // + stream
  kBarX = kBarOEmpty + 2,
  kBarDrain = kBarX + 1,
  kNumBars = kBarDrain + 1
};
static_assert(kNumBars * 8 + 16 <= 256, "barrier area");

__device__ __forceinline__ void decode_work(const AttnArgs& a, int w, int& b, int& h, int& i, int& row) {
  const int bh_count = a.B * a.Hq;
  i = a.nqb - 1 - w / bh_count;
  const int bh = w % bh_count;
  b = bh / a.Hq;
  h = bh % a.Hq;
  row = bh * a.nqb + i;
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
  constexpr int kStreamWarps = 4;  // softmax warps per stream; their barriers count one arrival per warp
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

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBarQFull + s), 1);
      mbar_init(bar(kBarQEmpty + s), 1);
      mbar_init(bar(kBarSFull + s), 1);
      mbar_init(bar(kBarPFull + s), kStreamWarps);
      mbar_init(bar(kBarOFull + s), 1);
      mbar_init(bar(kBarOEmpty + s), 2 * kStreamWarps);
    }
    for (int s = 0; s < kNS; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarVEmpty + s), 1);
    }
    mbar_init(bar(kBarX), 2 * kStreamWarps);
    mbar_init(bar(kBarDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
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
      const int empty0 = isK ? kBarKEmpty : kBarVEmpty;
      tma_prefetch_desc(map);
      if (isK) tma_prefetch_desc(&a.tmQ);
      uint32_t nf = 0, nq = 0;  // ring fills, Q fills issued
      bool ok = true;
      for (Work x = next_work(a, blockIdx.x); x.w < a.num_rows && ok; x = next_work(a, x.w + gridDim.x)) {
        int j_next = __ldg(a.col_idx + x.beg);
        if (isK) {
          const int qb = nq & 1;
          if (nq >= 2 && !mbar_wait(bar(kBarQEmpty + qb), ((nq >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(kBarQFull + qb), BQ * 256);
          tma_load_4d(sQ + qb * L::kQBytes, &a.tmQ, bar(kBarQFull + qb), 0, x.h, x.i * BQ, x.b);
          tma_load_4d(sQ + qb * L::kQBytes + 128 * 128, &a.tmQ, bar(kBarQFull + qb), 64, x.h, x.i * BQ, x.b);
          ++nq;
        }
        const int kvh = x.h / (a.Hq / a.Hkv);
        for (int t = 0; t < x.n; ++t) {
          int j = j_next;
          if (t + 1 < x.n) j_next = __ldg(a.col_idx + x.beg + t + 1);
          if (j < 0 || j >= a.nkb) j = 0;
          const int s = nf % kNS;
          if (nf >= kNS && !mbar_wait(bar(empty0 + s), ((nf / kNS) & 1) ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(full0 + s), BK * 256);
          tma_load_4d(ring + s * L::kKVBytes, map, bar(full0 + s), 0, kvh, j * BK, x.b);
          tma_load_4d(ring + s * L::kKVBytes + BK * 128, map, bar(full0 + s), 64, kvh, j * BK, x.b);
          ++nf;
        }
      }
      // drain: every load issued must land before the CTA exits.  Buffer s
      // was filled at fill numbers s, s + depth, ...; its last fill completes
      // phase (uses - 1).
      for (uint32_t s = 0; s < kNS; ++s)
        if (s < nf) mbar_drain(bar(full0 + s), ((nf - s + kNS - 1) / kNS - 1) & 1);
      if (isK)
        for (uint32_t s = 0; s < 2; ++s)
          if (s < nq) mbar_drain(bar(kBarQFull + s), ((nq - s + 1) / 2 - 1) & 1);
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------ MMA issuer
    {  // the whole warp runs the loop; one elected lane issues each tcgen05 instruction
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
      uint32_t kit = 0, vit = 0, item = 0, nP[2] = {0, 0};
      bool ok = true;
      for (Work x = next_work(a, blockIdx.x); x.w < a.num_rows && ok; x = next_work(a, x.w + gridDim.x)) {
        const int qb = item & 1, n = x.n;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(kBarQFull + qb), (item >> 1) & 1, abort_flag))) break;
        tc_fence_after();
        const uint64_t qd = qdesc0 + qb * kQUnits;
        auto issue_s = [&](int t) -> bool {
          const int st = t & 1, s = kit % kNS;
          if (!__all_sync(0xffffffffu, mbar_wait(bar(kBarKFull + s), (kit / kNS) & 1, abort_flag))) return false;
          tc_fence_after();
          const uint64_t kd = kdesc0 + s * kStageUnits;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t offq = (kk >> 2) * kQHalf + (kk & 3) * 2, offk = (kk >> 2) * kKHalf + (kk & 3) * 2;
            umma_ss_warp(tmem + L::col_s(st), qd + offq, kd + offk, idS, kk > 0 ? 1u : 0u);
          }
          umma_commit_warp(bar(kBarSFull + st));
          umma_commit_warp(bar(kBarKEmpty + s));
          if (t == n - 1) umma_commit_warp(bar(kBarQEmpty + qb));
          ++kit;
          return true;
        };
        auto issue_pv = [&](int t) -> bool {
          const int st = t & 1, s = vit % kNS;
          const bool first = t < 2;  // first tile of this stream in the row
          if (!__all_sync(0xffffffffu, mbar_wait(bar(kBarPFull + st), nP[st] & 1, abort_flag))) return false;
          if (!__all_sync(0xffffffffu, mbar_wait(bar(kBarVFull + s), (vit / kNS) & 1, abort_flag))) return false;
          if (first && item > 0 && !__all_sync(0xffffffffu, mbar_wait(bar(kBarOEmpty + st), (item - 1) & 1, abort_flag))) return false;
          tc_fence_after();
          const uint64_t vd = vdesc0 + s * kStageUnits;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_ts_warp(tmem + L::col_o(st), tmem + L::col_s(st) + kk * 8, vd + kk * (2048 >> 4), idPV,
                    (first && kk == 0) ? 0u : 1u);
          umma_commit_warp(bar(kBarVEmpty + s));
          if (t >= n - 2) umma_commit_warp(bar(kBarOFull + st));  // the stream's last tile of this row
          ++vit;
          ++nP[st];
          return true;
        };
        ok = issue_s(0) && (n < 2 || issue_s(1));
        for (int t = 0; t < n && ok; ++t) ok = issue_pv(t) && (t + 2 >= n || issue_s(t + 2));
        ++item;
      }
      // drain all outstanding tensor-core work before TMEM is freed
      umma_commit_warp(bar(kBarDrain));
      mbar_drain(bar(kBarDrain), 0);
    }
  } else {
    // ------------------------------------------------------------ softmax streams (warps 0-7)
    const int st = warp >> 2;  // stream: tiles st, st + 2, ...; epilogue dims [64 st, 64 st + 64)
    const int r = tid & 127;   // query row within the tile == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const float c = a.scale_log2;
    auto warp_arrive = [&](int k) {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(k));
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
          reinterpret_cast<uint4*>(a.O + eb * a.ob + qrow * a.os + eh * a.oh)[k & 15] = make_uint4(0, 0, 0, 0);
        }
        if (a.lse != nullptr)
          for (int k = lane; k < BQ; k += 32)
            a.lse[(static_cast<int64_t>(eb) * a.Hq + eh) * a.Lq + static_cast<int64_t>(ei) * BQ + k] = -INFINITY;
      }
    }

    uint32_t nS = 0, nO[2] = {0, 0}, item = 0;
    bool ok = true;
    for (Work x = next_work(a, blockIdx.x); x.w < a.num_rows && ok; x = next_work(a, x.w + gridDim.x)) {
      const int n = x.n;
      const int gi = x.i + a.q_block_off;
      float m_used = -INFINITY;  // this stream's running max, in log2 units (score * c)
      float2 l2 = make_float2(0.f, 0.f);
      int j_next = st < n ? __ldg(a.col_idx + x.beg + st) : 0;
      for (int t = st; t < n; t += 2) {
        const int j = j_next;
        if (t + 2 < n) j_next = __ldg(a.col_idx + x.beg + t + 2);
        if (!__all_sync(0xffffffffu, mbar_wait(bar(kBarSFull + st), nS & 1, abort_flag))) { ok = false; break; }
        ++nS;
        tc_fence_after();
        const bool bad = j < 0 || j >= a.nkb;
        const bool dead = bad || (a.causal && j > gi);
        const bool diag = a.causal && j == gi;
        if (dead && r == 0) raise_error(bad ? RBS_DEVERR_BLOCK_INDEX : RBS_DEVERR_NONCAUSAL);
        // tile column c is masked when c > r (diagonal block) or always (dead block)
        auto mask64 = [&](uint32_t(&v)[2][32], int base) {
          if (dead || diag) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const int lim = dead ? -1 : r - (base + 32 * q);
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (e > lim) v[q][e] = __float_as_uint(-INFINITY);
            }
          }
        };
        // pass 1: the row maximum, 64 columns at a time
        float mx = -INFINITY;
#pragma unroll
        for (int h64 = 0; h64 < BK / 64; ++h64) {
          uint32_t v[2][32];
          tmem_ld32(lane_base + L::col_s(st) + 64 * h64, v[0]);
          tmem_ld32(lane_base + L::col_s(st) + 64 * h64 + 32, v[1]);
          tmem_wait_ld();
          mask64(v, 64 * h64);
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            float m0 = __uint_as_float(v[q][0]);
#pragma unroll
            for (int e = 1; e < 31; e += 2) m0 = fmax3(m0, __uint_as_float(v[q][e]), __uint_as_float(v[q][e + 1]));
            mx = fmax3(mx, m0, __uint_as_float(v[q][31]));
          }
        }
        const float m_new = fmaxf(m_used, mx * c);
        float factor = 1.f;
        bool rescale = false;
        if (t < 2) {
          m_used = m_new;
        } else if (m_new - m_used > 8.f) {
          factor = ptx_exp2(m_used - m_new);
          m_used = m_new;
          rescale = true;
        }
        const float m_exp = m_used == -INFINITY ? 0.f : m_used;
        l2.x *= factor;
        l2.y *= factor;
        // this stream's previous PV is complete (S_t was issued after it): O is stable
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t v[32];
            tmem_ld32(lane_base + L::col_o(st) + 32 * q, v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * factor);
            tmem_st32(lane_base + L::col_o(st) + 32 * q, v);
          }
        }
        // pass 2: P = exp2(s*c - m), 64 columns at a time, written as packed
        // bf16 pairs over S columns this thread has already consumed
        const float2 c2 = make_float2(c, c), nm2 = make_float2(-m_exp, -m_exp);
        float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int h64 = 0; h64 < BK / 64; ++h64) {
          uint32_t v[2][32];
          tmem_ld32(lane_base + L::col_s(st) + 64 * h64, v[0]);
          tmem_ld32(lane_base + L::col_s(st) + 64 * h64 + 32, v[1]);
          tmem_wait_ld();
          mask64(v, 64 * h64);
          uint32_t pw[32];
#pragma unroll
          for (int e = 0; e < 64; e += 2) {
            const float2 sv = make_float2(__uint_as_float(v[e >> 5][e & 31]), __uint_as_float(v[e >> 5][(e & 31) + 1]));
            const float2 arg = ffma2(sv, c2, nm2);
            const int pi = (e >> 1) & 7;  // pairs 1, 4 and 6 of every 8 on the FMA pipe
            const float2 p = (pi == 1 || pi == 4 || pi == 6) ? exp2_fma2(arg)
                                                               : make_float2(ptx_exp2(arg.x), ptx_exp2(arg.y));
            acc[(e >> 1) & 1] = fadd2(acc[(e >> 1) & 1], p);
            pw[e >> 1] = pack_bf16x2(p.x, p.y);
          }
          tmem_st32(lane_base + L::col_s(st) + 32 * h64, pw);
        }
        l2 = fadd2(l2, fadd2(acc[0], acc[1]));
        tmem_wait_st();
        tc_fence_before();
        warp_arrive(kBarPFull + st);
      }
      if (!ok) break;

      // ---- epilogue: merge the two streams, O / l -> bf16, LSE
      float* xb = xch + (item & 1) * 512;  // [2 streams][m, l][128 rows]
      xb[st * 256 + r] = m_used;
      xb[st * 256 + 128 + r] = l2.x + l2.y;
      warp_arrive(kBarX);
      if (!__all_sync(0xffffffffu, mbar_wait(bar(kBarX), item & 1, abort_flag))) { ok = false; break; }
      const bool hasB = n > 1;  // stream B has tiles only when the row has two or more
      const float mA = xb[r], lA = xb[128 + r];
      const float mB = hasB ? xb[256 + r] : -INFINITY, lB = hasB ? xb[384 + r] : 0.f;
      const float m = fmaxf(mA, mB);
      const float wA = lA > 0.f ? ptx_exp2(mA - m) : 0.f;
      const float wB = lB > 0.f ? ptx_exp2(mB - m) : 0.f;
      const float lt = lA * wA + lB * wB;
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      bool okw = mbar_wait(bar(kBarOFull + 0), nO[0] & 1, abort_flag);
      if (hasB && okw) okw = mbar_wait(bar(kBarOFull + 1), nO[1] & 1, abort_flag);
      if (!__all_sync(0xffffffffu, okw)) { ok = false; break; }
      ++nO[0];
      if (hasB) ++nO[1];
      tc_fence_after();
      const int64_t qrow = static_cast<int64_t>(x.i) * BQ + r;
      uint4* dst = reinterpret_cast<uint4*>(a.O + x.b * a.ob + qrow * a.os + x.h * a.oh) + 8 * st;
      const float sa = wA * inv, sb = wB * inv;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint32_t va[32], vb[32];
        tmem_ld32(lane_base + L::col_o(0) + 64 * st + 32 * q, va);
        if (hasB) tmem_ld32(lane_base + L::col_o(1) + 64 * st + 32 * q, vb);
        tmem_wait_ld();
        float o[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          o[e] = __uint_as_float(va[e]) * sa;
          if (hasB) o[e] = fmaf(__uint_as_float(vb[e]), sb, o[e]);
        }
        if (r < BQ) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            dst[4 * q + k] = make_uint4(pack_bf16x2(o[8 * k], o[8 * k + 1]), pack_bf16x2(o[8 * k + 2], o[8 * k + 3]),
                                        pack_bf16x2(o[8 * k + 4], o[8 * k + 5]),
                                        pack_bf16x2(o[8 * k + 6], o[8 * k + 7]));
        }
      }
      if (st == 0 && a.lse != nullptr && r < BQ) {
        a.lse[(static_cast<int64_t>(x.b) * a.Hq + x.h) * a.Lq + qrow] =
            lt > 0.f ? (m + __log2f(lt)) * 0.69314718055994530942f : -INFINITY;
      }
      tc_fence_before();
      warp_arrive(kBarOEmpty + 0);
      warp_arrive(kBarOEmpty + 1);
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
