// Block-sparse prefill attention on the 5th-generation tensor core.
// ([RBS-en] "The Fix": exact softmax attention over the selected key blocks,
// compatible with standard multi-head / grouped-query attention.)
//
// Work item = one list row (batch b, q head h, query block i): a 128-row
// query tile (BQ valid rows) against the row's listed key blocks, in list
// order.  Persistent CTAs take non-empty work items round-robin in an order
// that starts with the last query blocks (the longest causal rows).
//
// Roles (NWG*128 + 96 threads, NWG = 2 or 4 softmax warpgroups):
//   warps 0 .. 4*NWG-1  softmax.  Thread r of warpgroup g owns query row r
//              and key columns [g*BK/NWG, (g+1)*BK/NWG) of every S tile (TMEM
//              lane r).  Every thread also reads the rest of its row from
//              TMEM to form the full row maximum itself, so all parts take
//              identical rescale decisions without exchanging anything; each
//              part keeps its own partial row sum until the epilogue.
//              P = exp2(S*c - m) (3 of every 8 element pairs on the FMA pipe,
//              see exp2_fma2, the rest on the SFU) goes back to TMEM as packed
//              bf16 pairs; O is rescaled in TMEM only when the
//              running max grows by more than 2^8 (the final normalisation
//              uses the same max, so this is exact).  Warpgroup g also loads
//              dims [g*128/NWG, (g+1)*128/NWG) of the next row's Q tile from
//              global memory into registers one row ahead, moves them into
//              TMEM, and writes those dims of every output row.
//   warp 4*NWG     K producer, warp 4*NWG+1  V producer (one thread each):
//              K_j / V_j tiles gathered by block index with TMA (4-D tensor
//              maps over [B, L, H, 128], 128B swizzle, no multicast) into
//              3-deep K and V rings; list indices fetched one tile ahead.
//   warp 4*NWG+2   TMEM allocator and MMA issuer (one thread):
//                S_t  = Q K_t^T   A = Q from TMEM, B = K_t (K-major smem)
//                O   += P_t V_t   A = P from TMEM, B = V_t (MN-major smem)
//              completion reported with tcgen05.commit on mbarriers.
// TMEM columns: S0 [0, BK), S1 [BK, 2BK), O [2BK, 2BK+128), Q (64 packed
// columns), P (BK/2 packed columns).  Issue order S_0, S_1, S_2, PV_0, S_3,
// PV_1, ...: S runs two tiles ahead of PV, so the softmax of tile t has two
// tile-periods to finish; the next row's S tiles start while the current
// row's output is written.
//
// Every mbarrier wait is bounded; on a timeout all roles unwind, in-flight
// TMA loads and MMAs are drained (bounded), TMEM is freed, and the device
// error word records RBS_DEVERR_TIMEOUT.  No named barriers are used after
// set-up, so an aborting warp can never strand another.
#pragma once

#include "common.cuh"

namespace rbs {

struct AttnArgs {
  CUtensorMap tmK, tmV;
  const __nv_bfloat16* Q;
  int64_t qb, qs, qh;
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

constexpr int kNS = 3;  // K and V ring depth

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
__host__ __device__ constexpr int attn_threads(int nwg) { return nwg * 128 + 96; }

template <int BK, int NWG>
struct AttnSmem {
  static constexpr int kKVBytes = BK * 128 * 2;  // BK rows x 128 dims (two 64-dim halves)
  static constexpr int kK = 0;
  static constexpr int kV = kK + kNS * kKVBytes;
  static constexpr int kLred = kV + kNS * kKVBytes;  // float [2 parity][NWG parts][128 rows]
  static constexpr int kBar = kLred + 2 * NWG * 128 * 4;
  static constexpr int kBarBytes = 256;
  static constexpr int kTotal = kBar + kBarBytes;
  static constexpr int kAlloc = kTotal + 1024;  // slack to align the base to 1024
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 2 * BK;
  static constexpr uint32_t kColQ = 2 * BK + 128;
  static constexpr uint32_t kColP = 2 * BK + 192;
  static_assert(kColP + BK / 2 <= kTmemCols, "TMEM budget");
};

// barrier slots (8 bytes each)
enum : int {
  kBarQTmem = 0,
  kBarKFull = 1,                 // + stage
  kBarKEmpty = kBarKFull + kNS,  // + stage
  kBarVFull = kBarKEmpty + kNS,
  kBarVEmpty = kBarVFull + kNS,
  kBarSFull = kBarVEmpty + kNS,  // + buffer (2)
  kBarSEmpty = kBarSFull + 2,
  kBarPFull = kBarSEmpty + 2,
  kBarPVDone = kBarPFull + 1,
  kBarOEmpty = kBarPVDone + 1,
  kBarL = kBarOEmpty + 1,
  kBarDrain = kBarL + 1,
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

template <int BQ, int BK, int NWG>
__global__ void __launch_bounds__(attn_threads(NWG), 1) bsa_prefill_kernel(const __grid_constant__ AttnArgs a) {
  using L = AttnSmem<BK, NWG>;
  constexpr int kThreads = attn_threads(NWG);
  constexpr int kSoftmaxWarps = NWG * 4;  // softmax-side barriers count one arrival per warp
  constexpr int COLS = BK / NWG;    // key columns per softmax warpgroup
  constexpr int DPW = 128 / NWG;    // head dims per softmax warpgroup (Q staging, O)
  constexpr int kKWarp = 4 * NWG, kVWarp = 4 * NWG + 1, kMmaWarp = 4 * NWG + 2;
  static_assert(COLS % 32 == 0 || COLS == 16, "columns per warpgroup");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sK = sbase + L::kK;
  const uint32_t sV = sbase + L::kV;
  float* lred = reinterpret_cast<float*>(smem + L::kLred);
  const uint32_t bars = sbase + L::kBar;
  auto bar = [&](int k) -> uint32_t { return bars + 8u * k; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kBar + kNumBars * 8 + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(bar(kBarQTmem), kSoftmaxWarps);
    for (int s = 0; s < kNS; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarVEmpty + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBarSFull + s), 1);
      mbar_init(bar(kBarSEmpty + s), kSoftmaxWarps);
    }
    mbar_init(bar(kBarPFull), kSoftmaxWarps);
    mbar_init(bar(kBarPVDone), 1);
    mbar_init(bar(kBarOEmpty), kSoftmaxWarps);
    mbar_init(bar(kBarL), kSoftmaxWarps);
    mbar_init(bar(kBarDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kKWarp || warp == kVWarp) {
    // ------------------------------------------------------------ K / V producers
    if (lane == 0) {
      const bool isK = warp == kKWarp;
      const CUtensorMap* map = isK ? &a.tmK : &a.tmV;
      const uint32_t ring = isK ? sK : sV;
      const int full0 = isK ? kBarKFull : kBarVFull;
      const int empty0 = isK ? kBarKEmpty : kBarVEmpty;
      tma_prefetch_desc(map);
      uint32_t nf = 0;  // fills issued
      bool ok = true;
      for (Work x = next_work(a, blockIdx.x); x.w < a.num_rows && ok; x = next_work(a, x.w + gridDim.x)) {
        const int kvh = x.h / (a.Hq / a.Hkv);
        int j_next = __ldg(a.col_idx + x.beg);
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
      // drain: every load issued must land before the CTA exits.  Stage s
      // was filled at fill numbers s, s + NS, ...; its last fill completes
      // phase (uses - 1).
      for (uint32_t s = 0; s < kNS; ++s)
        if (s < nf) mbar_drain(bar(full0 + s), ((nf - s + kNS - 1) / kNS - 1) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, BK, 0, 0);
      constexpr uint32_t idPV = idesc_bf16_f32(128, 128, 0, 1);
      // Descriptors are built once per ring stage; a k-step only adds its
      // start-address offset (16-byte units) to the low field, so issuing an
      // MMA costs one 64-bit add.  Addresses stay below 256 KB: no carry out
      // of the 14-bit field.
      const uint64_t kdesc0 = smem_desc(sK, 16, 1024, kLayoutSW128);
      const uint64_t vdesc0 = smem_desc(sV, BK * 128, 1024, kLayoutSW128);
      constexpr uint32_t kStageUnits = L::kKVBytes >> 4;
      uint32_t kv_base = 0, g = 0, item = 0;
      bool ok = true;
      for (Work x = next_work(a, blockIdx.x); x.w < a.num_rows && ok; x = next_work(a, x.w + gridDim.x)) {
        if (!mbar_wait(bar(kBarQTmem), item & 1, abort_flag)) break;
        tc_fence_after();
        const int n = x.n;
        int sS = kv_base % kNS, sPV = kv_base % kNS;  // ring stages of the next S and PV
        for (int t = 0; t < n + 2; ++t) {
          if (t < n) {
            const uint32_t it = kv_base + t;
            const uint32_t gt = g + t;
            const int sb = gt & 1;
            if (!mbar_wait(bar(kBarKFull + sS), (it / kNS) & 1, abort_flag)) { ok = false; break; }
            if (gt >= 2 && !mbar_wait(bar(kBarSEmpty + sb), ((gt >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t dS = tmem + sb * BK;
            const uint64_t kd = kdesc0 + static_cast<uint32_t>(sS) * kStageUnits;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              constexpr uint32_t kHalf = (BK * 128) >> 4;
              umma_ts(dS, tmem + L::kColQ + kk * 8, kd + ((kk >> 2) * kHalf + (kk & 3) * 2), idS, kk > 0 ? 1u : 0u);
            }
            umma_commit(bar(kBarSFull + sb));
            umma_commit(bar(kBarKEmpty + sS));
            sS = sS + 1 == kNS ? 0 : sS + 1;
          }
          if (t >= 2) {
            const int tp = t - 2;
            const uint32_t it = kv_base + tp;
            const uint32_t gt = g + tp;
            if (!mbar_wait(bar(kBarPFull), gt & 1, abort_flag)) { ok = false; break; }
            if (!mbar_wait(bar(kBarVFull + sPV), (it / kNS) & 1, abort_flag)) { ok = false; break; }
            if (tp == 0 && item > 0 && !mbar_wait(bar(kBarOEmpty), (item - 1) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint64_t vd = vdesc0 + static_cast<uint32_t>(sPV) * kStageUnits;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma_ts(tmem + L::kColO, tmem + L::kColP + kk * 8, vd + kk * (2048 >> 4), idPV,
                      (tp > 0 || kk > 0) ? 1u : 0u);
            umma_commit(bar(kBarVEmpty + sPV));
            umma_commit(bar(kBarPVDone));
            sPV = sPV + 1 == kNS ? 0 : sPV + 1;
          }
        }
        kv_base += n;
        g += n;
        ++item;
      }
      // drain all outstanding tensor-core work before TMEM is freed
      umma_commit(bar(kBarDrain));
      mbar_drain(bar(kBarDrain), 0);
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0 .. 4*NWG-1)
    const int wg = tid >> 7;  // warpgroup: key columns [wg*COLS, ..), dims [wg*DPW, ..)
    const int r = tid & 127;  // query row within the tile == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const float c = a.scale_log2;
    // one arrival per warp: every lane's prior shared-memory writes and (fenced)
    // tcgen05 operations are ordered before lane 0's arrive by the warp sync
    auto warp_arrive = [&](int k) {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(k));
    };

    // rows with no (or a corrupt) list: zeros and LSE = -inf, no pipeline work
    for (int w = blockIdx.x; w < a.num_rows; w += gridDim.x) {
      int b, h, i, row, beg;
      decode_work(a, w, b, h, i, row);
      const int n = row_extent(a, row, beg);
      if (n > 0) continue;
      if (n < 0 && tid == 0) raise_error(RBS_DEVERR_ROW_PTR);
      if (r < BQ) {
        const int64_t qrow = static_cast<int64_t>(i) * BQ + r;
        uint4* dst = reinterpret_cast<uint4*>(a.O + b * a.ob + qrow * a.os + h * a.oh) + (DPW / 8) * wg;
#pragma unroll
        for (int k = 0; k < DPW / 8; ++k) dst[k] = make_uint4(0, 0, 0, 0);
        if (wg == 0 && a.lse != nullptr) a.lse[(static_cast<int64_t>(b) * a.Hq + h) * a.Lq + qrow] = -INFINITY;
      }
    }

    // dims [wg*DPW, (wg+1)*DPW) of Q row r: global -> registers (one row ahead) -> TMEM
    uint4 qv[DPW / 8];
    auto load_q = [&](const Work& y) {
      if (y.w < a.num_rows && r < BQ) {
        const __nv_bfloat16* src =
            a.Q + y.b * a.qb + (static_cast<int64_t>(y.i) * BQ + r) * a.qs + y.h * a.qh + wg * DPW;
#pragma unroll
        for (int k = 0; k < DPW / 8; ++k) qv[k] = ldg_stream(src + 8 * k);
      } else {
#pragma unroll
        for (int k = 0; k < DPW / 8; ++k) qv[k] = make_uint4(0, 0, 0, 0);
      }
    };
    auto stage_q = [&]() {
      uint32_t v[DPW / 2];
#pragma unroll
      for (int k = 0; k < DPW / 8; ++k) {
        v[4 * k + 0] = qv[k].x;
        v[4 * k + 1] = qv[k].y;
        v[4 * k + 2] = qv[k].z;
        v[4 * k + 3] = qv[k].w;
      }
      if constexpr (DPW == 64) {
        tmem_st32(lane_base + L::kColQ + 32 * wg, v);
      } else {
        tmem_st16(lane_base + L::kColQ + 16 * wg, v);
      }
      tmem_wait_st();
      tc_fence_before();
      warp_arrive(kBarQTmem);
    };

    uint32_t g = 0, item = 0;
    bool ok = true;
    Work x = next_work(a, blockIdx.x);
    if (x.w < a.num_rows) {
      load_q(x);
      stage_q();
    }
    while (ok && x.w < a.num_rows) {
      const Work xn = next_work(a, x.w + gridDim.x);
      load_q(xn);  // the next row's Q streams in while this row runs
      const int n = x.n;
      const int gi = x.i + a.q_block_off;
      float m_used = -INFINITY;  // running max, in log2 units (score * c)
      float2 l2 = make_float2(0.f, 0.f);  // this part's partial row sum (two lanes)
      int j_next = __ldg(a.col_idx + x.beg);
      for (int t = 0; t < n; ++t) {
        const uint32_t gt = g + t;
        const int sb = gt & 1;
        const int j = j_next;
        if (t + 1 < n) j_next = __ldg(a.col_idx + x.beg + t + 1);
        if (!__all_sync(0xffffffffu, mbar_wait(bar(kBarSFull + sb), (gt >> 1) & 1, abort_flag))) { ok = false; break; }
        tc_fence_after();
        // the whole row of S: this part's columns are kept, the other parts'
        // columns only contribute to the row maximum (read one 32-column chunk
        // at a time to bound register use)
        constexpr int NO = COLS / 32, NX = (BK - COLS) / 32;
        uint32_t own[NO][32], tmp[32];
#pragma unroll
        for (int q = 0; q < NO; ++q) tmem_ld32(lane_base + sb * BK + wg * COLS + 32 * q, own[q]);
        const bool bad = j < 0 || j >= a.nkb;
        const bool dead = bad || (a.causal && j > gi);
        const bool diag = a.causal && j == gi;
        if (dead && tid == 0) raise_error(bad ? RBS_DEVERR_BLOCK_INDEX : RBS_DEVERR_NONCAUSAL);
        // masking: token-causal on the diagonal, nothing visible past it.  A
        // column c is masked when c > r: chunk base b masks its lanes e > r - b.
        float mx = -INFINITY;
        auto fold = [&](uint32_t(&w)[32], int base) {
          if (dead || diag) {
            const int lim = dead ? -1 : r - base;
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (e > lim) w[e] = __float_as_uint(-INFINITY);
          }
          float m0 = __uint_as_float(w[0]);
#pragma unroll
          for (int e = 1; e < 31; e += 2) m0 = fmax3(m0, __uint_as_float(w[e]), __uint_as_float(w[e + 1]));
          mx = fmax3(mx, m0, __uint_as_float(w[31]));
        };
#pragma unroll
        for (int q = 0; q < NX; ++q) {
          const int part = q / NO + (q / NO >= wg ? 1 : 0);
          const int base = part * COLS + 32 * (q % NO);
          tmem_ld32(lane_base + sb * BK + base, tmp);
          tmem_wait_ld();
          if (q == 0) {
#pragma unroll
            for (int qo = 0; qo < NO; ++qo) fold(own[qo], wg * COLS + 32 * qo);
          }
          fold(tmp, base);
        }
        if constexpr (NX == 0) {
          tmem_wait_ld();
#pragma unroll
          for (int qo = 0; qo < NO; ++qo) fold(own[qo], wg * COLS + 32 * qo);
        }
        tc_fence_before();
        warp_arrive(kBarSEmpty + sb);
        float s[COLS];
#pragma unroll
        for (int e = 0; e < COLS; ++e) s[e] = __uint_as_float(own[e / 32][e % 32]);

        const float m_new = fmaxf(m_used, mx * c);
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
        const float2 c2 = make_float2(c, c), nm2 = make_float2(-m_exp, -m_exp);
        uint32_t pw[COLS / 2];
        float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int e = 0; e < COLS; e += 2) {
          const float2 arg = ffma2(make_float2(s[e], s[e + 1]), c2, nm2);
          const int pi = (e >> 1) & 7;  // pairs 1, 4 and 6 of every 8 on the FMA pipe
          const float2 p = (pi == 1 || pi == 4 || pi == 6) ? exp2_fma2(arg)
                                                             : make_float2(ptx_exp2(arg.x), ptx_exp2(arg.y));
          acc[(e >> 1) & 1] = fadd2(acc[(e >> 1) & 1], p);
          pw[e >> 1] = pack_bf16x2(p.x, p.y);
        }
        l2 = fadd2(l2, fadd2(acc[0], acc[1]));
        // the previous PV must be complete: it frees the P columns and fixes O
        if (!__all_sync(0xffffffffu, gt == 0 || mbar_wait(bar(kBarPVDone), (gt - 1) & 1, abort_flag))) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int q = 0; q < DPW / 32; ++q) {
            uint32_t v[32];
            tmem_ld32(lane_base + L::kColO + DPW * wg + 32 * q, v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * factor);
            tmem_st32(lane_base + L::kColO + DPW * wg + 32 * q, v);
          }
        }
        if constexpr (COLS == 64) {
          tmem_st32(lane_base + L::kColP + 32 * wg, pw);
        } else {
          tmem_st16(lane_base + L::kColP + 16 * wg, pw);
        }
        tmem_wait_st();
        tc_fence_before();
        warp_arrive(kBarPFull);
      }
      if (!ok) break;

      // all of this row's MMAs are complete once its last PV is
      const uint32_t glast = g + n - 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(kBarPVDone), glast & 1, abort_flag))) { ok = false; break; }
      tc_fence_after();
      // stage the next row's Q so the tensor core can start it during this epilogue
      if (xn.w < a.num_rows) stage_q();
      // epilogue: full row sum, O / l -> bf16 (this warpgroup's dims), LSE
      float* lb = lred + (item & 1) * (NWG * 128);
      lb[wg * 128 + r] = l2.x + l2.y;
      warp_arrive(kBarL);
      if (!__all_sync(0xffffffffu, mbar_wait(bar(kBarL), item & 1, abort_flag))) { ok = false; break; }
      float lt = lb[r] + lb[128 + r];
      if constexpr (NWG == 4) lt += lb[256 + r] + lb[384 + r];
      const float inv_l = lt > 0.f ? 1.f / lt : 0.f;
      const int64_t qrow = static_cast<int64_t>(x.i) * BQ + r;
      uint4* dst = reinterpret_cast<uint4*>(a.O + x.b * a.ob + qrow * a.os + x.h * a.oh) + (DPW / 8) * wg;
#pragma unroll
      for (int q = 0; q < DPW / 32; ++q) {
        uint32_t v[32];
        tmem_ld32(lane_base + L::kColO + DPW * wg + 32 * q, v);
        tmem_wait_ld();
        if (r < BQ) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            dst[4 * q + k] = make_uint4(
                pack_bf16x2(__uint_as_float(v[8 * k + 0]) * inv_l, __uint_as_float(v[8 * k + 1]) * inv_l),
                pack_bf16x2(__uint_as_float(v[8 * k + 2]) * inv_l, __uint_as_float(v[8 * k + 3]) * inv_l),
                pack_bf16x2(__uint_as_float(v[8 * k + 4]) * inv_l, __uint_as_float(v[8 * k + 5]) * inv_l),
                pack_bf16x2(__uint_as_float(v[8 * k + 6]) * inv_l, __uint_as_float(v[8 * k + 7]) * inv_l));
          }
        }
      }
      if (wg == 0 && a.lse != nullptr && r < BQ) {
        a.lse[(static_cast<int64_t>(x.b) * a.Hq + x.h) * a.Lq + qrow] =
            lt > 0.f ? (m_used + __log2f(lt)) * 0.69314718055994530942f : -INFINITY;
      }
      tc_fence_before();
      warp_arrive(kBarOEmpty);
      g += n;
      ++item;
      x = xn;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace rbs
