// Two-branch selection in three kernels (the mean-query scores on the tensor
// core), used when the caller's workspace holds the score matrix, after
// select_prep_kernel (beta, and the centroids' bf16 hi / lo parts):
//
//   pool_split_kernel   qbar_i = mean of query block i's queries for every
//                       (batch, q head), streamed from HBM through a 4-stage
//                       ring of 8-row TMA chunks by a producer warp and
//                       reduced by four consumer warps; written as bf16 hi /
//                       lo parts (qbar = hi + lo to about 2^-17) and |qbar|.
//   score_gemm_kernel   s_c(i, j) = qbar_i . c_j for every visible (i, j) as
//                       128 x 128 x 128 MMAs: A = 128 centroids (K-major, the
//                       bf16 hi / lo parts of rbs_block_stats' fp32
//                       centroids), B = 128 pooled queries (R q heads of one
//                       KV head x 128 / R query blocks), D in TMEM, three
//                       products hi.hi + lo.hi + hi.lo accumulated in fp32;
//                       eight epilogue warps (two per TMEM lane quarter, one
//                       key block per thread, half the columns each) write
//                       the scores to the workspace.  Persistent CTAs take
//                       the items in a snake over the longest-first order.
//   topk_rows_kernel    one warp per row: both branches' exact top-k
//                       (select_row) from the stored scores, the rescue score
//                       s_r = s_c + |qbar| r_j beta_j formed on the fly; or,
//                       for per-token-max scoring, from both branches' keys
//                       as select_tokmax_kernel stored them.
//
// ([RBS-en] "The Fix: A Radius-Adaptive Rescue Branch"; [RBS-id]
// "Dual-Branch Selection".)  The mask words, counts and tile sums they leave
// are the ones the fused select_rows_kernel writes; the tile scan and the
// compaction follow unchanged.
#pragma once

#include "common.cuh"
#include "select.cuh"

namespace rbs {

// ---------------------------------------------------------------------------
// Pooling

constexpr int kPoolKThreads = 160;  // warps 0-3 consume, warp 4 produces
constexpr int kPoolKStages = 4;

struct PoolArgs {
  int B, Hq, nqb, R, items, Lq, seq_inner;
  __nv_bfloat16* qhi;  // [B, Hq, nqb, 128]
  __nv_bfloat16* qlo;
  float* qnorm;        // [B, Hq, nqb]
};

// Item w -> (batch, query block, first q head of a group of R).
__device__ __forceinline__ void pool_item(const PoolArgs& a, int w, int& b, int& i, int& hq0) {
  const int nh = a.Hq / a.R;
  b = w / (a.nqb * nh);
  const int rem = w % (a.nqb * nh);
  i = rem / nh;
  hq0 = (rem % nh) * a.R;
}

template <int BQ>
__global__ void __launch_bounds__(kPoolKThreads) pool_split_kernel(const __grid_constant__ CUtensorMap qmap,
                                                                   PoolArgs a) {
  extern __shared__ __align__(128) uint8_t pool_smem[];
  __shared__ __align__(8) uint64_t full_bar[kPoolKStages], empty_bar[kPoolKStages];
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int R = a.R;
  constexpr int kChunks = BQ / kPoolRows;
  const int nitems = a.items > static_cast<int>(blockIdx.x)
                         ? (a.items - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                         : 0;
  const int total = nitems * kChunks;
  if (tid == 0) {
    for (int s = 0; s < kPoolKStages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 4);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 4) {
    // producer: chunk g = k * kChunks + c of item k into stage g % kPoolKStages
    if ((tid & 31) == 0) {
      tma_prefetch_desc(&qmap);
      const uint32_t chunk_bytes = static_cast<uint32_t>(kPoolRows * R * 128 * 2);
      int g = 0;
      for (; g < total; ++g) {
        const int s = g % kPoolKStages;
        // the stage's previous chunk, g - kPoolKStages, must be consumed
        if (g >= kPoolKStages &&
            !mbar_wait(smem_u32(&empty_bar[s]), ((g / kPoolKStages) - 1) & 1, &abort_flag))
          break;
        int b, i, hq0;
        pool_item(a, static_cast<int>(blockIdx.x) + (g / kChunks) * static_cast<int>(gridDim.x), b, i, hq0);
        const int row0 = i * BQ + (g % kChunks) * kPoolRows;
        const int c1 = a.seq_inner ? row0 : hq0, c2 = a.seq_inner ? hq0 : row0;
        const uint32_t bar = smem_u32(&full_bar[s]);
        const uint32_t dst = smem_u32(pool_smem + s * kPoolChunkBytes);
        mbar_arrive_expect_tx(bar, chunk_bytes);
        tma_load_4d(dst, &qmap, bar, 0, c1, c2, b);
        tma_load_4d(dst + chunk_bytes / 2, &qmap, bar, 64, c1, c2, b);
      }
      // every load issued must land before the CTA exits
      for (int s = 0; s < kPoolKStages; ++s)
        if (s < g) mbar_drain(smem_u32(&full_bar[s]), ((g - s + kPoolKStages - 1) / kPoolKStages - 1) & 1);
    }
    return;
  }

  // consumers: thread (h, dc) sums dims 8 dc .. 8 dc + 7 of head h over the rows
  const int h = tid >> 4, dc = tid & 15, lane = tid & 31;
  // element offset of row r: [half][row][head][64] for token-major Q,
  // [half][head][row][64] for head-major Q
  const int hoff = (dc >> 3) * (kPoolRows * R * 64) + (a.seq_inner ? h * kPoolRows * 64 : h * 64) + (dc & 7) * 8;
  const int rstride = a.seq_inner ? 64 : R * 64;
  for (int k = 0; k < nitems; ++k) {
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    for (int c = 0; c < kChunks; ++c) {
      const int g = k * kChunks + c, s = g % kPoolKStages;
      const bool ok = mbar_wait(smem_u32(&full_bar[s]), (g / kPoolKStages) & 1, &abort_flag);
      if (ok && h < R) {
        const __nv_bfloat16* chunk = reinterpret_cast<const __nv_bfloat16*>(pool_smem + s * kPoolChunkBytes) + hoff;
#pragma unroll
        for (int r = 0; r < kPoolRows; ++r) {
          const uint4 v = *reinterpret_cast<const uint4*>(chunk + r * rstride);
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            acc[2 * q] += bf16lo(w[q]);
            acc[2 * q + 1] += bf16hi(w[q]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty_bar[s]));
    }
    int b, i, hq0;
    pool_item(a, static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x), b, i, hq0);
    const int nq = min(BQ, a.Lq - i * BQ);  // rows past Lq were loaded as zeros
    const float inv_n = nq == BQ ? 1.0f / BQ : 1.0f / nq;
    float s2 = 0.f;
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float m0 = acc[2 * q] * inv_n, m1 = acc[2 * q + 1] * inv_n;
      s2 = fmaf(m0, m0, s2);
      s2 = fmaf(m1, m1, s2);
      const __nv_bfloat16 h0 = __float2bfloat16_rn(m0), h1 = __float2bfloat16_rn(m1);
      hi[q] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
      lo[q] = pack_bf16x2(m0 - __bfloat162float(h0), m1 - __bfloat162float(h1));
    }
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);  // the 16 threads of head h
    if (h < R) {
      const int64_t row = (static_cast<int64_t>(b) * a.Hq + hq0 + h) * a.nqb + i;
      reinterpret_cast<uint4*>(a.qhi + row * RBS_HEAD_DIM)[dc] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      reinterpret_cast<uint4*>(a.qlo + row * RBS_HEAD_DIM)[dc] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      if (dc == 0) a.qnorm[row] = sqrtf(s2);
    }
  }
}

// ---------------------------------------------------------------------------
// Scores on the tensor core

constexpr int kGemmThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2-9 epilogue

struct GemmSmem {
  static constexpr int kHalf = 128 * 128;        // 128 rows x 64 dims, bf16
  static constexpr int kPart = 2 * kHalf;        // 128 rows x 128 dims
  static constexpr int kB = 0;                   // pooled queries: hi, lo
  static constexpr int kA = kB + 2 * kPart;      // centroid stages: hi, lo each
  static constexpr int kAStage = 2 * kPart;
  static constexpr int kCols = kA + 2 * kAStage;  // per D column: score row (int), visible blocks (int)
  static constexpr int kBar = kCols + 2 * 128 * 4;
  static constexpr int kTotal = kBar + 256;
  static constexpr int kAlloc = kTotal + 1024;
  static constexpr uint32_t kTmemCols = 256;     // two D buffers of 128 columns
};

enum : int {
  kGmBFull = 0,
  kGmBEmpty = 1,
  kGmAFull = 2,                 // + stage (2)
  kGmAEmpty = kGmAFull + 2,
  kGmDFull = kGmAEmpty + 2,     // + buffer (2)
  kGmDEmpty = kGmDFull + 2,
  kGmNumBars = kGmDEmpty + 2
};

struct GemmArgs {
  CUtensorMap tmChi, tmClo;  // centroid parts as [B, nkb "tokens", Hkv "heads", 128]
  CUtensorMap tmQhi, tmQlo;  // pooled parts [B, Hq, nqb, 128]: box 64 dims x QB blocks x R heads
  float* scores;             // [B * Hq * nqb, nkbp] centroid-branch scores
  int B, Hq, Hkv, nqb, nkb, nkbp, R, QB, ngroups, items;
  int q_block_offset, causal;
};

// Item w -> (batch, first q head hq0 of a group of R, first query block i0 of
// a group of QB): the last query-block groups (the longest rows) first.
__device__ __forceinline__ void gemm_item(const GemmArgs& a, int w, int& b, int& hq0, int& i0) {
  const int nh = a.Hq / a.R;
  const int per_g = a.B * nh;
  const int g = a.ngroups - 1 - w / per_g;
  const int rem = w % per_g;
  b = rem / nh;
  hq0 = (rem % nh) * a.R;
  i0 = g * a.QB;
}

// The k-th item of CTA c of G: a snake over the longest-first item order
// (c, 2G - 1 - c, 2G + c, 4G - 1 - c, ...), so a CTA that takes one of the
// longest items of a round takes one of the shortest of the next: the items'
// tile counts fall from 8 to 1 at 128K, and the busiest CTA's total drops
// from half again the mean (round-robin) to about the mean.  Increasing in k.
__device__ __forceinline__ int gemm_work(int k, int c, int G) { return (k & 1) ? (k + 1) * G - 1 - c : k * G + c; }

__device__ __forceinline__ int gemm_tiles(const GemmArgs& a, int i0) {
  const int i_last = min(a.nqb - 1, i0 + a.QB - 1);
  const int n = a.causal ? min(a.nkb, i_last + a.q_block_offset + 1) : a.nkb;
  return (n + 127) / 128;
}

__global__ void __launch_bounds__(kGemmThreads, 1) score_gemm_kernel(const __grid_constant__ GemmArgs a) {
  using L = GemmSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sB = sbase + L::kB, sA = sbase + L::kA;
  const uint32_t bars = sbase + L::kBar;
  auto bar = [&](int k) -> uint32_t { return bars + 8u * k; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + kGmNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kBar + kGmNumBars * 8 + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.Hq / a.Hkv;
  const int cta = static_cast<int>(blockIdx.x), grid = static_cast<int>(gridDim.x);
  int nitems = 0;
  while (gemm_work(nitems, cta, grid) < a.items) ++nitems;

  if (tid == 0) {
    mbar_init(bar(kGmBFull), 1);
    mbar_init(bar(kGmBEmpty), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kGmAFull + s), 1);
      mbar_init(bar(kGmAEmpty + s), 1);
      mbar_init(bar(kGmDFull + s), 1);
      mbar_init(bar(kGmDEmpty + s), 8);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t b_bytes = static_cast<uint32_t>(a.R * a.QB * 128 * 2);  // one part, both halves

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&a.tmChi);
      tma_prefetch_desc(&a.tmClo);
      tma_prefetch_desc(&a.tmQhi);
      tma_prefetch_desc(&a.tmQlo);
      uint32_t gt = 0, nb = 0;
      bool ok = true;
      for (int k = 0; k < nitems && ok; ++k) {
        int b, hq0, i0;
        gemm_item(a, gemm_work(k, cta, grid), b, hq0, i0);
        if (k > 0 && !mbar_wait(bar(kGmBEmpty), (k - 1) & 1, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(bar(kGmBFull), 2 * b_bytes);
        // box rows (R heads x QB blocks) land as 128-byte rows h * QB + ii of each half
        tma_load_4d(sB, &a.tmQhi, bar(kGmBFull), 0, i0, hq0, b);
        tma_load_4d(sB + L::kHalf, &a.tmQhi, bar(kGmBFull), 64, i0, hq0, b);
        tma_load_4d(sB + L::kPart, &a.tmQlo, bar(kGmBFull), 0, i0, hq0, b);
        tma_load_4d(sB + L::kPart + L::kHalf, &a.tmQlo, bar(kGmBFull), 64, i0, hq0, b);
        ++nb;
        const int kvh = hq0 / G;
        const int T = gemm_tiles(a, i0);
        for (int m = 0; m < T; ++m, ++gt) {
          const int s = gt & 1;
          if (gt >= 2 && !mbar_wait(bar(kGmAEmpty + s), ((gt >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
          const uint32_t dst = sA + s * L::kAStage;
          mbar_arrive_expect_tx(bar(kGmAFull + s), L::kAStage);
          tma_load_4d(dst, &a.tmChi, bar(kGmAFull + s), 0, m * 128, kvh, b);
          tma_load_4d(dst + L::kHalf, &a.tmChi, bar(kGmAFull + s), 64, m * 128, kvh, b);
          tma_load_4d(dst + L::kPart, &a.tmClo, bar(kGmAFull + s), 0, m * 128, kvh, b);
          tma_load_4d(dst + L::kPart + L::kHalf, &a.tmClo, bar(kGmAFull + s), 64, m * 128, kvh, b);
        }
      }
      for (uint32_t s = 0; s < 2; ++s)
        if (s < gt) mbar_drain(bar(kGmAFull + s), ((gt - s + 1) / 2 - 1) & 1);
      if (nb > 0) mbar_drain(bar(kGmBFull), (nb - 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (whole warp, one elected lane)
    constexpr uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
    const uint64_t adesc0 = smem_desc(sA, 16, 1024, kLayoutSW128);
    const uint64_t bdesc0 = smem_desc(sB, 16, 1024, kLayoutSW128);
    constexpr uint32_t kHalfU = L::kHalf >> 4, kPartU = L::kPart >> 4, kStageU = L::kAStage >> 4;
    auto wait = [&](int k, uint32_t parity) { return __all_sync(0xffffffffu, mbar_wait(bar(k), parity, abort_flag)); };
    uint32_t gt = 0;
    bool ok = true;
    for (int k = 0; k < nitems && ok; ++k) {
      int b, hq0, i0;
      gemm_item(a, gemm_work(k, cta, grid), b, hq0, i0);
      if (!wait(kGmBFull, k & 1)) break;
      const int T = gemm_tiles(a, i0);
      for (int m = 0; m < T; ++m, ++gt) {
        const int s = gt & 1, db = gt & 1;
        if (!wait(kGmAFull + s, (gt >> 1) & 1)) { ok = false; break; }
        if (gt >= 2 && !wait(kGmDEmpty + db, ((gt >> 1) - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        // D = A_hi B_hi + A_lo B_hi + A_hi B_lo
#pragma unroll
        for (int p = 0; p < 3; ++p) {
          const uint32_t apart = p == 1 ? kPartU : 0u, bpart = p == 2 ? kPartU : 0u;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kHalfU + (kk & 3) * 2;
            umma_ss_warp(tmem + db * 128, adesc0 + s * kStageU + apart + off, bdesc0 + bpart + off, idesc,
                         (p | kk) != 0 ? 1u : 0u);
          }
        }
        umma_commit_warp(bar(kGmAEmpty + s));
        umma_commit_warp(bar(kGmDFull + db));
      }
      if (ok) umma_commit_warp(bar(kGmBEmpty));
    }
  } else {
    // ------------------------------------------------------------ epilogue: scores to the workspace
    // warps 2-9: lane quarter warp % 4, columns [64 * ((warp - 2) / 4), + 64)
    const int quarter = warp & 3, chalf = (warp - 2) >> 2;
    const int etid = tid - 64;  // 0..255
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    int* col_row = reinterpret_cast<int*>(smem + L::kCols);  // score row of column c (-1: none)
    int* col_n = col_row + 128;                              // its visible key blocks
    // After a timeout (ok false) every epilogue warp still walks the items and
    // meets the named barriers, so none waits there for a warp that left.
    uint32_t gt = 0;
    bool ok = true;
    for (int k = 0; k < nitems; ++k) {
      int b, hq0, i0;
      gemm_item(a, gemm_work(k, cta, grid), b, hq0, i0);
      const int T = gemm_tiles(a, i0);
      named_bar_sync(1, 256);  // the previous item's columns are no longer read
      if (etid < 128) {
        // column c = hh * QB + ii holds row (hq0 + hh, i0 + ii)
        const int c = etid, hh = c / a.QB, i = i0 + c % a.QB;
        const bool valid = hh < a.R && i < a.nqb;
        col_row[c] = valid ? ((b * a.Hq + hq0 + hh) * a.nqb + i) : -1;
        col_n[c] = valid ? (a.causal ? min(a.nkb, i + a.q_block_offset + 1) : a.nkb) : 0;
      }
      named_bar_sync(1, 256);
      for (int m = 0; m < T && ok; ++m, ++gt) {
        const int db = gt & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(kGmDFull + db), (gt >> 1) & 1, abort_flag))) { ok = false; break; }
        tc_fence_after();
        const int j = m * 128 + quarter * 32 + lane;
        // both 32-column chunks of this warp's half in flight before one wait
        uint32_t va[32], vb[32];
        tmem_ld32(lane_base + db * 128 + 64 * chalf, va);
        tmem_ld32(lane_base + db * 128 + 64 * chalf + 32, vb);
        tmem_wait_ld();
#pragma unroll
        for (int e4 = 0; e4 < 16; ++e4) {
          // the column tables four columns at a time (broadcast reads)
          const int4 rw = reinterpret_cast<const int4*>(col_row + 64 * chalf)[e4];
          const int4 nn = reinterpret_cast<const int4*>(col_n + 64 * chalf)[e4];
          const int rows4[4] = {rw.x, rw.y, rw.z, rw.w}, ns4[4] = {nn.x, nn.y, nn.z, nn.w};
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (j < ns4[q])
              a.scores[static_cast<int64_t>(rows4[q]) * a.nkbp + j] =
                  __uint_as_float(e4 < 8 ? va[4 * e4 + q] : vb[4 * (e4 - 8) + q]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kGmDEmpty + db));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Top-k from the stored scores

struct TopkArgs {
  SelectArgs s;
  const float* scores;  // [rows, nkbp]
  const float* qnorm;   // [rows]
  // instead of scores: [rows][2 branches][nkbp] order-preserving keys of
  // both branches' scores (per-token-max scoring), or null
  const uint32_t* keys;
  int nkbp, rows;
  // grid (B * nhg, nqb): x = (batch, group of kTopkWarps q heads), y = the
  // query block counted from the last; reciprocals for exact small-integer
  // division, (x + 0.5) * (1 / d) (launch_topk_rows sets these)
  int nhg;
  float inv_nhg, inv_g;
  int y0;  // the query-block index (from the last) of blockIdx.y = 0 (launches of at most 65535 rows of the grid)
};

// Rows (one warp each) per CTA of topk_rows_kernel.  The kernel is bound by
// instruction issue, so the more warps an SM holds the better; its shared
// memory (two key rows per warp) and registers cap that near 20 warps, which
// CTAs of four warps reach (five per SM) and CTAs of eight (two) do not.
constexpr int kTopkWarps = 4;

// Shared memory of topk_rows_kernel: per warp the row's scores and the KV
// head's r_j beta_j (nkbp floats each), then per warp the top-k scratch.
__host__ __device__ constexpr size_t topk_smem_bytes(int nkbp, int nwords) {
  return static_cast<size_t>(kTopkWarps) * (2 * nkbp + sel_topk_scratch_words(nwords)) * 4;
}

template <int KPL>
__global__ void __launch_bounds__(kTopkWarps * 32) topk_rows_kernel(TopkArgs t) {
  extern __shared__ __align__(16) float topk_smem[];
  const SelectArgs& a = t.s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // rows with the last query blocks (the longest) first; no integer
  // division: (x + 0.5) / d is at least 0.5 / d from the next integer, far
  // beyond the float error for these sizes
  const int bx = static_cast<int>(blockIdx.x);
  const int b = __float2int_rz((static_cast<float>(bx) + 0.5f) * t.inv_nhg);
  const int hq = (bx - b * t.nhg) * kTopkWarps + warp;
  if (hq >= a.Hq) return;
  const int i = a.nqb - 1 - (t.y0 + static_cast<int>(blockIdx.y));
  const int kvh = __float2int_rz((static_cast<float>(hq) + 0.5f) * t.inv_g);
  const int gi = i + a.q_block_offset;
  const int n = a.causal ? min(a.nkb, gi + 1) : a.nkb;
  const int64_t row = (static_cast<int64_t>(b) * a.Hq + hq) * a.nqb + i;
  const int64_t kv_off = static_cast<int64_t>(b * a.Hkv + kvh) * a.nkb;
  float* ssc = topk_smem + warp * 2 * t.nkbp;
  float* srb = ssc + t.nkbp;
  uint32_t* scratch =
      reinterpret_cast<uint32_t*>(topk_smem + kTopkWarps * 2 * t.nkbp) + warp * sel_topk_scratch_words(a.nwords);
  // both branches' order-preserving keys of blocks 0 .. n-1, in place
  uint32_t* kcs = reinterpret_cast<uint32_t*>(ssc);
  uint32_t* krs = reinterpret_cast<uint32_t*>(srb);
  if (t.keys != nullptr) {
    // the keys as stored, 16 bytes at a time (each row starts 128-byte
    // aligned; 4 ceil(n / 4) <= nkbp)
    const uint4* srcc = reinterpret_cast<const uint4*>(t.keys + row * 2 * t.nkbp);
    const uint4* srcr = reinterpret_cast<const uint4*>(t.keys + row * 2 * t.nkbp + t.nkbp);
    for (int q = lane; q < (n + 3) / 4; q += 32) {
      reinterpret_cast<uint4*>(kcs)[q] = srcc[q];
      reinterpret_cast<uint4*>(krs)[q] = srcr[q];
    }
  } else {
    // The row's keys of s_c and of s_r = s_c + |qbar| r_j beta_j, into
    // shared memory.  Every global load of a chunk of up to 32 x 4 key blocks
    // is issued before any is used (one memory round trip per chunk, not
    // per key block): the scores with 16-byte loads (each row starts 128-byte
    // aligned and is padded to nkbp), r_j and beta_j with 16-byte loads when
    // their rows are 16-byte aligned (nkb a multiple of 4), else 4-byte ones.
    const float4* src = reinterpret_cast<const float4*>(t.scores + row * t.nkbp);
    const float qn = t.qnorm[row];
    const int nq4 = (n + 3) / 4;
    // float4 per lane per chunk: as many as the longest row of this
    // instantiation needs, at most 4 (512 key blocks); a longer row takes
    // several chunks.  Every slot of a chunk issues its instructions whether
    // or not it holds a block, so a larger chunk would cost the shorter rows
    // of an instantiation more than the extra round trip costs the longest.
    constexpr int kU = KPL / 4 < 1 ? 1 : (KPL / 4 > 4 ? 4 : KPL / 4);
    const bool vec = (a.nkb & 3) == 0;
    for (int base = 0; base < nq4; base += 32 * kU) {
      float4 s4[kU], r4[kU], b4[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int q = base + lane + 32 * u;
        s4[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        r4[u] = b4[u] = s4[u];
        if (q < nq4) {
          s4[u] = src[q];
          if (vec) {
            r4[u] = reinterpret_cast<const float4*>(a.rad + kv_off)[q];
            b4[u] = reinterpret_cast<const float4*>(a.beta + kv_off)[q];
          } else {
            const int j0 = 4 * q;
            r4[u] = make_float4(a.rad[kv_off + j0], j0 + 1 < n ? a.rad[kv_off + j0 + 1] : 0.f,
                                j0 + 2 < n ? a.rad[kv_off + j0 + 2] : 0.f, j0 + 3 < n ? a.rad[kv_off + j0 + 3] : 0.f);
            b4[u] = make_float4(a.beta[kv_off + j0], j0 + 1 < n ? a.beta[kv_off + j0 + 1] : 0.f,
                                j0 + 2 < n ? a.beta[kv_off + j0 + 2] : 0.f,
                                j0 + 3 < n ? a.beta[kv_off + j0 + 3] : 0.f);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int q = base + lane + 32 * u;
        if (q < nq4) {
          const float sv[4] = {s4[u].x, s4[u].y, s4[u].z, s4[u].w};
          const float rv[4] = {r4[u].x * b4[u].x, r4[u].y * b4[u].y, r4[u].z * b4[u].z, r4[u].w * b4[u].w};
          uint4 kc, kr;
          kc.x = order_key(sv[0]); kc.y = order_key(sv[1]); kc.z = order_key(sv[2]); kc.w = order_key(sv[3]);
          kr.x = order_key(fmaf(qn, rv[0], sv[0]));
          kr.y = order_key(fmaf(qn, rv[1], sv[1]));
          kr.z = order_key(fmaf(qn, rv[2], sv[2]));
          kr.w = order_key(fmaf(qn, rv[3], sv[3]));
          reinterpret_cast<uint4*>(kcs)[q] = kc;
          reinterpret_cast<uint4*>(krs)[q] = kr;
        }
      }
    }
  }
  __syncwarp();
  if (a.threshold_mode == 1) {
    // the scores back from their keys (an exact inverse)
    auto fc = [&](int j) { return key_to_float(kcs[j]); };
    auto fr = [&](int j) { return key_to_float(krs[j]); };
    select_row<2, KPL>(a, fc, fr, row, lane, gi, n, scratch);  // no key slots used in this mode
    return;
  }
  auto kc = [&](int s) -> uint32_t {
    const int j = 32 * s + lane;
    return j < n ? kcs[j] : 0u;
  };
  auto kr = [&](int s) -> uint32_t {
    const int j = 32 * s + lane;
    return j < n ? krs[j] : 0u;
  };
  if (KPL > 2 && n <= 64) select_row_keys<2, KPL>(a, kc, kr, row, lane, gi, n, scratch);
  else if (KPL > 8 && n <= 256) select_row_keys<8, KPL>(a, kc, kr, row, lane, gi, n, scratch);
  else if (KPL > 16 && n <= 512) select_row_keys<16, KPL>(a, kc, kr, row, lane, gi, n, scratch);
  else if (KPL > 32 && n <= 1024) select_row_keys<32, KPL>(a, kc, kr, row, lane, gi, n, scratch);
  else select_row_keys<KPL, KPL>(a, kc, kr, row, lane, gi, n, scratch);
}

}  // namespace rbs
