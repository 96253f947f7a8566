// Per-token-max scoring of the two branches on the tensor core
// ([RBS-en] "The Fix" scores a key block against a query q; here q runs over
// the query block's tokens and the block keeps each branch's best token):
//   s_c(i, j) = max_t q_t . c_j
//   s_r(i, j) = max_t (q_t . c_j + |q_t| r_j beta_j)
// over the (valid) tokens t of query block i.  The dot products of a query
// block's BQ tokens with 128 centroids at a time are one 128 x BQ x 128 MMA:
// A = the centroid tile (128 key blocks x 128 dims, K-major), B = the query
// tile (BQ tokens x 128 dims, K-major), D = 128 key blocks (TMEM lanes) x BQ
// tokens (columns), fp32.  The fp32 centroids enter as two bf16 parts, c =
// hi + lo with hi = bf16(c), lo = bf16(c - hi), and both products accumulate
// into D, so with bf16 queries every product is exact and only the fp32
// accumulation and lo's rounding (2^-17 of c) remain.  Each epilogue thread
// owns one key block (its TMEM lane) and takes the two maxima over half of
// its row of BQ columns in registers.  Selection then proceeds as for the
// mean query.
//
// Roles (384 threads, one CTA per SM, persistent over rows (batch, q head,
// query block), longest rows first):
//   warps 0-7  token norms |q_t| from the query tile in shared memory (the
//              four warps of a token half a quarter each, shared through a
//              double-buffered array), then per key tile the two maxima over
//              half the tokens (two warps per TMEM lane quarter); the halves
//              meet through atomicMax on order-preserving keys in a
//              double-buffered shared row
//   warp 8     TMA producer: the query tile (once per row) and the hi / lo
//              centroid tiles (2-stage ring), no multicast
//   warp 9     TMEM allocation and the MMA issue (one elected lane)
//   warps 10-11 alternate rows: with a key matrix in the workspace they copy
//              the row's keys there (topk_rows_kernel selects from them
//              afterwards, eight rows per CTA); without one they run both
//              branches' top-k of the row themselves
#pragma once

#include "common.cuh"
#include "select.cuh"
#include "stats.cuh"

namespace rbs {

constexpr int kTokThreads = 384;
constexpr int kTokCStages = 2;
constexpr int kTokMaxKV = 2048;  // key blocks per sequence in this mode

template <int BQ>
struct TokSmem {
  static constexpr int kQBytes = BQ * 256;       // BQ tokens x 128 dims (two 64-dim halves of BQ x 128 B)
  static constexpr int kCHalf = 128 * 128;       // 128 key blocks x 64 dims, bf16
  static constexpr int kCPart = 2 * kCHalf;      // one part (hi or lo): 32 KB
  static constexpr int kCStage = 2 * kCPart;     // hi then lo
  static constexpr int kQ = 0;
  static constexpr int kC = kQ + kQBytes;        // 1024-aligned: kQBytes is 16 or 32 KB
  static constexpr int kScores = kC + kTokCStages * kCStage;  // uint32 keys [2 rows][2 branches][kTokMaxKV]
  static constexpr int kQn = kScores + 2 * 2 * kTokMaxKV * 4;  // token norms, float [2 row buffers][128 tokens]
  static constexpr int kScratch = kQn + 8 * 64 * 4;            // top-k scratch of warps 10 and 11
  static constexpr int kScratchWords = sel_topk_scratch_words(kTokMaxKV / 32);
  static constexpr int kBar = kScratch + 2 * kScratchWords * 4;
  static constexpr int kBarBytes = 256;
  static constexpr int kTotal = kBar + kBarBytes;
  static constexpr int kAlloc = kTotal + 1024;  // slack to align the base to 1024
  static constexpr uint32_t kTmemCols = 256;    // two D buffers of BQ columns
};

enum : int {
  kTokQFull = 0,
  kTokQEmpty = 1,                   // MMA commit + 8 epilogue warps
  kTokCFull = 2,                    // + stage
  kTokCEmpty = kTokCFull + kTokCStages,
  kTokDFull = kTokCEmpty + kTokCStages,  // + D buffer
  kTokDEmpty = kTokDFull + 2,
  kTokSFull = kTokDEmpty + 2,       // + score row buffer
  kTokSEmpty = kTokSFull + 2,
  kTokNFull = kTokSEmpty + 2,       // + 2 * token half + norm buffer: the half's 4 epilogue warps
  kTokNumBars = kTokNFull + 4
};

struct TokArgs {
  CUtensorMap tmQ, tmChi, tmClo;  // Q [B, Lq, Hq, 128]; centroid parts [B, Hkv, nkb, 128] (token index = block)
  SelectArgs s;
  int rows;  // work items: B * Hq * nqb
  // [rows][2 branches][nkbp] order-preserving keys of the blocks' maxima
  // (row as for the masks), or null to select inside this kernel
  uint32_t* keys_out;
  int nkbp;  // multiple of 32, >= nkb
};

// Row w -> (batch, q head, query block): the last query blocks first.
__device__ __forceinline__ void tok_item(const SelectArgs& a, int w, int& b, int& hq, int& i) {
  const int per_i = a.B * a.Hq;
  i = a.nqb - 1 - w / per_i;
  const int rem = w % per_i;
  b = rem / a.Hq;
  hq = rem % a.Hq;
}

template <int BQ, int KPL>
__global__ void __launch_bounds__(kTokThreads, 1) select_tokmax_kernel(const __grid_constant__ TokArgs ta) {
  using L = TokSmem<BQ>;
  const SelectArgs& a = ta.s;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + L::kQ, sC = sbase + L::kC;
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem + L::kScores);
  float* qn_s = reinterpret_cast<float*>(smem + L::kQn);
  const uint32_t bars = sbase + L::kBar;
  auto bar = [&](int k) -> uint32_t { return bars + 8u * k; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + kTokNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kBar + kTokNumBars * 8 + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.Hq / a.Hkv;
  const int nitems = ta.rows > static_cast<int>(blockIdx.x)
                         ? (ta.rows - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                         : 0;
  auto visible = [&](int i) { return a.causal ? min(a.nkb, i + a.q_block_offset + 1) : a.nkb; };

  if (tid == 0) {
    mbar_init(bar(kTokQFull), 1);
    mbar_init(bar(kTokQEmpty), 1 + 8);
    for (int s = 0; s < kTokCStages; ++s) {
      mbar_init(bar(kTokCFull + s), 1);
      mbar_init(bar(kTokCEmpty + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kTokDFull + s), 1);
      mbar_init(bar(kTokDEmpty + s), 8);
      mbar_init(bar(kTokSFull + s), 8);
      mbar_init(bar(kTokSEmpty + s), 1);
    }
    for (int s = 0; s < 4; ++s) mbar_init(bar(kTokNFull + s), 4);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // the key rows start at 0 (below every float's key); the top-k warps
  // clear each row they consume
  for (int o = tid; o < 2 * 2 * kTokMaxKV; o += kTokThreads) keys[o] = 0u;
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&ta.tmQ);
      tma_prefetch_desc(&ta.tmChi);
      tma_prefetch_desc(&ta.tmClo);
      uint32_t gt = 0, nq = 0;  // centroid tiles and query tiles issued
      bool ok = true;
      for (int k = 0; k < nitems && ok; ++k) {
        int b, hq, i;
        tok_item(a, static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x), b, hq, i);
        // the previous row's MMAs and token norms are done with the query tile
        if (k > 0 && !mbar_wait(bar(kTokQEmpty), (k - 1) & 1, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(bar(kTokQFull), BQ * 256);
        tma_load_4d(sQ, &ta.tmQ, bar(kTokQFull), 0, hq, i * BQ, b);
        tma_load_4d(sQ + BQ * 128, &ta.tmQ, bar(kTokQFull), 64, hq, i * BQ, b);
        ++nq;
        const int kvh = hq / G;
        const int T = (visible(i) + 127) / 128;
        for (int m = 0; m < T; ++m, ++gt) {
          const int s = gt % kTokCStages;
          // the stage's previous tile, gt - 2, must be consumed by its MMAs
          if (gt >= kTokCStages && !mbar_wait(bar(kTokCEmpty + s), ((gt / kTokCStages) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t dst = sC + s * L::kCStage;
          mbar_arrive_expect_tx(bar(kTokCFull + s), L::kCStage);
          tma_load_4d(dst, &ta.tmChi, bar(kTokCFull + s), 0, m * 128, kvh, b);
          tma_load_4d(dst + L::kCHalf, &ta.tmChi, bar(kTokCFull + s), 64, m * 128, kvh, b);
          tma_load_4d(dst + L::kCPart, &ta.tmClo, bar(kTokCFull + s), 0, m * 128, kvh, b);
          tma_load_4d(dst + L::kCPart + L::kCHalf, &ta.tmClo, bar(kTokCFull + s), 64, m * 128, kvh, b);
        }
      }
      // every load issued must land before the CTA exits: stage s was filled
      // at tile numbers s, s + 2, ...; its last fill completes phase (uses - 1)
      for (uint32_t s = 0; s < kTokCStages; ++s)
        if (s < gt) mbar_drain(bar(kTokCFull + s), ((gt - s + kTokCStages - 1) / kTokCStages - 1) & 1);
      if (nq > 0) mbar_drain(bar(kTokQFull), (nq - 1) & 1);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer (whole warp, one elected lane)
    constexpr uint32_t idesc = idesc_bf16_f32(128, BQ, 0, 0);
    const uint64_t cdesc0 = smem_desc(sC, 16, 1024, kLayoutSW128);
    const uint64_t qdesc0 = smem_desc(sQ, 16, 1024, kLayoutSW128);
    constexpr uint32_t kCHalfU = L::kCHalf >> 4, kCPartU = L::kCPart >> 4, kCStageU = L::kCStage >> 4;
    constexpr uint32_t kQHalfU = (BQ * 128) >> 4;
    auto wait = [&](int k, uint32_t parity) { return __all_sync(0xffffffffu, mbar_wait(bar(k), parity, abort_flag)); };
    uint32_t gt = 0;
    bool ok = true;
    for (int k = 0; k < nitems && ok; ++k) {
      int b, hq, i;
      tok_item(a, static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x), b, hq, i);
      if (!wait(kTokQFull, k & 1)) break;
      const int T = (visible(i) + 127) / 128;
      for (int m = 0; m < T; ++m, ++gt) {
        const int s = gt % kTokCStages, db = gt & 1;
        if (!wait(kTokCFull + s, (gt / kTokCStages) & 1)) { ok = false; break; }
        // D buffer db held tile gt - 2: its epilogue must have read it
        if (gt >= 2 && !wait(kTokDEmpty + db, ((gt >> 1) - 1) & 1)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int part = 0; part < 2; ++part) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t ad = cdesc0 + s * kCStageU + part * kCPartU + (kk >> 2) * kCHalfU + (kk & 3) * 2;
            const uint64_t bd = qdesc0 + (kk >> 2) * kQHalfU + (kk & 3) * 2;
            umma_ss_warp(tmem + db * BQ, ad, bd, idesc, (part | kk) != 0 ? 1u : 0u);
          }
        }
        umma_commit_warp(bar(kTokCEmpty + s));
        umma_commit_warp(bar(kTokDFull + db));
      }
      if (ok) umma_commit_warp(bar(kTokQEmpty));
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ token norms and the per-block maxima
    const int quarter = warp & 3, thalf = warp >> 2;  // TMEM lane quarter, half of the tokens
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    uint32_t gt = 0;
    bool ok = true;
    for (int k = 0; k < nitems && ok; ++k) {
      int b, hq, i;
      tok_item(a, static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x), b, hq, i);
      const int n = visible(i), T = (n + 127) / 128;
      const int nq = min(BQ, a.Lq - i * BQ);  // valid tokens of this query block
      const int kvh = hq / G;
      const int64_t kv_off = static_cast<int64_t>(b * a.Hkv + kvh) * a.nkb;
      // this row's token norms, shared by the four warps of a token half
      // through norm buffer k & 1: warp (quarter q) takes tokens
      // t0 + q TPW .. t0 + q TPW + TPW - 1, LPT lanes per token, each lane
      // summing CPL of the token's sixteen 16-byte chunks (two 64-dim halves)
      constexpr int TPW = BQ / 8, LPT = 32 / TPW, CPL = 16 / LPT;
      const int t0 = thalf * (BQ / 2), nb = k & 1;
      float* qn = qn_s + nb * 128;  // qn[t] for the tokens t of this row
      if (!__all_sync(0xffffffffu, mbar_wait(bar(kTokQFull), k & 1, abort_flag))) break;
      {
        const int t = t0 + quarter * TPW + lane / LPT, sl = lane % LPT;
        float s2 = 0.f;
#pragma unroll
        for (int cc = 0; cc < CPL; ++cc) {
          // chunk c of the token's 128-byte row in half h sits at chunk
          // position c ^ (t % 8) (128-byte swizzle)
          const int chunk = sl * CPL + cc, h = chunk >> 3, c = chunk & 7;
          const uint4 v =
              *reinterpret_cast<const uint4*>(smem + L::kQ + h * BQ * 128 + t * 128 + ((c ^ (t & 7)) << 4));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            s2 = fmaf(bf16lo(w[q]), bf16lo(w[q]), s2);
            s2 = fmaf(bf16hi(w[q]), bf16hi(w[q]), s2);
          }
        }
#pragma unroll
        for (int o = 1; o < LPT; o <<= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
        if (sl == 0) qn[t] = sqrtf(s2);
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(kTokQEmpty));
        mbar_arrive(bar(kTokNFull + 2 * thalf + nb));
      }
      const int sb = k & 1;
      uint32_t* kc = keys + sb * 2 * kTokMaxKV;
      uint32_t* kr = kc + kTokMaxKV;
      // the top-k of row k - 2 must be done with this score buffer
      if (k >= 2 && !__all_sync(0xffffffffu, mbar_wait(bar(kTokSEmpty + sb), ((k >> 1) - 1) & 1, abort_flag))) break;
      // the other three warps' norms of this half.  Norm buffer nb is written
      // again two rows later, by a warp past the next row's wait: all four
      // warps have finished this row by then.
      if (!__all_sync(0xffffffffu, mbar_wait(bar(kTokNFull + 2 * thalf + nb), (k >> 1) & 1, abort_flag))) break;
      for (int m = 0; m < T; ++m, ++gt) {
        const int db = gt & 1;
        const int j = m * 128 + quarter * 32 + lane;
        const float rho = j < n ? a.rad[kv_off + j] * a.beta[kv_off + j] : 0.f;  // in flight during the wait
        if (!__all_sync(0xffffffffu, mbar_wait(bar(kTokDFull + db), (gt >> 1) & 1, abort_flag))) { ok = false; break; }
        tc_fence_after();
        float mc = -INFINITY, mr = -INFINITY;
#pragma unroll
        for (int c = thalf * (BQ / 64); c < (thalf + 1) * (BQ / 64); ++c) {
          uint32_t v[32];
          tmem_ld32(lane_base + db * BQ + 32 * c, v);
          tmem_wait_ld();
          if (32 * c + 32 <= nq) {
            // all 32 tokens valid (every query block but a short last one):
            // two tokens per 3-input max, four norms per shared load
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              const float4 q4 = *reinterpret_cast<const float4*>(qn + 32 * c + e);
              const float d0 = __uint_as_float(v[e]), d1 = __uint_as_float(v[e + 1]);
              const float d2 = __uint_as_float(v[e + 2]), d3 = __uint_as_float(v[e + 3]);
              mc = fmax3(mc, d0, d1);
              mc = fmax3(mc, d2, d3);
              mr = fmax3(mr, fmaf(q4.x, rho, d0), fmaf(q4.y, rho, d1));
              mr = fmax3(mr, fmaf(q4.z, rho, d2), fmaf(q4.w, rho, d3));
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              if (32 * c + e < nq) {
                const float d = __uint_as_float(v[e]);
                mc = fmaxf(mc, d);
                mr = fmaxf(mr, fmaf(qn[32 * c + e], rho, d));
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kTokDEmpty + db));
        if (j < n) {  // the other half of the tokens meets this one here
          atomicMax(&kc[j], order_key(mc));
          atomicMax(&kr[j], order_key(mr));
        }
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kTokSFull + sb));
    }
  } else {
    // ------------------------------------------------------------ alternate rows: key copy-out or top-k
    const int tk = warp - 10;
    uint32_t* scratch = reinterpret_cast<uint32_t*>(smem + L::kScratch) + tk * L::kScratchWords;
    for (int k = tk; k < nitems; k += 2) {
      int b, hq, i;
      tok_item(a, static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x), b, hq, i);
      const int sb = k & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(kTokSFull + sb), (k >> 1) & 1, abort_flag))) break;
      uint32_t* kc = keys + sb * 2 * kTokMaxKV;
      uint32_t* kr = kc + kTokMaxKV;
      const int n = visible(i), gi = i + a.q_block_offset;
      const int64_t row = (static_cast<int64_t>(b) * a.Hq + hq) * a.nqb + i;
      if (ta.keys_out != nullptr) {
        // both key rows, 16 bytes at a time: slots n .. 4 ceil(n / 4) - 1
        // hold 0 (never raised), and 4 ceil(n / 4) <= nkbp
        uint4* dc = reinterpret_cast<uint4*>(ta.keys_out + row * 2 * ta.nkbp);
        uint4* dr = reinterpret_cast<uint4*>(ta.keys_out + row * 2 * ta.nkbp + ta.nkbp);
        for (int q = lane; q < (n + 3) >> 2; q += 32) {
          dc[q] = reinterpret_cast<const uint4*>(kc)[q];
          dr[q] = reinterpret_cast<const uint4*>(kr)[q];
        }
      } else if (a.threshold_mode == 1) {
        auto fc = [&](int j) { return key_to_float(kc[j]); };
        auto fr = [&](int j) { return key_to_float(kr[j]); };
        select_row<2, KPL>(a, fc, fr, row, lane, gi, n, scratch);  // no key slots used in this mode
      } else {
        auto sc = [&](int s) -> uint32_t {
          const int j = 32 * s + lane;
          return j < n ? kc[j] : 0u;
        };
        auto sr = [&](int s) -> uint32_t {
          const int j = 32 * s + lane;
          return j < n ? kr[j] : 0u;
        };
        if (KPL > 2 && n <= 64) select_row_keys<2, KPL>(a, sc, sr, row, lane, gi, n, scratch);
        else if (KPL > 8 && n <= 256) select_row_keys<8, KPL>(a, sc, sr, row, lane, gi, n, scratch);
        else if (KPL > 16 && n <= 512) select_row_keys<16, KPL>(a, sc, sr, row, lane, gi, n, scratch);
        else if (KPL > 32 && n <= 1024) select_row_keys<32, KPL>(a, sc, sr, row, lane, gi, n, scratch);
        else select_row_keys<KPL, KPL>(a, sc, sr, row, lane, gi, n, scratch);
      }
      __syncwarp();
      for (int j = lane; j < n; j += 32) kc[j] = kr[j] = 0u;  // ready for the buffer's next row
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kTokSEmpty + sb));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// The selection's first launch when it scores on the tensor core: beta of
// every (batch, KV head) in CTAs 0 .. nbeta - 1 (block_beta_body, nbeta =
// B Hkv), in the rest the centroids' bf16 parts c -> (hi, lo): hi = bf16(c),
// lo = bf16(c - hi), both rounded to nearest even, so hi + lo carries c to
// about 2^-17 of its size.
__global__ void __launch_bounds__(1024) select_prep_kernel(const __grid_constant__ BetaArgs ba, int nbeta,
                                                           const float* __restrict__ C, int64_t n,
                                                           __nv_bfloat16* __restrict__ hi,
                                                           __nv_bfloat16* __restrict__ lo) {
  extern __shared__ float prep_sort[];
  if (static_cast<int>(blockIdx.x) < nbeta) {
    block_beta_body(ba, static_cast<int>(blockIdx.x) % ba.H, static_cast<int>(blockIdx.x) / ba.H, prep_sort);
    return;
  }
  const int64_t stride = static_cast<int64_t>(gridDim.x - nbeta) * 1024;
  for (int64_t k = static_cast<int64_t>(blockIdx.x - nbeta) * 1024 + threadIdx.x; k < n; k += stride) {
    const float c = C[k];
    const __nv_bfloat16 h = __float2bfloat16_rn(c);
    hi[k] = h;
    lo[k] = __float2bfloat16_rn(c - __bfloat162float(h));
  }
}

}  // namespace rbs
