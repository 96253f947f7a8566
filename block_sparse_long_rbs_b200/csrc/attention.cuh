// Block-sparse prefill attention on the 5th-generation tensor core.
// ([RBS-en] "The Fix": exact softmax attention over the selected key blocks,
// compatible with standard multi-head / grouped-query attention.)
//
// Work item = one list row (batch b, q head h, query block i): a 128-row
// query tile (BQ valid rows) against the row's listed key blocks, in list
// order.  Persistent CTAs take work items round-robin in an order that
// starts with the last query blocks (the longest causal rows).
//
// Roles (192 threads):
//   warps 0-3  softmax: thread r owns query row r.  Reads S = Q K^T from
//              TMEM, applies the token-level causal mask on the diagonal
//              block, keeps a running max (rescaling O in TMEM only when the
//              max grows by more than 2^8), writes P = exp2(S*c - m) as bf16
//              into a 128B-swizzled shared-memory tile, and finally
//              normalises O and writes it (and the LSE) out.
//   warp 4     TMA producer: Q tile, then K_j and V_j tiles gathered by block
//              index (4-D tensor maps over [B, L, H, 128], 128B swizzle, no
//              multicast), into NS-deep K and V rings.
//   warp 5     TMEM allocator and MMA issuer (one thread): S_t = Q K_t^T into
//              one of two TMEM S buffers, O += P_{t-1} V_{t-1} into the TMEM
//              O accumulator; completion reported with tcgen05.commit.
// Issue order S_0, S_1, PV_0, S_2, PV_1, ... lets the softmax of tile t
// overlap the tensor core's work on tiles t-1 and t+1.
//
// Every mbarrier wait is bounded; on a timeout all roles unwind, in-flight
// TMA loads and MMAs are drained (bounded), TMEM is freed, and the device
// error word records RBS_DEVERR_TIMEOUT.
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

constexpr int kAttnThreads = 192;
constexpr int kNS = 2;  // K and V ring depth

template <int BK>
struct AttnSmem {
  static constexpr int kQBytes = 128 * 128 * 2;  // 128 rows x 128 dims (two 64-dim halves)
  static constexpr int kKVBytes = BK * 128 * 2;  // BK rows x 128 dims (two halves)
  static constexpr int kPBytes = 128 * BK * 2;   // 128 rows x BK keys
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQBytes;
  static constexpr int kV = kK + kNS * kKVBytes;
  static constexpr int kP = kV + kNS * kKVBytes;
  static constexpr int kBar = kP + kPBytes;
  static constexpr int kBarBytes = 256;
  static constexpr int kTotal = kBar + kBarBytes;
  static constexpr int kAlloc = kTotal + 1024;  // slack to align the base to 1024
  static constexpr uint32_t kTmemCols = BK == 128 ? 512 : 256;
  static constexpr uint32_t kColO = 2 * BK;
};

// barrier slots (8 bytes each) in the barrier area
enum : int {
  kBarQFull = 0,
  kBarQEmpty = 1,
  kBarKFull = 2,                // + stage
  kBarKEmpty = kBarKFull + kNS,  // + stage
  kBarVFull = kBarKEmpty + kNS,
  kBarVEmpty = kBarVFull + kNS,
  kBarSFull = kBarVEmpty + kNS,  // + buffer (2)
  kBarSEmpty = kBarSFull + 2,
  kBarPFull = kBarSEmpty + 2,
  kBarPVDone = kBarPFull + 1,
  kBarOEmpty = kBarPVDone + 1,
  kBarDrain = kBarOEmpty + 1,
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

// Row extent with validation (identical in every role).
__device__ __forceinline__ int row_extent(const AttnArgs& a, int row, int& beg) {
  beg = __ldg(a.row_ptr + row);
  const int end = __ldg(a.row_ptr + row + 1);
  if (beg < 0 || end < beg || end > a.capacity) return -1;
  return end - beg;
}

template <int BQ, int BK>
__global__ void __launch_bounds__(kAttnThreads, 1) bsa_prefill_kernel(const __grid_constant__ AttnArgs a) {
  using L = AttnSmem<BK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + L::kQ;
  const uint32_t sK = sbase + L::kK;
  const uint32_t sV = sbase + L::kV;
  const uint32_t sP = sbase + L::kP;
  const uint32_t bars = sbase + L::kBar;
  auto bar = [&](int k) -> uint32_t { return bars + 8u * k; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kBar + kNumBars * 8 + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(bar(kBarQFull), 1);
    mbar_init(bar(kBarQEmpty), 1);
    for (int s = 0; s < kNS; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarVEmpty + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBarSFull + s), 1);
      mbar_init(bar(kBarSEmpty + s), 128);
    }
    mbar_init(bar(kBarPFull), 128);
    mbar_init(bar(kBarPVDone), 1);
    mbar_init(bar(kBarOEmpty), 128);
    mbar_init(bar(kBarDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (BQ < 128) {
    // rows BQ..127 of the Q tile are never loaded: make them zeros once
    uint4* q4 = reinterpret_cast<uint4*>(smem + L::kQ);
    for (int k = tid; k < L::kQBytes / 16; k += kAttnThreads) q4[k] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&a.tmQ);
      tma_prefetch_desc(&a.tmK);
      tma_prefetch_desc(&a.tmV);
      uint32_t nk = 0, nv = 0, item = 0;  // K fills, V fills, Q fills issued
      bool ok = true;
      for (int w = blockIdx.x; w < a.num_rows && ok; w += gridDim.x) {
        int b, h, i, row, beg;
        decode_work(a, w, b, h, i, row);
        const int n = row_extent(a, row, beg);
        if (n <= 0) continue;
        if (item > 0 && !mbar_wait(bar(kBarQEmpty), (item - 1) & 1, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(bar(kBarQFull), BQ * 256);
        tma_load_4d(sQ, &a.tmQ, bar(kBarQFull), 0, h, i * BQ, b);
        tma_load_4d(sQ + 128 * 128, &a.tmQ, bar(kBarQFull), 64, h, i * BQ, b);
        ++item;
        const int kvh = h / (a.Hq / a.Hkv);
        for (int t = 0; t < n; ++t) {
          int j = __ldg(a.col_idx + beg + t);
          if (j < 0 || j >= a.nkb) j = 0;
          const int s = nk % kNS;
          const uint32_t ph = (nk / kNS) & 1;
          if (nk >= kNS && !mbar_wait(bar(kBarKEmpty + s), ph ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(kBarKFull + s), BK * 256);
          tma_load_4d(sK + s * L::kKVBytes, &a.tmK, bar(kBarKFull + s), 0, kvh, j * BK, b);
          tma_load_4d(sK + s * L::kKVBytes + BK * 128, &a.tmK, bar(kBarKFull + s), 64, kvh, j * BK, b);
          ++nk;
          if (nv >= kNS && !mbar_wait(bar(kBarVEmpty + s), ph ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(kBarVFull + s), BK * 256);
          tma_load_4d(sV + s * L::kKVBytes, &a.tmV, bar(kBarVFull + s), 0, kvh, j * BK, b);
          tma_load_4d(sV + s * L::kKVBytes + BK * 128, &a.tmV, bar(kBarVFull + s), 64, kvh, j * BK, b);
          ++nv;
        }
      }
      // drain: every load issued must land before the CTA exits.  Stage s
      // was filled at fill numbers s, s + NS, ...; its last fill completes
      // phase (uses - 1).
      if (item > 0) mbar_drain(bar(kBarQFull), (item - 1) & 1);
      for (uint32_t s = 0; s < kNS; ++s) {
        if (s < nk) mbar_drain(bar(kBarKFull + s), ((nk - s + kNS - 1) / kNS - 1) & 1);
        if (s < nv) mbar_drain(bar(kBarVFull + s), ((nv - s + kNS - 1) / kNS - 1) & 1);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, BK, 0, 0);
      constexpr uint32_t idPV = idesc_bf16_f32(128, 128, 0, 1);
      uint32_t kv_base = 0, g = 0, item = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < a.num_rows && ok; w += gridDim.x) {
        int b, h, i, row, beg;
        decode_work(a, w, b, h, i, row);
        const int n = row_extent(a, row, beg);
        if (n <= 0) continue;
        if (!mbar_wait(bar(kBarQFull), item & 1, abort_flag)) break;
        tc_fence_after();
        for (int t = 0; t <= n; ++t) {
          if (t < n) {
            const uint32_t it = kv_base + t;
            const int s = it % kNS;
            const uint32_t gt = g + t;
            const int sb = gt & 1;
            if (!mbar_wait(bar(kBarKFull + s), (it / kNS) & 1, abort_flag)) { ok = false; break; }
            if (gt >= 2 && !mbar_wait(bar(kBarSEmpty + sb), ((gt >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t dS = tmem + sb * BK;
            const uint32_t kbase = sK + s * L::kKVBytes;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t half = kk >> 2, off = (kk & 3) * 32;
              const uint64_t ad = smem_desc(sQ + half * (128 * 128) + off, 16, 1024, kLayoutSW128);
              const uint64_t bd = smem_desc(kbase + half * (BK * 128) + off, 16, 1024, kLayoutSW128);
              umma_ss(dS, ad, bd, idS, kk > 0 ? 1u : 0u);
            }
            umma_commit(bar(kBarSFull + sb));
            umma_commit(bar(kBarKEmpty + s));
            if (t == n - 1) umma_commit(bar(kBarQEmpty));
          }
          if (t >= 1) {
            const int tp = t - 1;
            const uint32_t it = kv_base + tp;
            const int s = it % kNS;
            const uint32_t gt = g + tp;
            if (!mbar_wait(bar(kBarPFull), gt & 1, abort_flag)) { ok = false; break; }
            if (!mbar_wait(bar(kBarVFull + s), (it / kNS) & 1, abort_flag)) { ok = false; break; }
            if (tp == 0 && item > 0 && !mbar_wait(bar(kBarOEmpty), (item - 1) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t dO = tmem + L::kColO;
            const uint32_t vbase = sV + s * L::kKVBytes;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint32_t half = kk >> 2, off = (kk & 3) * 32;
              const uint64_t ad = smem_desc(sP + half * (128 * 128) + off, 16, 1024, kLayoutSW128);
              const uint64_t bd = smem_desc(vbase + kk * 2048, BK * 128, 1024, kLayoutSW128);
              umma_ss(dO, ad, bd, idPV, (tp > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(bar(kBarVEmpty + s));
            umma_commit(bar(kBarPVDone));
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
    // ------------------------------------------------------------ softmax (warps 0-3)
    const int r = tid;  // query row within the tile == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float c = a.scale_log2;
    uint32_t g = 0, item = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < a.num_rows && ok; w += gridDim.x) {
      int b, h, i, row, beg;
      decode_work(a, w, b, h, i, row);
      const int n = row_extent(a, row, beg);
      const int gi = i + a.q_block_off;
      const int64_t qrow = static_cast<int64_t>(i) * BQ + r;
      if (n <= 0) {
        if (n < 0 && r == 0) raise_error(RBS_DEVERR_ROW_PTR);
        if (r < BQ) {
          uint4* dst = reinterpret_cast<uint4*>(a.O + b * a.ob + qrow * a.os + h * a.oh);
#pragma unroll
          for (int k = 0; k < 16; ++k) dst[k] = make_uint4(0, 0, 0, 0);
          if (a.lse != nullptr) a.lse[(static_cast<int64_t>(b) * a.Hq + h) * a.Lq + qrow] = -INFINITY;
        }
        continue;
      }
      float m_used = -INFINITY;  // running max, in log2 units (score * c)
      float l = 0.f;
      for (int t = 0; t < n; ++t) {
        const uint32_t gt = g + t;
        const int sb = gt & 1;
        const int j = __ldg(a.col_idx + beg + t);
        bool okw = mbar_wait(bar(kBarSFull + sb), (gt >> 1) & 1, abort_flag);
        if (!__all_sync(0xffffffffu, okw)) { ok = false; break; }
        tc_fence_after();
        float s[BK];
#pragma unroll
        for (int q = 0; q < BK / 32; ++q) {
          uint32_t v[32];
          tmem_ld32(lane_base + sb * BK + 32 * q, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) s[32 * q + e] = __uint_as_float(v[e]);
        }
        tc_fence_before();
        mbar_arrive(bar(kBarSEmpty + sb));

        // masking: token-causal on the diagonal, nothing visible past it
        const bool bad = j < 0 || j >= a.nkb;
        if (bad || (a.causal && j > gi)) {
          if (r == 0) raise_error(bad ? RBS_DEVERR_BLOCK_INDEX : RBS_DEVERR_NONCAUSAL);
#pragma unroll
          for (int e = 0; e < BK; ++e) s[e] = -INFINITY;
        } else if (a.causal && j == gi) {
#pragma unroll
          for (int e = 0; e < BK; ++e)
            if (e > r) s[e] = -INFINITY;
        }
        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < BK; ++e) mx = fmaxf(mx, s[e]);
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
        l *= factor;

        // the previous PV must be complete: it frees the P tile and fixes O
        okw = gt == 0 || mbar_wait(bar(kBarPVDone), (gt - 1) & 1, abort_flag);
        if (!__all_sync(0xffffffffu, okw)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t v[32];
            tmem_ld32(lane_base + L::kColO + 32 * q, v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * factor);
            tmem_st32(lane_base + L::kColO + 32 * q, v);
          }
          tmem_wait_st();
        }
        // P = exp2(s*c - m) as bf16 into the 128B-swizzled K-major tile
#pragma unroll
        for (int ch = 0; ch < BK / 8; ++ch) {
          float p[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            p[e] = ptx_exp2(fmaf(s[8 * ch + e], c, -m_exp));
            l += p[e];
          }
          const uint32_t half = ch >> 3, chl = ch & 7;
          const uint32_t addr = sP + half * (128 * 128) + r * 128 + ((chl ^ (r & 7)) << 4);
          st_shared_v4(addr, pack_bf16x2(p[0], p[1]), pack_bf16x2(p[2], p[3]), pack_bf16x2(p[4], p[5]),
                       pack_bf16x2(p[6], p[7]));
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(kBarPFull));
      }
      if (!ok) break;
      // epilogue: O / l -> bf16, LSE
      {
        const uint32_t glast = g + n - 1;
        const bool okw = mbar_wait(bar(kBarPVDone), glast & 1, abort_flag);
        if (!__all_sync(0xffffffffu, okw)) { ok = false; break; }
        tc_fence_after();
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
        uint4* dst = reinterpret_cast<uint4*>(a.O + b * a.ob + qrow * a.os + h * a.oh);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t v[32];
          tmem_ld32(lane_base + L::kColO + 32 * q, v);
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
        if (a.lse != nullptr && r < BQ) {
          a.lse[(static_cast<int64_t>(b) * a.Hq + h) * a.Lq + qrow] =
              l > 0.f ? (m_used + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
        }
        tc_fence_before();
        mbar_arrive(bar(kBarOEmpty));
      }
      g += n;
      ++item;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace rbs
