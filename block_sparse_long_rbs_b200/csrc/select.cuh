// Two-branch block selection ([RBS-en] "The Fix: A Radius-Adaptive Rescue
// Branch"; [RBS-id] "Dual-Branch Selection"):
//   s_c(i, j) = qbar_i . c_j
//   s_r(i, j) = s_c(i, j) + |qbar_i| * r_j * beta_j
// each branch keeps its own top ceil(rho * n_i) of the n_i visible key
// blocks (ties to the lower index), the kept sets are OR-ed with the forced
// blocks, and the rows are compacted into CSR lists.
//
// Kernels:
//   select_rows_kernel  one CTA per (query block, group of R q heads of one
//                       KV head, batch).  Scores for all visible blocks are
//                       computed into shared memory (centroid tiles staged
//                       through shared memory, 256 blocks x 32 dims at a
//                       time), then warp w < R finds the exact k-th largest
//                       score of its row's branch by a 32-step bitwise search
//                       over order-preserving keys held in registers, breaks
//                       ties by block index with warp ballots, and emits one
//                       32-bit mask word per 32 blocks (bit = lane).
//   scan_counts_kernel  exclusive scan of the per-row counts -> row_ptr.
//   compact_lists_kernel one warp per row turns mask words into ascending
//                       block indices and per-entry branch flags.
#pragma once

#include "common.cuh"

namespace rbs {

struct SelectArgs {
  const float* qbar;   // [B, Hq, nqb, 128]
  const float* qnorm;  // [B, Hq, nqb]
  const float* C;      // [B, Hkv, nkb, 128]
  const float* rad;    // [B, Hkv, nkb]
  const float* beta;   // [B, Hkv, nkb]
  int Hq, Hkv, nqb, nkb, R, nwords;
  int q_block_offset, causal, force_diag, force_sink;
  float rho_c, rho_r;
  uint32_t* mask_c;  // [rows, nwords]
  uint32_t* mask_r;  // [rows, nwords]
  int* counts;       // [rows]
};

constexpr int kSelThreads = 256;
constexpr int kSelMaxR = 8;
constexpr int kStageJ = 256;  // key blocks per staged centroid tile
constexpr int kStageD = 32;   // dims per staged centroid tile
constexpr int kStagePitch = kStageD + 1;

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ int keep_count(float rho, int n) {
  // k = ceil(rho * n) within [1, n]; rho is the float32 parameter widened to
  // double, and the 1e-4 slack absorbs its float32 representation error.
  int k = static_cast<int>(ceil(static_cast<double>(rho) * n - 1e-4));
  return k < 1 ? 1 : (k > n ? n : k);
}

// Exact top-k of the warp's keys (key 0 = not a candidate; k <= #candidates):
// returns, per lane, the mask words this lane owns (word t is owned by lane
// t % 32) with bit `lane` of word t set iff block 32t + lane is kept.
template <int KPL>
__device__ __forceinline__ void warp_topk_words(const uint32_t (&key)[KPL], int k, int lane,
                                                uint32_t (&own)[(KPL + 31) / 32]) {
  uint32_t T = 0;
#pragma unroll 1
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    int cnt = 0;
#pragma unroll
    for (int t = 0; t < KPL; ++t) cnt += key[t] >= cand ? 1 : 0;
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (cnt >= k) T = cand;
  }
  int gt = 0;
#pragma unroll
  for (int t = 0; t < KPL; ++t) gt += key[t] > T ? 1 : 0;
  gt = __reduce_add_sync(0xffffffffu, gt);
  const int need = k - gt;  // ties at T to keep, lowest block index first
  const uint32_t lt_mask = (1u << lane) - 1u;
  int base = 0;
#pragma unroll
  for (int t = 0; t < (KPL + 31) / 32; ++t) own[t] = 0;
#pragma unroll
  for (int t = 0; t < KPL; ++t) {
    const bool tie = key[t] == T;
    const uint32_t bal = __ballot_sync(0xffffffffu, tie);
    const int rank = base + __popc(bal & lt_mask);
    const bool sel = key[t] > T || (tie && rank < need);
    const uint32_t word = __ballot_sync(0xffffffffu, sel);
    if (lane == (t & 31)) own[t >> 5] = word;
    base += __popc(bal);
  }
}

template <int KPL>
__global__ void __launch_bounds__(kSelThreads) select_rows_kernel(SelectArgs a) {
  extern __shared__ __align__(16) float sm[];
  const int i = blockIdx.x, hblk = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int R = a.R;
  const int G = a.Hq / a.Hkv;
  const int hq0 = hblk * R;
  const int kvh = hq0 / G;
  const int gi = i + a.q_block_offset;
  const int n = a.causal ? min(a.nkb, gi + 1) : a.nkb;
  const int npad = (a.nkb + 31) & ~31;

  float* qs = sm;                         // [R][128]
  float* rb = qs + kSelMaxR * 128;        // [npad]  r_j * beta_j
  float* sc = rb + npad;                  // [R][npad] centroid-branch scores
  float* cs = sc + kSelMaxR * npad;       // [kStageJ][kStagePitch]
  __shared__ float qn[kSelMaxR];

  const int64_t kv_off = static_cast<int64_t>(b * a.Hkv + kvh) * a.nkb;
  for (int idx = tid; idx < R * 128; idx += kSelThreads) {
    const int h = idx >> 7, d = idx & 127;
    qs[idx] = a.qbar[(static_cast<int64_t>(b * a.Hq + hq0 + h) * a.nqb + i) * 128 + d];
  }
  if (tid < R) qn[tid] = a.qnorm[static_cast<int64_t>(b * a.Hq + hq0 + tid) * a.nqb + i];
  for (int j = tid; j < n; j += kSelThreads) rb[j] = a.rad[kv_off + j] * a.beta[kv_off + j];

  // ---- scores s_c for j < n
  const float* Cb = a.C + kv_off * 128;
  for (int j0 = 0; j0 < n; j0 += kStageJ) {
    const int jn = min(kStageJ, n - j0);
    float acc[kSelMaxR];
#pragma unroll
    for (int h = 0; h < kSelMaxR; ++h) acc[h] = 0.f;
    for (int d0 = 0; d0 < 128; d0 += kStageD) {
      __syncthreads();
#pragma unroll
      for (int u = 0; u < (kStageJ * kStageD / 4) / kSelThreads; ++u) {
        const int idx = tid + kSelThreads * u;
        const int jl = idx >> 3, d4 = idx & 7;
        if (jl < jn) {
          const float4 v = *reinterpret_cast<const float4*>(Cb + static_cast<int64_t>(j0 + jl) * 128 + d0 + 4 * d4);
          float* dst = cs + jl * kStagePitch + 4 * d4;
          dst[0] = v.x;
          dst[1] = v.y;
          dst[2] = v.z;
          dst[3] = v.w;
        }
      }
      __syncthreads();
      if (tid < jn) {
        const float* crow = cs + tid * kStagePitch;
#pragma unroll 4
        for (int d = 0; d < kStageD; d += 4) {
          const float c0 = crow[d], c1 = crow[d + 1], c2 = crow[d + 2], c3 = crow[d + 3];
#pragma unroll
          for (int h = 0; h < kSelMaxR; ++h) {
            if (h < R) {
              const float4 q = *reinterpret_cast<const float4*>(qs + h * 128 + d0 + d);
              acc[h] = fmaf(q.x, c0, acc[h]);
              acc[h] = fmaf(q.y, c1, acc[h]);
              acc[h] = fmaf(q.z, c2, acc[h]);
              acc[h] = fmaf(q.w, c3, acc[h]);
            }
          }
        }
      }
    }
    if (tid < jn) {
#pragma unroll
      for (int h = 0; h < kSelMaxR; ++h)
        if (h < R) sc[h * npad + j0 + tid] = acc[h];
    }
  }
  __syncthreads();

  // ---- per-branch top-k, one warp per row
  if (warp < R) {
    const int hq = hq0 + warp;
    const int64_t row = (static_cast<int64_t>(b) * a.Hq + hq) * a.nqb + i;
    const float qnv = qn[warp];
    constexpr int NO = (KPL + 31) / 32;
    uint32_t own_c[NO], own_r[NO];
    {
      uint32_t key[KPL];
#pragma unroll
      for (int t = 0; t < KPL; ++t) {
        const int j = 32 * t + lane;
        key[t] = j < n ? order_key(sc[warp * npad + j]) : 0u;
      }
      warp_topk_words<KPL>(key, keep_count(a.rho_c, n), lane, own_c);
    }
    {
      uint32_t key[KPL];
#pragma unroll
      for (int t = 0; t < KPL; ++t) {
        const int j = 32 * t + lane;
        key[t] = j < n ? order_key(fmaf(qnv, rb[j], sc[warp * npad + j])) : 0u;
      }
      warp_topk_words<KPL>(key, keep_count(a.rho_r, n), lane, own_r);
    }
    int cnt = 0;
#pragma unroll
    for (int q = 0; q < NO; ++q) {
      const int t = 32 * q + lane;
      if (t < a.nwords) {
        uint32_t f = 0;
        if (a.force_diag && gi < a.nkb && (gi >> 5) == t) f |= 1u << (gi & 31);
        if (a.force_sink && t == 0) f |= 1u;
        cnt += __popc(own_c[q] | own_r[q] | f);
        a.mask_c[row * a.nwords + t] = own_c[q];
        a.mask_r[row * a.nwords + t] = own_r[q];
      }
    }
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (lane == 0) a.counts[row] = cnt;
  }
}

// Exclusive scan of per-row counts into row_ptr (one CTA of 1024 threads).
__global__ void __launch_bounds__(1024) scan_counts_kernel(const int* __restrict__ counts, int rows,
                                                           int* __restrict__ row_ptr, int64_t capacity) {
  __shared__ long long wsum[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (rows + 1023) / 1024;
  const int s0 = min(rows, tid * per), s1 = min(rows, s0 + per);
  long long local = 0;
  for (int r = s0; r < s1; ++r) local += counts[r];
  long long incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    long long w = wsum[lane];
    long long wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long v = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += v;
    }
    wsum[lane] = wi - w;
  }
  __syncthreads();
  long long run = wsum[warp] + incl - local;
  for (int r = s0; r < s1; ++r) {
    row_ptr[r] = static_cast<int>(run);
    run += counts[r];
  }
  if (tid == 1023) {
    row_ptr[rows] = static_cast<int>(run);
    if (run > capacity) raise_error(RBS_DEVERR_ROW_PTR);
  }
}

struct CompactArgs {
  const uint32_t* mask_c;
  const uint32_t* mask_r;
  const int* row_ptr;
  int32_t* col_idx;
  uint8_t* flags;
  int64_t capacity;
  int rows, nqb, nkb, nwords, q_block_offset, force_diag, force_sink;
};

__global__ void __launch_bounds__(256) compact_lists_kernel(CompactArgs a) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= a.rows) return;
  const int gi = row % a.nqb + a.q_block_offset;
  const int beg = a.row_ptr[row], end = a.row_ptr[row + 1];
  if (beg < 0 || end < beg || end > a.capacity) {
    if (lane == 0) raise_error(RBS_DEVERR_ROW_PTR);
    return;
  }
  int run = beg;
  const int64_t mbase = static_cast<int64_t>(row) * a.nwords;
  for (int w0 = 0; w0 < a.nwords; w0 += 32) {
    const int t = w0 + lane;
    uint32_t c = 0, r = 0, f = 0;
    if (t < a.nwords) {
      c = a.mask_c[mbase + t];
      r = a.mask_r[mbase + t];
      if (a.force_diag && gi < a.nkb && (gi >> 5) == t) f |= 1u << (gi & 31);
      if (a.force_sink && t == 0) f |= 1u;
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
