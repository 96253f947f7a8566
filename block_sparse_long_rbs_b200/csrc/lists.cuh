// Device list builders: every causally visible block (the dense reference
// point), and the Block-attention mask ([BA] 2.1 Main idea, 2.2 Block
// segmentation, 2.4 Block fine-tune): a query block of passage s sees the key
// blocks of passage s up to itself, a query block of the final block sees
// every key block up to itself.  Row pointers are closed forms, so one warp
// per row writes its own entries with no scan.
#pragma once

#include "common.cuh"

namespace rbs {

// Causal-full rows: row (bh, i) lists 0 .. i + off.
__global__ void __launch_bounds__(256) lists_causal_full_kernel(int rows, int nqb, int off, int32_t* row_ptr,
                                                                int32_t* col_idx, uint8_t* flags) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int64_t bh = row / nqb, i = row % nqb;
  const int64_t per_head = static_cast<int64_t>(nqb) * (nqb - 1) / 2 + static_cast<int64_t>(nqb) * (off + 1);
  const int64_t start = bh * per_head + i * (i - 1) / 2 + i * (off + 1);
  const int cnt = static_cast<int>(i + off + 1);
  if (lane == 0) {
    row_ptr[row] = static_cast<int32_t>(start);
    if (row == rows - 1) row_ptr[rows] = static_cast<int32_t>(start + cnt);
  }
  for (int k = lane; k < cnt; k += 32) {
    col_idx[start + k] = k;
    if (flags != nullptr) flags[start + k] = 0;
  }
}

struct SegmentTable {
  int n;                           // passages
  int final_blk;                   // first block of the final block
  int start_blk[RBS_MAX_SEGMENTS];  // first block of each passage, ascending, start_blk[0] == 0
};

// First visible key block of global query block g.
__device__ __forceinline__ int ba_first(const SegmentTable& s, int g) {
  if (g >= s.final_blk) return 0;
  int lo = 0, hi = s.n - 1;  // last passage whose start <= g
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s.start_blk[mid] <= g) lo = mid; else hi = mid - 1;
  }
  return s.start_blk[lo];
}

// Entries of global query blocks 0 .. x-1 (one head).
__device__ __forceinline__ int64_t ba_prefix(const SegmentTable& s, int x) {
  int64_t tot = 0;
  for (int p = 0; p < s.n; ++p) {
    const int a = s.start_blk[p];
    const int e = p + 1 < s.n ? s.start_blk[p + 1] : s.final_blk;
    const int64_t m = static_cast<int64_t>(min(max(x, a), e) - a);
    tot += m * (m + 1) / 2;
  }
  const int64_t mf = static_cast<int64_t>(max(0, x - s.final_blk));
  tot += mf * (s.final_blk + 1) + mf * (mf - 1) / 2;
  return tot;
}

__global__ void __launch_bounds__(256) lists_block_attention_kernel(const __grid_constant__ SegmentTable seg,
                                                                    int rows, int q_first, int q_num,
                                                                    int32_t* row_ptr, int32_t* col_idx,
                                                                    uint8_t* flags) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int64_t bh = row / q_num;
  const int g = q_first + row % q_num;
  const int64_t base0 = ba_prefix(seg, q_first);
  const int64_t per_head = ba_prefix(seg, q_first + q_num) - base0;
  const int64_t start = bh * per_head + ba_prefix(seg, g) - base0;
  const int first = ba_first(seg, g);
  const int cnt = g - first + 1;
  if (lane == 0) {
    row_ptr[row] = static_cast<int32_t>(start);
    if (row == rows - 1) row_ptr[rows] = static_cast<int32_t>(start + cnt);
  }
  for (int k = lane; k < cnt; k += 32) {
    col_idx[start + k] = first + k;
    if (flags != nullptr) flags[start + k] = 0;
  }
}

}  // namespace rbs
