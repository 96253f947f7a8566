// Device list builders: every causally visible block (the dense reference
// point), and the Block-attention mask ([BA] 2.1 Main idea, 2.2 Block
// segmentation, 2.4 Block fine-tune): a query block of passage s sees the key
// blocks of passage s up to itself, a query block of the final block sees
// every key block up to itself.  Passages may start at any token: a query
// block then lists every key block holding a key one of its tokens may see,
// and bsa_prefill_segments masks the other passages' keys token by token.
// Row pointers are closed forms, so one warp per row writes its own entries
// with no scan.
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
  int n;                            // passages
  int block;                        // block size (tokens)
  int final_start;                  // first token of the final block
  int start_tok[RBS_MAX_SEGMENTS];  // first token of each passage, ascending, start_tok[0] == 0
};

// First visible key block of global query block g: the block of the smallest
// first-visible-key over g's tokens.  Its first token carries the smallest
// passage start; a block holding a token of the final block sees key 0.
__device__ __forceinline__ int ba_first(const SegmentTable& s, int g) {
  if (static_cast<int64_t>(g + 1) * s.block > s.final_start) return 0;
  const int64_t p = static_cast<int64_t>(g) * s.block;
  int lo = 0, hi = s.n - 1;  // last passage whose start <= p
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s.start_tok[mid] <= p) lo = mid; else hi = mid - 1;
  }
  return s.start_tok[lo] / s.block;
}

// Entries of global query blocks 0 .. x-1 (one head): the sum over g < x of
// g - ba_first(g) + 1, in closed form per passage.  Passage s owns the query
// blocks whose first token it holds, g in [ceil(a_s / B), ceil(a_{s+1} / B)),
// each listing from block floor(a_s / B); blocks from floor(final_start / B)
// on hold a token of the final block and list from block 0.
__device__ __host__ __forceinline__ int64_t ba_prefix(const SegmentTable& s, int64_t x) {
  const int64_t B = s.block;
  const int64_t fb = s.final_start / B;
  const int64_t cap = x < fb ? x : fb;
  int64_t tot = 0;
  for (int p = 0; p < s.n; ++p) {
    const int64_t a = s.start_tok[p];
    const int64_t e = p + 1 < s.n ? s.start_tok[p + 1] : s.final_start;
    int64_t lo = (a + B - 1) / B, hi = (e + B - 1) / B;
    if (hi > cap) hi = cap;
    if (hi <= lo) continue;
    const int64_t f = a / B;
    tot += (hi * (hi + 1) / 2 - lo * (lo + 1) / 2) - f * (hi - lo);
  }
  if (x > fb) tot += x * (x + 1) / 2 - fb * (fb + 1) / 2;
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
