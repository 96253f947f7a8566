// Key-block statistics ([RBS-en] "The Standard Approach and Its Blind
// Spot"): centroid c_b = mean of the block's keys, radius r_b = max over the
// block's keys of ||k - c_b||_2.  When the sequence length L is not a block
// multiple the last block holds the L - (nkb - 1) BK remaining keys (n_b of
// them), and its mean and maximum run over those keys only.
//
// One 128-thread CTA per (key block, KV head, batch).  The block's BK key
// rows (256 bytes each) are read once with 16-byte streaming loads and kept
// in registers: thread t owns 16-byte chunk (t % 16) of rows (t / 16) + 8r.
// Sums reduce across the 8 row groups (shuffle + shared memory), the centroid
// is broadcast through shared memory, and the squared distances of the
// register-resident rows reduce across each row's 16 threads by shuffles.
#pragma once

#include "common.cuh"

namespace rbs {

// The same unpacking as opaque instructions: a kernel that reads packed data
// held in registers twice uses these in its second pass, so the compiler does
// not keep the first pass's unpacked floats alive (twice the registers).
__device__ __forceinline__ float bf16lo_again(uint32_t v) {
  uint32_t u;
  asm volatile("shl.b32 %0, %1, 16;" : "=r"(u) : "r"(v));
  return __uint_as_float(u);
}
__device__ __forceinline__ float bf16hi_again(uint32_t v) {
  uint32_t u;
  asm volatile("and.b32 %0, %1, 0xFFFF0000;" : "=r"(u) : "r"(v));
  return __uint_as_float(u);
}

template <int BK>
__global__ void __launch_bounds__(128) block_stats_kernel(const __nv_bfloat16* __restrict__ K, int64_t sb,
                                                          int64_t ss, int64_t sh, int nkb, int H, int L,
                                                          float* __restrict__ C, float* __restrict__ R) {
  constexpr int RPT = BK / 8;  // rows per thread
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int nb = min(BK, L - j * BK);  // keys in this block
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int chunk = tid & 15;
  const int rgrp = tid >> 4;
  __shared__ float part[4][128];
  __shared__ float cen[128];
  __shared__ float wmax[4];

  const char* base = reinterpret_cast<const char*>(K + b * sb + static_cast<int64_t>(j) * BK * ss + h * sh) +
                     chunk * 16;
  uint4 v[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r)
    v[r] = rgrp + 8 * r < nb ? ldg_stream(base + static_cast<int64_t>(rgrp + 8 * r) * ss * 2) : make_uint4(0, 0, 0, 0);

  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const uint32_t w[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      acc[2 * q] += bf16lo(w[q]);
      acc[2 * q + 1] += bf16hi(w[q]);
    }
  }
  // lanes l and l ^ 16 hold the same chunk for row groups 2w and 2w+1
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
  if (lane < 16) {
#pragma unroll
    for (int e = 0; e < 8; ++e) part[warp][chunk * 8 + e] = acc[e];
  }
  __syncthreads();
  const float c = ((part[0][tid] + part[1][tid]) + (part[2][tid] + part[3][tid])) * (nb == BK ? 1.0f / BK : 1.0f / nb);
  cen[tid] = c;
  C[(static_cast<int64_t>(b * H + h) * nkb + j) * RBS_HEAD_DIM + tid] = c;
  __syncthreads();

  float cl[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) cl[e] = cen[chunk * 8 + e];
  float m = 0.f;
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const uint32_t w[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
    float d2 = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float a = bf16lo_again(w[q]) - cl[2 * q];
      const float bb = bf16hi_again(w[q]) - cl[2 * q + 1];
      d2 = fmaf(a, a, d2);
      d2 = fmaf(bb, bb, d2);
    }
    // the 16 lanes of a row share (lane >> 4)
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) d2 += __shfl_xor_sync(0xffffffffu, d2, o);
    if (rgrp + 8 * r < nb) m = fmaxf(m, d2);
  }
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
  if (lane == 0) wmax[warp] = m;
  __syncthreads();
  if (tid == 0) {
    const float mm = fmaxf(fmaxf(wmax[0], wmax[1]), fmaxf(wmax[2], wmax[3]));
    R[static_cast<int64_t>(b * H + h) * nkb + j] = sqrtf(mm);
  }
}

// ---------------------------------------------------------------------------
// Rescue coefficient beta ([RBS-en] "The Fix"; [RBS-id] "Dual-Branch
// Selection"): per (batch, KV head), beta_b = clamp((r_b - R_lo) /
// (R_hi - R_lo), 0, 1) with R_lo / R_hi linear-interpolation quantiles of that
// head's radii (a bitonic sort of the radii in shared memory), or a constant.

struct BetaArgs {
  const float* R;
  int nkb, H, mode;
  float beta_const, p_lo, p_hi;
  float* beta;
  float* range;
};

// beta of KV head h of batch entry b; the whole CTA (up to 1024 threads)
// takes part, with s[] holding a power of two >= nkb floats for the sort.
__device__ __forceinline__ void block_beta_body(const BetaArgs& ba, int h, int b, float* s) {
  const float* __restrict__ R = ba.R;
  const int nkb = ba.nkb, H = ba.H, mode = ba.mode;
  const float beta_const = ba.beta_const, p_lo = ba.p_lo, p_hi = ba.p_hi;
  float* __restrict__ beta = ba.beta;
  float* __restrict__ range = ba.range;
  __shared__ float lo_hi[2];
  const int tid = threadIdx.x;
  const int64_t off = static_cast<int64_t>(b * H + h) * nkb;
  if (mode == 1) {
    for (int j = tid; j < nkb; j += blockDim.x) beta[off + j] = beta_const;
    if (range != nullptr && tid == 0) {
      range[2 * (b * H + h)] = 0.f;
      range[2 * (b * H + h) + 1] = 0.f;
    }
    return;
  }
  if (p_lo <= 0.f && p_hi == 1.f) {
    // quantile 0 is the minimum and quantile 1 the maximum: no sort needed
    // (p_lo < 0 means R_lo = 0, handled below)
    float mn = INFINITY, mx = -INFINITY;
    for (int j = tid; j < nkb; j += blockDim.x) {
      const float r = R[off + j];
      mn = fminf(mn, r);
      mx = fmaxf(mx, r);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    __shared__ float wmn[32], wmx[32];
    if ((tid & 31) == 0) {
      wmn[tid >> 5] = mn;
      wmx[tid >> 5] = mx;
    }
    __syncthreads();
    if (tid == 0) {
      for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) {
        mn = fminf(mn, wmn[w]);
        mx = fmaxf(mx, wmx[w]);
      }
      lo_hi[0] = p_lo < 0.f ? 0.f : mn;
      lo_hi[1] = mx;
      if (range != nullptr) {
        range[2 * (b * H + h)] = lo_hi[0];
        range[2 * (b * H + h) + 1] = lo_hi[1];
      }
    }
    __syncthreads();
  } else {
  int n2 = 1;
  while (n2 < nkb) n2 <<= 1;
  for (int i = tid; i < n2; i += blockDim.x) s[i] = i < nkb ? R[off + i] : __int_as_float(0x7f800000);
  __syncthreads();
  for (int k = 2; k <= n2; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int i = tid; i < n2; i += blockDim.x) {
        const int ixj = i ^ jj;
        if (ixj > i) {
          const float a = s[i], c = s[ixj];
          const bool up = (i & k) == 0;
          if ((a > c) == up) {
            s[i] = c;
            s[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  if (tid == 0) {
    float q[2];
    const float ps[2] = {p_lo, p_hi};
    for (int t = 0; t < 2; ++t) {
      if (t == 0 && ps[0] < 0.f) {
        q[0] = 0.f;
        continue;
      }
      const double hpos = static_cast<double>(nkb - 1) * static_cast<double>(ps[t]);
      int lo = static_cast<int>(floor(hpos));
      lo = lo < 0 ? 0 : (lo > nkb - 1 ? nkb - 1 : lo);
      const int hi = lo + 1 < nkb ? lo + 1 : nkb - 1;
      const double fr = hpos - lo;
      q[t] = static_cast<float>(static_cast<double>(s[lo]) + fr * (static_cast<double>(s[hi]) - s[lo]));
    }
    lo_hi[0] = q[0];
    lo_hi[1] = q[1];
    if (range != nullptr) {
      range[2 * (b * H + h)] = q[0];
      range[2 * (b * H + h) + 1] = q[1];
    }
  }
  __syncthreads();
  }
  const float rlo = lo_hi[0], rhi = lo_hi[1];
  const bool degenerate = (rhi - rlo) <= 1e-12f * fmaxf(rhi, 1e-30f);
  const float inv = degenerate ? 0.f : 1.f / (rhi - rlo);
  for (int j = tid; j < nkb; j += blockDim.x) {
    const float r = R[off + j];
    beta[off + j] = degenerate ? 1.f : fminf(fmaxf((r - rlo) * inv, 0.f), 1.f);
  }
}

__global__ void __launch_bounds__(1024) block_beta_kernel(const __grid_constant__ BetaArgs ba) {
  extern __shared__ float beta_sort[];
  block_beta_body(ba, blockIdx.x, blockIdx.y, beta_sort);
}

// ---------------------------------------------------------------------------
// Query-block representative: qbar = mean of the block's BQ queries (of the
// remaining L - (nqb - 1) BQ queries for a last, partial block) and its
// norm.  One 256-thread CTA per (query block, group of 4 q heads, batch):
// thread t owns 16-byte chunk (t % 16) of head (t / 16) % 4 and rows
// (t / 64) + 4r.  Deterministic reduction order.

template <int BQ>
__global__ void __launch_bounds__(256) pool_queries_kernel(const __nv_bfloat16* __restrict__ Q, int64_t sb,
                                                           int64_t ss, int64_t sh, int Hq, int nqb, int L,
                                                           float* __restrict__ qbar, float* __restrict__ qnorm) {
  constexpr int RPT = BQ / 4;
  const int i = blockIdx.x, hg = blockIdx.y, b = blockIdx.z;
  const int nq = min(BQ, L - i * BQ);  // queries in this block
  const float inv_n = nq == BQ ? 1.0f / BQ : 1.0f / nq;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int col = tid & 63;
  const int hl = col >> 4, chunk = col & 15, rg = tid >> 6;
  const int hq = hg * 4 + hl;
  __shared__ float part[4][512];
  __shared__ float sq[8];

  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  if (hq < Hq) {
    const char* base =
        reinterpret_cast<const char*>(Q + b * sb + static_cast<int64_t>(i) * BQ * ss + hq * sh) + chunk * 16;
#pragma unroll
    for (int r0 = 0; r0 < RPT; r0 += 8) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        v[u] = rg + 4 * (r0 + u) < nq ? ldg_stream(base + static_cast<int64_t>(rg + 4 * (r0 + u)) * ss * 2)
                                      : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[2 * q] += bf16lo(w[q]);
          acc[2 * q + 1] += bf16hi(w[q]);
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[rg][col * 8 + e] = acc[e];
  __syncthreads();
  // thread t produces outputs 2t, 2t+1 (head t / 64, elements 2(t % 64) ..)
  const int o = 2 * tid;
  const int oh = tid >> 6;
  const float m0 = ((part[0][o] + part[1][o]) + (part[2][o] + part[3][o])) * inv_n;
  const float m1 = ((part[0][o + 1] + part[1][o + 1]) + (part[2][o + 1] + part[3][o + 1])) * inv_n;
  float s2 = m0 * m0 + m1 * m1;
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, w);
  if (lane == 0) sq[warp] = s2;
  const int ohq = hg * 4 + oh;
  if (ohq < Hq) {
    float2* dst = reinterpret_cast<float2*>(qbar + (static_cast<int64_t>(b * Hq + ohq) * nqb + i) * RBS_HEAD_DIM);
    dst[tid & 63] = make_float2(m0, m1);
  }
  __syncthreads();
  if (tid < 4 && hg * 4 + tid < Hq) {
    qnorm[static_cast<int64_t>(b * Hq + hg * 4 + tid) * nqb + i] = sqrtf(sq[2 * tid] + sq[2 * tid + 1]);
  }
}

}  // namespace rbs
