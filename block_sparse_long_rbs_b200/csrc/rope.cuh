// RoPE position re-encoding ([BA] 2.3 Position re-encoding, 2.5 Inference):
// a key cached with RoPE at old_pos is reset to position 0 and rotated to
// new_pos.  Rotations compose, so this is one rotation of every pair by
// (new_pos - old_pos) * inv_freq_m.  The angle is formed and its sine/cosine
// evaluated in fp64 once per (token, m) and shared by all heads of the token;
// the rotation is applied in fp32 and rounded once to bf16.
//
// One 256-thread CTA per 16 tokens of one batch entry.  Rotate-half pairs
// (m, m + 64): a thread task is (token, head, chunk c in 0..7) and moves the
// two 16-byte chunks c and c + 8 of the head's row.  Interleaved pairs
// (2m, 2m + 1): a task is (token, head, chunk c in 0..15) and moves chunk c.
#pragma once

#include "common.cuh"

namespace rbs {

struct RopeArgs {
  const __nv_bfloat16* x;
  __nv_bfloat16* y;
  int64_t xb, xs, xh, yb, ys, yh;
  const int32_t* old_pos;
  const int32_t* new_pos;
  int L, H;
  double inv_freq[64];
};

constexpr int kRopeTokens = 16;

__device__ __forceinline__ void rot8(const uint4& a, const uint4& bsrc, const float* c, const float* s, uint4& oa,
                                     uint4& ob) {
  const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
  const uint32_t bw[4] = {bsrc.x, bsrc.y, bsrc.z, bsrc.w};
  uint32_t ra[4], rb[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float a0 = bf16lo(aw[q]), a1 = bf16hi(aw[q]);
    const float b0 = bf16lo(bw[q]), b1 = bf16hi(bw[q]);
    const float c0 = c[2 * q], c1 = c[2 * q + 1], s0 = s[2 * q], s1 = s[2 * q + 1];
    ra[q] = pack_bf16x2(fmaf(a0, c0, -b0 * s0), fmaf(a1, c1, -b1 * s1));
    rb[q] = pack_bf16x2(fmaf(a0, s0, b0 * c0), fmaf(a1, s1, b1 * c1));
  }
  oa = make_uint4(ra[0], ra[1], ra[2], ra[3]);
  ob = make_uint4(rb[0], rb[1], rb[2], rb[3]);
}

// Tasks per thread and pass: their loads are issued together, and the first
// pass's loads before the sine/cosine table is formed, so the table's fp64
// arithmetic runs under the memory latency instead of ahead of it.  The
// output is stored with the default policy: the attention pass that follows
// reads it, and it may still be in L2.
constexpr int kRopeUnroll = 4;

template <int STYLE>
__global__ void __launch_bounds__(256) rope_reencode_kernel(const __grid_constant__ RopeArgs a) {
  __shared__ float cs[kRopeTokens][64];
  __shared__ float sn[kRopeTokens][64];
  __shared__ double inv[64];
  const int t0 = blockIdx.x * kRopeTokens, b = blockIdx.y, tid = threadIdx.x;
  constexpr int CPH = STYLE == 0 ? 8 : 16;  // tasks per head
  const int tasks = kRopeTokens * a.H * CPH;
  // task k -> (token tl, head h, chunk c); false past the last token
  auto task = [&](int k, int& tl, int& h, int& c) {
    c = k % CPH;
    h = (k / CPH) % a.H;
    tl = k / (CPH * a.H);
    return k < tasks && t0 + tl < a.L;
  };
  uint4 va[kRopeUnroll], vb[kRopeUnroll];
  auto load = [&](int base) {
#pragma unroll
    for (int u = 0; u < kRopeUnroll; ++u) {
      int tl, h, c;
      if (task(base + tid + 256 * u, tl, h, c)) {
        const uint4* src = reinterpret_cast<const uint4*>(a.x + b * a.xb + (t0 + tl) * a.xs + h * a.xh);
        va[u] = src[c];
        if (STYLE == 0) vb[u] = src[c + 8];
      }
    }
  };
  load(0);
  // the frequency table to shared memory with uniform (non-divergent) reads of
  // the parameter block
  if (tid < 64) {
    double f = 0.0;
#pragma unroll
    for (int m = 0; m < 64; ++m)
      if (m == tid) f = a.inv_freq[m];
    inv[tid] = f;
  }
  // When every token of the CTA moves by the same offset (a passage moved as
  // a whole), one sine/cosine per m serves all of them.
  const int tme = t0 + tid % kRopeTokens;
  const int d0 = a.new_pos[t0] - a.old_pos[t0];
  const bool uniform = __syncthreads_and(tme >= a.L || a.new_pos[tme] - a.old_pos[tme] == d0);
  if (uniform) {
    if (tid < 64) {
      double sv, cv;
      sincos(static_cast<double>(d0) * inv[tid], &sv, &cv);
#pragma unroll
      for (int tl = 0; tl < kRopeTokens; ++tl) {
        cs[tl][tid] = static_cast<float>(cv);
        sn[tl][tid] = static_cast<float>(sv);
      }
    }
  } else {
    for (int k = tid; k < kRopeTokens * 64; k += blockDim.x) {
      const int tl = k >> 6, m = k & 63, t = t0 + tl;
      double sv = 0.0, cv = 1.0;
      if (t < a.L) {
        const double phi = static_cast<double>(a.new_pos[t] - a.old_pos[t]) * inv[m];
        sincos(phi, &sv, &cv);
      }
      cs[tl][m] = static_cast<float>(cv);
      sn[tl][m] = static_cast<float>(sv);
    }
  }
  __syncthreads();
  for (int base = 0; base < tasks; base += 256 * kRopeUnroll) {
    if (base > 0) load(base);
#pragma unroll
    for (int u = 0; u < kRopeUnroll; ++u) {
      int tl, h, c;
      if (!task(base + tid + 256 * u, tl, h, c)) continue;
      uint4* dst = reinterpret_cast<uint4*>(a.y + b * a.yb + (t0 + tl) * a.ys + h * a.yh);
      if (STYLE == 0) {
        uint4 olo, ohi;
        rot8(va[u], vb[u], &cs[tl][8 * c], &sn[tl][8 * c], olo, ohi);
        dst[c] = olo;
        dst[c + 8] = ohi;
      } else {
        // chunk c holds pairs (2m, 2m+1), m = 4c .. 4c+3: even lanes are the
        // first member of a pair, odd lanes the second.
        const uint32_t w[4] = {va[u].x, va[u].y, va[u].z, va[u].w};
        uint32_t r[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int m = 4 * c + q;
          const float x0 = bf16lo(w[q]), x1 = bf16hi(w[q]);
          const float cv = cs[tl][m], sv = sn[tl][m];
          r[q] = pack_bf16x2(fmaf(x0, cv, -x1 * sv), fmaf(x0, sv, x1 * cv));
        }
        dst[c] = make_uint4(r[0], r[1], r[2], r[3]);
      }
    }
  }
}

}  // namespace rbs
