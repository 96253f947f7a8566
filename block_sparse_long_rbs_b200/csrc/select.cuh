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
//                       KV head, batch), longest rows (last query blocks)
//                       first.  The CTA first pools its query block (mean of
//                       the BQ queries of each of its R heads, streamed from
//                       HBM with 16-byte loads), then computes the scores of
//                       all visible blocks into shared memory (centroid tiles
//                       of 256 blocks x 32 dims staged through shared memory,
//                       the next tile's loads in flight while one is used),
//                       then warp w < R finds, for both branches at
//                       once, the exact k-th largest score of its row by a
//                       32-step bitwise search over order-preserving keys held
//                       in registers, breaks ties by block index with warp
//                       ballots, and emits one 32-bit mask word per 32 blocks
//                       (bit = lane).
//   scan_counts_kernel  exclusive scan of the per-row counts -> row_ptr.
//   compact_lists_kernel one warp per row turns mask words into ascending
//                       block indices and per-entry branch flags.
#pragma once

#include "common.cuh"

namespace rbs {

struct SelectArgs {
  const __nv_bfloat16* Q;  // [B, Lq, Hq, 128]
  int64_t qb, qs, qh;      // element strides
  const float* C;      // [B, Hkv, nkb, 128]
  const float* rad;    // [B, Hkv, nkb]
  const float* beta;   // [B, Hkv, nkb]
  int Hq, Hkv, nqb, nkb, R, nwords;
  int q_block_offset, causal, force_diag, force_sink;
  float rho_c, rho_r;
  int threshold_mode;    // 0 = top-k fraction, 1 = within delta of the row maximum
  float delta_c, delta_r;
  uint32_t* mask_c;  // [rows, nwords]
  uint32_t* mask_r;  // [rows, nwords]
  int* counts;       // [rows]
};

constexpr int kSelThreads = 256;
constexpr int kSelMaxR = 8;
constexpr int kStageJ = 256;  // key blocks per staged centroid tile (one per thread)
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

// Exact top-k of the warp's keys for two branches at once (key 0 = not a
// candidate; k <= #candidates).  The k-th largest key T is built bit by bit
// from the top (the largest T with at least k keys >= T); keys above T are
// kept, and of the keys equal to T the ones with the lowest block index.
// Returns, per lane, the mask words this lane owns (word t is owned by lane
// t % 32) with bit `lane` of word t set iff block 32t + lane is kept.
template <int KPL>
__device__ __forceinline__ void warp_topk2(const uint32_t (&kc)[KPL], const uint32_t (&kr)[KPL], int k_c, int k_r,
                                           int lane, uint32_t (&own_c)[(KPL + 31) / 32],
                                           uint32_t (&own_r)[(KPL + 31) / 32]) {
  uint32_t Tc = 0, Tr = 0;
#pragma unroll 1
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cc = Tc | (1u << bit), cr = Tr | (1u << bit);
    int nc2[2] = {0, 0}, nr2[2] = {0, 0};  // two partial counts per branch (shorter add chains)
#pragma unroll
    for (int t = 0; t < KPL; ++t) {
      nc2[t & 1] += kc[t] >= cc ? 1 : 0;
      nr2[t & 1] += kr[t] >= cr ? 1 : 0;
    }
    const int nc = __reduce_add_sync(0xffffffffu, nc2[0] + nc2[1]);
    const int nr = __reduce_add_sync(0xffffffffu, nr2[0] + nr2[1]);
    if (nc >= k_c) Tc = cc;
    if (nr >= k_r) Tr = cr;
  }
  int gc = 0, gr = 0;
#pragma unroll
  for (int t = 0; t < KPL; ++t) {
    gc += kc[t] > Tc ? 1 : 0;
    gr += kr[t] > Tr ? 1 : 0;
  }
  const int need_c = k_c - __reduce_add_sync(0xffffffffu, gc);  // ties at T to keep, lowest index first
  const int need_r = k_r - __reduce_add_sync(0xffffffffu, gr);
  const uint32_t lt_mask = (1u << lane) - 1u;
  int base_c = 0, base_r = 0;
#pragma unroll
  for (int t = 0; t < (KPL + 31) / 32; ++t) own_c[t] = own_r[t] = 0;
#pragma unroll
  for (int t = 0; t < KPL; ++t) {
    const bool tie_c = kc[t] == Tc, tie_r = kr[t] == Tr;
    const uint32_t bc = __ballot_sync(0xffffffffu, tie_c), br = __ballot_sync(0xffffffffu, tie_r);
    const bool sel_c = kc[t] > Tc || (tie_c && base_c + __popc(bc & lt_mask) < need_c);
    const bool sel_r = kr[t] > Tr || (tie_r && base_r + __popc(br & lt_mask) < need_r);
    const uint32_t wc = __ballot_sync(0xffffffffu, sel_c), wr = __ballot_sync(0xffffffffu, sel_r);
    if (lane == (t & 31)) {
      own_c[t >> 5] = wc;
      own_r[t >> 5] = wr;
    }
    base_c += __popc(bc);
    base_r += __popc(br);
  }
}

// Exact top-k of both branches by pruning, for k <= 64 (key(t) = this
// lane's key in slot t, block 32 t + lane, read from shared memory).  Each
// lane's two largest keys form a 64-key subset of the row.  L is the largest
// key with its low 16 bits clear such that at least k keys of the subset are
// >= L; it is at most the subset's k-th largest key, hence at most the row's
// k-th largest key T, so every key >= T is a candidate (key >= L).  When at
// most 64 keys are candidates they are compacted in ascending block order
// into shared memory, T is found among them by a bitwise search (the largest
// T with at least k candidates >= T), the keys above T are kept and of the
// ties at T the lowest block indices, and the kept blocks are OR-ed into
// words[0, nwords) (cleared first).  Returns false, having written nothing
// the caller uses, when k > 64 or more than 64 keys of a branch are
// candidates (many near-equal keys); the caller then runs the full search.
// Both branches advance together so their reduction chains overlap.
// Warp-uniform.
template <int KP, typename KeyC, typename KeyR>
__device__ __forceinline__ bool warp_topk2_pruned(KeyC key_c, KeyR key_r, int k_c, int k_r, int lane, int nwords,
                                                  uint32_t* scratch, uint32_t* words_c, uint32_t* words_r) {
  if (k_c > 64 || k_r > 64) return false;
  uint32_t* ck_c = scratch;  // candidate keys [64] and blocks [64] of each branch
  int* ci_c = reinterpret_cast<int*>(scratch + 64);
  uint32_t* ck_r = scratch + 128;
  int* ci_r = reinterpret_cast<int*>(scratch + 192);
  uint32_t c1 = 0, c2 = 0, r1 = 0, r2 = 0;  // this lane's two largest keys per branch
#pragma unroll 4
  for (int t = 0; t < KP; ++t) {
    const uint32_t uc = key_c(t), ur = key_r(t);
    c2 = max(c2, min(c1, uc));
    c1 = max(c1, uc);
    r2 = max(r2, min(r1, ur));
    r1 = max(r1, ur);
  }
  // The subset holds at least k keys that are not absent (rows interleave
  // blocks over the lanes), and a present key is >= 2^16, so L > 0 and no
  // absent slot (key 0) becomes a candidate.
  uint32_t Lc = 0, Lr = 0;
#pragma unroll 1
  for (int bit = 31; bit >= 16; --bit) {
    const uint32_t xc = Lc | (1u << bit), xr = Lr | (1u << bit);
    const int nc = __reduce_add_sync(0xffffffffu, (c1 >= xc ? 1 : 0) + (c2 >= xc ? 1 : 0));
    const int nr = __reduce_add_sync(0xffffffffu, (r1 >= xr ? 1 : 0) + (r2 >= xr ? 1 : 0));
    if (nc >= k_c) Lc = xc;
    if (nr >= k_r) Lr = xr;
  }
  const uint32_t lt_mask = (1u << lane) - 1u;
  int base_c = 0, base_r = 0;
#pragma unroll 4
  for (int t = 0; t < KP; ++t) {
    const uint32_t uc = key_c(t), ur = key_r(t);
    const bool cand_c = uc >= Lc, cand_r = ur >= Lr;
    const uint32_t bc = __ballot_sync(0xffffffffu, cand_c), br = __ballot_sync(0xffffffffu, cand_r);
    const int pc = base_c + __popc(bc & lt_mask), pr = base_r + __popc(br & lt_mask);
    if (cand_c && pc < 64) {
      ck_c[pc] = uc;
      ci_c[pc] = 32 * t + lane;
    }
    if (cand_r && pr < 64) {
      ck_r[pr] = ur;
      ci_r[pr] = 32 * t + lane;
    }
    base_c += __popc(bc);
    base_r += __popc(br);
  }
  if (base_c > 64 || base_r > 64) return false;
  __syncwarp();
  const uint32_t a0 = lane < base_c ? ck_c[lane] : 0u, a1 = lane + 32 < base_c ? ck_c[lane + 32] : 0u;
  const uint32_t b0 = lane < base_r ? ck_r[lane] : 0u, b1 = lane + 32 < base_r ? ck_r[lane + 32] : 0u;
  const int ia0 = lane < base_c ? ci_c[lane] : 0, ia1 = lane + 32 < base_c ? ci_c[lane + 32] : 0;
  const int ib0 = lane < base_r ? ci_r[lane] : 0, ib1 = lane + 32 < base_r ? ci_r[lane + 32] : 0;
  uint32_t Tc = 0, Tr = 0;
#pragma unroll 1
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t xc = Tc | (1u << bit), xr = Tr | (1u << bit);
    const int nc = __reduce_add_sync(0xffffffffu, (a0 >= xc ? 1 : 0) + (a1 >= xc ? 1 : 0));
    const int nr = __reduce_add_sync(0xffffffffu, (b0 >= xr ? 1 : 0) + (b1 >= xr ? 1 : 0));
    if (nc >= k_c) Tc = xc;
    if (nr >= k_r) Tr = xr;
  }
  // candidate position p (= lane, lane + 32) is in ascending block order, so
  // a tie's rank is the number of ties at lower positions
  const int need_c = k_c - __reduce_add_sync(0xffffffffu, (a0 > Tc ? 1 : 0) + (a1 > Tc ? 1 : 0));
  const int need_r = k_r - __reduce_add_sync(0xffffffffu, (b0 > Tr ? 1 : 0) + (b1 > Tr ? 1 : 0));
  const bool ta0 = a0 == Tc, ta1 = a1 == Tc, tb0 = b0 == Tr, tb1 = b1 == Tr;
  const uint32_t ba0 = __ballot_sync(0xffffffffu, ta0), ba1 = __ballot_sync(0xffffffffu, ta1);
  const uint32_t bb0 = __ballot_sync(0xffffffffu, tb0), bb1 = __ballot_sync(0xffffffffu, tb1);
  const bool sa0 = a0 > Tc || (ta0 && __popc(ba0 & lt_mask) < need_c);
  const bool sa1 = a1 > Tc || (ta1 && __popc(ba0) + __popc(ba1 & lt_mask) < need_c);
  const bool sb0 = b0 > Tr || (tb0 && __popc(bb0 & lt_mask) < need_r);
  const bool sb1 = b1 > Tr || (tb1 && __popc(bb0) + __popc(bb1 & lt_mask) < need_r);
  for (int w = lane; w < nwords; w += 32) words_c[w] = words_r[w] = 0u;
  __syncwarp();
  if (sa0) atomicOr(&words_c[ia0 >> 5], 1u << (ia0 & 31));
  if (sa1) atomicOr(&words_c[ia1 >> 5], 1u << (ia1 & 31));
  if (sb0) atomicOr(&words_r[ib0 >> 5], 1u << (ib0 & 31));
  if (sb1) atomicOr(&words_r[ib1 >> 5], 1u << (ib1 & 31));
  __syncwarp();
  return true;
}

// Both branches' top-k of one row (warp-wide) -> mask words and the row's
// union count.  Keys hold KP slots per lane (block 32t + lane in slot t); the
// row's mask words cover all nwords <= (KPMAX + 31) / 32 * 32 words.
template <int KP, int KPMAX>
__device__ __forceinline__ void select_topk_row(const SelectArgs& a, const float* sc, const float* rb,
                                                const float* qn, int warp, int lane, int hq0, int b, int i, int gi,
                                                int n, int npad, uint32_t* scratch) {
  const int hq = hq0 + warp;
  const int64_t row = (static_cast<int64_t>(b) * a.Hq + hq) * a.nqb + i;
  const float qnv = qn[warp];
  // per-warp scratch: candidates of both branches [256], mask words of both branches
  uint32_t* words_c = scratch + 256;
  uint32_t* words_r = words_c + a.nwords;
  const float* srow = sc + warp * npad;
  auto key_c = [&](int t) -> uint32_t {
    const int j = 32 * t + lane;
    return j < n ? order_key(srow[j]) : 0u;
  };
  auto key_r = [&](int t) -> uint32_t {
    const int j = 32 * t + lane;
    return j < n ? order_key(fmaf(qnv, rb[j], srow[j])) : 0u;
  };
  if (a.threshold_mode == 1) {
    // Each branch keeps every visible block scoring at least its row maximum
    // minus delta; the threshold is formed in fp32 from the maximum score.
    float mc = -INFINITY, mr = -INFINITY;
    for (int j = lane; j < n; j += 32) {
      mc = fmaxf(mc, srow[j]);
      mr = fmaxf(mr, fmaf(qnv, rb[j], srow[j]));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, o));
      mr = fmaxf(mr, __shfl_xor_sync(0xffffffffu, mr, o));
    }
    const uint32_t tc = order_key(mc - a.delta_c), tr = order_key(mr - a.delta_r);
    for (int w = lane; w < a.nwords; w += 32) {
      uint32_t wc = 0, wr = 0;
      for (int bit = 0; bit < 32; ++bit) {
        const int j = 32 * w + bit;
        if (j < n) {
          const float sv = srow[j];
          if (order_key(sv) >= tc) wc |= 1u << bit;
          if (order_key(fmaf(qnv, rb[j], sv)) >= tr) wr |= 1u << bit;
        }
      }
      words_c[w] = wc;
      words_r[w] = wr;
    }
    __syncwarp();
  } else {
    const int k_c = keep_count(a.rho_c, n), k_r = keep_count(a.rho_r, n);
    const bool done = warp_topk2_pruned<KP>(key_c, key_r, k_c, k_r, lane, a.nwords, scratch, words_c, words_r);
    if (!done) {
      uint32_t kc[KP], kr[KP];
#pragma unroll
      for (int t = 0; t < KP; ++t) {
        kc[t] = key_c(t);
        kr[t] = key_r(t);
      }
      constexpr int NO = (KP + 31) / 32;
      uint32_t own_c[NO], own_r[NO];
      warp_topk2<KP>(kc, kr, k_c, k_r, lane, own_c, own_r);
      for (int w = lane; w < a.nwords; w += 32) {
        const bool mine = w < KP;  // word w is owned by lane w % 32 as own[w / 32]
        words_c[w] = mine ? own_c[(w >> 5) < NO ? (w >> 5) : 0] : 0u;
        words_r[w] = mine ? own_r[(w >> 5) < NO ? (w >> 5) : 0] : 0u;
      }
      __syncwarp();
    }
  }
  int cnt = 0;
  for (int t = lane; t < a.nwords; t += 32) {
    const uint32_t wc = words_c[t], wr = words_r[t];
    uint32_t f = 0;
    if (a.force_diag && gi < a.nkb && (gi >> 5) == t) f |= 1u << (gi & 31);
    if (a.force_sink && t == 0) f |= 1u;
    cnt += __popc(wc | wr | f);
    a.mask_c[row * a.nwords + t] = wc;
    a.mask_r[row * a.nwords + t] = wr;
  }
  cnt = __reduce_add_sync(0xffffffffu, cnt);
  if (lane == 0) a.counts[row] = cnt;
}

template <int KPL, int BQ>
__global__ void __launch_bounds__(kSelThreads, KPL <= 32 ? 3 : 1) select_rows_kernel(SelectArgs a) {
  extern __shared__ __align__(16) float sm[];
  const int i = a.nqb - 1 - static_cast<int>(blockIdx.x);  // longest rows first
  const int hblk = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int R = a.R;
  const int G = a.Hq / a.Hkv;
  const int hq0 = hblk * R;
  const int kvh = hq0 / G;
  const int gi = i + a.q_block_offset;
  const int n = a.causal ? min(a.nkb, gi + 1) : a.nkb;
  const int npad = (a.nkb + 31) & ~31;

  float* qs = sm;                         // [128][8] pooled queries, dim-major (heads >= R are 0)
  float* rb = qs + kSelMaxR * 128;        // [npad]  r_j * beta_j
  float* sc = rb + npad;                  // [R][npad] centroid-branch scores
  float* cs = sc + kSelMaxR * npad;       // [kStageJ][kStagePitch]; first holds pooling partial sums
  __shared__ float qn[kSelMaxR];

  const int64_t kv_off = static_cast<int64_t>(b * a.Hkv + kvh) * a.nkb;
  for (int j = tid; j < n; j += kSelThreads) rb[j] = a.rad[kv_off + j] * a.beta[kv_off + j];

  // ---- pooled query of each of the R heads: mean of the BQ queries of block i.
  // Thread (rg, col): 16-byte chunk col % 16 of head col / 16, rows rg, rg + RG, ...
  {
    const int cols = R * 16;
    const int RG = kSelThreads / cols;
    const int col = tid % cols, rg = tid / cols;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    if (rg < RG) {
      const char* base = reinterpret_cast<const char*>(a.Q + b * a.qb + static_cast<int64_t>(i) * BQ * a.qs +
                                                       (hq0 + col / 16) * a.qh) + (col % 16) * 16;
      for (int r0 = rg; r0 < BQ; r0 += 8 * RG) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int row = r0 + u * RG;
          v[u] = row < BQ ? ldg_stream(base + static_cast<int64_t>(row) * a.qs * 2) : make_uint4(0, 0, 0, 0);
        }
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
#pragma unroll
      for (int e = 0; e < 8; ++e) cs[rg * (R * 128) + col * 8 + e] = acc[e];
    }
    __syncthreads();
    for (int o = tid; o < kSelMaxR * 128; o += kSelThreads) {
      const int h = o >> 7, d = o & 127;  // o = h * 128 + d, the pooling sums' order
      float sum = 0.f;
      if (h < R)
        for (int g2 = 0; g2 < RG; ++g2) sum += cs[g2 * (R * 128) + o];
      qs[d * kSelMaxR + h] = sum * (1.0f / BQ);
    }
    __syncthreads();
    if (warp < R) {
      float s2 = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float v = qs[(lane + 32 * e) * kSelMaxR + warp];
        s2 = fmaf(v, v, s2);
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
      if (lane == 0) qn[warp] = sqrtf(s2);
    }
  }

  // ---- scores s_c for j < n: thread t owns block j0 + t of each 256-block tile.
  // Stage (j-tile, 32-dim slice) k's global loads are issued while stage k-1
  // is being used.
  const float* Cb = a.C + kv_off * 128;
  const int nstages = ((n + kStageJ - 1) / kStageJ) * (128 / kStageD);
  constexpr int kLoads = (kStageJ * kStageD / 4) / kSelThreads;  // float4 per thread per stage
  float4 pre[kLoads];
  auto load_stage = [&](int st) {
    const int j0 = (st / (128 / kStageD)) * kStageJ, d0 = (st % (128 / kStageD)) * kStageD;
    const int jn = min(kStageJ, n - j0);
#pragma unroll
    for (int u = 0; u < kLoads; ++u) {
      const int idx = tid + kSelThreads * u;
      const int jl = idx >> 3, d4 = idx & 7;
      pre[u] = jl < jn ? *reinterpret_cast<const float4*>(Cb + static_cast<int64_t>(j0 + jl) * 128 + d0 + 4 * d4)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  // four head pairs per thread, accumulated with paired FMAs (the heads of a
  // pair share the centroid value)
  float2 acc[kSelMaxR / 2];
  load_stage(0);
  for (int st = 0; st < nstages; ++st) {
    const int j0 = (st / (128 / kStageD)) * kStageJ, d0 = (st % (128 / kStageD)) * kStageD;
    const int jn = min(kStageJ, n - j0);
    if (d0 == 0) {
#pragma unroll
      for (int h = 0; h < kSelMaxR / 2; ++h) acc[h] = make_float2(0.f, 0.f);
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kLoads; ++u) {
      const int idx = tid + kSelThreads * u;
      float* dst = cs + (idx >> 3) * kStagePitch + 4 * (idx & 7);
      dst[0] = pre[u].x;
      dst[1] = pre[u].y;
      dst[2] = pre[u].z;
      dst[3] = pre[u].w;
    }
    __syncthreads();
    if (st + 1 < nstages) load_stage(st + 1);
    if (tid < jn) {
      const float* crow = cs + tid * kStagePitch;
      const float* qd = qs + d0 * kSelMaxR;
      if (R > 4) {
#pragma unroll 8
        for (int d = 0; d < kStageD; ++d) {
          const float2 cc = make_float2(crow[d], crow[d]);
          const float4 qa = *reinterpret_cast<const float4*>(qd + d * kSelMaxR);
          const float4 qb = *reinterpret_cast<const float4*>(qd + d * kSelMaxR + 4);
          acc[0] = ffma2(make_float2(qa.x, qa.y), cc, acc[0]);
          acc[1] = ffma2(make_float2(qa.z, qa.w), cc, acc[1]);
          acc[2] = ffma2(make_float2(qb.x, qb.y), cc, acc[2]);
          acc[3] = ffma2(make_float2(qb.z, qb.w), cc, acc[3]);
        }
      } else {
#pragma unroll 8
        for (int d = 0; d < kStageD; ++d) {
          const float2 cc = make_float2(crow[d], crow[d]);
          const float4 qa = *reinterpret_cast<const float4*>(qd + d * kSelMaxR);
          acc[0] = ffma2(make_float2(qa.x, qa.y), cc, acc[0]);
          acc[1] = ffma2(make_float2(qa.z, qa.w), cc, acc[1]);
        }
      }
    }
    if (d0 + kStageD == 128 && tid < jn) {
#pragma unroll
      for (int h = 0; h < kSelMaxR; ++h)
        if (h < R) sc[h * npad + j0 + tid] = (h & 1) ? acc[h >> 1].y : acc[h >> 1].x;
    }
  }
  __syncthreads();

  // ---- per-branch top-k (both branches together), one warp per row, with
  // as few key slots per lane as this row needs
  if (warp < R) {
    // the staging area is free after the scores: per-warp top-k scratch
    uint32_t* scratch = reinterpret_cast<uint32_t*>(cs) + warp * (256 + 2 * a.nwords);
    if (KPL > 8 && n <= 64) select_topk_row<2, KPL>(a, sc, rb, qn, warp, lane, hq0, b, i, gi, n, npad, scratch);
    else if (KPL > 8 && n <= 256) select_topk_row<8, KPL>(a, sc, rb, qn, warp, lane, hq0, b, i, gi, n, npad, scratch);
    else select_topk_row<KPL, KPL>(a, sc, rb, qn, warp, lane, hq0, b, i, gi, n, npad, scratch);
  }
}

// Exclusive scan of per-row counts into row_ptr (one CTA of 1024 threads;
// each thread owns a contiguous run of rows, read and written 4 at a time).
__global__ void __launch_bounds__(1024) scan_counts_kernel(const int* __restrict__ counts, int rows,
                                                           int* __restrict__ row_ptr, int64_t capacity) {
  __shared__ long long wsum[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = ((rows + 1023) / 1024 + 3) & ~3;  // multiple of 4
  const int s0 = min(rows, tid * per), s1 = min(rows, s0 + per);
  long long local = 0;
  int r = s0;
  for (; r + 4 <= s1; r += 4) {
    const int4 c4 = *reinterpret_cast<const int4*>(counts + r);
    local += static_cast<long long>(c4.x) + c4.y + c4.z + c4.w;
  }
  for (; r < s1; ++r) local += counts[r];
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
  r = s0;
  for (; r + 4 <= s1; r += 4) {
    const int4 c4 = *reinterpret_cast<const int4*>(counts + r);
    int4 o;
    o.x = static_cast<int>(run);
    o.y = static_cast<int>(run += c4.x);
    o.z = static_cast<int>(run += c4.y);
    o.w = static_cast<int>(run += c4.z);
    run += c4.w;
    *reinterpret_cast<int4*>(row_ptr + r) = o;
  }
  for (; r < s1; ++r) {
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
