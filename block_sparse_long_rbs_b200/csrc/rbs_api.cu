// librbs: the C ABI declared in include/rbs.h.  Host-side validation,
// workspace carving, TMA tensor-map encoding and kernel launches.  No call
// here allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "attention.cuh"
#include "common.cuh"
#include "lists.cuh"
#include "rope.cuh"
#include "select.cuh"
#include "stats.cuh"
#include "select_mma.cuh"
#include "tokmax.cuh"

using namespace rbs;

namespace {

thread_local char g_last_error[512] = "";

rbs_status fail(rbs_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

#define RBS_REQUIRE(cond, status, ...)       \
  do {                                       \
    if (!(cond)) return fail(status, __VA_ARGS__); \
  } while (0)

rbs_status check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(RBS_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return RBS_OK;
}

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  int sms = 0;
  bool attrs_set = false;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

rbs_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return fail(RBS_ERR_CUDA, "cudaGetDevice failed");
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (d.sms == 0) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0) return fail(RBS_ERR_UNSUPPORTED, "device %d is sm_%d%d; this build is sm_100a only", dev, major, minor);
    cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
  }
  if (!d.attrs_set) {
    cudaError_t e = cudaSuccess;
    e = e ? e : cudaFuncSetAttribute(bsa_prefill_kernel<128, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     AttnSmem<128>::kAlloc);
    e = e ? e : cudaFuncSetAttribute(bsa_prefill_kernel<64, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     AttnSmem<64>::kAlloc);
#define RBS_SEL_ATTR(KPL)                                                                                  \
  e = e ? e : cudaFuncSetAttribute(select_rows_kernel<KPL, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize,  \
                                   static_cast<int>(sel_smem_bytes(RBS_MAX_KV_BLOCKS)));                     \
  e = e ? e : cudaFuncSetAttribute(select_rows_kernel<KPL, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                   static_cast<int>(sel_smem_bytes(RBS_MAX_KV_BLOCKS)));
    RBS_SEL_ATTR(2)
    RBS_SEL_ATTR(8)
    RBS_SEL_ATTR(32)
    RBS_SEL_ATTR(64)
    RBS_SEL_ATTR(128)
#undef RBS_SEL_ATTR
#define RBS_TOK_ATTR(KPL)                                                                                      \
  e = e ? e : cudaFuncSetAttribute(select_tokmax_kernel<64, KPL>, cudaFuncAttributeMaxDynamicSharedMemorySize,  \
                                   TokSmem<64>::kAlloc);                                                        \
  e = e ? e : cudaFuncSetAttribute(select_tokmax_kernel<128, KPL>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                   TokSmem<128>::kAlloc);
    RBS_TOK_ATTR(8)
    RBS_TOK_ATTR(32)
    RBS_TOK_ATTR(64)
#undef RBS_TOK_ATTR
    e = e ? e : cudaFuncSetAttribute(pool_split_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kPoolKStages * kPoolChunkBytes);
    e = e ? e : cudaFuncSetAttribute(pool_split_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kPoolKStages * kPoolChunkBytes);
    e = e ? e : cudaFuncSetAttribute(score_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, GemmSmem::kAlloc);
    for (auto kern : {topk_rows_kernel<2>, topk_rows_kernel<8>, topk_rows_kernel<32>, topk_rows_kernel<64>})
      e = e ? e : cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(topk_smem_bytes(kTokMaxKV, kTokMaxKV / 32)));
    e = e ? e : cudaFuncSetAttribute(block_beta_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, RBS_MAX_KV_BLOCKS * 4);
    e = e ? e : cudaFuncSetAttribute(select_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, RBS_MAX_KV_BLOCKS * 4);
    if (e != cudaSuccess) return fail(RBS_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    d.attrs_set = true;
  }
  *out = &d;
  return RBS_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

rbs_status check_tensor(const rbs_bf16_tensor* t, const char* name) {
  RBS_REQUIRE(t != nullptr && t->data != nullptr, RBS_ERR_INVALID_ARG, "%s: null tensor", name);
  RBS_REQUIRE(t->batch > 0 && t->seqlen > 0 && t->heads > 0, RBS_ERR_INVALID_ARG, "%s: empty shape", name);
  RBS_REQUIRE(t->head_dim == RBS_HEAD_DIM, RBS_ERR_UNSUPPORTED, "%s: head_dim %lld != 128", name,
              static_cast<long long>(t->head_dim));
  RBS_REQUIRE(aligned16(t->data), RBS_ERR_INVALID_ARG, "%s: base pointer not 16-byte aligned", name);
  RBS_REQUIRE(t->stride_b > 0 && t->stride_s > 0 && t->stride_h > 0, RBS_ERR_INVALID_ARG, "%s: non-positive stride", name);
  RBS_REQUIRE(t->stride_b % 8 == 0 && t->stride_s % 8 == 0 && t->stride_h % 8 == 0, RBS_ERR_INVALID_ARG,
              "%s: strides must be multiples of 8 elements", name);
  RBS_REQUIRE(t->seqlen < (1ll << 31) && t->heads < (1 << 16) && t->batch < (1 << 16), RBS_ERR_UNSUPPORTED,
              "%s: shape too large", name);
  return RBS_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                    const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

PFN_encodeTiled encode_fn() {
  static PFN_encodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(p);
  });
  return fn;
}

// 4-D map over [B, L, H, 128] bf16 with a box of `rows` tokens x 64 dims of
// one head, 128-byte swizzle.  The token and head dimensions are ordered by
// stride (*seq_inner = 1 when the token stride is the smaller one).
rbs_status make_tensor_map(const rbs_bf16_tensor* t, int rows, CUtensorMap* map, int* seq_inner) {
  PFN_encodeTiled enc = encode_fn();
  if (enc == nullptr) return fail(RBS_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const bool si = t->stride_s < t->stride_h;
  *seq_inner = si ? 1 : 0;
  cuuint64_t dims[4], strides[3];
  cuuint32_t box[4], estr[4] = {1, 1, 1, 1};
  dims[0] = RBS_HEAD_DIM;
  box[0] = 64;
  if (si) {
    dims[1] = t->seqlen; strides[0] = t->stride_s * 2; box[1] = rows;
    dims[2] = t->heads; strides[1] = t->stride_h * 2; box[2] = 1;
  } else {
    dims[1] = t->heads; strides[0] = t->stride_h * 2; box[1] = 1;
    dims[2] = t->seqlen; strides[1] = t->stride_s * 2; box[2] = rows;
  }
  dims[3] = t->batch;
  strides[2] = t->stride_b * 2;
  box[3] = 1;
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, t->data, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(RBS_ERR_INVALID_ARG, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return RBS_OK;
}

// 4-D map over [B, L, H, 128] bf16 for the selection's pooling: a box of
// 64 dims x R heads x kPoolRows tokens, no swizzle (the token and head
// dimensions ordered by stride as above).
rbs_status make_pool_tensor_map(const rbs_bf16_tensor* t, int R, CUtensorMap* map, int* seq_inner) {
  PFN_encodeTiled enc = encode_fn();
  if (enc == nullptr) return fail(RBS_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const bool si = t->stride_s < t->stride_h;
  *seq_inner = si ? 1 : 0;
  cuuint64_t dims[4], strides[3];
  cuuint32_t box[4], estr[4] = {1, 1, 1, 1};
  dims[0] = RBS_HEAD_DIM;
  box[0] = 64;
  if (si) {
    dims[1] = t->seqlen; strides[0] = t->stride_s * 2; box[1] = kPoolRows;
    dims[2] = t->heads; strides[1] = t->stride_h * 2; box[2] = R;
  } else {
    dims[1] = t->heads; strides[0] = t->stride_h * 2; box[1] = R;
    dims[2] = t->seqlen; strides[1] = t->stride_s * 2; box[2] = kPoolRows;
  }
  dims[3] = t->batch;
  strides[2] = t->stride_b * 2;
  box[3] = 1;
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, t->data, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(RBS_ERR_INVALID_ARG, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return RBS_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct SelectLayout {
  size_t mask_c, mask_r, counts, beta, tiles, c_hi, c_lo, q_hi, q_lo, qnorm, scores;
  int64_t ntiles;  // partial sums of the row-pointer scan (kScanTile rows each)
  size_t base;   // bytes the fused mean-query kernel needs
  size_t total;  // bytes of the full layout
};

// The parts every path uses, then the bf16 hi / lo centroids (per-token and
// tensor-core mean scoring) and, for the tensor-core mean scoring, the pooled
// queries' parts and norms and the score matrix [rows, nkb rounded up to 32].
SelectLayout select_layout(int64_t B, int64_t Hq, int64_t nqb, int64_t Hkv, int64_t nkb, bool token_max) {
  SelectLayout l{};
  const int64_t rows = B * Hq * nqb;
  const int64_t nwords = (nkb + 31) / 32;
  size_t off = 0;
  l.mask_c = off; off += align256(rows * nwords * 4);
  l.mask_r = off; off += align256(rows * nwords * 4);
  l.counts = off; off += align256(rows * 4);
  l.beta = off; off += align256(B * Hkv * nkb * 4);
  l.ntiles = (rows + kScanTile - 1) / kScanTile;  // list rows <= rows
  l.tiles = off; off += align256(2 * l.ntiles * 4);  // the sums, then their exclusive prefixes
  l.base = off;
  l.c_hi = off; off += align256(B * Hkv * nkb * RBS_HEAD_DIM * 2);
  l.c_lo = off; off += align256(B * Hkv * nkb * RBS_HEAD_DIM * 2);
  if (token_max) {
    l.base = off;  // the per-token kernel needs the centroid parts
    l.scores = off; off += align256(rows * 2 * nwords * 32 * 4);  // both branches' keys, for the separate top-k
  } else {
    l.q_hi = off; off += align256(rows * RBS_HEAD_DIM * 2);
    l.q_lo = off; off += align256(rows * RBS_HEAD_DIM * 2);
    l.qnorm = off; off += align256(rows * 4);
    l.scores = off; off += align256(rows * nwords * 32 * 4);
  }
  l.total = off;
  return l;
}

// Both branches' top-k of every row from the stored scores or keys, kTopkWarps
// rows per CTA, with as many key slots per lane as the longest row needs.
void launch_topk_rows(const TopkArgs& t0, int64_t nkb, rbs_stream_t stream) {
  TopkArgs t = t0;
  const size_t tsm = topk_smem_bytes(t.nkbp, t.s.nwords);
  t.nhg = (t.s.Hq + kTopkWarps - 1) / kTopkWarps;
  t.inv_nhg = 1.0f / static_cast<float>(t.nhg);
  t.inv_g = 1.0f / static_cast<float>(t.s.Hq / t.s.Hkv);
  constexpr int kThreads = kTopkWarps * 32;
  for (int y0 = 0; y0 < t.s.nqb; y0 += 65535) {
    t.y0 = y0;
    const dim3 tgrid(static_cast<unsigned>(t.s.B * t.nhg), static_cast<unsigned>(std::min(65535, t.s.nqb - y0)));
    if (nkb <= 64) topk_rows_kernel<2><<<tgrid, kThreads, tsm, stream>>>(t);
    else if (nkb <= 256) topk_rows_kernel<8><<<tgrid, kThreads, tsm, stream>>>(t);
    else if (nkb <= 1024) topk_rows_kernel<32><<<tgrid, kThreads, tsm, stream>>>(t);
    else topk_rows_kernel<64><<<tgrid, kThreads, tsm, stream>>>(t);
  }
}

// Per-token-max selection scores (query_pool TOKEN_MAX): split the centroids
// into bf16 hi / lo parts in the workspace, then one persistent CTA per SM
// scores rows (select_tokmax_kernel).  With room in the workspace for both
// branches' key matrix the kernel stores the keys and topk_rows_kernel
// selects from them; otherwise two warps of each CTA select in place.  Both
// write the same mask words and counts as the mean-query kernels.
rbs_status launch_token_max(const rbs_bf16_tensor* Q, const float* centroids, int64_t B, int32_t Hkv, int64_t nkb,
                            const rbs_select_params* p, const SelectArgs& sa, uint8_t* c_hi, uint8_t* c_lo,
                            uint32_t* keys, DeviceInfo* di, rbs_stream_t stream) {
  rbs_status st;
  TokArgs ta;
  int si = 0;
  if ((st = make_tensor_map(Q, p->block_q, &ta.tmQ, &si)) != RBS_OK) return st;
  RBS_REQUIRE(si == 0, RBS_ERR_UNSUPPORTED,
              "query_pool TOKEN_MAX needs Q with the head stride no larger than the token stride");
  // the centroid parts as [B, nkb "tokens", Hkv "heads", 128]: block j of KV head h at (j, h)
  for (int part = 0; part < 2; ++part) {
    rbs_bf16_tensor v;
    v.data = part == 0 ? c_hi : c_lo;
    v.batch = B;
    v.seqlen = nkb;
    v.heads = Hkv;
    v.head_dim = RBS_HEAD_DIM;
    v.stride_b = Hkv * nkb * RBS_HEAD_DIM;
    v.stride_s = RBS_HEAD_DIM;
    v.stride_h = nkb * RBS_HEAD_DIM;
    if ((st = make_tensor_map(&v, 128, part == 0 ? &ta.tmChi : &ta.tmClo, &si)) != RBS_OK) return st;
  }
  ta.s = sa;
  ta.rows = static_cast<int>(B * sa.Hq * sa.nqb);
  ta.keys_out = keys;
  ta.nkbp = static_cast<int>((nkb + 31) & ~31ll);
  const int grid = static_cast<int>(std::min<int64_t>(ta.rows, di->sms));
#define RBS_TOK_LAUNCH(KPL)                                                                                  \
  do {                                                                                                       \
    if (p->block_q == 128)                                                                                   \
      select_tokmax_kernel<128, KPL><<<grid, kTokThreads, TokSmem<128>::kAlloc, stream>>>(ta);               \
    else                                                                                                     \
      select_tokmax_kernel<64, KPL><<<grid, kTokThreads, TokSmem<64>::kAlloc, stream>>>(ta);                 \
  } while (0)
  if (nkb <= 256) RBS_TOK_LAUNCH(8);
  else if (nkb <= 1024) RBS_TOK_LAUNCH(32);
  else RBS_TOK_LAUNCH(64);
#undef RBS_TOK_LAUNCH
  if ((st = check_launch("select_tokmax_kernel")) != RBS_OK || keys == nullptr) return st;
  // the stored keys -> masks and counts, one warp per row
  TopkArgs tk;
  tk.s = sa;
  tk.scores = nullptr;
  tk.qnorm = nullptr;
  tk.keys = keys;
  tk.nkbp = ta.nkbp;
  tk.rows = ta.rows;
  launch_topk_rows(tk, nkb, stream);
  return check_launch("topk_rows_kernel");
}

// 4-D map over a contiguous [B, H, n, 128] bf16 array with a box of 64 dims x
// rows x heads (128-byte swizzle): the pooled-query parts, R heads x QB blocks.
rbs_status make_rows_heads_map(void* data, int64_t B, int64_t H, int64_t n, int rows, int heads, CUtensorMap* map) {
  PFN_encodeTiled enc = encode_fn();
  if (enc == nullptr) return fail(RBS_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[4] = {RBS_HEAD_DIM, static_cast<cuuint64_t>(n), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {RBS_HEAD_DIM * 2, static_cast<cuuint64_t>(n) * RBS_HEAD_DIM * 2,
                                 static_cast<cuuint64_t>(H * n) * RBS_HEAD_DIM * 2};
  const cuuint32_t box[4] = {64, static_cast<cuuint32_t>(rows), static_cast<cuuint32_t>(heads), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, data, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(RBS_ERR_INVALID_ARG, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return RBS_OK;
}

// Mean-query scores on the tensor core: pool the query blocks into bf16 hi /
// lo parts, split the centroids, one 128 x 128 x 128 MMA tile per (128 pooled
// queries, 128 key blocks) into the score matrix, then one warp per row for
// the top-k (pool_split_kernel, score_gemm_kernel, topk_rows_kernel).
rbs_status launch_mma_select(const rbs_bf16_tensor* Q, const float* centroids, int64_t B, int32_t Hkv, int64_t nkb,
                             const rbs_select_params* p, const SelectArgs& sa, int R, uint8_t* ws,
                             const SelectLayout& lay, DeviceInfo* di, rbs_stream_t stream) {
  rbs_status st;
  const int64_t Hq = Q->heads, nqb = sa.nqb, rows = B * Hq * nqb;
  const int npad = static_cast<int>((nkb + 31) & ~31ll);
  auto* c_hi = reinterpret_cast<__nv_bfloat16*>(ws + lay.c_hi);
  auto* c_lo = reinterpret_cast<__nv_bfloat16*>(ws + lay.c_lo);
  auto* q_hi = reinterpret_cast<__nv_bfloat16*>(ws + lay.q_hi);
  auto* q_lo = reinterpret_cast<__nv_bfloat16*>(ws + lay.q_lo);
  float* qnorm = reinterpret_cast<float*>(ws + lay.qnorm);
  float* scores = reinterpret_cast<float*>(ws + lay.scores);


  // pooling
  PoolArgs pa;
  CUtensorMap qmap;
  int seq_inner = 0;
  if ((st = make_pool_tensor_map(Q, R, &qmap, &seq_inner)) != RBS_OK) return st;
  pa.B = static_cast<int>(B);
  pa.Hq = static_cast<int>(Hq);
  pa.nqb = static_cast<int>(nqb);
  pa.R = R;
  pa.items = static_cast<int>(B * nqb * (Hq / R));
  pa.Lq = static_cast<int>(Q->seqlen);
  pa.seq_inner = seq_inner;
  pa.qhi = q_hi;
  pa.qlo = q_lo;
  pa.qnorm = qnorm;
  {
    const size_t smem = kPoolKStages * kPoolChunkBytes;
    auto launch = [&](auto kern) -> rbs_status {
      int per_sm = 0;
      const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kPoolKThreads, smem);
      if (e != cudaSuccess || per_sm < 1) return fail(RBS_ERR_CUDA, "pool_split_kernel does not fit on an SM");
      const int grid = static_cast<int>(std::min<int64_t>(pa.items, static_cast<int64_t>(per_sm) * di->sms));
      kern<<<grid, kPoolKThreads, smem, stream>>>(qmap, pa);
      return check_launch("pool_split_kernel");
    };
    st = p->block_q == 128 ? launch(pool_split_kernel<128>) : launch(pool_split_kernel<64>);
    if (st != RBS_OK) return st;
  }

  // scores
  GemmArgs ga;
  for (int part = 0; part < 2; ++part) {
    rbs_bf16_tensor v;
    v.data = part == 0 ? static_cast<void*>(c_hi) : static_cast<void*>(c_lo);
    v.batch = B;
    v.seqlen = nkb;
    v.heads = Hkv;
    v.head_dim = RBS_HEAD_DIM;
    v.stride_b = Hkv * nkb * RBS_HEAD_DIM;
    v.stride_s = RBS_HEAD_DIM;
    v.stride_h = nkb * RBS_HEAD_DIM;
    int si = 0;
    if ((st = make_tensor_map(&v, 128, part == 0 ? &ga.tmChi : &ga.tmClo, &si)) != RBS_OK) return st;
  }
  const int QB = 128 / R;
  if ((st = make_rows_heads_map(q_hi, B, Hq, nqb, QB, R, &ga.tmQhi)) != RBS_OK) return st;
  if ((st = make_rows_heads_map(q_lo, B, Hq, nqb, QB, R, &ga.tmQlo)) != RBS_OK) return st;
  ga.scores = scores;
  ga.B = static_cast<int>(B);
  ga.Hq = static_cast<int>(Hq);
  ga.Hkv = Hkv;
  ga.nqb = static_cast<int>(nqb);
  ga.nkb = static_cast<int>(nkb);
  ga.nkbp = npad;
  ga.R = R;
  ga.QB = QB;
  ga.ngroups = static_cast<int>((nqb + QB - 1) / QB);
  ga.items = static_cast<int>(B * (Hq / R) * ga.ngroups);
  ga.q_block_offset = p->q_block_offset;
  ga.causal = p->causal;
  score_gemm_kernel<<<static_cast<unsigned>(std::min<int64_t>(ga.items, di->sms)), kGemmThreads, GemmSmem::kAlloc,
                      stream>>>(ga);
  if ((st = check_launch("score_gemm_kernel")) != RBS_OK) return st;

  // top-k
  TopkArgs ta;
  ta.s = sa;
  ta.scores = scores;
  ta.qnorm = qnorm;
  ta.keys = nullptr;
  ta.nkbp = npad;
  ta.rows = static_cast<int>(rows);
  launch_topk_rows(ta, nkb, stream);
  return check_launch("topk_rows_kernel");
}

int keep_count_host(float rho, int64_t n) {
  int64_t k = static_cast<int64_t>(std::ceil(static_cast<double>(rho) * static_cast<double>(n) - 1e-4));
  if (k < 1) k = 1;
  if (k > n) k = n;
  return static_cast<int>(k);
}

rbs_status check_lists(const rbs_block_lists* out, int64_t rows) {
  RBS_REQUIRE(out != nullptr && out->row_ptr != nullptr && out->col_idx != nullptr, RBS_ERR_INVALID_ARG,
              "lists: null pointer");
  RBS_REQUIRE(out->num_rows == rows, RBS_ERR_INVALID_ARG, "lists: num_rows %d != %lld", out->num_rows,
              static_cast<long long>(rows));
  RBS_REQUIRE(out->capacity >= 0 && out->capacity < (1ll << 31), RBS_ERR_UNSUPPORTED, "lists: capacity out of int32 range");
  return RBS_OK;
}

}  // namespace

extern "C" {

int32_t rbs_abi_version(void) { return RBS_ABI_VERSION; }

const char* rbs_status_string(rbs_status s) {
  switch (s) {
    case RBS_OK: return "ok";
    case RBS_ERR_INVALID_ARG: return "invalid argument";
    case RBS_ERR_UNSUPPORTED: return "unsupported";
    case RBS_ERR_CAPACITY: return "capacity";
    case RBS_ERR_CUDA: return "cuda error";
    case RBS_ERR_DEVICE: return "device error";
  }
  return "unknown status";
}

const char* rbs_last_error(void) { return g_last_error; }

void rbs_select_params_default(rbs_select_params* p) {
  if (p == nullptr) return;
  p->block_q = 128;
  p->block_k = 128;
  p->rho_centroid = 0.05f;
  p->rho_rescue = 0.05f;
  p->beta_mode = 0;
  p->beta_const = 1.0f;
  p->beta_p_lo = 0.0f;
  p->beta_p_hi = 1.0f;
  p->force_diag = 1;
  p->force_sink = 0;
  p->causal = 1;
  p->q_block_offset = 0;
  p->threshold_mode = 0;
  p->delta_centroid = 0.0f;
  p->delta_rescue = 0.0f;
  p->list_mode = 0;
  p->query_pool = 0;
}

rbs_status rbs_get_device_error(int32_t* code_host, rbs_stream_t stream) {
  RBS_REQUIRE(code_host != nullptr, RBS_ERR_INVALID_ARG, "null code pointer");
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_device_error, sizeof(int), 0, cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  const int zero = 0;
  if (e == cudaSuccess) e = cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return fail(RBS_ERR_CUDA, "device error word: %s", cudaGetErrorString(e));
  *code_host = v;
  if (v != 0) return fail(RBS_ERR_DEVICE, "device error word 0x%x", v);
  return RBS_OK;
}

// ---------------------------------------------------------------------------

rbs_status rbs_block_stats(const rbs_bf16_tensor* K, int32_t block_k, float* centroids, float* radii,
                           rbs_stream_t stream) {
  rbs_status st = check_tensor(K, "K");
  if (st != RBS_OK) return st;
  RBS_REQUIRE(block_k == 64 || block_k == 128, RBS_ERR_UNSUPPORTED, "block_k must be 64 or 128");
  RBS_REQUIRE(centroids != nullptr && radii != nullptr, RBS_ERR_INVALID_ARG, "null output");
  RBS_REQUIRE(aligned16(centroids), RBS_ERR_INVALID_ARG, "centroids not 16-byte aligned");
  DeviceInfo* di;
  if ((st = device_info(&di)) != RBS_OK) return st;
  const int nkb = static_cast<int>((K->seqlen + block_k - 1) / block_k);
  const int L = static_cast<int>(K->seqlen);
  const dim3 grid(nkb, static_cast<unsigned>(K->heads), static_cast<unsigned>(K->batch));
  const __nv_bfloat16* k = static_cast<const __nv_bfloat16*>(K->data);
  if (block_k == 128)
    block_stats_kernel<128><<<grid, 128, 0, stream>>>(k, K->stride_b, K->stride_s, K->stride_h, nkb,
                                                      static_cast<int>(K->heads), L, centroids, radii);
  else
    block_stats_kernel<64><<<grid, 128, 0, stream>>>(k, K->stride_b, K->stride_s, K->stride_h, nkb,
                                                     static_cast<int>(K->heads), L, centroids, radii);
  return check_launch("block_stats_kernel");
}

}  // extern "C"

// Validates the beta parameters, then launches beta alone (block_beta_kernel)
// or, with split_n > 0, beta and the centroids' bf16 hi / lo split as one
// launch (select_prep_kernel).
rbs_status launch_beta(const float* radii, int64_t batch, int64_t kv_heads, int64_t num_blocks,
                       const rbs_select_params* p, float* beta, float* radius_range, const float* centroids,
                       int64_t split_n, void* c_hi, void* c_lo, rbs_stream_t stream) {
  RBS_REQUIRE(radii != nullptr && beta != nullptr && p != nullptr, RBS_ERR_INVALID_ARG, "null argument");
  RBS_REQUIRE(batch > 0 && kv_heads > 0 && num_blocks > 0, RBS_ERR_INVALID_ARG, "empty shape");
  RBS_REQUIRE(num_blocks <= RBS_MAX_KV_BLOCKS, RBS_ERR_UNSUPPORTED, "num_blocks > %d", RBS_MAX_KV_BLOCKS);
  RBS_REQUIRE(p->beta_mode == 0 || p->beta_mode == 1, RBS_ERR_INVALID_ARG, "beta_mode");
  RBS_REQUIRE(p->beta_mode == 1 || (p->beta_p_hi >= 0.f && p->beta_p_hi <= 1.f && p->beta_p_lo <= 1.f),
              RBS_ERR_INVALID_ARG, "beta quantiles out of range");
  RBS_REQUIRE(kv_heads < 65536 && batch < 65536, RBS_ERR_UNSUPPORTED, "shape too large");
  DeviceInfo* di;
  rbs_status st = device_info(&di);
  if (st != RBS_OK) return st;
  int n2 = 1;
  while (n2 < num_blocks) n2 <<= 1;
  BetaArgs ba;
  ba.R = radii;
  ba.nkb = static_cast<int>(num_blocks);
  ba.H = static_cast<int>(kv_heads);
  ba.mode = p->beta_mode;
  ba.beta_const = p->beta_const;
  ba.p_lo = p->beta_p_lo;
  ba.p_hi = p->beta_p_hi;
  ba.beta = beta;
  ba.range = radius_range;
  if (split_n == 0) {
    block_beta_kernel<<<dim3(static_cast<unsigned>(kv_heads), static_cast<unsigned>(batch)), 1024, n2 * 4, stream>>>(
        ba);
    return check_launch("block_beta_kernel");
  }
  const int64_t nbeta = batch * kv_heads;
  const int64_t nsplit = std::min<int64_t>((split_n + 1023) / 1024, di->sms);
  select_prep_kernel<<<static_cast<unsigned>(nbeta + nsplit), 1024, n2 * 4, stream>>>(
      ba, static_cast<int>(nbeta), centroids, split_n, static_cast<__nv_bfloat16*>(c_hi),
      static_cast<__nv_bfloat16*>(c_lo));
  return check_launch("select_prep_kernel");
}

extern "C" {

rbs_status rbs_block_beta(const float* radii, int64_t batch, int64_t kv_heads, int64_t num_blocks,
                          const rbs_select_params* p, float* beta, float* radius_range, rbs_stream_t stream) {
  return launch_beta(radii, batch, kv_heads, num_blocks, p, beta, radius_range, nullptr, 0, nullptr, nullptr, stream);
}

rbs_status rbs_pool_queries(const rbs_bf16_tensor* Q, int32_t block_q, float* qbar, float* qnorm,
                            rbs_stream_t stream) {
  rbs_status st = check_tensor(Q, "Q");
  if (st != RBS_OK) return st;
  RBS_REQUIRE(block_q == 64 || block_q == 128, RBS_ERR_UNSUPPORTED, "block_q must be 64 or 128");
  RBS_REQUIRE(qbar != nullptr && qnorm != nullptr && aligned16(qbar), RBS_ERR_INVALID_ARG, "bad output");
  DeviceInfo* di;
  if ((st = device_info(&di)) != RBS_OK) return st;
  const int nqb = static_cast<int>((Q->seqlen + block_q - 1) / block_q);
  const int L = static_cast<int>(Q->seqlen);
  const int Hq = static_cast<int>(Q->heads);
  const dim3 grid(nqb, (Hq + 3) / 4, static_cast<unsigned>(Q->batch));
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(Q->data);
  if (block_q == 128)
    pool_queries_kernel<128><<<grid, 256, 0, stream>>>(q, Q->stride_b, Q->stride_s, Q->stride_h, Hq, nqb, L, qbar,
                                                       qnorm);
  else
    pool_queries_kernel<64><<<grid, 256, 0, stream>>>(q, Q->stride_b, Q->stride_s, Q->stride_h, Hq, nqb, L, qbar,
                                                      qnorm);
  return check_launch("pool_queries_kernel");
}

int64_t rbs_select_capacity(int64_t batch, int64_t heads_q, int64_t num_q_blocks, int64_t num_kv_blocks,
                            const rbs_select_params* p) {
  if (p == nullptr || batch <= 0 || heads_q <= 0 || num_q_blocks <= 0 || num_kv_blocks <= 0) return -1;
  int64_t per_head = 0;
  for (int64_t i = 0; i < num_q_blocks; ++i) {
    const int64_t gi = i + p->q_block_offset;
    const int64_t n = p->causal ? std::min<int64_t>(num_kv_blocks, gi + 1) : num_kv_blocks;
    if (n <= 0) continue;
    // MAX_RELATIVE keeps an unbounded number: every visible block may be kept
    int64_t c = p->threshold_mode == 1 ? n
                                       : keep_count_host(p->rho_centroid, n) + keep_count_host(p->rho_rescue, n);
    c += (p->force_diag && gi < num_kv_blocks) ? 1 : 0;
    c += p->force_sink ? 1 : 0;
    per_head += std::min<int64_t>(n, c);
  }
  return per_head * batch * heads_q;
}

size_t rbs_select_workspace_bytes(int64_t batch, int64_t heads_q, int64_t num_q_blocks, int64_t kv_heads,
                                  int64_t num_kv_blocks, const rbs_select_params* p) {
  (void)p;
  if (batch <= 0 || heads_q <= 0 || num_q_blocks <= 0 || kv_heads <= 0 || num_kv_blocks <= 0) return 0;
  return select_layout(batch, heads_q, num_q_blocks, kv_heads, num_kv_blocks, p != nullptr && p->query_pool == 1).total;
}

rbs_status rbs_select(const rbs_bf16_tensor* Q, const float* centroids, const float* radii, int32_t kv_heads,
                      int64_t num_kv_blocks, const rbs_select_params* p, void* workspace, size_t workspace_bytes,
                      rbs_block_lists* out, float* beta_out, rbs_stream_t stream) {
  rbs_status st = check_tensor(Q, "Q");
  if (st != RBS_OK) return st;
  RBS_REQUIRE(p != nullptr && centroids != nullptr && radii != nullptr, RBS_ERR_INVALID_ARG, "null argument");
  RBS_REQUIRE(p->block_q == p->block_k && (p->block_q == 64 || p->block_q == 128), RBS_ERR_UNSUPPORTED,
              "block_q must equal block_k, 64 or 128");
  RBS_REQUIRE(kv_heads > 0 && Q->heads % kv_heads == 0, RBS_ERR_INVALID_ARG, "heads_q %% kv_heads != 0");
  RBS_REQUIRE(num_kv_blocks > 0 && num_kv_blocks <= RBS_MAX_KV_BLOCKS, RBS_ERR_UNSUPPORTED,
              "num_kv_blocks must be in [1, %d]", RBS_MAX_KV_BLOCKS);
  RBS_REQUIRE(p->threshold_mode == 0 || p->threshold_mode == 1, RBS_ERR_INVALID_ARG, "threshold_mode must be 0 or 1");
  RBS_REQUIRE(p->threshold_mode == 1 ||
                  (p->rho_centroid > 0.f && p->rho_centroid <= 1.f && p->rho_rescue > 0.f && p->rho_rescue <= 1.f),
              RBS_ERR_INVALID_ARG, "rho must be in (0, 1]");
  RBS_REQUIRE(p->threshold_mode == 0 || (p->delta_centroid >= 0.f && p->delta_rescue >= 0.f),
              RBS_ERR_INVALID_ARG, "delta must be >= 0 (and not NaN)");
  RBS_REQUIRE(p->q_block_offset >= 0, RBS_ERR_INVALID_ARG, "q_block_offset < 0");
  RBS_REQUIRE(p->list_mode == 0 || p->list_mode == 1, RBS_ERR_INVALID_ARG, "list_mode must be 0 or 1");
  RBS_REQUIRE(p->query_pool == 0 || p->query_pool == 1, RBS_ERR_INVALID_ARG, "query_pool must be 0 or 1");
  RBS_REQUIRE(p->query_pool == 0 || num_kv_blocks <= kTokMaxKV, RBS_ERR_UNSUPPORTED,
              "query_pool TOKEN_MAX takes at most %d key blocks", kTokMaxKV);
  RBS_REQUIRE(aligned16(centroids), RBS_ERR_INVALID_ARG, "centroids not 16-byte aligned");
  const int64_t B = Q->batch, Hq = Q->heads, nqb = (Q->seqlen + p->block_q - 1) / p->block_q, nkb = num_kv_blocks;
  const int64_t rows = B * Hq * nqb;                                       // one per q head
  const int64_t list_rows = p->list_mode == 1 ? B * kv_heads * nqb : rows;  // rows of the output lists
  if ((st = check_lists(out, list_rows)) != RBS_OK) return st;
  const int64_t cap = rbs_select_capacity(B, Hq, nqb, nkb, p);
  RBS_REQUIRE(out->capacity >= cap, RBS_ERR_CAPACITY, "list capacity %lld < %lld", static_cast<long long>(out->capacity),
              static_cast<long long>(cap));
  const SelectLayout lay = select_layout(B, Hq, nqb, kv_heads, nkb, p->query_pool == 1);
  // the full layout enables the tensor-core mean scoring; a workspace of at
  // least the base part runs the fused kernel
  RBS_REQUIRE(workspace != nullptr && workspace_bytes >= lay.base, RBS_ERR_CAPACITY, "workspace %zu < %zu bytes",
              workspace_bytes, lay.base);
  const bool mma_path = p->query_pool == 0 && workspace_bytes >= lay.total && nkb <= kTokMaxKV;
  RBS_REQUIRE((reinterpret_cast<uintptr_t>(workspace) & 255u) == 0, RBS_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  DeviceInfo* di;
  if ((st = device_info(&di)) != RBS_OK) return st;

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* beta = beta_out != nullptr ? beta_out : reinterpret_cast<float*>(ws + lay.beta);
  // the tensor-core and per-token scoring need the centroids' bf16 hi / lo
  // parts: split them in the same launch as beta
  const int64_t split_n = (p->query_pool == 1 || mma_path) ? B * kv_heads * nkb * RBS_HEAD_DIM : 0;
  if ((st = launch_beta(radii, B, kv_heads, nkb, p, beta, nullptr, centroids, split_n, ws + lay.c_hi, ws + lay.c_lo,
                        stream)) != RBS_OK)
    return st;

  const int G = static_cast<int>(Hq / kv_heads);
  int R = 1;
  for (int r = 1; r <= kSelMaxR; ++r)
    if (G % r == 0) R = r;
  CUtensorMap qmap;
  int seq_inner = 0;
  if (p->query_pool == 0 && (st = make_pool_tensor_map(Q, R, &qmap, &seq_inner)) != RBS_OK) return st;
  SelectArgs sa;
  sa.C = centroids;
  sa.rad = radii;
  sa.beta = beta;
  sa.B = static_cast<int>(B);
  sa.Hq = static_cast<int>(Hq);
  sa.Hkv = kv_heads;
  sa.items = static_cast<int>(B * nqb * (Hq / R));
  sa.Lq = static_cast<int>(Q->seqlen);
  sa.seq_inner = seq_inner;
  sa.nqb = static_cast<int>(nqb);
  sa.nkb = static_cast<int>(nkb);
  sa.R = R;
  sa.nwords = static_cast<int>((nkb + 31) / 32);
  sa.q_block_offset = p->q_block_offset;
  sa.causal = p->causal;
  sa.force_diag = p->force_diag;
  sa.force_sink = p->force_sink;
  sa.threshold_mode = p->threshold_mode;
  sa.delta_c = p->delta_centroid;
  sa.delta_r = p->delta_rescue;
  sa.rho_c = p->rho_centroid;
  sa.rho_r = p->rho_rescue;
  sa.mask_c = reinterpret_cast<uint32_t*>(ws + lay.mask_c);
  sa.mask_r = reinterpret_cast<uint32_t*>(ws + lay.mask_r);
  sa.counts = reinterpret_cast<int*>(ws + lay.counts);
  int* tile_sums = reinterpret_cast<int*>(ws + lay.tiles);
  int* tile_prefix = tile_sums + lay.ntiles;
  const int64_t list_tiles = (list_rows + kScanTile - 1) / kScanTile;
  // KV_GROUP lists sum the group unions' counts instead (group_counts_kernel)
  sa.tile_sums = p->list_mode == 1 ? nullptr : tile_sums;
  if (cudaMemsetAsync(tile_sums, 0, static_cast<size_t>(list_tiles) * 4, stream) != cudaSuccess)
    return fail(RBS_ERR_CUDA, "cudaMemsetAsync failed");
  if (p->query_pool == 1) {
    uint32_t* keys = workspace_bytes >= lay.total ? reinterpret_cast<uint32_t*>(ws + lay.scores) : nullptr;
    if ((st = launch_token_max(Q, centroids, B, kv_heads, nkb, p, sa, ws + lay.c_hi, ws + lay.c_lo, keys, di,
                               stream)) != RBS_OK)
      return st;
  } else if (mma_path) {
    if ((st = launch_mma_select(Q, centroids, B, kv_heads, nkb, p, sa, R, ws, lay, di, stream)) != RBS_OK) return st;
  } else {
    const int npad = static_cast<int>((nkb + 31) & ~31ll);
    const size_t smem = sel_smem_bytes(npad);
    // persistent: as many CTAs as fit on the device at once, each walking the
    // work items with a stride of the grid
    auto launch = [&](auto kern) -> rbs_status {
      int per_sm = 0;
      const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kSelThreads, smem);
      if (e != cudaSuccess || per_sm < 1) return fail(RBS_ERR_CUDA, "select_rows_kernel does not fit on an SM");
      const int grid = static_cast<int>(std::min<int64_t>(sa.items, static_cast<int64_t>(per_sm) * di->sms));
      kern<<<grid, kSelThreads, smem, stream>>>(qmap, sa);
      return check_launch("select_rows_kernel");
    };
#define RBS_SEL_LAUNCH(KPL) \
    st = p->block_q == 128 ? launch(select_rows_kernel<KPL, 128>) : launch(select_rows_kernel<KPL, 64>)
    if (nkb <= 64) RBS_SEL_LAUNCH(2);
    else if (nkb <= 256) RBS_SEL_LAUNCH(8);
    else if (nkb <= 1024) RBS_SEL_LAUNCH(32);
    else if (nkb <= 2048) RBS_SEL_LAUNCH(64);
    else RBS_SEL_LAUNCH(128);
#undef RBS_SEL_LAUNCH
    if (st != RBS_OK) return st;
  }

  CompactArgs ca;
  ca.mask_c = sa.mask_c;
  ca.mask_r = sa.mask_r;
  ca.col_idx = out->col_idx;
  ca.flags = out->flags;
  ca.capacity = out->capacity;
  ca.rows = static_cast<int>(list_rows);
  ca.nqb = static_cast<int>(nqb);
  ca.nkb = static_cast<int>(nkb);
  ca.nwords = sa.nwords;
  ca.q_block_offset = p->q_block_offset;
  ca.force_diag = p->force_diag;
  ca.force_sink = p->force_sink;
  ca.Hq = static_cast<int>(Hq);
  ca.Hl = p->list_mode == 1 ? kv_heads : static_cast<int>(Hq);
  ca.glist = p->list_mode == 1 ? G : 1;
  const unsigned list_grid = static_cast<unsigned>((list_rows + 7) / 8);
  if (p->list_mode == 1) {
    // the per-head counts written by the selection are replaced by the
    // counts of the group unions (list_rows <= rows entries)
    group_counts_kernel<<<list_grid, 256, 0, stream>>>(ca, sa.counts, tile_sums);
    if ((st = check_launch("group_counts_kernel")) != RBS_OK) return st;
  }
  scan_tiles_kernel<<<1, 1024, 0, stream>>>(tile_sums, static_cast<int>(list_tiles), tile_prefix, out->row_ptr,
                                            static_cast<int>(list_rows), out->capacity);
  if ((st = check_launch("scan_tiles_kernel")) != RBS_OK) return st;
  compact_lists_kernel<<<list_grid, 256, 0, stream>>>(ca, sa.counts, tile_prefix, out->row_ptr);
  return check_launch("compact_lists_kernel");
}

// ---------------------------------------------------------------------------
// Selection without any allocation by the caller.  The scratch that
// rbs_select normally takes as a workspace is instead a fixed buffer in this
// library's own device image (RBS_NOALLOC_SCRATCH_BYTES on every device that
// loads the library, held until the process exits).  Host code cannot use the
// array's name as a device address: its address on the current device is
// looked up on every call (a runtime query that allocates nothing), so no
// cached address can outlive a context that was torn down and rebuilt.

}  // extern "C"

static __device__ __align__(256) uint8_t g_noalloc_scratch[RBS_NOALLOC_SCRATCH_BYTES];

namespace {
rbs_status noalloc_scratch(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || p == nullptr)
    return fail(RBS_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
  *out = p;
  return RBS_OK;
}
}  // namespace

extern "C" {

rbs_status rbs_select_noalloc(const rbs_bf16_tensor* Q, const float* centroids, const float* radii,
                              int32_t kv_heads, int64_t num_kv_blocks, const rbs_select_params* p,
                              rbs_block_lists* out, float* beta_out, rbs_stream_t stream) {
  // The size check needs only the shapes, so it comes first: a selection too
  // large for the built-in buffer is refused whatever the pointers are.
  RBS_REQUIRE(Q != nullptr && Q->batch > 0 && Q->seqlen > 0 && Q->heads > 0, RBS_ERR_INVALID_ARG,
              "Q: null tensor or empty shape");
  RBS_REQUIRE(p != nullptr && (p->block_q == 64 || p->block_q == 128), RBS_ERR_UNSUPPORTED,
              "block_q must be 64 or 128");
  RBS_REQUIRE(kv_heads > 0 && num_kv_blocks > 0, RBS_ERR_INVALID_ARG, "empty KV shape");
  const size_t need = select_layout(Q->batch, Q->heads, (Q->seqlen + p->block_q - 1) / p->block_q, kv_heads,
                                    num_kv_blocks, p->query_pool == 1).base;
  RBS_REQUIRE(need <= RBS_NOALLOC_SCRATCH_BYTES, RBS_ERR_CAPACITY,
              "this selection needs %zu bytes of scratch; the built-in buffer holds %zu (use rbs_select with a "
              "workspace)", need, static_cast<size_t>(RBS_NOALLOC_SCRATCH_BYTES));
  rbs_status st = check_tensor(Q, "Q");
  if (st != RBS_OK) return st;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != RBS_OK) return st;
  return rbs_select(Q, centroids, radii, kv_heads, num_kv_blocks, p, scratch, RBS_NOALLOC_SCRATCH_BYTES, out,
                    beta_out, stream);
}

// ---------------------------------------------------------------------------

int64_t rbs_lists_causal_full_nnz(int32_t batch, int32_t heads_q, int32_t num_q_blocks, int32_t q_block_offset) {
  if (batch <= 0 || heads_q <= 0 || num_q_blocks <= 0 || q_block_offset < 0) return -1;
  const int64_t n = num_q_blocks;
  return static_cast<int64_t>(batch) * heads_q * (n * (n - 1) / 2 + n * (q_block_offset + 1));
}

rbs_status rbs_lists_causal_full(int32_t batch, int32_t heads_q, int32_t num_q_blocks, int32_t q_block_offset,
                                 rbs_block_lists* out, rbs_stream_t stream) {
  RBS_REQUIRE(batch > 0 && heads_q > 0 && num_q_blocks > 0 && q_block_offset >= 0, RBS_ERR_INVALID_ARG, "bad shape");
  const int64_t rows = static_cast<int64_t>(batch) * heads_q * num_q_blocks;
  rbs_status st = check_lists(out, rows);
  if (st != RBS_OK) return st;
  const int64_t nnz = rbs_lists_causal_full_nnz(batch, heads_q, num_q_blocks, q_block_offset);
  RBS_REQUIRE(out->capacity >= nnz, RBS_ERR_CAPACITY, "list capacity %lld < %lld", static_cast<long long>(out->capacity),
              static_cast<long long>(nnz));
  lists_causal_full_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(
      static_cast<int>(rows), num_q_blocks, q_block_offset, out->row_ptr, out->col_idx, out->flags);
  return check_launch("lists_causal_full_kernel");
}

namespace {
// Passage starts (host array) -> the device segment table.  Starts are token
// offsets in any position: ascending, the first 0, the final block after the
// last passage.
rbs_status segment_table(const int32_t* seg_start, int32_t num_segments, int32_t final_start, int32_t block,
                         SegmentTable* t) {
  RBS_REQUIRE(seg_start != nullptr && num_segments > 0 && num_segments <= RBS_MAX_SEGMENTS, RBS_ERR_INVALID_ARG,
              "segments: need 1..%d host offsets", RBS_MAX_SEGMENTS);
  RBS_REQUIRE(block == 64 || block == 128, RBS_ERR_UNSUPPORTED, "block must be 64 or 128");
  RBS_REQUIRE(seg_start[0] == 0, RBS_ERR_INVALID_ARG, "seg_start[0] must be 0");
  t->n = num_segments;
  t->block = block;
  for (int s = 0; s < num_segments; ++s) {
    RBS_REQUIRE(s == 0 || seg_start[s] > seg_start[s - 1], RBS_ERR_INVALID_ARG, "segment starts must ascend");
    t->start_tok[s] = seg_start[s];
  }
  RBS_REQUIRE(final_start > seg_start[num_segments - 1], RBS_ERR_INVALID_ARG,
              "final_start must come after the last passage start");
  t->final_start = final_start;
  return RBS_OK;
}
}  // namespace

int64_t rbs_lists_block_attention_nnz(const int32_t* seg_start, int32_t num_segments, int32_t final_start,
                                      int32_t block, int32_t batch, int32_t heads_q, int32_t q_first_block,
                                      int32_t q_num_blocks) {
  SegmentTable t;
  if (segment_table(seg_start, num_segments, final_start, block, &t) != RBS_OK) return -1;
  if (batch <= 0 || heads_q <= 0 || q_first_block < 0 || q_num_blocks <= 0) return -1;
  return static_cast<int64_t>(batch) * heads_q *
         (ba_prefix(t, static_cast<int64_t>(q_first_block) + q_num_blocks) - ba_prefix(t, q_first_block));
}

rbs_status rbs_lists_block_attention(const int32_t* seg_start, int32_t num_segments, int32_t final_start,
                                     int32_t block, int32_t batch, int32_t heads_q, int32_t q_first_block,
                                     int32_t q_num_blocks, rbs_block_lists* out, rbs_stream_t stream) {
  SegmentTable t;
  rbs_status st = segment_table(seg_start, num_segments, final_start, block, &t);
  if (st != RBS_OK) return st;
  RBS_REQUIRE(batch > 0 && heads_q > 0 && q_first_block >= 0 && q_num_blocks > 0, RBS_ERR_INVALID_ARG, "bad shape");
  const int64_t rows = static_cast<int64_t>(batch) * heads_q * q_num_blocks;
  if ((st = check_lists(out, rows)) != RBS_OK) return st;
  const int64_t nnz = rbs_lists_block_attention_nnz(seg_start, num_segments, final_start, block, batch, heads_q,
                                                    q_first_block, q_num_blocks);
  RBS_REQUIRE(out->capacity >= nnz, RBS_ERR_CAPACITY, "list capacity %lld < %lld", static_cast<long long>(out->capacity),
              static_cast<long long>(nnz));
  lists_block_attention_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(
      t, static_cast<int>(rows), q_first_block, q_num_blocks, out->row_ptr, out->col_idx, out->flags);
  return check_launch("lists_block_attention_kernel");
}

// ---------------------------------------------------------------------------

}  // extern "C"

namespace {

// bsa_prefill and its rescue-weighted form: flags == nullptr gives every
// block weight 1; otherwise rescue-only entries get log2(w) = rescue_bias.
// Extra controls of one attention launch: the Block-attention segment mask
// (null: none) and, for the library's own tests, the wait limit and a
// producer that stops early.
struct BsaExtra {
  const SegmentTable* seg = nullptr;
  uint64_t wait_ns = kWaitLimitNs;
  int stall_after = -1;
};

rbs_status launch_bsa(const rbs_bf16_tensor* Q, const rbs_bf16_tensor* K, const rbs_bf16_tensor* V,
                      const rbs_block_lists* lists, int32_t block_q, int32_t block_k, int64_t q_offset,
                      float softmax_scale, int32_t causal, const uint8_t* flags, float rescue_bias,
                      rbs_bf16_tensor* O, float* lse, rbs_stream_t stream, const BsaExtra& ex = BsaExtra()) {
  rbs_status st;
  if ((st = check_tensor(Q, "Q")) != RBS_OK) return st;
  if ((st = check_tensor(K, "K")) != RBS_OK) return st;
  if ((st = check_tensor(V, "V")) != RBS_OK) return st;
  if ((st = check_tensor(O, "O")) != RBS_OK) return st;
  RBS_REQUIRE(block_q == block_k && (block_q == 64 || block_q == 128), RBS_ERR_UNSUPPORTED,
              "block_q must equal block_k, 64 or 128");
  RBS_REQUIRE(K->batch == Q->batch && V->batch == Q->batch && O->batch == Q->batch, RBS_ERR_INVALID_ARG, "batch mismatch");
  RBS_REQUIRE(K->seqlen == V->seqlen && K->heads == V->heads, RBS_ERR_INVALID_ARG, "K/V shape mismatch");
  RBS_REQUIRE(O->seqlen == Q->seqlen && O->heads == Q->heads, RBS_ERR_INVALID_ARG, "O shape != Q shape");
  RBS_REQUIRE(Q->heads % K->heads == 0, RBS_ERR_INVALID_ARG, "heads_q %% heads_kv != 0");
  RBS_REQUIRE(q_offset >= 0 && q_offset % block_k == 0, RBS_ERR_UNSUPPORTED, "q_offset must be a non-negative block multiple");
  const int64_t nqb = (Q->seqlen + block_q - 1) / block_q;
  const int64_t rows = Q->batch * Q->heads * nqb;  // work items: one per (batch, q head, query block)
  // one list per q head, or one per KV head shared by its q heads
  const bool group_lists = lists != nullptr && Q->heads != K->heads && lists->num_rows == Q->batch * K->heads * nqb;
  if ((st = check_lists(lists, group_lists ? Q->batch * K->heads * nqb : rows)) != RBS_OK) return st;
  DeviceInfo* di;
  if ((st = device_info(&di)) != RBS_OK) return st;

  AttnArgs a;
  int siq = 0, sik = 0, siv = 0;
  if ((st = make_tensor_map(Q, block_q, &a.tmQ, &siq)) != RBS_OK) return st;
  if ((st = make_tensor_map(K, block_k, &a.tmK, &sik)) != RBS_OK) return st;
  if ((st = make_tensor_map(V, block_k, &a.tmV, &siv)) != RBS_OK) return st;
  RBS_REQUIRE(siq == 0 && sik == 0 && siv == 0, RBS_ERR_UNSUPPORTED,
              "Q/K/V must have the head stride no larger than the token stride ([B, L, H, 128] order)");
  a.row_ptr = lists->row_ptr;
  a.col_idx = lists->col_idx;
  a.capacity = lists->capacity;
  a.O = static_cast<__nv_bfloat16*>(O->data);
  a.ob = O->stride_b;
  a.os = O->stride_s;
  a.oh = O->stride_h;
  a.lse = lse;
  a.B = static_cast<int>(Q->batch);
  a.Hq = static_cast<int>(Q->heads);
  a.Hkv = static_cast<int>(K->heads);
  a.nqb = static_cast<int>(nqb);
  a.nkb = static_cast<int>((K->seqlen + block_k - 1) / block_k);
  a.k_tail = static_cast<int>(K->seqlen - static_cast<int64_t>(a.nkb - 1) * block_k);
  a.Lq = static_cast<int>(Q->seqlen);
  a.q_block_off = static_cast<int>(q_offset / block_k);
  a.causal = causal ? 1 : 0;
  a.num_rows = static_cast<int>(rows);
  a.group_lists = group_lists ? 1 : 0;
  a.flags = flags;
  a.rescue_bias = rescue_bias;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf(static_cast<float>(RBS_HEAD_DIM));
  a.scale_log2 = scale * 1.4426950408889634f;
  a.wait_ns = ex.wait_ns;
  a.stall_after = ex.stall_after;
  a.seg_n = 0;
  a.seg_final = 0;
  if (ex.seg != nullptr) {
    a.seg_n = ex.seg->n;
    a.seg_final = ex.seg->final_start;
    for (int k = 0; k < ex.seg->n; ++k) a.seg_start[k] = ex.seg->start_tok[k];
  }
  // persistent: one CTA per SM
  const int grid = static_cast<int>(std::min<int64_t>(rows, di->sms));
  if (block_q == 128)
    bsa_prefill_kernel<128, 128><<<grid, kAttnThreads, AttnSmem<128>::kAlloc, stream>>>(a);
  else
    bsa_prefill_kernel<64, 64><<<grid, kAttnThreads, AttnSmem<64>::kAlloc, stream>>>(a);
  return check_launch("bsa_prefill_kernel");
}

}  // namespace

extern "C" {

rbs_status bsa_prefill(const rbs_bf16_tensor* Q, const rbs_bf16_tensor* K, const rbs_bf16_tensor* V,
                       const rbs_block_lists* lists, int32_t block_q, int32_t block_k, int64_t q_offset,
                       float softmax_scale, int32_t causal, rbs_bf16_tensor* O, float* lse, rbs_stream_t stream) {
  return launch_bsa(Q, K, V, lists, block_q, block_k, q_offset, softmax_scale, causal, nullptr, 0.f, O, lse, stream);
}

rbs_status bsa_prefill_rescue_weighted(const rbs_bf16_tensor* Q, const rbs_bf16_tensor* K, const rbs_bf16_tensor* V,
                                       const rbs_block_lists* lists, int32_t block_q, int32_t block_k,
                                       int64_t q_offset, float softmax_scale, int32_t causal, float rescue_weight,
                                       rbs_bf16_tensor* O, float* lse, rbs_stream_t stream) {
  RBS_REQUIRE(rescue_weight >= 0.f && std::isfinite(rescue_weight), RBS_ERR_INVALID_ARG,
              "rescue_weight must be finite and >= 0");
  if (rescue_weight == 1.f)
    return launch_bsa(Q, K, V, lists, block_q, block_k, q_offset, softmax_scale, causal, nullptr, 0.f, O, lse, stream);
  RBS_REQUIRE(lists != nullptr && lists->flags != nullptr, RBS_ERR_INVALID_ARG,
              "rescue weighting needs the lists' branch flags");
  const float bias = rescue_weight > 0.f ? std::log2(rescue_weight) : -INFINITY;
  return launch_bsa(Q, K, V, lists, block_q, block_k, q_offset, softmax_scale, causal, lists->flags, bias, O, lse,
                    stream);
}

rbs_status bsa_prefill_segments(const rbs_bf16_tensor* Q, const rbs_bf16_tensor* K, const rbs_bf16_tensor* V,
                                const rbs_block_lists* lists, int32_t block_q, int32_t block_k, int64_t q_offset,
                                const int32_t* seg_start, int32_t num_segments, int32_t final_start,
                                float softmax_scale, rbs_bf16_tensor* O, float* lse, rbs_stream_t stream) {
  SegmentTable t;
  const rbs_status st = segment_table(seg_start, num_segments, final_start, block_k, &t);
  if (st != RBS_OK) return st;
  BsaExtra ex;
  ex.seg = &t;
  return launch_bsa(Q, K, V, lists, block_q, block_k, q_offset, softmax_scale, 1, nullptr, 0.f, O, lse, stream, ex);
}

rbs_status rbs_testing_bsa_prefill_stalled(const rbs_bf16_tensor* Q, const rbs_bf16_tensor* K,
                                           const rbs_bf16_tensor* V, const rbs_block_lists* lists, int32_t block_q,
                                           int32_t block_k, uint64_t wait_ns, int32_t stall_after,
                                           rbs_bf16_tensor* O, rbs_stream_t stream) {
  RBS_REQUIRE(wait_ns >= 100000ull && wait_ns <= kWaitLimitNs, RBS_ERR_INVALID_ARG,
              "wait_ns must be in [1e5, %llu]", static_cast<unsigned long long>(kWaitLimitNs));
  RBS_REQUIRE(stall_after >= 0, RBS_ERR_INVALID_ARG, "stall_after must be >= 0");
  BsaExtra ex;
  ex.wait_ns = wait_ns;
  ex.stall_after = stall_after;
  return launch_bsa(Q, K, V, lists, block_q, block_k, 0, 0.f, 1, nullptr, 0.f, O, nullptr, stream, ex);
}

rbs_status rbs_testing_exp2(const float* x, float* y, int64_t n, rbs_stream_t stream) {
  RBS_REQUIRE(x != nullptr && y != nullptr && n > 0 && n < (1ll << 31), RBS_ERR_INVALID_ARG, "bad exp2 test buffers");
  const int64_t pairs = (n + 1) / 2;
  exp2_test_kernel<<<static_cast<unsigned>((pairs + 255) / 256), 256, 0, stream>>>(x, y, n);
  return check_launch("exp2_test_kernel");
}

// ---------------------------------------------------------------------------

rbs_status rope_reencode(const rbs_bf16_tensor* x_in, rbs_bf16_tensor* x_out, const int32_t* old_pos,
                         const int32_t* new_pos, float theta, int32_t rope_style, rbs_stream_t stream) {
  rbs_status st;
  if ((st = check_tensor(x_in, "x_in")) != RBS_OK) return st;
  if ((st = check_tensor(x_out, "x_out")) != RBS_OK) return st;
  RBS_REQUIRE(x_in->batch == x_out->batch && x_in->seqlen == x_out->seqlen && x_in->heads == x_out->heads,
              RBS_ERR_INVALID_ARG, "x_out shape != x_in shape");
  RBS_REQUIRE(old_pos != nullptr && new_pos != nullptr, RBS_ERR_INVALID_ARG, "null positions");
  RBS_REQUIRE(theta > 0.f, RBS_ERR_INVALID_ARG, "theta must be positive");
  RBS_REQUIRE(rope_style == 0 || rope_style == 1, RBS_ERR_INVALID_ARG, "rope_style must be 0 or 1");
  const bool alias = x_in->data == x_out->data;
  RBS_REQUIRE(!alias || (x_in->stride_b == x_out->stride_b && x_in->stride_s == x_out->stride_s &&
                         x_in->stride_h == x_out->stride_h),
              RBS_ERR_INVALID_ARG, "in-place re-encoding needs identical strides");
  DeviceInfo* di;
  if ((st = device_info(&di)) != RBS_OK) return st;
  RopeArgs a;
  a.x = static_cast<const __nv_bfloat16*>(x_in->data);
  a.y = static_cast<__nv_bfloat16*>(x_out->data);
  a.xb = x_in->stride_b; a.xs = x_in->stride_s; a.xh = x_in->stride_h;
  a.yb = x_out->stride_b; a.ys = x_out->stride_s; a.yh = x_out->stride_h;
  a.old_pos = old_pos;
  a.new_pos = new_pos;
  a.L = static_cast<int>(x_in->seqlen);
  a.H = static_cast<int>(x_in->heads);
  for (int m = 0; m < 64; ++m)
    a.inv_freq[m] = std::pow(static_cast<double>(theta), -2.0 * m / static_cast<double>(RBS_HEAD_DIM));
  const dim3 grid(static_cast<unsigned>((a.L + kRopeTokens - 1) / kRopeTokens), static_cast<unsigned>(x_in->batch));
  if (rope_style == 0) rope_reencode_kernel<0><<<grid, 256, 0, stream>>>(a);
  else rope_reencode_kernel<1><<<grid, 256, 0, stream>>>(a);
  return check_launch("rope_reencode_kernel");
}

}  // extern "C"
