/*
 * rbs.h -- C ABI of librbs: block-sparse prefill attention with
 * radius-bounded block selection (RBS) and the Block-attention mask, for
 * NVIDIA B200 (sm_100a).
 *
 * Sources the operations follow (web pages, cited by title and section):
 *   [RBS-en] "RBS-Attention: How a Geometric Rescue Branch Fixes Sparse
 *            Prefill for Long-Context LLMs": "The Standard Approach and Its
 *            Blind Spot" (block centroid and radius), "The Fix: A
 *            Radius-Adaptive Rescue Branch" (two scoring branches, independent
 *            thresholds, combined mask, block-sparse attention).
 *   [RBS-id] "RBS-Attention Bikin Prefill LLM Gede 20x Lebih Cepat, Tanpa
 *            Training Lagi?": "Dual-Branch Selection: Centroid Base + Rescue
 *            Branch" (radius distribution per prompt / layer / head).
 *   [BA]     "Block-Attention for Efficient Prefilling": 2.1 Main idea,
 *            2.2 Block segmentation, 2.3 Position re-encoding, 2.4 Block
 *            fine-tune, 2.5 Inference.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every pointer is a DEVICE pointer owned by the caller unless the argument
 *   says "host".  The library never allocates device memory; calls that need
 *   scratch take a caller-provided workspace whose size a *_workspace_bytes
 *   query returns.
 * - Every call is asynchronous on the given stream (a cudaStream_t; NULL is
 *   the legacy default stream).  Results are valid once the stream reaches
 *   the point after the call.
 * - Host-side validation runs before any launch; a failed check returns its
 *   status and launches nothing.  A CUDA launch error returns
 *   RBS_ERR_CUDA.  rbs_last_error() gives a one-line reason for the last
 *   non-OK status returned on the calling thread.
 * - A data inconsistency found on the device (a block index out of range, a
 *   row pointer beyond the list capacity, a pipeline wait that ran out of
 *   time) never traps: the kernel skips the affected work, records a code in
 *   the library's device error word and returns.  rbs_get_device_error()
 *   reads and clears that word.
 * - Tensors are bf16 [batch, seqlen, heads, head_dim] with head_dim == 128
 *   contiguous (stride 1) and explicit element strides for the other three
 *   dimensions; the base pointer and every stride must be 16-byte aligned
 *   (strides a multiple of 8 elements).
 * - Block lists ("rows") are CSR with one row per (batch, q head, query
 *   block), ordered batch-major, then q head, then query block; each row's
 *   key-block indices are ascending, so a row's diagonal block, when present,
 *   is its last entry.
 */
#ifndef RBS_H_
#define RBS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define RBS_API __attribute__((visibility("default")))
#else
#define RBS_API
#endif

#define RBS_ABI_VERSION 5
#define RBS_HEAD_DIM 128
#define RBS_MAX_SEGMENTS 512 /* Block-attention segments per call */
#define RBS_MAX_KV_BLOCKS 4096 /* key blocks per sequence for rbs_select */

typedef struct CUstream_st* rbs_stream_t; /* identical to cudaStream_t */

typedef enum {
  RBS_OK = 0,
  RBS_ERR_INVALID_ARG = 1, /* null pointer, bad shape, misaligned stride */
  RBS_ERR_UNSUPPORTED = 2, /* valid but outside what this build implements */
  RBS_ERR_CAPACITY = 3,    /* output list or workspace too small */
  RBS_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed */
  RBS_ERR_DEVICE = 5       /* the device error word was set (see below) */
} rbs_status;

/* Device error word bits (rbs_get_device_error). */
#define RBS_DEVERR_BLOCK_INDEX 0x1   /* a list entry outside [0, num_kv_blocks) */
#define RBS_DEVERR_ROW_PTR 0x2       /* row_ptr not monotone or beyond capacity */
#define RBS_DEVERR_TIMEOUT 0x4       /* a pipeline wait ran out of time */
#define RBS_DEVERR_NONCAUSAL 0x8     /* a causal row lists a block after its diagonal */

typedef struct {
  void* data; /* device pointer to the element at [0, 0, 0, 0] */
  int64_t batch, seqlen, heads, head_dim;
  int64_t stride_b, stride_s, stride_h; /* in elements; the head_dim stride is 1 */
} rbs_bf16_tensor;

/*
 * Selection parameters.  Every point the sources leave open is a field
 * (defaults from rbs_select_params_default):
 *   block_q, block_k   query / key block size, 64 or 128, equal (128)
 *   rho_centroid       centroid branch: keep ceil(rho * n_i) of the n_i
 *   rho_rescue         rescue branch: same rule, its own rho ([RBS-en] "The
 *                      Fix": the branches are thresholded independently) (0.05)
 *   beta_mode          0 = RANGE: beta_b = clamp((r_b - R_lo)/(R_hi - R_lo), 0, 1)
 *                      with R_lo, R_hi the beta_p_lo / beta_p_hi quantiles
 *                      (linear interpolation) of the radii of that prompt and
 *                      KV head ([RBS-id]: per prompt, per head), a degenerate
 *                      range giving beta = 1; 1 = CONST: beta_b = beta_const (0)
 *   beta_const         CONST value; 1 gives the Cauchy-Schwarz bound (1.0)
 *   beta_p_lo/hi       RANGE quantiles; beta_p_lo < 0 means R_lo = 0 (0, 1)
 *   force_diag         always keep the query block's own (diagonal) key block (1)
 *   force_sink         always keep key block 0 (0)
 *   causal             query block i (global index i + q_block_offset) may
 *                      select key blocks 0 .. i + q_block_offset only (1)
 *   q_block_offset     global key-block index of query block 0 (0)
 *   threshold_mode     0 = TOPK_FRACTION: each branch keeps its top
 *                      ceil(rho * n_i) as above; 1 = MAX_RELATIVE: each branch
 *                      keeps every visible block whose score is at least the
 *                      row's maximum score minus delta_centroid / delta_rescue
 *                      (no ranking; [RBS-en] "How This Fits Into the Broader
 *                      Sparse Attention Landscape") (0)
 *   delta_centroid, delta_rescue  MAX_RELATIVE margins in raw score units,
 *                      >= 0 (0, 0)
 *   list_mode          0 = PER_HEAD: one list per (batch, q head, query
 *                      block); 1 = KV_GROUP: one list per (batch, KV head,
 *                      query block), the union of the lists of the Hq / Hkv
 *                      q heads that share the KV head, so that those heads
 *                      attend to the same key blocks (grouped-query attention,
 *                      [RBS-en] "How This Fits Into the Broader Sparse
 *                      Attention Landscape"; shared key blocks across queries,
 *                      [QUILT] Abstract) (0)
 *   query_pool         the query side of the scores: 0 = MEAN: the mean of
 *                      the query block's queries, qbar (as above); 1 =
 *                      TOKEN_MAX: each branch takes the best token of the
 *                      block, s_c = max_t q_t . c_j and s_r = max_t (q_t . c_j
 *                      + ||q_t|| r_j beta_j) ([RBS-en] "The Fix" scores a query
 *                      q; here q runs over the block's tokens).  TOKEN_MAX
 *                      needs num_kv_blocks <= 2048, Q with stride_h <=
 *                      stride_s, and a larger workspace: the split
 *                      centroids at least; the full size adds both
 *                      branches' per-block maxima, so a separate top-k
 *                      kernel can select from them (0)
 * Scores are raw dot products (no 1/sqrt(d)); ties between equal scores go
 * to the lower block index.  Forced blocks do not count toward a branch's k.
 */
typedef struct {
  int32_t block_q, block_k;
  float rho_centroid, rho_rescue;
  int32_t beta_mode;
  float beta_const;
  float beta_p_lo, beta_p_hi;
  int32_t force_diag, force_sink, causal;
  int32_t q_block_offset;
  int32_t threshold_mode;
  float delta_centroid, delta_rescue;
  int32_t list_mode;
  int32_t query_pool;
} rbs_select_params;

/* Per-query-block key-block lists in CSR form (all device memory). */
typedef struct {
  int32_t* row_ptr; /* [num_rows + 1]; row r spans col_idx[row_ptr[r] .. row_ptr[r+1]) */
  int32_t* col_idx; /* [capacity] key-block indices, ascending within a row */
  uint8_t* flags;   /* [capacity] or NULL: bit0 centroid branch kept the block,
                       bit1 rescue branch kept it, bit2 forced (diagonal/sink);
                       in KV_GROUP lists a bit is set when it holds for any
                       q head of the group */
  int64_t capacity; /* entries col_idx (and flags) can hold */
  int32_t num_rows; /* batch * heads * num_q_blocks, rows ordered (batch, head,
                       query block); heads = heads_q (one list per q head) or
                       heads_kv (one list per KV head, shared by its q heads) */
} rbs_block_lists;

/* ---- housekeeping ------------------------------------------------------ */

RBS_API int32_t rbs_abi_version(void);
RBS_API const char* rbs_status_string(rbs_status s);
/* One-line reason for the last non-OK status returned on this host thread. */
RBS_API const char* rbs_last_error(void);
/* Fill *p with the defaults listed above. */
RBS_API void rbs_select_params_default(rbs_select_params* p);
/* Read (synchronising the stream) and clear the device error word.
 * *code_host receives the RBS_DEVERR_* bits; returns RBS_ERR_DEVICE when
 * any bit was set, RBS_OK otherwise. */
RBS_API rbs_status rbs_get_device_error(int32_t* code_host, rbs_stream_t stream);

/* ---- block statistics  ([RBS-en] "The Standard Approach and Its Blind Spot")
 * For every key block b of block_k consecutive tokens of every (batch, KV
 * head): centroid c_b = mean of the block's keys, radius r_b = max over the
 * block's keys of ||k - c_b||_2.  fp32 accumulation of the bf16 keys.  With
 * nKB = ceil(L / block_k), a last block shorter than block_k (L not a block
 * multiple) has the mean and maximum of its L - (nKB - 1) block_k keys.
 *   K          [B, L, Hkv, 128] bf16, block_k 64 or 128
 *   centroids  out [B, Hkv, nKB, 128] fp32, contiguous
 *   radii      out [B, Hkv, nKB] fp32, contiguous
 */
RBS_API rbs_status rbs_block_stats(const rbs_bf16_tensor* K, int32_t block_k, float* centroids, float* radii,
                           rbs_stream_t stream);

/* ---- rescue coefficient  ([RBS-en] "The Fix"; [RBS-id] "Dual-Branch Selection")
 * beta [B, Hkv, nKB] from radii [B, Hkv, nKB] per p->beta_mode (see the
 * parameter block above).  radius_range, when not NULL, receives (R_lo, R_hi)
 * per (batch, KV head) as [B, Hkv, 2] fp32.  nKB <= RBS_MAX_KV_BLOCKS. */
RBS_API rbs_status rbs_block_beta(const float* radii, int64_t batch, int64_t kv_heads, int64_t num_blocks,
                          const rbs_select_params* p, float* beta, float* radius_range, rbs_stream_t stream);

/* ---- query-block representative  ([RBS-en] "The Fix": the q of q^T c_b)
 * qbar [B, Hq, nQB, 128] fp32 = mean of each query block's queries (nQB =
 * ceil(L / block_q); a last, shorter block averages its own queries);
 * qnorm [B, Hq, nQB] fp32 = ||qbar||_2.  Both contiguous. */
RBS_API rbs_status rbs_pool_queries(const rbs_bf16_tensor* Q, int32_t block_q, float* qbar, float* qnorm,
                            rbs_stream_t stream);

/* ---- selection  ([RBS-en] "The Fix"; [RBS-id] "Dual-Branch Selection")
 * For every (batch, q head h, query block i), with KV head h / (Hq / Hkv):
 *   s_c(j) = qbar_i . c_j                      (centroid branch)
 *   s_r(j) = s_c(j) + ||qbar_i|| * r_j * beta_j  (rescue branch)
 * over the visible key blocks j (j <= i + q_block_offset when causal); each
 * branch keeps its own top ceil(rho * n_i) blocks (or, in MAX_RELATIVE mode,
 * the blocks within its delta of the row maximum); the row's list is the
 * union of both kept sets plus the forced blocks, ascending.
 *   Q            [B, Lq, Hq, 128] bf16; nQB = ceil(Lq / block_q) query blocks,
 *                the last one shorter when Lq is not a block multiple
 *   centroids    [B, Hkv, num_kv_blocks, 128] fp32 (rbs_block_stats)
 *   radii        [B, Hkv, num_kv_blocks] fp32
 *   workspace    device scratch, 256-byte aligned, contents need no
 *                initialisation.  rbs_select_workspace_bytes(...) bytes
 *                enable the tensor-core scoring of the mean query (the score
 *                matrix lives there) when num_kv_blocks <= 2048; a smaller
 *                workspace, or more key blocks, runs the fused
 *                CUDA-core scoring kernel, down to the masks and counts it
 *                needs (RBS_ERR_CAPACITY below that).  For TOKEN_MAX the
 *                full size holds both branches' per-block maxima for the
 *                separate top-k kernel; down to the split centroids the
 *                scoring kernel selects in place.  Both choices give the
 *                same lists.
 *   out          lists with num_rows = B * Hq * nQB (B * Hkv * nQB when
 *                list_mode is KV_GROUP) and capacity >=
 *                rbs_select_capacity(...), which bounds both modes;
 *                row_ptr, col_idx and flags written
 *   beta_out     optional [B, Hkv, num_kv_blocks] fp32 copy of beta (or NULL)
 * Requires Hq % Hkv == 0, num_kv_blocks <= RBS_MAX_KV_BLOCKS. */
RBS_API int64_t rbs_select_capacity(int64_t batch, int64_t heads_q, int64_t num_q_blocks, int64_t num_kv_blocks,
                            const rbs_select_params* p);
RBS_API size_t rbs_select_workspace_bytes(int64_t batch, int64_t heads_q, int64_t num_q_blocks, int64_t kv_heads,
                                  int64_t num_kv_blocks, const rbs_select_params* p);
RBS_API rbs_status rbs_select(const rbs_bf16_tensor* Q, const float* centroids, const float* radii, int32_t kv_heads,
                      int64_t num_kv_blocks, const rbs_select_params* p, void* workspace, size_t workspace_bytes,
                      rbs_block_lists* out, float* beta_out, rbs_stream_t stream);

/* ---- selection with no caller-provided scratch
 * No counterpart in the papers: this is a convenience of the library.  Some
 * callers cannot hand the library a device workspace -- for example code
 * running inside a host framework that owns all device memory and forbids raw
 * allocations, or a serving loop where any allocation could stall other
 * streams.  This variant of rbs_select allocates nothing: its scratch is a
 * fixed buffer of RBS_NOALLOC_SCRATCH_BYTES compiled into the library, which
 * every GPU that loads the library holds until the process exits.
 * The caller still passes all inputs and outputs (same meaning as
 * rbs_select).  The buffer is handed to rbs_select as its workspace, so
 * the same rule picks the scoring path: when the full workspace
 * (rbs_select_workspace_bytes) fits in RBS_NOALLOC_SCRATCH_BYTES (and
 * num_kv_blocks <= 2048) the tensor-core scoring runs, otherwise the fused
 * CUDA-core scoring kernel,
 * which needs only the masks, counts and beta.  Only a selection whose masks,
 * counts and beta alone (plus the split centroids, for per-token-max query
 * scoring) exceed the buffer returns RBS_ERR_CAPACITY and launches nothing.
 * Every call looks up the buffer's address on the current device (a CUDA
 * runtime query that allocates nothing); the first call on a device may
 * also load the library's device code there, so make that first call before
 * any stream capture.  The size check uses only the shapes: a selection too
 * large for the buffer is refused before any pointer is looked at.  All
 * calls on a device share the one buffer:
 * every scratch region is fully written before it is read, so nothing needs
 * clearing between calls, but two calls that may overlap on the GPU (other
 * streams, other host threads) race on it and must be serialised by the
 * caller. */
#define RBS_NOALLOC_SCRATCH_BYTES (32u << 20)
RBS_API rbs_status rbs_select_noalloc(const rbs_bf16_tensor* Q, const float* centroids, const float* radii,
                                      int32_t kv_heads, int64_t num_kv_blocks, const rbs_select_params* p,
                                      rbs_block_lists* out, float* beta_out, rbs_stream_t stream);

/* ---- list builders (device kernels; no host copies)
 * Every causally visible block: row (b, h, i) lists 0 .. i + q_block_offset.
 * Capacity needed: batch * heads_q * sum_i (i + q_block_offset + 1). */
RBS_API int64_t rbs_lists_causal_full_nnz(int32_t batch, int32_t heads_q, int32_t num_q_blocks, int32_t q_block_offset);
RBS_API rbs_status rbs_lists_causal_full(int32_t batch, int32_t heads_q, int32_t num_q_blocks, int32_t q_block_offset,
                                 rbs_block_lists* out, rbs_stream_t stream);

/* Block-attention mask ([BA] 2.1, 2.2, 2.4): passage s covers tokens
 * [seg_start[s], seg_start[s+1]) (the last passage ends at final_start); the
 * final block (the user query) covers [final_start, end).  A query block of
 * passage s lists the key blocks of passage s up to itself; a query block of
 * the final block lists every key block up to itself.  Rows are query blocks
 * q_first_block .. q_first_block + q_num_blocks - 1 (global block indices) of
 * every (batch, q head).  seg_start is a HOST array of num_segments <=
 * RBS_MAX_SEGMENTS ascending token offsets, seg_start[0] == 0, final_start
 * after the last of them.  Offsets need not be block multiples: a query
 * block then lists every key block holding a key one of its tokens may see
 * (from the block of the smallest passage start among its tokens, or block
 * 0 when it holds a token of the final block), and bsa_prefill_segments
 * applies the mask token by token. */
RBS_API int64_t rbs_lists_block_attention_nnz(const int32_t* seg_start, int32_t num_segments, int32_t final_start,
                                      int32_t block, int32_t batch, int32_t heads_q, int32_t q_first_block,
                                      int32_t q_num_blocks);
RBS_API rbs_status rbs_lists_block_attention(const int32_t* seg_start, int32_t num_segments, int32_t final_start,
                                     int32_t block, int32_t batch, int32_t heads_q, int32_t q_first_block,
                                     int32_t q_num_blocks, rbs_block_lists* out, rbs_stream_t stream);

/* ---- block-sparse prefill attention  ([RBS-en] "The Fix": exact attention over
 * the selected blocks, standard multi-head / grouped-query attention)
 * For query token t of row (b, h, i) at position t + q_offset:
 *   O[b, t, h] = sum_s softmax_s(scale * q_t . k_s) v_s
 * over the key tokens s of the row's listed blocks, with s <= t + q_offset
 * when causal; KV head = h / (Hq / Hkv).  bf16 tensor-core products, fp32
 * accumulation and softmax.
 *   Q         [B, Lq, Hq, 128] bf16; K, V [B, Lk, Hkv, 128] bf16; each with
 *             stride_h <= stride_s (heads inside tokens, as in a packed QKV
 *             projection; else RBS_ERR_UNSUPPORTED)
 *   lists     num_rows = B * Hq * nQB (row (b, h, i) serves q head h) or
 *             B * Hkv * nQB (row (b, g, i) serves every q head of KV head
 *             g), nQB = ceil(Lq / block_q); indices in [0, ceil(Lk / block_k))
 *   block_q == block_k, 64 or 128; q_offset a multiple of block_k.  Lq and
 *             Lk need not be block multiples: query rows past Lq are not
 *             written and keys past Lk are never attended.
 *   softmax_scale  <= 0 selects 1/sqrt(128)
 *   O         out [B, Lq, Hq, 128] bf16 (may not alias Q, K or V)
 *   lse       optional out [B, Hq, Lq] fp32 = ln sum_s exp(scale q_t.k_s)
 *             (-inf for an empty row, whose O is 0)
 * Uses no workspace.  Lists are read, never written. */
RBS_API rbs_status bsa_prefill(const rbs_bf16_tensor* Q, const rbs_bf16_tensor* K, const rbs_bf16_tensor* V,
                       const rbs_block_lists* lists, int32_t block_q, int32_t block_k, int64_t q_offset,
                       float softmax_scale, int32_t causal, rbs_bf16_tensor* O, float* lse, rbs_stream_t stream);

/* ---- rescue blocks with a controlled contribution  ([RBS-id] "Dual-Branch
 * Selection": regular blocks through the block-sparse pass, rescue blocks
 * handled separately, their contribution controllable)
 * A list entry is a rescue block when its flags have the rescue bit and
 * neither the centroid nor the forced bit; every other entry is regular.  With
 * x_s = scale * q_t . k_s and w = rescue_weight:
 *   O[b, t, h] = (sum_{s regular} e^{x_s} v_s + w sum_{s rescue} e^{x_s} v_s)
 *              / (sum_{s regular} e^{x_s}     + w sum_{s rescue} e^{x_s})
 * i.e. the regular and the rescue partial attentions merged with the rescue
 * partial's softmax mass scaled by w; lse = ln of that denominator (-inf and
 * O = 0 when it is 0).  w = 1 is bsa_prefill; w = 0 keeps the regular blocks
 * only.  Arguments, layouts and errors as bsa_prefill, plus:
 *   rescue_weight  finite, >= 0 (else RBS_ERR_INVALID_ARG)
 *   lists->flags   required unless rescue_weight == 1 (else RBS_ERR_INVALID_ARG)
 * One pass: the kernel adds log2(w) to the scaled scores of the rescue
 * blocks' tiles, which weights their softmax mass by w. */
RBS_API rbs_status bsa_prefill_rescue_weighted(const rbs_bf16_tensor* Q, const rbs_bf16_tensor* K,
                                       const rbs_bf16_tensor* V, const rbs_block_lists* lists, int32_t block_q,
                                       int32_t block_k, int64_t q_offset, float softmax_scale, int32_t causal,
                                       float rescue_weight, rbs_bf16_tensor* O, float* lse, rbs_stream_t stream);

/* ---- Block-attention with passages at any token offset  ([BA] 2.2 Block
 * segmentation: each retrieved passage is a block, the user query is the
 * final block; 2.4 Block fine-tune: a token of a passage attends only to
 * earlier tokens of its own passage, a token of the final block to every
 * earlier token)
 * bsa_prefill with the Block-attention mask applied token by token: the
 * query token at key position p = t + q_offset sees key s when
 *   lo(p) <= s <= p,  lo(p) = the last seg_start <= p   (p < final_start)
 *                     lo(p) = 0                          (p >= final_start).
 * seg_start / num_segments / final_start as for rbs_lists_block_attention
 * (a HOST array; offsets need not be block multiples), and lists must hold
 * every key block a row's tokens may see (rbs_lists_block_attention with the
 * same segments builds them: a query block straddling a passage boundary
 * lists both passages' blocks and the bound above removes the keys its
 * tokens may not see).  Always causal.  Other arguments, layouts and errors
 * as bsa_prefill. */
RBS_API rbs_status bsa_prefill_segments(const rbs_bf16_tensor* Q, const rbs_bf16_tensor* K, const rbs_bf16_tensor* V,
                                        const rbs_block_lists* lists, int32_t block_q, int32_t block_k,
                                        int64_t q_offset, const int32_t* seg_start, int32_t num_segments,
                                        int32_t final_start, float softmax_scale, rbs_bf16_tensor* O, float* lse,
                                        rbs_stream_t stream);

/* ---- RoPE position re-encoding  ([BA] 2.3 Position re-encoding, 2.5 Inference)
 * Keys cached with RoPE at old_pos are moved to new_pos: the rotation is reset
 * to position 0 and applied again at the new position, done as one rotation by
 * (new_pos - old_pos) * inv_freq_m, inv_freq_m = theta^(-2m/128).  The angle
 * is formed and reduced in fp64; the rotation is applied in fp32 and rounded
 * to bf16 once.
 *   x_in, x_out  [B, L, H, 128] bf16, same shape; x_out may alias x_in
 *   old_pos, new_pos  [L] int32 token positions (shared by batch and heads)
 *   rope_style   0 = rotate-half pairs (m, m + 64); 1 = interleaved (2m, 2m+1)
 * Re-encoding from old_pos = 0 is plain RoPE encoding. */
RBS_API rbs_status rope_reencode(const rbs_bf16_tensor* x_in, rbs_bf16_tensor* x_out, const int32_t* old_pos,
                         const int32_t* new_pos, float theta, int32_t rope_style, rbs_stream_t stream);

/* ---- testing hooks (no counterpart in the papers; used by the library's
 * own tests to reach code paths that correct inputs never reach)
 * rbs_testing_bsa_prefill_stalled: bsa_prefill (causal, default scale, no
 *   LSE) with every pipeline wait limited to wait_ns (1e5 .. 2e9 ns; the
 *   product limit is 2e9) and the K/Q producer stopping for good after
 *   stall_after key tiles.  The waits for the tiles never loaded run out:
 *   the kernel must set RBS_DEVERR_TIMEOUT, leave no copy or MMA in flight,
 *   free its tensor memory and return.  O is left partly written.
 * rbs_testing_exp2: y[i] = the attention kernel's software base-2
 *   exponential (the FMA-pipe polynomial) of x[i], n values (device). */
RBS_API rbs_status rbs_testing_bsa_prefill_stalled(const rbs_bf16_tensor* Q, const rbs_bf16_tensor* K,
                                                   const rbs_bf16_tensor* V, const rbs_block_lists* lists,
                                                   int32_t block_q, int32_t block_k, uint64_t wait_ns,
                                                   int32_t stall_after, rbs_bf16_tensor* O, rbs_stream_t stream);
RBS_API rbs_status rbs_testing_exp2(const float* x, float* y, int64_t n, rbs_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* RBS_H_ */
