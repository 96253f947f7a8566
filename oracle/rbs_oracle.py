"""Plain CPU float64 oracle for RBS block selection, block-sparse prefill
attention, Block-attention lists and RoPE position re-encoding.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
this module.  It shares no code with the CUDA library: it reads the same bf16
input bytes (widened exactly to float64) and computes every step from its
plain definition with numpy, one step per function, in the order the sources
give them.  It is slow on purpose.

Sources (web pages; cited by title and section):

* [RBS-en] "RBS-Attention: How a Geometric Rescue Branch Fixes Sparse Prefill
  for Long-Context LLMs" -- sections "The Standard Approach and Its Blind
  Spot" (centroid = average of the block's keys; radius = largest distance of
  a key from the centroid) and "The Fix: A Radius-Adaptive Rescue Branch"
  (centroid branch q^T c_b; rescue branch q^T c_b + |q|_2 r_b beta_b with
  beta_b in [0, 1] taken from the radius distribution; branches thresholded
  independently, masks combined; Cauchy-Schwarz bound; exact block-sparse
  attention on the result).
* [RBS-id] "RBS-Attention Bikin Prefill LLM Gede 20x Lebih Cepat, Tanpa
  Training Lagi?" -- section "Dual-Branch Selection: Centroid Base + Rescue
  Branch" (radius distribution per prompt, per layer, per head; the two
  branches thresholded independently; masks merged).
* [BA] "Block-Attention for Efficient Prefilling" -- 2.1 Main idea, 2.2 Block
  segmentation, 2.3 Position re-encoding, 2.4 Block fine-tune (mask), 2.5
  Inference.

Readings of points the pages leave open (each is a parameter here):
  query representative = mean of the query block's queries; raw dot-product
  scores (no 1/sqrt(d)); beta = per (prompt, KV head) min-max normalisation of
  the radii with quantiles (p_lo, p_hi) (type-7, linear interpolation), a
  degenerate range giving beta = 1; per-branch threshold = keep the
  k_i = ceil(rho * n_i) best of the n_i causally visible blocks, ties to the
  lower block index; the diagonal block is always kept and does not count
  toward k_i; RoPE = rotate-half pairs (m, m + d/2) with
  inv_freq_m = theta^(-2m/d).

Pins: every function here is checked in tests/test_oracle_pins.py against a
closed form, a library routine, an invariant the pages state, or brute force.
Parity unpinned: none of the functions below.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

# ----------------------------------------------------------------------------
# bf16 storage -> float64


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def as_f64(x: np.ndarray) -> np.ndarray:
    """Accept either bf16 bits (uint16) or floating arrays; return float64."""
    if x.dtype == np.uint16:
        return bf16_to_f64(x)
    return np.asarray(x, dtype=np.float64)


# ----------------------------------------------------------------------------
# Parameters of the selection (mirrors the C struct field by field)


@dataclasses.dataclass
class SelectParams:
    block_q: int = 128
    block_k: int = 128
    rho_centroid: float = 0.05
    rho_rescue: float = 0.05
    beta_mode: int = 0  # 0 = RANGE (quantile min-max of the radii), 1 = CONST
    beta_const: float = 1.0
    beta_p_lo: float = 0.0  # < 0 means R_lo = 0
    beta_p_hi: float = 1.0
    force_diag: int = 1
    force_sink: int = 0
    causal: int = 1
    q_block_offset: int = 0  # global index of query block 0 (in key blocks)
    # threshold rule per branch: 0 = TOPK_FRACTION (keep the top k_i), 1 =
    # MAX_RELATIVE (keep every visible block scoring at least the row's
    # maximum minus delta, no ranking)
    threshold_mode: int = 0
    delta_centroid: float = 0.0
    delta_rescue: float = 0.0
    # list layout: 0 = one list per (batch, q head, query block); 1 = one list
    # per (batch, KV head, query block), the union of the lists of the q heads
    # that share the KV head (they then attend to the same key blocks)
    list_mode: int = 0
    # query representative: 0 = MEAN (the mean of the query block's queries);
    # 1 = TOKEN_MAX (each branch scores a key block by its best query token)
    query_pool: int = 0


FLAG_CENTROID = 1
FLAG_RESCUE = 2
FLAG_FORCED = 4


# ----------------------------------------------------------------------------
# Block statistics  [RBS-en, "The Standard Approach and Its Blind Spot"]


def block_stats(K: np.ndarray, block_k: int):
    """Centroid and radius of every key block.

    K: [B, L, Hkv, d] (bf16 bits or float).  Block b holds keys
    b*block_k .. min((b+1)*block_k, L) - 1, so n_b = block_k except for a
    last, shorter block when L is not a multiple of block_k.
    c_b = (1/n_b) sum_{k in b} k ;  r_b = max_{k in b} ||k - c_b||_2.
    Returns centroids [B, Hkv, nKB, d] and radii [B, Hkv, nKB], float64,
    nKB = ceil(L / block_k).
    """
    B, L, H, d = K.shape
    nkb = -(-L // block_k)
    C = np.empty((B, H, nkb, d))
    R = np.empty((B, H, nkb))
    for b in range(B):
        for h in range(H):
            x = as_f64(K[b, :, h, :])
            for j in range(nkb):
                kb = x[j * block_k:min((j + 1) * block_k, L)]
                c = kb.sum(axis=0) / kb.shape[0]
                C[b, h, j] = c
                R[b, h, j] = np.sqrt(((kb - c) ** 2).sum(axis=1)).max()
    return C, R


# ----------------------------------------------------------------------------
# Rescue coefficient beta_b  [RBS-en "The Fix"; RBS-id "Dual-Branch Selection"]


def quantile_type7(x: np.ndarray, p: float) -> float:
    """Linear-interpolation sample quantile (Hyndman-Fan type 7)."""
    xs = np.sort(np.asarray(x, dtype=np.float64).ravel())
    n = xs.size
    h = (n - 1) * p
    lo = int(math.floor(h))
    hi = min(lo + 1, n - 1)
    return float(xs[lo] + (h - lo) * (xs[hi] - xs[lo]))


def rescue_beta(R: np.ndarray, p: SelectParams):
    """beta [B, Hkv, nKB] in [0, 1] and the (R_lo, R_hi) range per (batch, KV head).

    RANGE mode: beta_b = clamp((r_b - R_lo) / (R_hi - R_lo), 0, 1) where
    R_lo, R_hi are the p_lo / p_hi quantiles of the radii of that prompt and
    KV head (R_lo = 0 when p_lo < 0); a range of (relative) width <= 1e-12
    gives beta = 1.  CONST mode: beta_b = beta_const.
    """
    B, H, nkb = R.shape
    beta = np.empty_like(R)
    rng = np.empty((B, H, 2))
    for b in range(B):
        for h in range(H):
            r = R[b, h]
            if p.beta_mode == 1:
                beta[b, h] = p.beta_const
                rng[b, h] = (0.0, 0.0)
                continue
            r_lo = 0.0 if p.beta_p_lo < 0 else quantile_type7(r, p.beta_p_lo)
            r_hi = quantile_type7(r, p.beta_p_hi)
            rng[b, h] = (r_lo, r_hi)
            if r_hi - r_lo <= 1e-12 * max(r_hi, 1e-30):
                beta[b, h] = 1.0
            else:
                beta[b, h] = np.clip((r - r_lo) / (r_hi - r_lo), 0.0, 1.0)
    return beta, rng


# ----------------------------------------------------------------------------
# Query-block representative  [RBS-en "The Fix": the q in q^T c_b]


def pooled_queries(Q: np.ndarray, block_q: int):
    """Mean query of every query block and its Euclidean norm.

    Q: [B, L, Hq, d].  Query block i holds queries i*block_q ..
    min((i+1)*block_q, L) - 1 (a last, shorter block when L is not a
    multiple of block_q).  Returns qbar [B, Hq, nQB, d] and qnorm [B, Hq, nQB],
    nQB = ceil(L / block_q).
    """
    B, L, H, d = Q.shape
    nqb = -(-L // block_q)
    qbar = np.empty((B, H, nqb, d))
    for b in range(B):
        for h in range(H):
            x = as_f64(Q[b, :, h, :])
            for i in range(nqb):
                blk = x[i * block_q:min((i + 1) * block_q, L)]
                qbar[b, h, i] = blk.sum(axis=0) / blk.shape[0]
    qnorm = np.sqrt((qbar ** 2).sum(axis=-1))
    return qbar, qnorm


# ----------------------------------------------------------------------------
# Branch scores, per-branch threshold, union  [RBS-en "The Fix"; RBS-id]


def keep_count(rho: float, n: int) -> int:
    """k = ceil(rho * n), at least 1 and at most n.

    rho is a float32 parameter (e.g. float32(0.05) = 0.0500000007...); the
    1e-4 slack keeps its representation error from adding a block
    (ceil(20 * float32(0.05)) would otherwise be 2, not 1).
    """
    return int(min(n, max(1, math.ceil(rho * n - 1e-4))))


def visible_blocks(i: int, nkb: int, p: SelectParams) -> int:
    """Number of key blocks query block i may select: 0..i+offset when causal, else all."""
    if p.causal:
        return min(nkb, i + p.q_block_offset + 1)
    return nkb


def top_k_desc(scores: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k best scores, best first: higher score first, ties to the lower index."""
    order = np.argsort(-scores, kind="stable")
    return order[:k]


def branch_scores(qbar: np.ndarray, qnorm: np.ndarray, C: np.ndarray, R: np.ndarray, beta: np.ndarray):
    """Centroid-branch and rescue-branch scores of one (prompt, q head).

    qbar [nQB, d], qnorm [nQB], C [nKB, d], R, beta [nKB] (the q head's KV head).
    s_c(i, j) = qbar_i . c_j ;  s_r(i, j) = s_c(i, j) + |qbar_i| * r_j * beta_j.
    """
    s_c = qbar @ C.T
    s_r = s_c + qnorm[:, None] * (R * beta)[None, :]
    return s_c, s_r


def token_max_scores(Qbh: np.ndarray, C: np.ndarray, R: np.ndarray, beta: np.ndarray, block_q: int):
    """Per-token scoring of one (prompt, q head): every query token scores the
    key blocks, and a query block keeps each branch's best token score.

    Qbh [L, d] (the q head's queries), C [nKB, d], R, beta [nKB].  For query
    block i (tokens i*block_q .. min((i+1)*block_q, L) - 1):
      s_c(i, j) = max_t q_t . c_j
      s_r(i, j) = max_t (q_t . c_j + |q_t| r_j beta_j)
    ([RBS-en] "The Fix" writes both branch scores for a query q; here q runs
    over the block's query tokens instead of their mean).
    """
    L = Qbh.shape[0]
    nqb = -(-L // block_q)
    q = as_f64(Qbh)
    rb = R * beta
    s_c = np.empty((nqb, C.shape[0]))
    s_r = np.empty((nqb, C.shape[0]))
    for i in range(nqb):
        qi = q[i * block_q:min((i + 1) * block_q, L)]
        dots = qi @ C.T  # [tokens, nKB]
        s_c[i] = dots.max(axis=0)
        s_r[i] = (dots + np.sqrt((qi ** 2).sum(axis=1))[:, None] * rb[None, :]).max(axis=0)
    return s_c, s_r


def branch_scores_for(Q, qbar, qnorm, C, R, beta, b: int, hq: int, kvh: int, p: SelectParams):
    """The two branches' scores of one (prompt, q head) under p.query_pool."""
    if p.query_pool == 1:
        return token_max_scores(Q[b, :, hq, :], C[b, kvh], R[b, kvh], beta[b, kvh], p.block_q)
    return branch_scores(qbar[b, hq], qnorm[b, hq], C[b, kvh], R[b, kvh], beta[b, kvh])


def select_blocks(Q: np.ndarray, C: np.ndarray, R: np.ndarray, p: SelectParams, keep_scores: bool = False):
    """Per-query-block KV-block lists (CSR), rows ordered (batch, q head, query block).

    For each row: both branches keep their own top-k_i of the visible blocks
    (k_i = keep_count(rho_branch, n_i)); the row's list is the union of the
    two kept sets plus the forced diagonal (and block 0 when force_sink),
    sorted ascending.  flags: bit0 centroid kept, bit1 rescue kept, bit2 forced.
    Also returns each row's per-branch threshold tau (the k_i-th kept score)
    and, with keep_scores, the score matrices (for the near-threshold rule).

    threshold_mode 1 replaces each branch's top-k by a threshold relative to
    the row maximum, tau = max_j s(i, j) - delta_branch: every visible block
    with s >= tau is kept (the max-based dynamic thresholding [RBS-en] "How
    This Fits Into the Broader Sparse Attention Landscape" describes as an
    alternative to ranking, with the rescue branch layered on it).  k then
    reports the kept count.

    list_mode 1 returns one list per (batch, KV head, query block) instead:
    the union of the lists of the G = Hq / Hkv q heads of that KV head, each
    entry's flags the OR of those heads' flags (grouped-query attention with
    the key blocks shared by the group, [RBS-en] "How This Fits Into the
    Broader Sparse Attention Landscape"; sharing selected KV entries across
    queries, [QUILT] Abstract).  tau and k stay per q head.
    """
    B, L, Hq, d = Q.shape
    _, Hkv, nkb, _ = C.shape
    G = Hq // Hkv
    beta, _ = rescue_beta(R, p)
    qbar, qnorm = pooled_queries(Q, p.block_q)
    nqb = qbar.shape[2]
    row_ptr = [0]
    cols, flags = [], []
    tau = np.zeros((B, Hq, nqb, 2))
    kept_k = np.zeros((B, Hq, nqb, 2), dtype=np.int64)
    scores = {} if keep_scores else None
    for b in range(B):
        for hq in range(Hq):
            kvh = hq // G
            s_c, s_r = branch_scores_for(Q, qbar, qnorm, C, R, beta, b, hq, kvh, p)
            if keep_scores:
                scores[(b, hq)] = (s_c, s_r)
            for i in range(nqb):
                n = visible_blocks(i, nkb, p)
                if p.threshold_mode == 1:
                    t_c = s_c[i, :n].max() - p.delta_centroid
                    t_r = s_r[i, :n].max() - p.delta_rescue
                    top_c = np.nonzero(s_c[i, :n] >= t_c)[0]
                    top_r = np.nonzero(s_r[i, :n] >= t_r)[0]
                    kc, kr = top_c.size, top_r.size
                    tau[b, hq, i] = (t_c, t_r)
                else:
                    kc = keep_count(p.rho_centroid, n)
                    kr = keep_count(p.rho_rescue, n)
                    top_c = top_k_desc(s_c[i, :n], kc)
                    top_r = top_k_desc(s_r[i, :n], kr)
                    tau[b, hq, i] = (s_c[i, top_c[-1]], s_r[i, top_r[-1]])
                kept_k[b, hq, i] = (kc, kr)
                f = np.zeros(nkb, dtype=np.uint8)
                f[top_c] |= FLAG_CENTROID
                f[top_r] |= FLAG_RESCUE
                diag = i + p.q_block_offset
                if p.force_diag and diag < nkb:
                    f[diag] |= FLAG_FORCED
                if p.force_sink:
                    f[0] |= FLAG_FORCED
                sel = np.nonzero(f)[0]
                cols.extend(sel.tolist())
                flags.extend(f[sel].tolist())
                row_ptr.append(len(cols))
    if p.list_mode == 1:
        row_ptr, cols, flags = group_union_lists(row_ptr, cols, flags, B, Hq, Hkv, nqb, nkb)
    out = {
        "row_ptr": np.asarray(row_ptr, dtype=np.int64),
        "col_idx": np.asarray(cols, dtype=np.int64),
        "flags": np.asarray(flags, dtype=np.uint8),
        "tau": tau,
        "k": kept_k,
        "beta": beta,
        "qbar": qbar,
        "qnorm": qnorm,
    }
    if keep_scores:
        out["scores"] = scores
    return out


def group_union_lists(row_ptr, cols, flags, B: int, Hq: int, Hkv: int, nqb: int, nkb: int):
    """Per-q-head CSR rows (b, hq, i) -> per-KV-head rows (b, g, i): the set union
    of the rows of q heads g*G .. g*G + G - 1, ascending, flags OR-ed."""
    G = Hq // Hkv
    out_ptr, out_cols, out_flags = [0], [], []
    for b in range(B):
        for g in range(Hkv):
            for i in range(nqb):
                f = np.zeros(nkb, dtype=np.uint8)
                for hq in range(g * G, (g + 1) * G):
                    r = (b * Hq + hq) * nqb + i
                    for e in range(row_ptr[r], row_ptr[r + 1]):
                        f[cols[e]] |= flags[e]
                sel = np.nonzero(f)[0]
                out_cols.extend(sel.tolist())
                out_flags.extend(f[sel].tolist())
                out_ptr.append(len(out_cols))
    return out_ptr, out_cols, out_flags


def list_density(row_ptr: np.ndarray, nqb: int, nkb: int, q_block_offset: int = 0, causal: int = 1) -> float:
    """Kept-block density: selected (row, block) pairs over visible pairs."""
    rows = row_ptr.size - 1
    per_head_visible = sum(min(nkb, i + q_block_offset + 1) if causal else nkb for i in range(nqb))
    return float(row_ptr[-1]) / (per_head_visible * (rows // nqb))


def union_ranks(Q, C, R, p: SelectParams):
    """For every row: each visible block's better rank over the two branches, and the forced mask.

    rank = position in the branch's best-first order (higher score first, ties
    to the lower index).  With both branches at the same rho, block j is kept
    iff min(rank_c, rank_r) < k_i(rho) or j is forced: the same set
    select_blocks builds.
    """
    B, L, Hq, d = Q.shape
    _, Hkv, nkb, _ = C.shape
    G = Hq // Hkv
    beta, _ = rescue_beta(R, p)
    qbar, qnorm = pooled_queries(Q, p.block_q)
    nqb = qbar.shape[2]
    rows = []
    for b in range(B):
        for hq in range(Hq):
            kvh = hq // G
            s_c, s_r = branch_scores_for(Q, qbar, qnorm, C, R, beta, b, hq, kvh, p)
            for i in range(nqb):
                n = visible_blocks(i, nkb, p)
                rank_c = np.empty(n, dtype=np.int64)
                rank_c[top_k_desc(s_c[i, :n], n)] = np.arange(n)
                rank_r = np.empty(n, dtype=np.int64)
                rank_r[top_k_desc(s_r[i, :n], n)] = np.arange(n)
                forced = np.zeros(n, dtype=bool)
                diag = i + p.q_block_offset
                if p.force_diag and diag < n:
                    forced[diag] = True
                if p.force_sink:
                    forced[0] = True
                rows.append((np.minimum(rank_c, rank_r), forced))
    return rows


def density_of(rows, rho: float) -> float:
    """Kept-union density at a shared per-branch rho, from union_ranks output."""
    kept = visible = 0
    for best, forced in rows:
        n = best.size
        kept += np.count_nonzero((best < keep_count(rho, n)) | forced)
        visible += n
    return kept / visible


def bisect_rho(Q, C, R, p: SelectParams, target: float, steps: int = 30):
    """Shared per-branch rho whose kept-union density is closest to ``target``.

    Density is monotone in rho (each branch's top-k sets are nested), so a
    bisection on [0, 1] converges.  Returns (rho, achieved density).
    """
    rows = union_ranks(Q, C, R, p)
    lo, hi = 0.0, 1.0
    best = None
    for _ in range(steps):
        mid = 0.5 * (lo + hi)
        dens = density_of(rows, mid)
        if best is None or abs(dens - target) < abs(best[1] - target):
            best = (mid, dens)
        if dens < target:
            lo = mid
        else:
            hi = mid
    return best


# ----------------------------------------------------------------------------
# List builders: causal-full and Block-attention  [BA 2.1, 2.2, 2.4]


def causal_full_lists(batch: int, heads_q: int, nqb: int, q_block_offset: int = 0):
    """Every causally visible block for every row: j in [0, i + offset]."""
    row_ptr = [0]
    cols = []
    for _ in range(batch * heads_q):
        for i in range(nqb):
            cols.extend(range(0, i + q_block_offset + 1))
            row_ptr.append(len(cols))
    return np.asarray(row_ptr, dtype=np.int64), np.asarray(cols, dtype=np.int64)


def block_attention_key_start(seg_start, final_start: int, positions) -> np.ndarray:
    """Lowest key position each query position may attend to under the
    Block-attention mask ([BA] 2.1 Main idea, 2.2 Block segmentation, 2.4
    Block fine-tune): a token of passage s (seg_start[s] <= p < next start,
    the last passage ending at final_start) sees only its own passage's
    keys, so the bound is its passage's first token; a token of the final
    block (p >= final_start) sees the whole prompt, bound 0.  Passage starts
    are token offsets; nothing requires them to be block multiples."""
    starts = [int(x) for x in seg_start]
    assert starts[0] == 0 and all(b > a for a, b in zip(starts, starts[1:])) and final_start > starts[-1]
    out = []
    for p in positions:
        p = int(p)
        if p >= final_start:
            out.append(0)
        else:
            out.append(max(a for a in starts if a <= p))
    return np.asarray(out, dtype=np.int64)


def block_attention_lists(seg_start, final_start: int, block: int, batch: int, heads_q: int,
                          q_first_block: int, q_num_blocks: int):
    """Block-attention mask as per-query-block lists.

    Segments: passage s covers tokens [seg_start[s], next start); the final
    block (the user query) starts at ``final_start`` and runs to the end.
    Query block g holds tokens [g * block, (g + 1) * block); its row lists
    every key block that holds a key one of those tokens may see: from the
    block of the smallest key_start over its tokens (block_attention_key_start)
    up to g itself (causal).  When passages start on block boundaries this is
    "the key blocks of the passage up to itself" for a passage block and
    "every key block up to itself" for a block of the final block; a block
    that straddles a boundary lists the union of its tokens' ranges, and the
    token-level mask (masked_attention's key_start) removes the keys of the
    other passage.  Rows cover query blocks q_first_block .. q_first_block +
    q_num_blocks - 1 (global block indices), for every (batch, q head).
    """
    row_ptr = [0]
    cols = []
    for _ in range(batch * heads_q):
        for gi in range(q_first_block, q_first_block + q_num_blocks):
            lo = block_attention_key_start(seg_start, final_start, range(gi * block, (gi + 1) * block)).min()
            cols.extend(range(int(lo) // block, gi + 1))
            row_ptr.append(len(cols))
    return np.asarray(row_ptr, dtype=np.int64), np.asarray(cols, dtype=np.int64)


# ----------------------------------------------------------------------------
# Exact block-sparse attention  [RBS-en "The Fix": exact attention over the
# selected blocks; standard multi-head / grouped-query attention]


def masked_attention(Q, K, V, row_ptr, col_idx, block_q: int, block_k: int, q_offset: int = 0,
                     scale: float | None = None, causal: int = 1, rows=None, key_start=None):
    """Softmax attention of each query token over the key tokens of its row's blocks.

    Q [B, Lq, Hq, d]; K, V [B, Lk, Hkv, d].  The lists hold one row per
    (b, hq, i), or, when they have B * Hkv * nqb rows (Hkv < Hq), one row per
    (b, KV head, i) that every q head of the KV head uses.  Query token t of
    query block i of q head hq sits at position t + q_offset and may see key
    position s of any listed block when s <= t + q_offset (causal).  The KV
    head of q head hq is hq // (Hq / Hkv).  Returns O [B, Lq, Hq, d] (NaN for
    rows not computed) and lse [B, Hq, Lq] = log sum_s exp(scale * q.k_s).
    ``rows``: optional iterable of (b, hq, i) numbers (b * Hq + hq) * nqb + i
    to compute (default: all).  ``key_start``: optional [Lq] array, the lowest
    key position query token t may see (the Block-attention token mask,
    block_attention_key_start of the token's position); keys below it are
    masked like keys after the query.
    """
    B, Lq, Hq, d = Q.shape
    Hkv = K.shape[2]
    G = Hq // Hkv
    Lk = K.shape[1]
    nqb = -(-Lq // block_q)  # a last, shorter query block when Lq is not a block multiple
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = np.full((B, Lq, Hq, d), np.nan)
    lse = np.full((B, Hq, Lq), np.nan)
    group_lists = Hkv < Hq and len(row_ptr) - 1 == B * Hkv * nqb
    if rows is None:
        rows = range(B * Hq * nqb)
    for row in rows:
        b, rem = divmod(int(row), Hq * nqb)
        hq, i = divmod(rem, nqb)
        kvh = hq // G
        lrow = (b * Hkv + kvh) * nqb + i if group_lists else row
        blocks = col_idx[row_ptr[lrow]:row_ptr[lrow + 1]]
        t0, t1 = i * block_q, min((i + 1) * block_q, Lq)
        q = as_f64(Q[b, t0:t1, hq, :])
        if len(blocks) == 0:
            O[b, t0:t1, hq] = 0.0
            lse[b, hq, t0:t1] = -np.inf
            continue
        # key positions of the listed blocks (a last, shorter block ends at Lk)
        kpos = np.concatenate([np.arange(j * block_k, min((j + 1) * block_k, Lk)) for j in blocks])
        k = as_f64(K[b, kpos, kvh, :])
        v = as_f64(V[b, kpos, kvh, :])
        logits = scale * (q @ k.T)
        if causal:
            qpos = np.arange(t0, t1) + q_offset
            logits = np.where(kpos[None, :] <= qpos[:, None], logits, -np.inf)
        if key_start is not None:
            lo = np.asarray(key_start, dtype=np.int64)[t0:t1]
            logits = np.where(kpos[None, :] >= lo[:, None], logits, -np.inf)
        m = logits.max(axis=1, keepdims=True)
        m = np.where(np.isfinite(m), m, 0.0)
        w = np.exp(logits - m)
        z = w.sum(axis=1, keepdims=True)
        with np.errstate(invalid="ignore", divide="ignore"):
            O[b, t0:t1, hq] = np.where(z > 0, (w @ v) / z, 0.0)
            lse[b, hq, t0:t1] = (np.log(z) + m)[:, 0]
    return O, lse


def split_regular_rescue(row_ptr, col_idx, flags):
    """Split lists into the regular blocks (kept by the centroid branch, or
    forced) and the rescue blocks (kept by the rescue branch alone), each in
    CSR form over the same rows ([RBS-id] "Dual-Branch Selection": regular
    blocks go through the standard block-sparse pass, rescue blocks are
    handled separately).  Entries without any flag count as regular."""
    reg_ptr, reg_idx, res_ptr, res_idx = [0], [], [0], []
    for r in range(len(row_ptr) - 1):
        for e in range(row_ptr[r], row_ptr[r + 1]):
            f = int(flags[e])
            rescue_only = (f & FLAG_RESCUE) and not (f & (FLAG_CENTROID | FLAG_FORCED))
            (res_idx if rescue_only else reg_idx).append(int(col_idx[e]))
        reg_ptr.append(len(reg_idx))
        res_ptr.append(len(res_idx))
    as_arr = lambda x: np.asarray(x, dtype=np.int64)
    return as_arr(reg_ptr), as_arr(reg_idx), as_arr(res_ptr), as_arr(res_idx)


def rescue_weighted_attention(Q, K, V, row_ptr, col_idx, flags, rescue_weight: float, block_q: int, block_k: int,
                              q_offset: int = 0, scale: float | None = None, causal: int = 1, rows=None):
    """Attention with the rescue blocks handled separately and their contribution
    scaled by rescue_weight (gamma >= 0) ([RBS-id] "Dual-Branch Selection": the
    rescue blocks' contribution can be controlled precisely).

    The regular blocks and the rescue blocks are each attended on their own
    (softmax partials O_reg, lse_reg and O_res, lse_res), and the partials are
    merged with the rescue partial's softmax mass multiplied by gamma:
      Z = exp(lse_reg) + gamma exp(lse_res)
      O = (exp(lse_reg) O_reg + gamma exp(lse_res) O_res) / Z,  lse = log Z.
    gamma = 1 is attention over the union of both sets; gamma = 0 is attention
    over the regular blocks alone.  A row with Z = 0 gives O = 0, lse = -inf.
    Arguments as masked_attention, plus the lists' flags.
    """
    reg_ptr, reg_idx, res_ptr, res_idx = split_regular_rescue(row_ptr, col_idx, flags)
    Oa, la = masked_attention(Q, K, V, reg_ptr, reg_idx, block_q, block_k, q_offset, scale, causal, rows)
    Ob, lb = masked_attention(Q, K, V, res_ptr, res_idx, block_q, block_k, q_offset, scale, causal, rows)
    m = np.maximum(la, lb)
    m = np.where(np.isfinite(m), m, 0.0)
    with np.errstate(invalid="ignore", over="ignore"):
        wa = np.where(np.isfinite(la), np.exp(la - m), 0.0)
        wb = np.where(np.isfinite(lb), rescue_weight * np.exp(lb - m), 0.0)
        z = wa + wb
        Oa0 = np.where(np.isfinite(la)[..., None].transpose(0, 2, 1, 3), Oa, 0.0)
        Ob0 = np.where(np.isfinite(lb)[..., None].transpose(0, 2, 1, 3), Ob, 0.0)
        wa_t, wb_t, z_t = (x.transpose(0, 2, 1)[..., None] for x in (wa, wb, z))
        O = np.where(z_t > 0, (wa_t * Oa0 + wb_t * Ob0) / np.where(z_t > 0, z_t, 1.0), 0.0)
        lse = np.where(z > 0, np.log(np.where(z > 0, z, 1.0)) + m, -np.inf)
    nan_rows = np.isnan(la)  # rows not computed stay NaN
    O = np.where(nan_rows.transpose(0, 2, 1)[..., None], np.nan, O)
    lse = np.where(nan_rows, np.nan, lse)
    return O, lse


def dense_causal_attention(Q, K, V, q_offset: int = 0, scale: float | None = None):
    """Textbook softmax(scale * Q K^T + causal mask) V per q head, full matrices (no blocks).

    Query row t sits at position t + q_offset and sees keys s <= t + q_offset.
    """
    B, Lq, Hq, d = Q.shape
    Lk, Hkv = K.shape[1], K.shape[2]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = np.empty((B, Lq, Hq, d))
    mask = np.arange(Lk)[None, :] > (np.arange(Lq)[:, None] + q_offset)
    for b in range(B):
        for hq in range(Hq):
            q = as_f64(Q[b, :, hq, :])
            k = as_f64(K[b, :, hq // G, :])
            v = as_f64(V[b, :, hq // G, :])
            s = scale * (q @ k.T)
            s[mask] = -np.inf
            s -= s.max(axis=1, keepdims=True)
            pmat = np.exp(s)
            pmat /= pmat.sum(axis=1, keepdims=True)
            O[b, :, hq] = pmat @ v
    return O


# ----------------------------------------------------------------------------
# RoPE and position re-encoding  [BA 2.3 Position re-encoding, 2.5 Inference]


def rope_inv_freq(d: int, theta: float) -> np.ndarray:
    """inv_freq_m = theta^(-2m/d), m = 0 .. d/2 - 1."""
    return theta ** (-2.0 * np.arange(d // 2) / d)


def rope_rotate(x: np.ndarray, pos, theta: float, style: int = 0) -> np.ndarray:
    """Rotate every (pair) of x [B, L, H, d] by the angle pos_t * inv_freq_m.

    style 0 (rotate-half): pairs (m, m + d/2).  style 1 (interleaved): pairs (2m, 2m+1).
    (a, b) -> (a cos phi - b sin phi, a sin phi + b cos phi).
    """
    x = as_f64(x)
    d = x.shape[-1]
    phi = np.asarray(pos, dtype=np.float64)[:, None] * rope_inv_freq(d, theta)[None, :]  # [L, d/2]
    cos = np.cos(phi)[None, :, None, :]
    sin = np.sin(phi)[None, :, None, :]
    out = np.empty_like(x)
    if style == 0:
        a, b = x[..., : d // 2], x[..., d // 2:]
        out[..., : d // 2] = a * cos - b * sin
        out[..., d // 2:] = a * sin + b * cos
    else:
        a, b = x[..., 0::2], x[..., 1::2]
        out[..., 0::2] = a * cos - b * sin
        out[..., 1::2] = a * sin + b * cos
    return out


def rope_reencode(x: np.ndarray, old_pos, new_pos, theta: float, style: int = 0) -> np.ndarray:
    """Re-encode keys cached at old_pos to new_pos: reset the rotation to position 0, then rotate to new_pos."""
    at_zero = rope_rotate(x, -np.asarray(old_pos, dtype=np.float64), theta, style)
    return rope_rotate(at_zero, new_pos, theta, style)
