"""Seeded synthetic Q/K/V generators for the five prefill workloads.

The pages measure on RULER / LongBench-v2 / InfiniteBench with trained
models; none of that is available, so these generators stand in for the
pages' 128K-context workloads with the same shapes and with key blocks whose
structure (compact vs dispersed blocks, isolated high-dot "planted" keys)
exercises the failure mode the RBS-Attention article describes ("The
Standard Approach and Its Blind Spot": a single relevant key diluted inside a
block of noise).

Storage: every tensor is returned as a numpy ``uint16`` array holding bf16
bit patterns, layout ``[B, L, H, d]`` with ``d`` contiguous.  Values are drawn
in float32 from ``numpy.random.Generator(PCG64(seed))`` and rounded once to
bf16 (round to nearest, ties to even).  The same bytes feed the GPU path and
the oracle.

Draw order (fixed, so a workload is reproducible from its seed): Q, key
structure (per-block centres and compact/dispersed flags, or block offsets),
K noise, V, planted keys.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

HEAD_DIM = 128
SEED_BASE = 20260


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return the bits as uint16."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    rounding = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float32 exactly."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic prefill workload (shapes, block size and selection budget)."""

    name: str
    seqlen: int
    heads_q: int
    heads_kv: int
    block: int
    kind: str  # "tiny", "mixture" or "block_attention"
    rho: float | None = None  # per-branch kept fraction, when fixed
    density_target: float | None = None  # kept-union density target, when bisected
    batch: int = 1
    head_dim: int = HEAD_DIM
    seed: int = SEED_BASE
    passages: int = 0
    passage_len: int = 0
    final_len: int = 0
    rope_theta: float = 0.0


WORKLOADS: dict[str, Workload] = {
    # 4K tokens, 2 q heads / 1 KV head, 64x64 blocks, top 25% per branch.
    "tiny_rbs_4k": Workload("tiny_rbs_4k", 4096, 2, 1, 64, "tiny", rho=0.25, seed=SEED_BASE + 0),
    # 32K tokens, 64 q / 8 KV heads, compact/dispersed key mixture, ~10% kept.
    "gqa_rbs_32k": Workload("gqa_rbs_32k", 32768, 64, 8, 128, "mixture", density_target=0.10, seed=SEED_BASE + 1),
    # 128K tokens, 32 q / 4 KV heads, same mixture, 5% per branch.
    "gqa_rbs_128k": Workload("gqa_rbs_128k", 131072, 32, 4, 128, "mixture", rho=0.05, seed=SEED_BASE + 2),
    # 16 passages x 2048 tokens + a 512-token final block, 32 q / 8 KV heads.
    "block_attention_rag_33k": Workload(
        "block_attention_rag_33k", 16 * 2048 + 512, 32, 8, 128, "block_attention",
        seed=SEED_BASE + 3, passages=16, passage_len=2048, final_len=512, rope_theta=500000.0),
    # 64K tokens, 32 q / 8 KV heads, mixture, kept density swept.
    "density_sweep_64k": Workload("density_sweep_64k", 65536, 32, 8, 128, "mixture", seed=SEED_BASE + 4),
}


def _normal_bf16(rng: np.random.Generator, shape, scale: float = 1.0, chunk_rows: int = 8192) -> np.ndarray:
    """Draw N(0, scale^2) float32 values in row chunks and round them to bf16 bits."""
    out = np.empty(shape, dtype=np.uint16)
    rows = shape[0] * shape[1]
    flat = out.reshape(rows, -1)
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        x = rng.standard_normal((r1 - r0, flat.shape[1]), dtype=np.float32)
        if scale != 1.0:
            x *= np.float32(scale)
        flat[r0:r1] = f32_to_bf16_bits(x)
    return out


def _plant(K: np.ndarray, Q: np.ndarray, b: int, kvh: int, pos_k: int, q_tok: int, q_head: int, logit: float) -> None:
    """Overwrite key ``pos_k`` with k* = (logit*sqrt(d)/|q|^2) q for the chosen query q.

    Then q . k* / sqrt(d) = logit: one isolated high-dot key for that query.
    """
    q = bf16_bits_to_f32(Q[b, q_tok, q_head]).astype(np.float64)
    d = q.shape[0]
    scale = logit * math.sqrt(d) / float(q @ q)
    K[b, pos_k, kvh] = f32_to_bf16_bits((scale * q).astype(np.float32))


def make_tied(L: int, Hq: int, Hkv: int, block: int, n_patterns: int, seed: int, batch: int = 1) -> dict:
    """Inputs whose block scores tie exactly: Q and K entries are integers in
    {-1, 0, 1} (exact in bf16), and the key blocks repeat n_patterns block
    contents (block j of each KV head takes pattern (7 j + h) % n_patterns).
    Centroids and pooled queries are then binary fractions, and blocks with
    the same content score the same, so each selection row holds about
    n / n_patterns exactly tied scores per value.  V is N(0, 1).
    """
    d = HEAD_DIM
    nb = L // block
    rng = np.random.Generator(np.random.PCG64(seed))
    Q = f32_to_bf16_bits(rng.integers(-1, 2, size=(batch, L, Hq, d)).astype(np.float32))
    pats = rng.integers(-1, 2, size=(batch, Hkv, n_patterns, block, d)).astype(np.float32)
    Kf = np.empty((batch, L, Hkv, d), dtype=np.float32)
    for b in range(batch):
        for h in range(Hkv):
            for j in range(nb):
                Kf[b, j * block:(j + 1) * block, h] = pats[b, h, (7 * j + h) % n_patterns]
    K = f32_to_bf16_bits(Kf)
    V = _normal_bf16(rng, (batch, L, Hkv, d))
    return {"Q": Q, "K": K, "V": V}


def make_tiny(L: int = 4096, Hq: int = 2, Hkv: int = 1, block: int = 64, seed: int = SEED_BASE + 0,
              batch: int = 1, offset_std: float = 0.5, plant_every: int = 16, logit: float = 8.0) -> dict:
    """Tiny RBS workload: N(0,1) Q/K/V, per-block N(0, offset_std^2) key offsets, planted keys.

    Every key block j with j % plant_every == 0 (and a later query block to
    aim at) gets one key, at a uniform position, replaced by a key aligned to
    a uniformly chosen query token of a later query block and a uniformly
    chosen q head of the KV group.
    """
    d = HEAD_DIM
    nb = L // block
    G = Hq // Hkv
    rng = np.random.Generator(np.random.PCG64(seed))
    Q = _normal_bf16(rng, (batch, L, Hq, d))
    offsets = rng.standard_normal((batch, Hkv, nb, d), dtype=np.float32) * np.float32(offset_std)
    Kf = rng.standard_normal((batch, L, Hkv, d), dtype=np.float32)
    Kf += np.repeat(offsets, block, axis=2).transpose(0, 2, 1, 3)
    K = f32_to_bf16_bits(Kf)
    del Kf
    V = _normal_bf16(rng, (batch, L, Hkv, d))
    plants = []
    for b in range(batch):
        for h in range(Hkv):
            for j in range(0, nb, plant_every):
                if j + 1 >= nb:
                    continue
                pos_k = j * block + int(rng.integers(0, block))
                qi = int(rng.integers(j + 1, nb))
                q_tok = qi * block + int(rng.integers(0, block))
                q_head = h * G + int(rng.integers(0, G))
                _plant(K, Q, b, h, pos_k, q_tok, q_head, logit)
                plants.append((b, h, j, pos_k, q_head, q_tok))
    return {"Q": Q, "K": K, "V": V, "plants": plants, "block": block}


def make_mixture(L: int, Hq: int, Hkv: int, block: int = 128, seed: int = SEED_BASE + 1, batch: int = 1,
                 centre_std: float = 0.5, compact_std: float = 0.2, dispersed_std: float = 1.5,
                 p_compact: float = 0.7, max_plants: int = 4, logit: float = 8.0) -> dict:
    """Compact/dispersed key-block mixture with planted keys in the dispersed blocks.

    Per (batch, KV head, key block): a centre mu ~ N(0, centre_std^2 I); the
    block is compact with probability p_compact (keys mu + compact_std*eps)
    and dispersed otherwise (keys mu + dispersed_std*eps).  Each dispersed
    block that has a later query block gets U{1..max_plants} planted keys,
    each aligned to a uniform query token of a uniform later query block and a
    uniform q head of the KV group.  Q and V are N(0, 1).
    """
    d = HEAD_DIM
    nb = -(-L // block)  # a last, shorter block when L is not a block multiple
    G = Hq // Hkv
    rng = np.random.Generator(np.random.PCG64(seed))
    Q = _normal_bf16(rng, (batch, L, Hq, d))
    centres = rng.standard_normal((batch, Hkv, nb, d), dtype=np.float32) * np.float32(centre_std)
    compact = rng.random((batch, Hkv, nb)) < p_compact
    sigma = np.where(compact, np.float32(compact_std), np.float32(dispersed_std)).astype(np.float32)
    K = np.empty((batch, L, Hkv, d), dtype=np.uint16)
    for b in range(batch):
        for j0 in range(0, nb, 64):
            j1 = min(nb, j0 + 64)
            eps = rng.standard_normal(((j1 - j0) * block, Hkv, d), dtype=np.float32)
            eps = eps.reshape(j1 - j0, block, Hkv, d)
            mu = centres[b, :, j0:j1].transpose(1, 0, 2)[:, None, :, :]
            sg = sigma[b, :, j0:j1].transpose(1, 0)[:, None, :, None]
            t1 = min(L, j1 * block)
            K[b, j0 * block:t1] = f32_to_bf16_bits((mu + sg * eps).reshape(-1, Hkv, d)[:t1 - j0 * block])
    V = _normal_bf16(rng, (batch, L, Hkv, d))
    plants = []
    for b in range(batch):
        for h in range(Hkv):
            for j in range(nb - 1):
                if compact[b, h, j]:
                    continue
                for _ in range(int(rng.integers(1, max_plants + 1))):
                    pos_k = j * block + int(rng.integers(0, block))
                    qi = int(rng.integers(j + 1, nb))
                    q_tok = qi * block + int(rng.integers(0, min(block, L - qi * block)))
                    q_head = h * G + int(rng.integers(0, G))
                    _plant(K, Q, b, h, pos_k, q_tok, q_head, logit)
                    plants.append((b, h, j, pos_k, q_head, q_tok))
    return {"Q": Q, "K": K, "V": V, "plants": plants, "compact": compact, "block": block}


def make_block_attention(passages: int = 16, passage_len: int = 2048, final_len: int = 512, Hq: int = 32,
                         Hkv: int = 8, block: int = 128, seed: int = SEED_BASE + 3, batch: int = 1,
                         passage_lens=None) -> dict:
    """RAG-shaped Block-attention workload: un-rotated Q/K/V ~ N(0,1) and the segment table.

    Passage p covers its own run of tokens: passage_len each, or the lengths
    in ``passage_lens`` (any token counts, not necessarily block multiples),
    one after the other; the final block (the user query) follows them.
    ``local_pos`` is each token's position inside its own passage (the
    position its cached key was encoded at); ``global_pos`` is its position
    in the assembled prompt.
    """
    d = HEAD_DIM
    lens = [int(x) for x in passage_lens] if passage_lens is not None else [passage_len] * passages
    seg_start = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int32)
    final_start = int(sum(lens))
    L = final_start + final_len
    rng = np.random.Generator(np.random.PCG64(seed))
    Q = _normal_bf16(rng, (batch, L, Hq, d))
    K = _normal_bf16(rng, (batch, L, Hkv, d))
    V = _normal_bf16(rng, (batch, L, Hkv, d))
    global_pos = np.arange(L, dtype=np.int32)
    local_pos = global_pos.copy()
    for a, n in zip(seg_start, lens):
        local_pos[a:a + n] = np.arange(n, dtype=np.int32)
    return {"Q": Q, "K": K, "V": V, "seg_start": seg_start, "final_start": final_start,
            "local_pos": local_pos, "global_pos": global_pos, "block": block}


def make_inputs(w: Workload, seqlen: int | None = None, heads_q: int | None = None,
                heads_kv: int | None = None) -> dict:
    """Inputs for a named workload, optionally at a reduced sequence length or head count."""
    L = seqlen or w.seqlen
    Hq = heads_q or w.heads_q
    Hkv = heads_kv or w.heads_kv
    if w.kind == "tiny":
        return make_tiny(L, Hq, Hkv, w.block, w.seed, w.batch)
    if w.kind == "mixture":
        return make_mixture(L, Hq, Hkv, w.block, w.seed, w.batch)
    if w.kind == "block_attention":
        return make_block_attention(w.passages, w.passage_len, w.final_len, Hq, Hkv, w.block, w.seed, w.batch)
    raise ValueError(w.kind)
