"""Plain, slow CPU oracle for the HISA hierarchical indexer and the flat DSA
indexer it replaces.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package; the library's product
path never calls it, and it shares no code with the CUDA path.

Sources.  The method is described in the abstract of "HISA: Efficient
Hierarchical Indexing for Fine-Grained Sparse Attention" (arXiv 2603.28458),
reproduced on several of the pages: DSA's lightweight indexer scores every key
of the prefix for every query and keeps a top-k subset; HISA first scores one
pooled key per block and keeps the best blocks, then runs the original indexer
only on the keys of the kept blocks, returning for each query a set of k token
indices (the claim list of one page states that the output has the same
structure as DSA's).  Key compression by a ratio of 4 and the
rule that the [queries, heads, keys] score tensor must never be materialised
come from the abstract of "StreamIndex: Memory-Bounded Compressed Sparse
Attention via Streaming Top-k" (arXiv 2605.02568).

The pages print no formula.  The indexer score used throughout is the DSA
lightning-indexer form fixed for this library,

    I[t, s] = sum_h w[t, h] * ReLU(q[t, h, :] . k[s, :]),

and blocks are represented by the arithmetic mean of their keys.  Readings of
points the pages leave open (all are listed in the design notes):

* A query at position p sees n_t keys 0..n_t-1.  Its current block is
  c_t = (n_t - 1) // B.  Only the blocks b < c_t are fully visible; they are
  scored, and the best m-1 of them join c_t, which is always kept.  When
  c_t + 1 <= m every visible block is kept.
* Ties at the m-th or k-th boundary go to the lower index.
* When fewer than k candidates exist, all are returned and the rest of the
  row is -1.
* Pooled keys are stored in the key dtype (bf16 / fp32 rounded once from the
  exact mean; e4m3 re-quantised with a per-block absmax/448 scale).

Everything is float64 except where a stored value is rounded to its storage
format, and the FP8 quantisation decision, which is made in float32 as the
CUDA path makes it (scale = absmax/448 in fp32, x/scale in fp32, then
round-to-nearest-even to E4M3).

Parity pins live in tests/test_oracle_pins.py (brute force on tiny inputs,
hand-worked fixtures under tests/golden/, closed forms, special cases and
invariants).  Parity unpinned: nothing in the pages fixes which blocks are the
"right" ones to retain, so block-selection *quality* is reported, not pinned.
"""
from __future__ import annotations

import numpy as np

from .ofp8 import bf16_round, e4m3_decode, e4m3_encode

# ---------------------------------------------------------------------------
# scoring


def indexer_scores(q_t: np.ndarray, w_t: np.ndarray, keys: np.ndarray) -> np.ndarray:
    """Indexer score of one query against a set of keys.

    q_t [H, d], w_t [H], keys [n, d]  ->  [n] float64 with
    I[s] = sum_h w[h] * max(0, q[h] . k[s]).
    """
    q_t = np.asarray(q_t, np.float64)
    w_t = np.asarray(w_t, np.float64)
    keys = np.asarray(keys, np.float64)
    if keys.shape[0] == 0:
        return np.zeros(0, np.float64)
    logits = keys @ q_t.T                        # [n, H]
    return np.maximum(logits, 0.0) @ w_t


# ---------------------------------------------------------------------------
# selection


def top_by_score(scores: np.ndarray, count: int) -> np.ndarray:
    """Positions of the ``count`` largest scores, ordered by (score desc,
    position asc); all positions when fewer exist."""
    scores = np.asarray(scores, np.float64)
    n = scores.shape[0]
    order = np.lexsort((np.arange(n), -scores))
    return order[:min(count, n)]


# ---------------------------------------------------------------------------
# key preprocessing


def round_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round exact float64 values once to bf16 or fp32 (returned as float64)."""
    if dtype == "bf16":
        return bf16_round(x)
    if dtype == "f32":
        return np.asarray(x, np.float64).astype(np.float32).astype(np.float64)
    raise ValueError(dtype)


def block_means(keys: np.ndarray, block: int) -> np.ndarray:
    """float64 mean of each run of ``block`` consecutive keys; a partial last
    run averages only the keys it has.  keys [L, d] -> [ceil(L/block), d]."""
    keys = np.asarray(keys, np.float64)
    L = keys.shape[0]
    nb = -(-L // block)
    out = np.empty((nb, keys.shape[1]), np.float64)
    for b in range(nb):
        out[b] = keys[b * block:min((b + 1) * block, L)].mean(axis=0)
    return out


def pool_blocks(keys: np.ndarray, block: int, dtype: str) -> np.ndarray:
    """HISA's pooled block keys for bf16/fp32 keys: the mean of each
    block, rounded once to the key dtype."""
    return round_storage(block_means(keys, block), dtype)


def compress_keys(keys: np.ndarray, ratio: int, dtype: str = "bf16") -> np.ndarray:
    """Compressed keys: the mean of each ``ratio`` consecutive raw keys, rounded
    to the key dtype; a trailing incomplete group is dropped (it is not yet a
    compressed key).  keys [S, d] -> [S // ratio, d]."""
    keys = np.asarray(keys, np.float64)
    T = keys.shape[0] // ratio
    return round_storage(block_means(keys[:T * ratio], ratio), dtype)


# ---------------------------------------------------------------------------
# FP8 (E4M3) with one fp32 scale per row


def quantize_e4m3_rows(x: np.ndarray):
    """Per-row E4M3 quantisation: scale = max|x| / 448 (1 when the row is all
    zero), code = E4M3(x / scale).  The scale, the division and the decision
    are taken in float32.  x [..., n] -> (codes uint8 [..., n], scale f32 [...])."""
    x32 = np.asarray(x, np.float32)
    amax = np.max(np.abs(x32), axis=-1)
    scale = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    ratio = (x32 / scale[..., None]).astype(np.float32)
    return e4m3_encode(ratio), scale


def dequantize_e4m3_rows(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """Exact float64 value of each quantised element: code value * row scale."""
    return e4m3_decode(codes) * np.asarray(scale, np.float64)[..., None]


def quantize_q_tokens(q: np.ndarray):
    """E4M3 q with one scale per query token, taken over all H*d values of the
    token (reading R10 of the task's per-token FP8 variant).
    q [Q, H, d] -> (codes uint8 [Q, H, d], scale f32 [Q])."""
    q = np.asarray(q)
    Qn, H, d = q.shape
    codes, scale = quantize_e4m3_rows(q.reshape(Qn, H * d).astype(np.float32))
    return codes.reshape(Qn, H, d), scale


def pool_blocks_e4m3(codes: np.ndarray, scale: np.ndarray, block: int):
    """Pooled blocks for E4M3 keys: the float64 mean of the dequantised keys of
    each block, rounded to float32, then re-quantised per block."""
    means = block_means(dequantize_e4m3_rows(codes, scale), block)
    return quantize_e4m3_rows(means.astype(np.float32))


# ---------------------------------------------------------------------------
# the two indexers, one query at a time


def current_block(n_t: int, block: int) -> int:
    """Block holding the last visible key; -1 when nothing is visible."""
    return (n_t - 1) // block if n_t > 0 else -1


def select_blocks(q_t, w_t, kpool, n_t: int, block: int, top_m: int) -> np.ndarray:
    """HISA coarse stage for one query: the retained blocks, ascending."""
    c = current_block(n_t, block)
    if c < 0:
        return np.zeros(0, np.int64)
    if c + 1 <= top_m:
        return np.arange(c + 1, dtype=np.int64)
    block_scores = indexer_scores(q_t, w_t, kpool[:c])
    kept = top_by_score(block_scores, top_m - 1)
    return np.sort(np.concatenate([kept, [c]])).astype(np.int64)


def candidate_keys(blocks: np.ndarray, n_t: int, block: int) -> np.ndarray:
    """Visible key positions inside the retained blocks, ascending."""
    parts = [np.arange(b * block, min((b + 1) * block, n_t)) for b in sorted(blocks)]
    return np.concatenate(parts).astype(np.int64) if parts else np.zeros(0, np.int64)


def refine_tokens(q_t, w_t, keys, cand: np.ndarray, top_k: int):
    """HISA fine stage: original indexer on the candidates, top-k of them.
    Returns (indices, scores) in (score desc, index asc) order."""
    scores = indexer_scores(q_t, w_t, keys[cand])
    pick = top_by_score(scores, top_k)
    return cand[pick], scores[pick]


def hisa_query(q_t, w_t, keys, kpool, n_t: int, block: int, top_m: int, top_k: int):
    """Whole HISA indexer for one query -> (blocks, indices, scores)."""
    blocks = select_blocks(q_t, w_t, kpool, n_t, block, top_m)
    cand = candidate_keys(blocks, n_t, block)
    idx, sc = refine_tokens(q_t, w_t, keys, cand, top_k)
    return blocks, idx, sc


def flat_query(q_t, w_t, keys, n_t: int, top_k: int):
    """Flat DSA indexer for one query: top-k over every visible key."""
    scores = indexer_scores(q_t, w_t, keys[:n_t])
    pick = top_by_score(scores, top_k)
    return pick.astype(np.int64), scores[pick]


# ------------------------------------------------------------ three levels
#
# Coarse-to-fine over three levels ("LongCat Sparse Attention" abstract,
# Hierarchical Indexing: a coarse-to-fine scoring scheme that narrows the
# candidate set step by step), read here as HISA's coarse step applied twice:
# super-blocks of `group` blocks are pooled from the keys like blocks are, the
# current super-block plus the best of the fully visible ones are kept, the
# fully visible blocks inside them are scored with their pooled keys, and the
# current block plus the best of those go to the token stage.

def candidate_blocks(superblocks: np.ndarray, c_t: int, group: int) -> np.ndarray:
    """Fully visible blocks (b < c_t) inside the retained super-blocks, ascending."""
    parts = [np.arange(u * group, min((u + 1) * group, c_t)) for u in sorted(superblocks)]
    return np.concatenate(parts).astype(np.int64) if parts else np.zeros(0, np.int64)


def select_blocks_among(q_t, w_t, kpool, cands: np.ndarray, c_t: int, top_m: int) -> np.ndarray:
    """Second level: the current block plus the top_m-1 best candidate blocks
    (every candidate when they fit), ascending; ties go to the lower block."""
    if c_t < 0:
        return np.zeros(0, np.int64)
    if len(cands) + 1 <= top_m:
        return np.sort(np.concatenate([cands, [c_t]])).astype(np.int64)
    scores = indexer_scores(q_t, w_t, kpool[cands])
    kept = cands[top_by_score(scores, top_m - 1)]
    return np.sort(np.concatenate([kept, [c_t]])).astype(np.int64)


def hisa3_query(q_t, w_t, keys, kpool, kpool2, n_t: int, block: int, group: int, top_m2: int,
                top_m: int, top_k: int):
    """Three-level indexer for one query -> (super-blocks, blocks, indices, scores).
    kpool2 holds the pooled super-blocks (block * group keys each)."""
    sb = select_blocks(q_t, w_t, kpool2, n_t, block * group, top_m2)
    c = current_block(n_t, block)
    blocks = select_blocks_among(q_t, w_t, kpool, candidate_blocks(sb, c, group), c, top_m)
    cand = candidate_keys(blocks, n_t, block)
    idx, sc = refine_tokens(q_t, w_t, keys, cand, top_k)
    return sb, blocks, idx, sc


def pad_row(values: np.ndarray, width: int, fill) -> np.ndarray:
    out = np.full(width, fill, dtype=np.asarray(values).dtype if len(values) else np.int64)
    out[:len(values)] = values
    return out
