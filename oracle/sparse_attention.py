"""Plain, slow CPU oracle for the consumer of the indexer's output: attention
restricted to each query's selected keys.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package; the library's product
path never calls it, and it shares no code with the CUDA path.

Sources.  The abstract of "HISA: Efficient Hierarchical Indexing for
Fine-Grained Sparse Attention" (arXiv 2603.28458) says DSA computes attention
only over the subset its indexer selects, and that HISA keeps the token-level
top-k index interface that the downstream Sparse MLA operator consumes.  The
pages give no formula for that operator.  The reading used here is the plain
one: softmax attention of each query head over the selected keys only,

    logit[h, j] = scale * q[t, h, :] . k[s_j, :]
    p[h, j]     = exp(logit[h, j]) / sum_j' exp(logit[h, j'])
    o[t, h, :]  = sum_j p[h, j] * v[s_j, :]
    lse[t, h]   = log sum_j exp(logit[h, j])

with one key and one value row per position shared by all heads (latent
attention keeps one compressed KV row per token for every head; a value row
may be a prefix of the key row).  The selected set is the index row with -1
entries, entries that name no key (outside 0..L-1) and repeats removed: the
indexer returns a set of key positions.  An empty set gives o = 0 and
lse = -inf.  Everything is float64.
"""
from __future__ import annotations

import numpy as np


def selected_positions(idx_row, num_keys=None) -> np.ndarray:
    """The set a row of indexer output denotes: -1 padding (and, given the key
    count, entries at or past it) dropped, repeats counted once, ascending."""
    r = np.asarray(idx_row, np.int64)
    keep = r >= 0
    if num_keys is not None:
        keep &= r < num_keys
    return np.unique(r[keep])


def sparse_attention_query(q_t: np.ndarray, keys: np.ndarray, values: np.ndarray, idx_row,
                           scale: float):
    """One query: q_t [H, dk], keys [L, dk], values [L, dv], idx_row [k] int.
    Returns (o [H, dv], lse [H])."""
    q_t = np.asarray(q_t, np.float64)
    s = selected_positions(idx_row, np.asarray(keys).shape[0])
    H = q_t.shape[0]
    dv = values.shape[1]
    if s.size == 0:
        return np.zeros((H, dv)), np.full(H, -np.inf)
    ks = np.asarray(keys, np.float64)[s]                 # [n, dk]
    vs = np.asarray(values, np.float64)[s]               # [n, dv]
    logits = scale * (q_t @ ks.T)                        # [H, n]
    m = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - m)
    z = e.sum(axis=1, keepdims=True)
    o = (e / z) @ vs
    lse = (m + np.log(z))[:, 0]
    return o, lse


def sparse_attention(q: np.ndarray, keys: np.ndarray, values: np.ndarray, idx: np.ndarray, scale: float):
    """All queries of one sequence: q [Q, H, dk], idx [Q, k] -> (o [Q, H, dv], lse [Q, H])."""
    Q, H = q.shape[:2]
    o = np.zeros((Q, H, values.shape[1]))
    lse = np.zeros((Q, H))
    for t in range(Q):
        o[t], lse[t] = sparse_attention_query(q[t], keys, values, idx[t], scale)
    return o, lse
