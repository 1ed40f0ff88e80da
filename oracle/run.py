"""Batch driver for the CPU oracle: takes one seeded draw from
``hierarchical_top_key_b200.synthetic`` and runs the per-query oracle over any
subset of queries.

TEST INFRASTRUCTURE ONLY (see the package docstring): used by the tests, by
``__graft_entry__.smoke()`` and by the CPU-baseline leg of ``bench.py``.
"""
from __future__ import annotations

import numpy as np

from . import hisa_oracle as ho


class Sequence:
    """The oracle's view of one sequence of a draw, in float64, with the key
    preprocessing (compression, FP8 quantisation, pooling) applied."""

    def __init__(self, inputs, b: int, fp8: bool = False):
        wl = inputs.workload
        self.workload = wl
        self.fp8 = fp8
        self.block = wl.block_size
        self.top_m = wl.top_m
        self.top_k = wl.top_k
        raw = inputs.keys[b].astype(np.float64)
        if wl.compress_ratio > 1:
            keys = ho.compress_keys(raw, wl.compress_ratio, wl.dtype)
        else:
            keys = raw
        q = inputs.q[b].astype(np.float64)                   # [Q, H, d]
        self.w = inputs.w[b].astype(np.float64)               # [Q, H]
        self.n_visible = inputs.n_visible[b].astype(np.int64)
        if fp8:
            Qn, H, d = q.shape
            qc, qs = ho.quantize_q_tokens(q)
            kc, ks = ho.quantize_e4m3_rows(keys.astype(np.float32))
            self.q_codes, self.q_scale = qc, qs
            self.k_codes, self.k_scale = kc, ks
            q = ho.dequantize_e4m3_rows(qc.reshape(Qn, H * d), qs).reshape(Qn, H, d)
            keys = ho.dequantize_e4m3_rows(kc, ks)
            pc, ps = ho.pool_blocks_e4m3(kc, ks, self.block)
            self.kpool_codes, self.kpool_scale = pc, ps
            self.kpool = ho.dequantize_e4m3_rows(pc, ps)
        else:
            self.kpool = ho.pool_blocks(keys, self.block, wl.dtype)
        self.q = q
        self.keys = keys

    def hisa(self, t: int, top_m: int | None = None, top_k: int | None = None):
        return ho.hisa_query(self.q[t], self.w[t], self.keys, self.kpool, int(self.n_visible[t]),
                             self.block, top_m or self.top_m, top_k or self.top_k)

    def flat(self, t: int, top_k: int | None = None):
        return ho.flat_query(self.q[t], self.w[t], self.keys, int(self.n_visible[t]),
                             top_k or self.top_k)

    def blocks(self, t: int, top_m: int | None = None):
        return ho.select_blocks(self.q[t], self.w[t], self.kpool, int(self.n_visible[t]),
                                self.block, top_m or self.top_m)

    def block_scores(self, t: int):
        c = ho.current_block(int(self.n_visible[t]), self.block)
        return ho.indexer_scores(self.q[t], self.w[t], self.kpool[:max(c, 0)])

    def token_stage(self, t: int, blocks, top_k: int | None = None):
        cand = ho.candidate_keys(np.asarray(blocks, np.int64), int(self.n_visible[t]), self.block)
        return ho.refine_tokens(self.q[t], self.w[t], self.keys, cand, top_k or self.top_k)

    def superblocks_pooled(self, group: int) -> np.ndarray:
        """Pooled super-blocks of `group` blocks (pooled from the keys like blocks)."""
        cache = self.__dict__.setdefault("_kpool2", {})
        if group not in cache:
            if self.fp8:
                pc, ps = ho.pool_blocks_e4m3(self.k_codes, self.k_scale, self.block * group)
                cache[group] = ho.dequantize_e4m3_rows(pc, ps)
            else:
                cache[group] = ho.pool_blocks(self.keys, self.block * group, self.workload.dtype)
        return cache[group]

    def hisa3(self, t: int, group: int, top_m2: int, top_m: int | None = None, top_k: int | None = None):
        return ho.hisa3_query(self.q[t], self.w[t], self.keys, self.kpool, self.superblocks_pooled(group),
                              int(self.n_visible[t]), self.block, group, top_m2, top_m or self.top_m,
                              top_k or self.top_k)

    def scores(self, t: int, positions) -> np.ndarray:
        """Oracle indexer score of query t at the given key positions."""
        return ho.indexer_scores(self.q[t], self.w[t], self.keys[np.asarray(positions, np.int64)])
