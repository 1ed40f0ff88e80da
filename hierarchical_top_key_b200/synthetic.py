"""Seeded synthetic inputs for the HISA / DSA indexer workloads.

This module only draws random numbers and lays them out; it holds none of the
indexer's arithmetic.  Both the CUDA path (through ``bench.py`` and the tests)
and the CPU oracle take their inputs from here, so the two sides always score
the same stored values.

The shapes and value distributions follow the five workloads the HISA and
StreamIndex pages benchmark on (DeepSeek-V3.2 / GLM-5 / V4-shaped indexers):

* ``tiny``        1 x 1024 keys, all 1024 causal queries, H=4, d=64, fp32.
* ``prefill_32k`` 1 x 32768 keys, all 32768 causal queries, H=64, d=128, bf16.
* ``chunk_64k``   65536-key prefix, 4096 queries at positions 61440..65535.
* ``decode_128k`` 64 sequences x 131072 keys, one query at the last position.
* ``compressed_256k`` 262144 raw keys (later compressed 4:1 by the method to
  65536), 8192 queries at the tail.

Recipe (the pages print no data, so every real activation is replaced by):

* q[t,h,:] i.i.d. N(0, sigma^2) across t, h and the feature dimension.
* keys: an AR(1) chain along the sequence, independently per feature,
  k_0 = e_0, k_s = rho*k_{s-1} + sqrt(1-rho^2)*e_s with e ~ N(0,1), times sigma.
* w[t,h] ~ U(0,1) * w_scale, kept in fp32 (U(w_low,1) * w_scale for the test
  cases with head weights of both signs).
* needles: distinct uniform key positions s; for each, a query t is drawn
  uniformly among those that can see s, and k[s] := q[t, 0, :] (the stored,
  already-rounded value), so the key is an exact copy of a query head.
* every stored value is rounded once to the storage dtype (bf16 round to
  nearest even through torch's CPU cast; fp32 kept as drawn).

Random streams: ``numpy.random.SeedSequence(seed).spawn`` gives independent
streams for q, keys, w and needles (and one set per sequence when batch > 1).
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import math
import os
from typing import Optional

import numpy as np
import scipy.signal
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_keys: int          # keys per sequence the indexer sees (after compression)
    num_queries: int       # queries per sequence
    heads: int
    head_dim: int
    block_size: int
    top_m: int
    top_k: int
    dtype: str             # "f32" or "bf16": storage dtype of q and k
    rho: float
    sigma: float
    w_scale: float
    needles: int           # per sequence
    first_query_pos: int   # position of query 0; queries occupy consecutive positions
    compress_ratio: int = 1
    raw_keys: int = 0      # keys before compression (== num_keys when ratio is 1)
    description: str = ""
    w_low: float = 0.0     # w ~ U(w_low, 1) * w_scale; below 0 the head weights take both signs

    @property
    def num_blocks(self) -> int:
        return -(-self.num_keys // self.block_size)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _c1_recipe():
    return dict(rho=0.9, sigma=1.0, w_scale=1.0)


WORKLOADS = {
    "tiny": Workload(
        "tiny", batch=1, num_keys=1024, num_queries=1024, heads=4, head_dim=64,
        block_size=64, top_m=4, top_k=128, dtype="f32", needles=8, first_query_pos=0,
        raw_keys=1024, description="1x1024 causal, H=4 d=64 fp32, B=64 m=4 k=128",
        **_c1_recipe()),
    "prefill_32k": Workload(
        "prefill_32k", batch=1, num_keys=32768, num_queries=32768, heads=64, head_dim=128,
        block_size=128, top_m=32, top_k=2048, dtype="bf16", rho=0.95,
        sigma=1.0 / math.sqrt(128.0), w_scale=1.0 / 64.0, needles=64, first_query_pos=0,
        raw_keys=32768, description="1x32768 causal prefill, H=64 d=128 bf16, B=128 m=32 k=2048"),
    "chunk_64k": Workload(
        "chunk_64k", batch=1, num_keys=65536, num_queries=4096, heads=64, head_dim=128,
        block_size=128, top_m=64, top_k=2048, dtype="bf16", needles=8,
        first_query_pos=61440, raw_keys=65536,
        description="65536-key prefix, 4096 queries at 61440..65535, H=64 d=128 bf16, B=128 m=64 k=2048",
        **_c1_recipe()),
    "decode_128k": Workload(
        "decode_128k", batch=64, num_keys=131072, num_queries=1, heads=64, head_dim=128,
        block_size=128, top_m=64, top_k=2048, dtype="bf16", needles=256,
        first_query_pos=131071, raw_keys=131072,
        description="64 sequences x 131072 keys, 1 query at the last position, H=64 d=128 bf16, B=128 m=64 k=2048",
        **_c1_recipe()),
    "compressed_256k": Workload(
        "compressed_256k", batch=1, num_keys=65536, num_queries=8192, heads=64, head_dim=128,
        block_size=64, top_m=64, top_k=1024, dtype="bf16", needles=0,
        first_query_pos=262144 - 8192, compress_ratio=4, raw_keys=262144,
        description="262144 raw keys -> 65536 (mean of 4), 8192 tail queries, H=64 d=128 bf16, B=64 m=64 k=1024",
        **_c1_recipe()),
}


@dataclasses.dataclass
class Inputs:
    """One seeded draw.  Float arrays are float32 holding values exactly
    representable in ``workload.dtype``; ``keys`` are the raw (uncompressed)
    keys, shape [batch, raw_keys, d]."""
    workload: Workload
    q: np.ndarray            # [batch, Q, H, d] float32
    keys: np.ndarray         # [batch, raw_keys, d] float32
    w: np.ndarray            # [batch, Q, H] float32
    positions: np.ndarray    # [batch, Q] int64 token position of each query
    n_visible: np.ndarray    # [batch, Q] int32 keys (after compression) visible to each query
    needle_pos: np.ndarray   # [batch, needles] int64 key positions that were overwritten
    needle_query: np.ndarray  # [batch, needles] int64 query index the needle copies


def round_to_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float data once to the storage dtype and return it as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "f32":
        return x
    if dtype == "bf16":
        return torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    raise ValueError(f"unknown storage dtype {dtype!r}")


def visible_keys(positions: np.ndarray, ratio: int) -> np.ndarray:
    """Keys a query at token position p may see: the p+1 raw keys of its prefix,
    or, after r:1 compression, the floor((p+1)/r) complete compressed keys."""
    return ((positions + 1) // ratio).astype(np.int32)


def _ar1_keys(rng: np.random.Generator, n: int, d: int, rho: float, sigma: float) -> np.ndarray:
    e = rng.standard_normal((d, n), dtype=np.float32).astype(np.float64)
    c = math.sqrt(1.0 - rho * rho)
    e[:, 0] /= c                    # so that k_0 = e_0 exactly (stationary start)
    y = scipy.signal.lfilter([c], [1.0, -rho], e, axis=1)
    return np.ascontiguousarray((y * sigma).T, dtype=np.float32)


def generate(workload: Workload | str, seed: int = 0, *, batch: Optional[int] = None) -> Inputs:
    """Draw the inputs of ``workload`` from ``seed``.  ``batch`` may lower the
    number of sequences (each sequence has its own random streams, so sequence
    i is the same whatever the batch)."""
    wl = WORKLOADS[workload] if isinstance(workload, str) else workload
    nb = wl.batch if batch is None else batch
    Q, H, d = wl.num_queries, wl.heads, wl.head_dim
    raw = wl.raw_keys if wl.raw_keys else wl.num_keys
    q = np.empty((nb, Q, H, d), np.float32)
    keys = np.empty((nb, raw, d), np.float32)
    w = np.empty((nb, Q, H), np.float32)
    positions = np.empty((nb, Q), np.int64)
    needle_pos = np.zeros((nb, wl.needles), np.int64)
    needle_query = np.zeros((nb, wl.needles), np.int64)
    root = np.random.SeedSequence(seed)
    seq_streams = root.spawn(wl.batch)

    def draw(b):
        # every value of sequence b comes from its own four streams, so the
        # sequences can be drawn in any order, or at the same time
        sq, sk, sw, sn = (np.random.default_rng(s) for s in seq_streams[b].spawn(4))
        qb = sq.standard_normal((Q, H, d), dtype=np.float32) * np.float32(wl.sigma)
        q[b] = round_to_storage(qb, wl.dtype)
        keys[b] = round_to_storage(_ar1_keys(sk, raw, d, wl.rho, wl.sigma), wl.dtype)
        u = sw.random((Q, H), dtype=np.float32)
        if wl.w_low:
            u = u * np.float32(1.0 - wl.w_low) + np.float32(wl.w_low)
        w[b] = (u * np.float32(wl.w_scale)).astype(np.float32)
        positions[b] = wl.first_query_pos + np.arange(Q, dtype=np.int64)
        if wl.needles:
            # a needle at raw position s is seen by queries whose prefix covers s
            s = sn.choice(raw, size=wl.needles, replace=False)
            s.sort()
            for j, sj in enumerate(s):
                eligible = np.nonzero(positions[b] >= sj)[0]
                t = eligible[sn.integers(len(eligible))]
                keys[b, sj] = q[b, t, 0]
                needle_pos[b, j] = sj
                needle_query[b, j] = t

    if nb > 1:
        with concurrent.futures.ThreadPoolExecutor(min(nb, os.cpu_count() or 1, 16)) as ex:
            list(ex.map(draw, range(nb)))
    else:
        for b in range(nb):
            draw(b)
    n_visible = visible_keys(positions, wl.compress_ratio)
    return Inputs(wl, q, keys, w, positions, n_visible, needle_pos, needle_query)


def small_case(*, batch=1, num_keys=300, num_queries=None, heads=4, head_dim=64,
               block_size=64, top_m=3, top_k=40, dtype="f32", first_query_pos=0,
               needles=4, rho=0.9, sigma=1.0, w_scale=1.0, compress_ratio=1,
               name="small", w_low=0.0) -> Workload:
    """A custom workload for tests (ragged sizes, odd shapes)."""
    raw = num_keys * compress_ratio
    if num_queries is None:
        num_queries = raw - first_query_pos
    return Workload(name, batch=batch, num_keys=num_keys, num_queries=num_queries,
                    heads=heads, head_dim=head_dim, block_size=block_size, top_m=top_m,
                    top_k=top_k, dtype=dtype, rho=rho, sigma=sigma, w_scale=w_scale,
                    needles=needles, first_query_pos=first_query_pos,
                    compress_ratio=compress_ratio, raw_keys=raw, w_low=w_low)


# ---------------------------------------------------------------- attention inputs
#
# The consumer of the indexer's output (attention over the selected keys) in
# latent form: one row of ATTN_DQK features per key position shared by every
# head (ATTN_DV latent features, which are also the value, then positional
# ones), and ATTN_HEADS query heads.  The pages give no dimensions for it; these
# are those of DeepSeek-V3.2's absorbed sparse MLA.  q and the rows are i.i.d.
# N(0, 1) rounded to bf16; the softmax scale is ATTN_SCALE.

ATTN_HEADS, ATTN_DQK, ATTN_DV = 128, 576, 512
ATTN_SCALE = 1.0 / math.sqrt(192.0)


def attention_inputs(batch: int, num_queries: int, num_keys: int, seed: int = 0, heads: int = ATTN_HEADS):
    """(q [batch, Q, heads, ATTN_DQK], kv [batch, L, ATTN_DQK]) as float32 arrays
    holding bf16 values, from two streams of SeedSequence(seed)."""
    sq, sk = (np.random.default_rng(s) for s in np.random.SeedSequence(seed).spawn(2))
    q = round_to_storage(sq.standard_normal((batch, num_queries, heads, ATTN_DQK), dtype=np.float32), "bf16")
    kv = round_to_storage(sk.standard_normal((batch, num_keys, ATTN_DQK), dtype=np.float32), "bf16")
    return q, kv


def attention_inputs_cuda(batch: int, num_queries: int, num_keys: int, seed: int = 0, heads: int = ATTN_HEADS,
                          device="cuda"):
    """The same distribution drawn directly on the GPU with torch's generator
    (a different draw from attention_inputs; for timing workloads too large to
    draw on the host): (q, kv) bf16 device tensors."""
    g = torch.Generator(device=device).manual_seed(seed)
    q = torch.randn((batch, num_queries, heads, ATTN_DQK), generator=g, device=device,
                    dtype=torch.float32).to(torch.bfloat16)
    kv = torch.randn((batch, num_keys, ATTN_DQK), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    return q, kv


def random_index_rows(batch: int, num_queries: int, num_keys: int, top_k: int, n_visible: np.ndarray,
                      seed: int = 0) -> np.ndarray:
    """Index rows shaped like an indexer's output: for query (b, t) min(top_k,
    n_visible[b, t]) distinct positions below n_visible[b, t] in random order,
    then -1 padding.  [batch, Q, top_k] int32."""
    rng = np.random.default_rng(np.random.SeedSequence(seed).spawn(3)[2])
    out = np.full((batch, num_queries, top_k), -1, np.int32)
    for b in range(batch):
        for t in range(num_queries):
            n = int(min(n_visible[b, t], num_keys))
            c = min(top_k, n)
            if c:
                out[b, t, :c] = rng.choice(n, size=c, replace=False)
    return out
