"""Attention over the selected keys (hisa_sparse_attention) against the CPU
oracle (oracle/sparse_attention.py) on the same inputs, element by element.

Tolerance, from the arithmetic: logits are exact bf16 products summed in
fp32; the softmax weights are rounded to bf16 before they multiply the values
(relative error 2^-9 each, so at most 2^-9 * max|v| on an output element) and
the output is stored in bf16 (2^-9 relative).  The test allows twice that:
|o - o_ref| <= 2^-8 * (|o_ref| + max|v|), and 2e-4 absolute on lse (fp32
log-sum-exp of O(10))."""
import numpy as np
import pytest
import torch

from oracle import sparse_attention as sa
from hierarchical_top_key_b200 import synthetic

pytestmark = pytest.mark.gpu

RT = 2.0 ** -8


def _check(q, kv, idx, o, lse, rows, what):
    """q [Q, H, dqk], kv [L, dqk] (float32 holding bf16), idx [Q, k]; o, lse from the GPU."""
    for t in rows:
        ro, rl = sa.sparse_attention_query(q[t], kv, kv[:, :synthetic.ATTN_DV], idx[t], synthetic.ATTN_SCALE)
        sel = sa.selected_positions(idx[t], kv.shape[0])
        if sel.size == 0:
            assert np.all(o[t] == 0) and np.all(np.isneginf(lse[t])), f"{what} query {t}: empty set"
            continue
        vmax = np.abs(kv[sel, :synthetic.ATTN_DV]).max()
        err = np.abs(o[t].astype(np.float64) - ro)
        bad = err > RT * (np.abs(ro) + vmax)
        assert not bad.any(), f"{what} query {t}: o off at {np.argwhere(bad)[:4].tolist()}, max err {err.max():.3g}"
        np.testing.assert_allclose(lse[t], rl, rtol=0, atol=2e-4, err_msg=f"{what} query {t}: lse")


def _run(q, kv, idx):
    from hierarchical_top_key_b200 import binding as hb
    dq = torch.from_numpy(q).cuda().to(torch.bfloat16)
    dkv = torch.from_numpy(kv).cuda().to(torch.bfloat16)
    didx = torch.from_numpy(idx).cuda()
    o, lse = hb.hisa_sparse_attention(dq, dkv, didx, scale=synthetic.ATTN_SCALE)
    hb.get_status()
    return o.float().cpu().numpy(), lse.cpu().numpy()


def test_small_with_padding_repeats_and_empty_rows(lib):
    B, Q, L, K = 2, 12, 3000, 300
    q, kv = synthetic.attention_inputs(B, Q, L, seed=5)
    nv = np.full((B, Q), L)
    nv[0, 3] = 40                                   # fewer positions than k: -1 padding
    idx = synthetic.random_index_rows(B, Q, L, K, nv, seed=5)
    idx[0, 5] = -1                                  # empty set
    idx[1, 2, 100:200] = idx[1, 2, :100]            # repeats count once
    idx[1, 4, ::3] = L + 7                          # out-of-range entries are dropped
    idx[1, 6, :] = 17                               # one key repeated: a single position
    o, lse = _run(q, kv, idx)
    for b in range(B):
        _check(q[b], kv[b], idx[b], o[b], lse[b], range(Q), f"small seq {b}")


@pytest.mark.parametrize("k", [64, 65, 2048, 4096])
def test_tile_tails(lib, k):
    """Index rows whose length is and is not a whole number of 64-key tiles."""
    Q, L = 6, 5000
    q, kv = synthetic.attention_inputs(1, Q, L, seed=k)
    idx = synthetic.random_index_rows(1, Q, L, k, np.full((1, Q), L), seed=k)
    o, lse = _run(q, kv, idx)
    _check(q[0], kv[0], idx[0], o[0], lse[0], range(Q), f"k={k}")


def test_prefill_32k_shape(lib):
    """The 32K-prefill shape: 32768 key rows, k = 2048 causal positions per
    query, 64 queries spread over the sequence (early ones padded)."""
    Q, L, K = 64, 32768, 2048
    q, kv = synthetic.attention_inputs(1, Q, L, seed=11)
    pos = np.sort(np.random.default_rng(11).choice(L, Q, replace=False))
    pos[:4] = [0, 5, 700, 2047]
    idx = synthetic.random_index_rows(1, Q, L, K, (pos + 1)[None], seed=11)
    o, lse = _run(q, kv, idx)
    _check(q[0], kv[0], idx[0], o[0], lse[0], range(Q), "prefill_32k shape")


def test_consumes_the_indexer_output(lib):
    """The drop-in interface: HISA's topk_idx goes straight into the attention."""
    from hierarchical_top_key_b200 import binding as hb
    wl = synthetic.small_case(num_keys=3000, num_queries=24, first_query_pos=2976, heads=64, head_dim=128,
                              block_size=64, top_m=8, top_k=256, dtype="bf16", needles=4, name="attn_chain")
    d = hb.to_device_inputs(synthetic.generate(wl))
    idx, _ = hb.HisaIndexer(wl.block_size, wl.top_m, wl.top_k)(d["q"], d["w"], d["k"], d["n_visible"])
    q, kv = synthetic.attention_inputs(1, wl.num_queries, wl.num_keys, seed=3)
    hidx = idx.cpu().numpy()
    o, lse = _run(q, kv, hidx)
    _check(q[0], kv[0], hidx[0], o[0], lse[0], range(wl.num_queries), "indexer -> attention")


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def test_output_rescaled_when_the_maximum_jumps(lib):
    """The online softmax moves its reference maximum only when a tile's
    maximum exceeds it by more than 8 (log2 units), and then rescales the
    output rows.  With i.i.d. N(0, 1) rows that never happens after the first
    tile, so here keys aligned with each query's mean head direction are
    planted at chosen places of its index row (tiles 2, 9 and 20), each
    raising the maximum by some tens; a few heads are anti-aligned and keep
    their reference, so rows of one warp rescale and others do not."""
    Q, L, K = 6, 4096, 2048
    q, kv = synthetic.attention_inputs(1, Q, L, seed=21)
    idx = synthetic.random_index_rows(1, Q, L, K, np.full((1, Q), L), seed=21)
    used = set()
    for t in range(Q):
        u = q[0, t].astype(np.float64).sum(axis=0)
        u /= np.linalg.norm(u)
        for place, c in ((2 * 64 + 7, 120.0), (9 * 64 + 33, 240.0), (20 * 64 + 63, 360.0)):
            pos = int(idx[0, t, place])
            if pos in used:
                continue
            used.add(pos)
            kv[0, pos] = _bf16(c * u)
    o, lse = _run(q, kv, idx)
    _check(q[0], kv[0], idx[0], o[0], lse[0], range(Q), "planted maxima")
    # the planted keys do dominate: lse far above what unplanted rows give
    assert np.median(lse[0]) > 30.0


def test_two_head_slices(lib):
    """256 query heads: two 128-head slices, each its own pair of CTAs."""
    Q, L, K = 5, 3000, 500
    q, kv = synthetic.attention_inputs(1, Q, L, seed=8, heads=256)
    idx = synthetic.random_index_rows(1, Q, L, K, np.full((1, Q), L), seed=8)
    o, lse = _run(q, kv, idx)
    assert o.shape == (1, Q, 256, synthetic.ATTN_DV) and lse.shape == (1, Q, 256)
    _check(q[0], kv[0], idx[0], o[0], lse[0], range(Q), "256 heads")
