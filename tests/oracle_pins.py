"""Checks that pin the CPU oracle to facts outside itself: hand-worked
fixtures (tests/golden), brute-force enumeration on tiny inputs with scores
computed by explicit loops, closed forms, special cases that reduce to a
library routine, and invariants of the method.

Each check is a plain function that raises AssertionError; the pytest module
test_oracle_pins.py runs them, and test_oracle_mutations.py plants mistakes in
the oracle and verifies that some check catches each one.
"""
from __future__ import annotations

import itertools
import json
import os

import numpy as np
import torch

from oracle import hisa_oracle as ho
from oracle import ofp8
from oracle import sparse_attention as sa
from oracle.run import Sequence
from hierarchical_top_key_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- golden


def pin_golden_flat():
    g = _load("flat_relu_weights.json")
    q, w, keys = (np.array(g[k], np.float64) for k in ("q", "w", "keys"))
    np.testing.assert_array_equal(ho.indexer_scores(q, w, keys), np.array(g["scores"], np.float64))
    for c in g["cases"]:
        idx, _ = ho.flat_query(q, w, keys, c["n_visible"], c["top_k"])
        assert list(idx) == c["indices"], (c, list(idx))


def _golden_hisa(name):
    g = _load(name)
    B = g["block_size"]
    q, w, keys = (np.array(g[k], np.float64) for k in ("q", "w", "keys"))
    kp = ho.pool_blocks(keys, B, "f32")
    np.testing.assert_array_equal(kp[:, 0], np.array(g["pooled"], np.float64))
    for c in g["cases"]:
        blocks, idx, _ = ho.hisa_query(q, w, keys, kp, c["n_visible"], B, c["top_m"], c["top_k"])
        assert list(blocks) == c["blocks"], (name, c, list(blocks))
        assert list(idx) == c["indices"], (name, c, list(idx))
    for c in g.get("flat_cases", []):
        idx, _ = ho.flat_query(q, w, keys, c["n_visible"], c["top_k"])
        assert list(idx) == c["indices"], (name, c, list(idx))


def pin_golden_hisa_blocks():
    _golden_hisa("hisa_blocks_1d.json")


def pin_golden_relu_of_mean():
    _golden_hisa("hisa_relu_of_mean.json")


def pin_golden_e4m3():
    g = _load("ofp8_e4m3.json")
    xs = np.array([e["x"] for e in g["encode"]])
    codes = np.array([e["code"] for e in g["encode"]], np.uint8)
    np.testing.assert_array_equal(ofp8.e4m3_encode(xs), codes)
    dc = np.array([e["code"] for e in g["decode"]], np.uint8)
    np.testing.assert_array_equal(ofp8.e4m3_decode(dc), np.array([e["x"] for e in g["decode"]]))
    assert np.all(np.isnan(ofp8.e4m3_decode(np.array(g["nan_codes"], np.uint8))))


def pin_golden_bf16():
    g = _load("bf16_round.json")
    xs = np.array([c["x"] for c in g["cases"]], np.float64)
    np.testing.assert_array_equal(ofp8.bf16_round(xs), np.array([c["bf16"] for c in g["cases"]]))


def _f32_from_bits(hexes):
    return np.array([int(h, 16) for h in hexes], np.uint32).view(np.float32)


def pin_golden_pool_e4m3():
    """Pooled E4M3 keys: exact mean of the dequantised keys, rounded to fp32,
    re-quantised per block with the fp32 decision (hand-worked cases)."""
    g = _load("pool_e4m3.json")
    for c in g["pool_cases"]:
        codes = np.array(c["codes"], np.uint8)
        scale = _f32_from_bits(c["scale_bits"])
        pc, ps = ho.pool_blocks_e4m3(codes, scale, c["block_size"])
        np.testing.assert_array_equal(pc, np.array(c["pooled_codes"], np.uint8), err_msg=c["name"])
        np.testing.assert_array_equal(np.asarray(ps, np.float32).view(np.uint32),
                                      _f32_from_bits(c["pooled_scale_bits"]).view(np.uint32), err_msg=c["name"])


def pin_golden_q_token_scale():
    """The oracle's E4M3 view of a sequence quantises q with one scale per
    token over all heads (hand-worked case, through run.Sequence)."""
    g = _load("pool_e4m3.json")
    for c in g["q_token_cases"]:
        q = np.array(c["q"], np.float32)
        Qn, H, d = q.shape
        wl = synthetic.small_case(num_keys=4, num_queries=Qn, first_query_pos=4 - Qn, heads=H, head_dim=d,
                                  block_size=2, top_m=1, top_k=1, dtype="f32", needles=0, name="q_token_golden")
        keys = np.ones((1, 4, d), np.float32)
        pos = np.arange(4 - Qn, 4, dtype=np.int64)[None]
        inp = synthetic.Inputs(wl, q[None], keys, np.ones((1, Qn, H), np.float32), pos,
                               synthetic.visible_keys(pos, 1), np.zeros((1, 0), np.int64), np.zeros((1, 0), np.int64))
        seq = Sequence(inp, 0, fp8=True)
        np.testing.assert_array_equal(seq.q_codes, np.array(c["q_codes"], np.uint8), err_msg=c["name"])
        np.testing.assert_array_equal(np.asarray(seq.q_scale, np.float32).view(np.uint32),
                                      _f32_from_bits(c["q_scale_bits"]).view(np.uint32), err_msg=c["name"])
        # the oracle scores with the dequantised values code * token scale
        deq = ofp8.e4m3_decode(np.array(c["q_codes"], np.uint8)) * \
            _f32_from_bits(c["q_scale_bits"]).astype(np.float64)[:, None, None]
        np.testing.assert_array_equal(seq.q, deq, err_msg=c["name"])


# ---------------------------------------------------------------- library special cases


def pin_e4m3_matches_torch_in_range():
    """Inside +-448 saturation plays no part, and E4M3 round-to-nearest-even
    is what torch's float8_e4m3fn cast does."""
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1, 30, 200)])
    x = np.clip(x, -447, 447).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ofp8.e4m3_encode(x), ref)
    allc = np.arange(256, dtype=np.uint8)
    fin = ~np.isnan(ofp8.e4m3_decode(allc))
    tv = torch.from_numpy(allc).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(ofp8.e4m3_decode(allc)[fin], tv[fin])


def pin_bf16_matches_torch_on_fp32_values():
    """For values already in fp32, one bf16 rounding equals torch's cast."""
    rng = np.random.default_rng(12)
    x = (rng.standard_normal(50000) * np.exp(rng.uniform(-20, 20, 50000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(ofp8.bf16_round(x.astype(np.float64)), ref)


def _loop_scores(q, w, keys):
    """Indexer scores by explicit loops (no matrix routines)."""
    H, d = q.shape
    out = []
    for s in range(keys.shape[0]):
        tot = 0.0
        for h in range(H):
            dot = 0.0
            for i in range(d):
                dot += float(q[h, i]) * float(keys[s, i])
            tot += float(w[h]) * max(dot, 0.0)
        out.append(tot)
    return np.array(out)


def pin_single_head_unit_weight_is_sort():
    """H=1, w=1: flat top-k is a stable descending sort of ReLU(q.k)."""
    rng = np.random.default_rng(13)
    for trial in range(20):
        n, d, k = int(rng.integers(1, 40)), int(rng.integers(1, 6)), int(rng.integers(1, 12))
        q = rng.integers(-3, 4, (1, d)).astype(np.float64)
        keys = rng.integers(-3, 4, (n, d)).astype(np.float64)
        s = np.maximum(keys @ q[0], 0)
        ref = np.argsort(-s, kind="stable")[:k]
        idx, sc = ho.flat_query(q, np.ones(1), keys, n, k)
        assert list(idx) == list(ref), (trial, list(idx), list(ref))
        np.testing.assert_array_equal(sc, s[ref])


# ---------------------------------------------------------------- brute force


def _brute_topk(scores, k):
    """Best-sum k-subset; among equal sums the lexicographically smallest
    sorted index tuple (ties go to lower indices)."""
    n = len(scores)
    k = min(k, n)
    best, best_sum = None, None
    for comb in itertools.combinations(range(n), k):
        s = sum(scores[i] for i in comb)
        if best_sum is None or s > best_sum:
            best, best_sum = comb, s
    return set(best) if best is not None else set()


def pin_brute_force_flat():
    rng = np.random.default_rng(14)
    for trial in range(60):
        n = int(rng.integers(1, 13))
        H, d = int(rng.integers(1, 3)), int(rng.integers(1, 4))
        k = int(rng.integers(1, 7))
        q = rng.integers(-2, 3, (H, d)).astype(np.float64)
        w = rng.integers(0, 3, H).astype(np.float64)
        keys = rng.integers(-2, 3, (n, d)).astype(np.float64)
        nt = int(rng.integers(0, n + 1))
        ref = _loop_scores(q, w, keys)
        np.testing.assert_array_equal(ho.indexer_scores(q, w, keys), ref)
        idx, _ = ho.flat_query(q, w, keys, nt, k)
        assert set(idx.tolist()) == _brute_topk(ref[:nt], k), (trial, idx, ref[:nt])
        assert len(idx) == min(k, nt)


def pin_brute_force_hisa():
    """Enumerate the m-1 blocks before the current one and the k candidates."""
    rng = np.random.default_rng(15)
    for trial in range(60):
        B = int(rng.integers(1, 4))
        L = int(rng.integers(1, 16))
        H, d = int(rng.integers(1, 3)), int(rng.integers(1, 3))
        m, k = int(rng.integers(1, 5)), int(rng.integers(1, 6))
        q = rng.integers(-2, 3, (H, d)).astype(np.float64)
        w = rng.integers(0, 3, H).astype(np.float64)
        keys = rng.integers(-3, 4, (L, d)).astype(np.float64)
        nt = int(rng.integers(1, L + 1))
        # pooled keys by explicit loops: block sums / counts (exact for these sizes)
        nb = -(-L // B)
        kp = np.zeros((nb, d))
        for b in range(nb):
            members = list(range(b * B, min((b + 1) * B, L)))
            for i in range(d):
                kp[b, i] = sum(keys[s, i] for s in members) / len(members)
        kp = kp.astype(np.float32).astype(np.float64)
        np.testing.assert_array_equal(ho.pool_blocks(keys, B, "f32"), kp)
        c = (nt - 1) // B
        bscore = _loop_scores(q, w, kp[:c])
        if c + 1 <= m:
            want_blocks = set(range(c + 1))
        else:
            want_blocks = _brute_topk(list(bscore), m - 1) | {c}
        blocks, idx, _ = ho.hisa_query(q, w, keys, kp, nt, B, m, k)
        assert set(blocks.tolist()) == want_blocks, (trial, blocks, want_blocks)
        cand = [s for b in sorted(want_blocks) for s in range(b * B, min((b + 1) * B, nt))]
        tok = _loop_scores(q, w, keys[cand]) if cand else np.zeros(0)
        want = {cand[i] for i in _brute_topk(list(tok), k)}
        assert set(idx.tolist()) == want, (trial, idx, want)


def pin_brute_force_hisa3():
    """Three levels on tiny inputs: every choice of m2-1 super-blocks, then of
    m-1 blocks among their fully visible blocks, then of k candidates."""
    rng = np.random.default_rng(21)
    for trial in range(60):
        B, S = int(rng.integers(1, 3)), int(rng.integers(1, 4))
        L = int(rng.integers(1, 19))
        H, d = int(rng.integers(1, 3)), int(rng.integers(1, 3))
        m2, m, k = int(rng.integers(1, 4)), int(rng.integers(1, 5)), int(rng.integers(1, 6))
        q = rng.integers(-2, 3, (H, d)).astype(np.float64)
        w = rng.integers(0, 3, H).astype(np.float64)
        keys = rng.integers(-3, 4, (L, d)).astype(np.float64)
        nt = int(rng.integers(1, L + 1))

        def pooled(size):
            nb = -(-L // size)
            out = np.zeros((nb, d))
            for b in range(nb):
                members = list(range(b * size, min((b + 1) * size, L)))
                for i in range(d):
                    out[b, i] = sum(keys[s, i] for s in members) / len(members)
            return out.astype(np.float32).astype(np.float64)

        kp, kp2 = pooled(B), pooled(B * S)
        c2, c = (nt - 1) // (B * S), (nt - 1) // B
        if c2 + 1 <= m2:
            want_sb = set(range(c2 + 1))
        else:
            want_sb = _brute_topk(list(_loop_scores(q, w, kp2[:c2])), m2 - 1) | {c2}
        cands = [b for u in sorted(want_sb) for b in range(u * S, min((u + 1) * S, c))]
        if len(cands) + 1 <= m:
            want_blocks = set(cands) | {c}
        else:
            bs = _loop_scores(q, w, kp[cands])
            want_blocks = {cands[i] for i in _brute_topk(list(bs), m - 1)} | {c}
        sb, blocks, idx, _ = ho.hisa3_query(q, w, keys, kp, kp2, nt, B, S, m2, m, k)
        assert set(sb.tolist()) == want_sb, (trial, sb, want_sb)
        assert set(blocks.tolist()) == want_blocks, (trial, blocks, want_blocks)
        cand = [s for b in sorted(want_blocks) for s in range(b * B, min((b + 1) * B, nt))]
        tok = _loop_scores(q, w, keys[cand]) if cand else np.zeros(0)
        assert set(idx.tolist()) == {cand[i] for i in _brute_topk(list(tok), k)}, trial


def pin_three_levels_reduce_to_two():
    """Every super-block kept, or super-blocks of one block with m2 = m: the
    three-level indexer is HISA exactly."""
    inp = synthetic.generate(synthetic.small_case(num_keys=700, heads=3, head_dim=8, block_size=16,
                                                  top_m=5, top_k=40, needles=3))
    seq = Sequence(inp, 0)
    for t in range(0, 700, 9):
        blocks, hi, hs = seq.hisa(t)
        _, b3, i3, s3 = seq.hisa3(t, group=4, top_m2=1000)
        assert list(b3) == list(blocks) and list(i3) == list(hi), t
        np.testing.assert_array_equal(s3, hs)
        _, b1, i1, _ = seq.hisa3(t, group=1, top_m2=5)
        assert list(b1) == list(blocks) and list(i1) == list(hi), t


def pin_three_levels_structure():
    """The kept blocks lie in the kept super-blocks, the current block is kept,
    and every candidate block left out scores no higher than the kept ones."""
    inp = synthetic.generate("tiny")
    seq = Sequence(inp, 0)
    B, S = inp.workload.block_size, 2
    for t in [0, 1, 63, 64, 200, 511, 700, 1023]:
        nt = int(seq.n_visible[t])
        sb, blocks, idx, _ = seq.hisa3(t, group=S, top_m2=3, top_m=3)
        c = ho.current_block(nt, B)
        assert c in set(blocks.tolist())
        assert all(b // S in set(sb.tolist()) for b in blocks.tolist())
        cands = ho.candidate_blocks(sb, c, S)
        kept = [b for b in blocks.tolist() if b != c]
        if len(cands) + 1 > 3 and kept:
            sc = ho.indexer_scores(seq.q[t], seq.w[t], seq.kpool[cands])
            low = min(sc[list(cands).index(b)] for b in kept)
            assert all(sc[i] <= low for i, b in enumerate(cands) if b not in kept), t
        assert set(idx.tolist()) <= set(ho.candidate_keys(blocks, nt, B).tolist())


# ---------------------------------------------------------------- closed forms / special cases


def pin_pool_closed_forms():
    rng = np.random.default_rng(16)
    keys = rng.standard_normal((37, 5)).astype(np.float32).astype(np.float64)
    # block size 1: pooled keys are the keys
    np.testing.assert_array_equal(ho.pool_blocks(keys, 1, "f32"), keys)
    # arithmetic progression along the sequence: block mean = midpoint
    ap = np.arange(40, dtype=np.float64)[:, None] * np.ones((1, 3)) * 2.0
    kp = ho.pool_blocks(ap, 8, "f32")
    np.testing.assert_array_equal(kp[:, 0], np.array([7, 23, 39, 55, 71], np.float64))
    # ragged tail: block of 5 keys (35..39) has mean 74
    kp = ho.pool_blocks(ap, 7, "f32")
    assert kp[-1, 0] == 74.0 and kp.shape[0] == 6
    # compression of constant groups
    const = np.repeat(np.arange(6, dtype=np.float64), 4)[:, None] * np.ones((1, 2))
    ck = ho.compress_keys(np.concatenate([const, np.ones((3, 2)) * 99]), 4, "bf16")
    np.testing.assert_array_equal(ck[:, 0], np.arange(6, dtype=np.float64))
    # mean rounded once to bf16: (1 + (1 + 2^-7)) / 2 = 1 + 2^-8 -> tie -> 1.0
    two = np.array([[1.0], [1.0 + 2 ** -7]])
    assert ho.pool_blocks(two, 2, "bf16")[0, 0] == 1.0


def pin_m_all_blocks_equals_flat():
    inp = synthetic.generate(synthetic.small_case(num_keys=333, heads=3, head_dim=8, block_size=16,
                                                  top_m=1000, top_k=25, needles=3))
    seq = Sequence(inp, 0)
    for t in range(0, 333, 7):
        _, hi, hs = seq.hisa(t)
        fi, fs = seq.flat(t)
        assert list(hi) == list(fi), t
        np.testing.assert_array_equal(hs, fs)


def pin_m_one_is_current_block():
    inp = synthetic.generate(synthetic.small_case(num_keys=200, heads=2, head_dim=4, block_size=10,
                                                  top_m=1, top_k=50, needles=0))
    seq = Sequence(inp, 0)
    for t in (0, 9, 10, 11, 57, 199):
        nt = int(seq.n_visible[t])
        blocks, idx, _ = seq.hisa(t)
        c = (nt - 1) // 10
        assert list(blocks) == [c]
        assert sorted(idx.tolist()) == list(range(c * 10, nt))     # k >= |C_t|: all returned


def pin_large_k_returns_all_candidates():
    inp = synthetic.generate(synthetic.small_case(num_keys=256, heads=2, head_dim=4, block_size=16,
                                                  top_m=3, top_k=48, needles=0))
    seq = Sequence(inp, 0)
    for t in (5, 40, 100, 255):
        blocks, idx, _ = seq.hisa(t)
        cand = ho.candidate_keys(blocks, int(seq.n_visible[t]), 16)
        assert sorted(idx.tolist()) == cand.tolist()


def pin_scale_invariance():
    """Positive rescaling of q, k or w (by powers of two, so exactly) leaves the
    selection unchanged and scales the scores."""
    inp = synthetic.generate(synthetic.small_case(num_keys=256, heads=3, head_dim=6, block_size=16,
                                                  top_m=4, top_k=20))
    seq = Sequence(inp, 0)
    for t in (30, 128, 255):
        b0, i0, s0 = seq.hisa(t)
        q, w, k, kp, nt = seq.q[t], seq.w[t], seq.keys, seq.kpool, int(seq.n_visible[t])
        b1, i1, s1 = ho.hisa_query(q * 2, w * 0.5, k * 4, kp * 4, nt, 16, 4, 20)
        assert list(b0) == list(b1) and list(i0) == list(i1)
        np.testing.assert_array_equal(s1, s0 * 4)


def pin_all_negative_gives_lowest_indices():
    """When every head's dot product is negative all scores are 0 and ties
    resolve to the lowest indices."""
    q = np.ones((2, 3))
    keys = -np.abs(np.random.default_rng(17).standard_normal((30, 3))) - 0.1
    idx, sc = ho.flat_query(q, np.ones(2), keys, 30, 7)
    assert list(idx) == list(range(7)) and np.all(sc == 0)


def pin_quantize_rows():
    rng = np.random.default_rng(18)
    x = rng.standard_normal((50, 64)).astype(np.float32)
    codes, scale = ho.quantize_e4m3_rows(x)
    amax = np.abs(x).max(axis=1)
    np.testing.assert_array_equal(scale, (amax / np.float32(448)).astype(np.float32))
    # the largest element of each row lands on +-448 (code 0x7E or 0xFE)
    arg = np.abs(x).argmax(axis=1)
    assert np.all((codes[np.arange(50), arg] & 0x7F) == 0x7E)
    # dequantised values are within half an E4M3 step (relative 2^-4) of the input
    deq = ho.dequantize_e4m3_rows(codes, scale)
    big = np.abs(x) >= scale[:, None] * 2 ** -6
    assert np.all(np.abs(deq - x)[big] <= np.abs(x)[big] * 2 ** -4 + 1e-12)
    # an all-zero row has scale 1 and zero codes
    c0, s0 = ho.quantize_e4m3_rows(np.zeros((1, 8), np.float32))
    assert s0[0] == 1.0 and np.all(c0 == 0)


# ---------------------------------------------------------------- invariants on a workload


def pin_tiny_workload_invariants():
    inp = synthetic.generate("tiny")
    wl = inp.workload
    seq = Sequence(inp, 0)
    rng = np.random.default_rng(19)
    ts = sorted(set([0, 1, 63, 64, 65, 127, 128, 511, 1023] + rng.integers(0, 1024, 40).tolist()))
    found_needles = 0
    for t in ts:
        nt = int(seq.n_visible[t])
        blocks, hi, hs = seq.hisa(t)
        fi, fs = seq.flat(t)
        cand = ho.candidate_keys(blocks, nt, wl.block_size)
        # structure: causal, unique, exactly min(k, |C_t|) / min(k, n_t)
        assert len(set(hi.tolist())) == len(hi) == min(wl.top_k, len(cand))
        assert len(set(fi.tolist())) == len(fi) == min(wl.top_k, nt)
        assert np.all(hi < nt) and np.all(fi < nt)
        # the token stage keeps every flat winner that is a candidate
        assert set(hi.tolist()) & set(fi.tolist()) == set(cand.tolist()) & set(fi.tolist())
        # recall against flat never drops as m grows (the candidate sets nest)
        rec = [len(set(seq.hisa(t, top_m=m)[1].tolist()) & set(fi.tolist())) for m in (1, 2, 4, 8, 16)]
        assert rec == sorted(rec), (t, rec)
        # m = every block: identical to flat
        assert list(seq.hisa(t, top_m=16)[1]) == list(fi)
    for s, t in zip(inp.needle_pos[0], inp.needle_query[0]):
        fi, _ = seq.flat(int(t))
        found_needles += int(s in set(fi.tolist()))
    assert found_needles >= len(inp.needle_pos[0]) - 1, found_needles



# ---------------------------------------------------------------- attention over the selected keys


def _attn_case(seed=3, H=3, L=9, dk=5, dv=4):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((H, dk)), rng.standard_normal((L, dk)), rng.standard_normal((L, dv)),
            float(1.0 / np.sqrt(dk)))


def pin_sparse_attention_brute_force():
    """Tiny inputs by explicit loops over a Python set of positions."""
    import math
    q, k, v, scale = _attn_case()
    for row in ([4], [0, 3, 8], [8, -1, 2, 2, -1, 5], [-1, -1], list(range(9)), [9, 2, 40, -1, 8, 9]):
        o, lse = sa.sparse_attention_query(q, k, v, row, scale)
        sel = sorted({i for i in row if 0 <= i < k.shape[0]})
        for h in range(q.shape[0]):
            if not sel:
                assert lse[h] == -math.inf and not np.any(o[h])
                continue
            logits = [scale * sum(q[h, i] * k[s, i] for i in range(k.shape[1])) for s in sel]
            z = sum(math.exp(x) for x in logits)
            assert abs(lse[h] - math.log(z)) < 1e-12
            for c in range(v.shape[1]):
                want = sum(math.exp(x) / z * v[s, c] for x, s in zip(logits, sel))
                assert abs(o[h, c] - want) < 1e-12, (row, h, c)


def pin_sparse_attention_closed_forms():
    q, k, v, scale = _attn_case(seed=5)
    # one selected key: its value row, whatever the query
    o, lse = sa.sparse_attention_query(q, k, v, [6, -1, 6], scale)
    np.testing.assert_array_equal(o, np.broadcast_to(v[6], o.shape))
    np.testing.assert_allclose(lse, scale * (q @ k[6]), rtol=0, atol=1e-14)
    # a zero query weighs every selected key equally: the mean value row, lse = log |S|
    sel = [1, 4, 4, 7, -1]
    o, lse = sa.sparse_attention_query(np.zeros_like(q), k, v, sel, scale)
    np.testing.assert_allclose(o, np.broadcast_to(v[[1, 4, 7]].mean(axis=0), o.shape), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, np.log(3.0), rtol=0, atol=1e-14)
    # affine maps of the values pass through (the weights sum to one)
    o1, _ = sa.sparse_attention_query(q, k, v, [0, 2, 5, 8], scale)
    o2, _ = sa.sparse_attention_query(q, k, 3.0 * v - 2.0, [0, 2, 5, 8], scale)
    np.testing.assert_allclose(o2, 3.0 * o1 - 2.0, rtol=1e-13, atol=1e-13)


def pin_sparse_attention_dense_special_case():
    """Every key selected is plain attention: torch's scaled_dot_product_attention
    in float64 (keys and values shared by the heads), causal and not; the lse
    is scipy's logsumexp of the selected logits."""
    from scipy.special import logsumexp
    q, k, v, scale = _attn_case(seed=7, H=4, L=11, dk=6, dv=3)
    Q = k.shape[0]
    qs = np.random.default_rng(8).standard_normal((Q, q.shape[0], q.shape[1]))
    tq = torch.from_numpy(qs).permute(1, 0, 2)[None]                  # [1, H, Q, dk]
    tk = torch.from_numpy(k)[None, None].expand(1, q.shape[0], -1, -1)
    tv = torch.from_numpy(v)[None, None].expand(1, q.shape[0], -1, -1)
    for causal in (False, True):
        want = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale)
        want = want[0].permute(1, 0, 2).numpy()                        # [Q, H, dv]
        idx = np.array([[s if (s <= t or not causal) else -1 for s in range(Q)] for t in range(Q)])
        o, lse = sa.sparse_attention(qs, k, v, idx, scale)
        np.testing.assert_allclose(o, want, rtol=1e-12, atol=1e-13)
        for t in range(Q):
            n = t + 1 if causal else Q
            np.testing.assert_allclose(lse[t], logsumexp(scale * qs[t] @ k[:n].T, axis=1), rtol=1e-13, atol=1e-13)


def pin_sparse_attention_is_a_function_of_the_set():
    q, k, v, scale = _attn_case(seed=9)
    base = sa.sparse_attention_query(q, k, v, [2, 5, 7], scale)
    for row in ([7, 5, 2], [5, -1, 2, 7, 7], [-1, 2, 2, 5, -1, 7, 5]):
        got = sa.sparse_attention_query(q, k, v, row, scale)
        np.testing.assert_array_equal(got[0], base[0])
        np.testing.assert_array_equal(got[1], base[1])


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
