"""Refinement and flat selection when a few keys score far above the rest:
the linear bins of the counting-scan selectors then crowd most candidates
into a few bins, and the selectors must still return the exact top-k."""
import numpy as np
import pytest

import parity
from oracle import hisa_oracle as ho
from oracle.run import Sequence
from hierarchical_top_key_b200 import synthetic

pytestmark = pytest.mark.gpu


def test_outlier_keys(lib):
    from hierarchical_top_key_b200 import binding as hb
    wl = synthetic.small_case(num_keys=4096, num_queries=256, first_query_pos=3840, heads=64, head_dim=128,
                              block_size=64, top_m=16, top_k=256, dtype="bf16", needles=0, name="outliers")
    inp = synthetic.generate(wl)
    rng = np.random.default_rng(5)
    hot = rng.choice(4096, 40, replace=False)
    inp.keys[0, hot, :] *= 64.0            # a power of two: exact in bf16
    dev = hb.to_device_inputs(inp)
    ix = hb.HisaIndexer(wl.block_size, wl.top_m, wl.top_k)
    _, _, blocks = ix(dev["q"], dev["w"], dev["k"], dev["n_visible"], return_blocks=True)
    seq = Sequence(inp, 0)
    # the refinement stage on the oracle's blocks, so every query is checked
    ob = np.full((1, wl.num_queries, wl.top_m), -1, np.int32)
    for t in range(wl.num_queries):
        b = seq.blocks(t)
        ob[0, t, :len(b)] = b
    import torch
    tok, tok_sc = hb.hisa_token_score_topk(dev["q"], dev["w"], dev["k"], dev["n_visible"],
                                           torch.from_numpy(ob).to(dev["q"].device), block_size=wl.block_size,
                                           top_k=wl.top_k, want_scores=True)
    flat, _ = hb.dsa_flat_indexer_topk(dev["q"], dev["w"], dev["k"], dev["n_visible"], top_k=wl.top_k)
    hb.get_status()
    tok, tok_sc, flat = tok.cpu().numpy(), tok_sc.cpu().numpy(), flat.cpu().numpy()
    hot_hit = 0
    for t in range(wl.num_queries):
        nt = int(seq.n_visible[t])
        cand = ho.candidate_keys(seq.blocks(t), nt, wl.block_size)
        cs = seq.scores(t, cand)
        hot_hit += int(len(set(hot.tolist()) & set(cand.tolist())) > 0)
        parity.check_selection(tok[0, t][tok[0, t] >= 0], cand, cs, wl.top_k, f"outliers query {t} tokens")
        parity.check_scores(tok[0, t], tok_sc[0, t], lambda ix: seq.scores(t, ix), parity.RTOL["bf16"],
                            f"outliers query {t} scores")
        fc = np.arange(nt)
        parity.check_selection(flat[0, t][flat[0, t] >= 0], fc, seq.scores(t, fc), wl.top_k,
                               f"outliers query {t} flat")
    assert hot_hit > wl.num_queries // 2    # the outliers really are among most queries' candidates
