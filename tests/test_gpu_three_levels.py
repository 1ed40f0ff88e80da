"""The three-level indexer (pooled super-blocks -> blocks -> tokens) on the GPU
against the oracle: super-block sets, block sets given the oracle's
super-blocks, and token sets given the oracle's blocks, under the same
tolerance rule as the two-level indexer."""
import numpy as np
import pytest

import parity
from oracle import hisa_oracle as ho
from oracle.run import Sequence
from hierarchical_top_key_b200 import synthetic

pytestmark = pytest.mark.gpu


def _check(inp, group, top_m2, queries=None, seqs=None):
    from hierarchical_top_key_b200 import binding as hb
    wl = inp.workload
    B = wl.block_size
    dev = hb.to_device_inputs(inp)
    ix = hb.HisaIndexer3(B, group, top_m2, wl.top_m, wl.top_k)
    idx, sb, blocks = ix(dev["q"], dev["w"], dev["k"], dev["n_visible"], return_blocks=True)
    hb.get_status()
    idx, sb, blocks = idx.cpu().numpy(), sb.cpu().numpy(), blocks.cpu().numpy()
    n_cmp = 0
    for b in (range(wl.batch) if seqs is None else seqs):
        seq = Sequence(inp, b)
        kp2 = seq.superblocks_pooled(group)
        for t in (range(wl.num_queries) if queries is None else queries):
            nt = int(seq.n_visible[t])
            what = f"{wl.name} seq {b} query {t} (n={nt})"
            o_sb, o_blocks, o_idx, _ = seq.hisa3(t, group, top_m2)
            # level 1: the coarse stage over pooled super-blocks
            g_sb = [int(x) for x in sb[b, t] if x >= 0]
            c2 = ho.current_block(nt, B * group)
            if c2 >= 0:
                assert c2 in g_sb, what
                parity.check_selection([x for x in g_sb if x != c2], np.arange(c2),
                                       ho.indexer_scores(seq.q[t], seq.w[t], kp2[:c2]), top_m2 - 1, what + " sb")
            # level 2, when both sides kept the same super-blocks
            g_bl = [int(x) for x in blocks[b, t] if x >= 0]
            c = ho.current_block(nt, B)
            if c >= 0:
                assert g_bl[0] == c, what
            if sorted(g_sb) == sorted(o_sb.tolist()):
                cands = ho.candidate_blocks(o_sb, c, group)
                assert set(g_bl) - {c} <= set(cands.tolist()), what
                if len(cands):
                    parity.check_selection([x for x in g_bl if x != c], cands,
                                           ho.indexer_scores(seq.q[t], seq.w[t], seq.kpool[cands]), wl.top_m - 1,
                                           what + " blocks")
                n_cmp += 1
            # level 3, when both sides kept the same blocks
            if sorted(g_bl) == sorted(o_blocks.tolist()):
                cand = ho.candidate_keys(o_blocks, nt, B)
                gi = idx[b, t]
                assert np.all(gi[min(wl.top_k, len(cand)):] == -1), what
                parity.check_selection(gi[gi >= 0], cand, seq.scores(t, cand) if len(cand) else np.zeros(0),
                                       wl.top_k, what + " tokens")
    assert n_cmp > 0


@pytest.mark.parametrize("group", [16, 4])
def test_three_levels_small(lib, group):
    # group 16 runs level two on the tensor-core refinement kernel, group 4 on the CUDA-core one
    wl = synthetic.small_case(num_keys=4096, num_queries=400, first_query_pos=3696, heads=64, head_dim=128,
                              block_size=64, top_m=6, top_k=100, dtype="bf16", needles=6, name=f"three_g{group}")
    _check(synthetic.generate(wl), group, top_m2=3)


def test_three_levels_early_queries(lib):
    # queries near the start: a single super-block, fewer candidates than m
    wl = synthetic.small_case(num_keys=2048, heads=64, head_dim=128, block_size=64, top_m=6, top_k=64,
                              dtype="bf16", needles=4, name="three_early")
    _check(synthetic.generate(wl), 16, top_m2=2, queries=list(range(0, 2048, 37)) + [2047])


def test_three_levels_decode_128k_sampled(lib):
    inp = synthetic.generate("decode_128k")
    _check(inp, 16, top_m2=8, seqs=[0, 31, 63])
