"""The flat indexer's sampled-threshold entry point (scores of every 16th key set a
per-query threshold; only keys at or above it are written back and selected)
against the oracle, including queries whose estimate fails and go through the
CUDA-core rescoring fallback."""
import numpy as np
import pytest

import parity
from oracle.run import Sequence
from hierarchical_top_key_b200 import synthetic

pytestmark = pytest.mark.gpu


def _flat_vs_oracle(inp, stride_boost=None):
    from hierarchical_top_key_b200 import binding as hb
    wl = inp.workload
    if stride_boost is not None:
        # the sampled keys (every 16th) scaled up by a power of two: their scores
        # dominate, the sample's threshold sits above almost every other key and
        # fewer than k keys pass it, so every query takes the fallback
        inp.keys[:, ::16, :] *= stride_boost
    dev = hb.to_device_inputs(inp)
    idx, sc = hb.dsa_flat_indexer_topk_sampled(dev["q"], dev["w"], dev["k"], dev["n_visible"], top_k=wl.top_k,
                                               want_scores=True)
    hb.get_status()
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    swaps = 0
    for b in range(wl.batch):
        seq = Sequence(inp, b)
        for t in range(wl.num_queries):
            nt = int(seq.n_visible[t])
            cand = np.arange(nt)
            cs = seq.scores(t, cand)
            gi = idx[b, t]
            what = f"{wl.name} seq {b} query {t} (n={nt})"
            assert np.all(gi[min(wl.top_k, nt):] == -1), what
            swaps += parity.check_selection(gi[gi >= 0], cand, cs, wl.top_k, what)
            parity.check_scores(gi, sc[b, t], lambda ix: seq.scores(t, ix), parity.RTOL[wl.dtype], what + " scores")
    return swaps


def test_threshold_path_matches_oracle(lib):
    wl = synthetic.small_case(batch=2, num_keys=4096, num_queries=96, first_query_pos=4000, heads=64, head_dim=128,
                              block_size=128, top_m=4, top_k=128, dtype="bf16", needles=8, name="flat_lite")
    _flat_vs_oracle(synthetic.generate(wl))


def test_failed_estimates_take_the_fallback(lib):
    wl = synthetic.small_case(num_keys=2048, num_queries=48, first_query_pos=2000, heads=64, head_dim=128,
                              block_size=128, top_m=4, top_k=256, dtype="bf16", needles=0, name="flat_fallback")
    _flat_vs_oracle(synthetic.generate(wl), stride_boost=8.0)


def test_threshold_path_with_signed_weights(lib):
    """Head weights of both signs: many scores are negative, so the sample's
    threshold and the selected keys fall on the sign half of the ordering keys."""
    wl = synthetic.small_case(batch=2, num_keys=4096, num_queries=64, first_query_pos=4032, heads=64, head_dim=128,
                              block_size=128, top_m=4, top_k=128, dtype="bf16", needles=8, w_low=-1.0,
                              name="flat_lite_signed")
    _flat_vs_oracle(synthetic.generate(wl))
