"""Edge cases of the indexer on the GPU against the oracle: empty and
over-long prefixes, adversarial block lists, all-equal scores, and the
largest candidate set the refinement stage takes (m * B = 16384)."""
import numpy as np
import pytest
import torch

import parity
from oracle import hisa_oracle as ho
from oracle.run import Sequence
from hierarchical_top_key_b200 import synthetic

pytestmark = pytest.mark.gpu


def _run(inp):
    from hierarchical_top_key_b200 import binding as hb
    wl = inp.workload
    dev = hb.to_device_inputs(inp)
    ix = hb.HisaIndexer(wl.block_size, wl.top_m, wl.top_k)
    idx, _, blocks = ix(dev["q"], dev["w"], dev["k"], dev["n_visible"], return_blocks=True)
    flat, _ = hb.dsa_flat_indexer_topk(dev["q"], dev["w"], dev["k"], dev["n_visible"], top_k=wl.top_k)
    hb.get_status()
    return dev, idx.cpu().numpy(), blocks.cpu().numpy(), flat.cpu().numpy()


def _check_rows(inp, idx, blocks, flat, rows):
    wl = inp.workload
    seq = Sequence(inp, 0)
    for t in rows:
        nt = int(min(max(seq.n_visible[t], 0), wl.num_keys))
        what = f"{wl.name} query {t} (n={nt})"
        ob = seq.blocks(t)
        gb = sorted(int(x) for x in blocks[0, t] if x >= 0)
        if nt == 0:
            assert gb == [] and np.all(idx[0, t] == -1) and np.all(flat[0, t] == -1), what
            continue
        c = ho.current_block(nt, wl.block_size)
        assert c in gb, what
        fc = np.arange(nt)
        parity.check_selection(flat[0, t][flat[0, t] >= 0], fc, seq.scores(t, fc), wl.top_k, what + " flat")
        if gb == sorted(ob.tolist()):
            cand = ho.candidate_keys(ob, nt, wl.block_size)
            parity.check_selection(idx[0, t][idx[0, t] >= 0], cand, seq.scores(t, cand), wl.top_k, what)


def test_empty_and_clamped_prefixes(lib):
    wl = synthetic.small_case(num_keys=1024, num_queries=64, first_query_pos=960, heads=64, head_dim=128,
                              block_size=64, top_m=4, top_k=100, dtype="bf16", needles=2, name="edge_prefix")
    inp = synthetic.generate(wl)
    nv = inp.n_visible
    nv[0, 0:4] = 0                      # nothing visible
    nv[0, 4:8] = [1, 63, 64, 65]        # one key; block edges
    nv[0, 8:12] = 5000                  # beyond the keys: clamped to L
    dev, idx, blocks, flat = _run(inp)
    # the oracle clamps the same way the kernels do
    inp.n_visible[0] = np.minimum(np.maximum(nv[0], 0), wl.num_keys)
    _check_rows(inp, idx, blocks, flat, range(16))


def test_adversarial_block_lists(lib):
    from hierarchical_top_key_b200 import binding as hb
    wl = synthetic.small_case(num_keys=1024, num_queries=16, first_query_pos=1008, heads=64, head_dim=128,
                              block_size=64, top_m=8, top_k=200, dtype="bf16", needles=2, name="edge_blocks")
    inp = synthetic.generate(wl)
    dev = hb.to_device_inputs(inp)
    seq = Sequence(inp, 0)
    rng = np.random.default_rng(4)
    lists = np.full((1, wl.num_queries, wl.top_m), -1, np.int32)
    for t in range(wl.num_queries):
        real = rng.choice(16, 4, replace=False)
        # repeats, -1 holes, indices past the last block, and the real blocks in any order
        lists[0, t] = [real[0], -1, real[1], real[0], 99, real[2], -7, real[3]]
    idx, _ = hb.hisa_token_score_topk(dev["q"], dev["w"], dev["k"], dev["n_visible"],
                                      torch.from_numpy(lists).to(dev["q"].device), block_size=wl.block_size,
                                      top_k=wl.top_k)
    hb.get_status()
    idx = idx.cpu().numpy()
    for t in range(wl.num_queries):
        nt = int(seq.n_visible[t])
        kept = np.unique([b for b in lists[0, t] if 0 <= b < 16])
        cand = ho.candidate_keys(kept, nt, wl.block_size)
        parity.check_selection(idx[0, t][idx[0, t] >= 0], cand, seq.scores(t, cand), wl.top_k, f"query {t}")


def test_all_equal_scores_pick_lowest_positions(lib):
    wl = synthetic.small_case(num_keys=512, num_queries=32, first_query_pos=480, heads=64, head_dim=128,
                              block_size=64, top_m=3, top_k=50, dtype="bf16", needles=0, name="edge_ties")
    inp = synthetic.generate(wl)
    inp.keys[:] = 0.0                   # every score is 0: ties everywhere
    dev, idx, blocks, flat = _run(inp)
    for t in range(wl.num_queries):
        nt = int(inp.n_visible[0, t])
        assert sorted(flat[0, t].tolist()) == list(range(50)), t
        c = (nt - 1) // 64
        assert sorted(int(x) for x in blocks[0, t] if x >= 0) == [0, 1, c], t
        assert sorted(idx[0, t].tolist()) == list(range(50)), t


def test_largest_candidate_set(lib):
    # top_m * B = 16384 candidates: past the tensor-core kernel's on-chip buffers,
    # served by the CUDA-core refinement kernel
    wl = synthetic.small_case(num_keys=20000, num_queries=8, first_query_pos=19992, heads=64, head_dim=128,
                              block_size=128, top_m=128, top_k=2048, dtype="bf16", needles=4, name="edge_max")
    inp = synthetic.generate(wl)
    dev, idx, blocks, flat = _run(inp)
    _check_rows(inp, idx, blocks, flat, range(8))
