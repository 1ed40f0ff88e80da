"""Scored output order: with a score output every entry point returns each
row sorted by (score desc, index asc), padding last, and the same index set
as without scores (the ScienceToStartup claim list: the output is a
per-query set of k token indices; the order is the one that defines the
top-k)."""
import numpy as np
import pytest
import torch

from hierarchical_top_key_b200 import synthetic

pytestmark = pytest.mark.gpu


def _assert_sorted(idx, sc, unscored, what):
    idx, sc, unscored = idx.cpu().numpy(), sc.cpu().numpy(), unscored.cpu().numpy()
    rows = idx.reshape(-1, idx.shape[-1])
    srows = sc.reshape(-1, idx.shape[-1])
    urows = unscored.reshape(-1, idx.shape[-1])
    for r in range(rows.shape[0]):
        i, s = rows[r], srows[r]
        n = int(np.sum(i >= 0))
        assert np.all(i[n:] == -1) and np.all(np.isneginf(s[n:])), f"{what} row {r}: padding not last"
        assert np.all(i[:n] >= 0)
        d = np.diff(s[:n].astype(np.float64))
        assert np.all(d <= 0), f"{what} row {r}: scores not descending"
        ties = d == 0
        assert np.all(np.diff(i[:n])[ties] > 0), f"{what} row {r}: equal scores not in index order"
        assert sorted(i[:n].tolist()) == sorted(x for x in urows[r].tolist() if x >= 0), f"{what} row {r}: set"


def _dev(wl):
    from hierarchical_top_key_b200 import binding as hb
    return hb.to_device_inputs(synthetic.generate(wl))


@pytest.mark.parametrize("case", [
    dict(num_keys=1000, heads=64, head_dim=128, block_size=64, top_m=5, top_k=100, dtype="bf16", name="s_tc"),
    dict(num_keys=700, heads=4, head_dim=64, block_size=64, top_m=3, top_k=50, dtype="f32", name="s_simt"),
    dict(batch=4, num_keys=2000, num_queries=2, first_query_pos=1998, heads=64, head_dim=128, block_size=64,
         top_m=8, top_k=100, dtype="bf16", name="s_split"),
    dict(num_keys=1000, heads=64, head_dim=128, block_size=64, top_m=5, top_k=100, dtype="bf16", w_low=-1.0,
         name="s_signed"),
], ids=lambda c: c["name"])
def test_refinement_and_flat_scores_sorted(lib, case):
    from hierarchical_top_key_b200 import binding as hb
    wl = synthetic.small_case(**case)
    d = _dev(wl)
    kp, kps = hb.hisa_pool_blocks(d["k"], wl.block_size)
    blocks = hb.hisa_block_score_topm(d["q"], d["w"], kp, d["n_visible"], num_keys=wl.num_keys,
                                      block_size=wl.block_size, top_m=wl.top_m)
    kw = dict(block_size=wl.block_size, top_k=wl.top_k)
    i1, s1 = hb.hisa_token_score_topk(d["q"], d["w"], d["k"], d["n_visible"], blocks, want_scores=True, **kw)
    i0, _ = hb.hisa_token_score_topk(d["q"], d["w"], d["k"], d["n_visible"], blocks, **kw)
    f1, fs1 = hb.dsa_flat_indexer_topk(d["q"], d["w"], d["k"], d["n_visible"], top_k=wl.top_k, want_scores=True)
    f0, _ = hb.dsa_flat_indexer_topk(d["q"], d["w"], d["k"], d["n_visible"], top_k=wl.top_k)
    hb.get_status()
    _assert_sorted(i1, s1, i0, wl.name + " refinement")
    _assert_sorted(f1, fs1, f0, wl.name + " flat")


def test_sampled_flat_and_paged_scores_sorted(lib):
    from hierarchical_top_key_b200 import binding as hb
    wl = synthetic.small_case(batch=2, num_keys=4096, num_queries=64, first_query_pos=4032, heads=64, head_dim=128,
                              block_size=128, top_m=4, top_k=128, dtype="bf16", needles=8, name="s_sampled")
    d = _dev(wl)
    f1, fs1 = hb.dsa_flat_indexer_topk_sampled(d["q"], d["w"], d["k"], d["n_visible"], top_k=wl.top_k,
                                               want_scores=True)
    f0, _ = hb.dsa_flat_indexer_topk_sampled(d["q"], d["w"], d["k"], d["n_visible"], top_k=wl.top_k)
    # paged keys: pages in reverse order
    nb = wl.num_keys // wl.block_size
    table = torch.arange(2 * nb - 1, -1, -1, dtype=torch.int32, device=d["k"].device).view(2, nb).contiguous()
    pages = torch.empty((2 * nb, wl.block_size, wl.head_dim), dtype=d["k"].dtype, device=d["k"].device)
    pages[table.view(-1).long()] = d["k"].view(2 * nb, wl.block_size, wl.head_dim)
    kp, _ = hb.hisa_pool_blocks(d["k"], wl.block_size)
    blocks = hb.hisa_block_score_topm(d["q"], d["w"], kp, d["n_visible"], num_keys=wl.num_keys,
                                      block_size=wl.block_size, top_m=wl.top_m)
    p1, ps1 = hb.hisa_token_score_topk_paged(d["q"], d["w"], pages, table, d["n_visible"], blocks,
                                             num_keys=wl.num_keys, top_k=wl.top_k, want_scores=True)
    p0, _ = hb.hisa_token_score_topk_paged(d["q"], d["w"], pages, table, d["n_visible"], blocks,
                                           num_keys=wl.num_keys, top_k=wl.top_k)
    hb.get_status()
    _assert_sorted(f1, fs1, f0, "sampled flat")
    _assert_sorted(p1, ps1, p0, "paged refinement")
