"""Paged keys (hisa_pool_blocks_paged, hisa_token_score_topk_paged): keys
scattered over shuffled fixed-size pages, with garbage in unused pages and in
the tail of the last page of each sequence, give the pooled keys and the
token top-k of the contiguous layout bit for bit, and the oracle's; a page
entry out of range is skipped and reported."""
import numpy as np
import pytest
import torch

import parity
from oracle import hisa_oracle as ho
from oracle.run import Sequence
from hierarchical_top_key_b200 import synthetic

pytestmark = pytest.mark.gpu


def _paginate(k, k_scale, B, extra_pages=5, seed=11):
    """Scatter k [batch, L, d] (and k_scale [batch, L]) into shuffled pages of B
    rows; returns (k_pages, page_scale or None, page_table [batch, nb] int32)."""
    b, L, d = k.shape
    nb = -(-L // B)
    total = b * nb + extra_pages
    rng = np.random.default_rng(seed)
    perm = torch.from_numpy(rng.permutation(total).astype(np.int32)).to(k.device)
    table = perm[: b * nb].reshape(b, nb).contiguous()
    g = torch.Generator(device="cpu").manual_seed(seed)
    if k.dtype == torch.uint8:
        pages = torch.randint(0, 0x7f, (total, B, d), dtype=torch.uint8, generator=g).to(k.device)
    else:
        pages = (torch.randn((total, B, d), generator=g) * 50).to(k.dtype).to(k.device)
    pscale = None
    if k_scale is not None:
        pscale = (torch.rand((total, B), generator=g) * 9 + 1).to(k.device)
    for s in range(b):
        for j in range(nb):
            r0, r1 = j * B, min(L, (j + 1) * B)
            pg = int(table[s, j])
            pages[pg, : r1 - r0] = k[s, r0:r1]
            if pscale is not None:
                pscale[pg, : r1 - r0] = k_scale[s, r0:r1]
    return pages.contiguous(), pscale, table


def _bits(t):
    return t.contiguous().view(torch.uint8).cpu().numpy()


@pytest.mark.parametrize("fp8", [False, True])
def test_paged_pooling_equals_contiguous_and_oracle(lib, fp8):
    from hierarchical_top_key_b200 import binding as hb
    wl = synthetic.small_case(batch=2, num_keys=1000, heads=4, head_dim=128, block_size=64, top_m=3, top_k=40,
                              dtype="bf16", needles=2, name="paged_pool")
    inp = synthetic.generate(wl)
    dev = hb.to_device_inputs(inp, fp8=fp8)
    k, ks = dev["k"], dev["k_scale"]
    B, nb = wl.block_size, -(-wl.num_keys // wl.block_size)
    full, full_s = hb.hisa_pool_blocks(k, B, ks)
    pages, pscale, table = _paginate(k, ks, B)
    cache = torch.zeros_like(full)
    cache_s = torch.zeros_like(full_s) if fp8 else None
    hb.hisa_pool_blocks_paged(pages, table, num_keys=wl.num_keys, first_block=0, block_count=nb - 3, kpool=cache,
                              k_page_scale=pscale, kpool_scale=cache_s)
    for j in range(nb - 3, nb):                     # the rest one block at a time, as a decoder fills them
        hb.hisa_pool_blocks_paged(pages, table, num_keys=wl.num_keys, first_block=j, block_count=1, kpool=cache,
                                  k_page_scale=pscale, kpool_scale=cache_s)
    hb.get_status()
    np.testing.assert_array_equal(_bits(cache), _bits(full))
    if fp8:
        np.testing.assert_array_equal(cache_s.cpu().numpy(), full_s.cpu().numpy())
    for b in range(wl.batch):
        seq = Sequence(inp, b, fp8=fp8)
        if fp8:
            np.testing.assert_array_equal(cache[b].cpu().numpy(), seq.kpool_codes)
        else:
            np.testing.assert_array_equal(cache[b].float().cpu().numpy().astype(np.float64), seq.kpool)


def _token_case(inp, fp8, want_scores=False, table_edit=None):
    """Blocks from the GPU coarse stage; the refinement on contiguous and on
    paged keys.  Returns (dev, blocks, contiguous idx, paged idx, paged scores)."""
    from hierarchical_top_key_b200 import binding as hb
    wl = inp.workload
    dev = hb.to_device_inputs(inp, fp8=fp8)
    ix = hb.HisaIndexer(wl.block_size, wl.top_m, wl.top_k)
    idx, _, blocks = ix(dev["q"], dev["w"], dev["k"], dev["n_visible"], q_scale=dev["q_scale"],
                        k_scale=dev["k_scale"], return_blocks=True)
    hb.get_status()
    pages, pscale, table = _paginate(dev["k"], dev["k_scale"], wl.block_size)
    if table_edit is not None:
        table_edit(table, pages.shape[0])
    pidx, psc = hb.hisa_token_score_topk_paged(dev["q"], dev["w"], pages, table, dev["n_visible"], blocks,
                                               num_keys=wl.num_keys, top_k=wl.top_k, q_scale=dev["q_scale"],
                                               k_page_scale=pscale, want_scores=want_scores)
    return dev, blocks.cpu().numpy(), idx.cpu().numpy(), pidx, psc


def _check_against_oracle(inp, fp8, blocks, got, rows, drop=None):
    wl = inp.workload
    for b, t in rows:
        seq = Sequence(inp, b, fp8=fp8)
        kept = [x for x in blocks[b, t] if x >= 0 and (drop is None or (b, x) not in drop)]
        cand = ho.candidate_keys(np.asarray(kept, np.int64), int(seq.n_visible[t]), wl.block_size)
        g = got[b, t]
        parity.check_selection(g[g >= 0], cand, seq.scores(t, cand), wl.top_k, f"seq {b} query {t}")


@pytest.mark.parametrize("fp8", [False, True])
def test_paged_refinement_equals_contiguous_and_oracle(lib, fp8):
    from hierarchical_top_key_b200 import binding as hb
    wl = synthetic.small_case(batch=2, num_keys=1000, num_queries=200, first_query_pos=800, heads=64,
                              head_dim=128, block_size=64, top_m=5, top_k=150, dtype="bf16", needles=4,
                              name="paged_token")
    inp = synthetic.generate(wl)
    _, blocks, idx, pidx, psc = _token_case(inp, fp8, want_scores=True)
    hb.get_status()
    got = pidx.cpu().numpy()
    np.testing.assert_array_equal(np.sort(got, axis=-1), np.sort(idx, axis=-1))
    assert np.all(np.isfinite(psc.cpu().numpy()[got >= 0]))
    _check_against_oracle(inp, fp8, blocks, got, [(b, t) for b in range(2) for t in (0, 37, 63, 64, 150, 199)])


def test_paged_refinement_split_queries(lib):
    """Few queries (a decode step): each query's blocks split over several
    CTAs reading pages, merged exactly."""
    from hierarchical_top_key_b200 import binding as hb
    wl = synthetic.small_case(batch=8, num_keys=4096, num_queries=1, first_query_pos=4095, heads=64,
                              head_dim=128, block_size=128, top_m=8, top_k=256, dtype="bf16", needles=4,
                              name="paged_decode")
    inp = synthetic.generate(wl)
    shape = hb.Shape(8, 4096, 1, 64, 128, 128, 8, 256, hb.HISA_BF16)
    assert hb.workspace_size(hb.OP_TOKEN, shape) > 0          # the split path is taken
    _, blocks, idx, pidx, _ = _token_case(inp, False)
    hb.get_status()
    got = pidx.cpu().numpy()
    np.testing.assert_array_equal(np.sort(got, axis=-1), np.sort(idx, axis=-1))
    _check_against_oracle(inp, False, blocks, got, [(b, 0) for b in range(8)])


def test_out_of_range_page_is_skipped_and_reported(lib):
    from hierarchical_top_key_b200 import binding as hb
    wl = synthetic.small_case(batch=2, num_keys=1000, num_queries=100, first_query_pos=900, heads=64,
                              head_dim=128, block_size=64, top_m=5, top_k=150, dtype="bf16", needles=4,
                              name="paged_bad")
    inp = synthetic.generate(wl)
    bad = {(0, 15), (1, 2)}

    def edit(table, num_pages):
        table[0, 15] = num_pages + 7          # the current block of sequence 0's queries at 960..999
        table[1, 2] = -3

    _, blocks, _, pidx, _ = _token_case(inp, False, table_edit=edit)
    with pytest.raises(hb.HisaError) as err:
        hb.get_status()
    assert err.value.status == 1               # HISA_ERR_INVALID_ARG
    hb.get_status()                            # the read cleared the word
    got = pidx.cpu().numpy()
    assert not np.any(got[0] >= 15 * 64)       # nothing from the skipped page
    rows = [(0, 0), (0, 50), (0, 60), (0, 99), (1, 3), (1, 99)]
    _check_against_oracle(inp, False, blocks, got, rows, drop=bad)
