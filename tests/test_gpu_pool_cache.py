"""Pooled keys kept as a cache (hisa_pool_blocks_range): a cache grown one
block at a time, as a decoder fills blocks, holds exactly the rows the
whole-context pooling writes (and the oracle computes); a range writes only
its own rows."""
import numpy as np
import pytest
import torch

from oracle.run import Sequence
from hierarchical_top_key_b200 import synthetic

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.contiguous().view(torch.uint8).cpu().numpy()


@pytest.mark.parametrize("fp8", [False, True])
def test_block_range_pooling_builds_the_same_cache(lib, fp8):
    from hierarchical_top_key_b200 import binding as hb
    wl = synthetic.small_case(batch=2, num_keys=1000, heads=4, head_dim=128, block_size=64, top_m=3, top_k=40,
                              dtype="bf16", needles=2, name="pool_cache")
    inp = synthetic.generate(wl)
    dev = hb.to_device_inputs(inp, fp8=fp8)
    k, ks = dev["k"], dev["k_scale"]
    B, nb = wl.block_size, -(-wl.num_keys // wl.block_size)
    full, full_s = hb.hisa_pool_blocks(k, B, ks)

    def blank():
        c = torch.full_like(full, 0x55) if fp8 else torch.full_like(full, 7.0)
        cs = torch.full((wl.batch, nb), -1.0, dtype=torch.float32, device=k.device) if fp8 else None
        return c, cs

    # grown one block at a time
    cache, cache_s = blank()
    for b in range(nb):
        hb.hisa_pool_blocks_range(k, B, b, 1, cache, ks, cache_s)
    hb.get_status()
    np.testing.assert_array_equal(_bits(cache), _bits(full))
    if fp8:
        np.testing.assert_array_equal(cache_s.cpu().numpy(), full_s.cpu().numpy())
    # a range writes its rows and nothing else; a range past the end is clipped
    for first, count, rows in [(5, 4, range(5, 9)), (14, 100, range(14, 16)), (nb + 3, 2, range(0))]:
        part, part_s = blank()
        untouched = _bits(part).copy()
        hb.hisa_pool_blocks_range(k, B, first, count, part, ks, part_s)
        hb.get_status()
        got, want = _bits(part), _bits(full)
        for r in range(nb):
            ref = want if r in rows else untouched
            np.testing.assert_array_equal(got[:, r], ref[:, r], err_msg=f"range ({first}, {count}) row {r}")
        if fp8:
            ps = part_s.cpu().numpy()
            assert np.all(ps[:, [r for r in range(nb) if r not in rows]] == -1.0)
            np.testing.assert_array_equal(ps[:, list(rows)], full_s.cpu().numpy()[:, list(rows)])
    # and the cache is the oracle's pooling
    for b in range(wl.batch):
        seq = Sequence(inp, b, fp8=fp8)
        if fp8:
            np.testing.assert_array_equal(cache[b].cpu().numpy(), seq.kpool_codes)
            np.testing.assert_array_equal(cache_s[b].cpu().numpy(), seq.kpool_scale)
        else:
            np.testing.assert_array_equal(cache[b].float().cpu().numpy().astype(np.float64), seq.kpool)


@pytest.mark.parametrize("fp8", [False, True])
def test_long_groups_pool_like_the_oracle(lib, fp8):
    """Super-block pooling (groups of 1024 keys, the one-CTA-per-row kernel),
    including a ragged last group, is the oracle's exact mean."""
    from hierarchical_top_key_b200 import binding as hb
    from oracle import hisa_oracle as ho
    wl = synthetic.small_case(batch=2, num_keys=3000, heads=4, head_dim=128, block_size=64, top_m=3, top_k=40,
                              dtype="bf16", needles=2, name="pool_long")
    inp = synthetic.generate(wl)
    dev = hb.to_device_inputs(inp, fp8=fp8)
    kp, kps = hb.hisa_pool_blocks(dev["k"], 1024, dev["k_scale"])
    hb.get_status()
    for b in range(wl.batch):
        seq = Sequence(inp, b, fp8=fp8)
        if fp8:
            pc, ps = ho.pool_blocks_e4m3(seq.k_codes, seq.k_scale, 1024)
            np.testing.assert_array_equal(kp[b].cpu().numpy(), pc)
            np.testing.assert_array_equal(kps[b].cpu().numpy(), ps)
        else:
            np.testing.assert_array_equal(kp[b].float().cpu().numpy().astype(np.float64),
                                          ho.pool_blocks(seq.keys, 1024, "bf16"))
