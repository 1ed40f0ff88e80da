"""Argument checks of the binding that run on the host before any launch
(no GPU needed)."""
import pytest
import torch

from hierarchical_top_key_b200 import binding as hb


def _host(b=1, Q=8, H=4, d=64, L=8, k=4):
    q = torch.zeros((b, Q, H, d), dtype=torch.bfloat16)
    w = torch.zeros((b, Q, H), dtype=torch.float32)
    keys = torch.zeros((b, L, d), dtype=torch.bfloat16)
    nv = torch.ones((b, Q), dtype=torch.int32)
    out = torch.zeros((b, Q, k), dtype=torch.int32)
    return q, w, keys, nv, out


def test_from_host_rejects_bad_host_tensors():
    ix = hb.HisaIndexer(block_size=4, top_m=2, top_k=4)
    q, w, keys, nv, out = _host()
    with pytest.raises(ValueError):                       # wrong output shape
        ix.from_host(q, w, keys, nv, torch.zeros((1, 8, 5), dtype=torch.int32))
    with pytest.raises(ValueError):                       # wrong output dtype
        ix.from_host(q, w, keys, nv, torch.zeros((1, 8, 4), dtype=torch.int64))
    with pytest.raises(ValueError):                       # non-contiguous q
        ix.from_host(q.transpose(2, 3), w, keys, nv, out)
    with pytest.raises(ValueError):                       # keys without the batch dimension
        ix.from_host(q, w, keys[0], nv, out)


def test_device_entry_points_reject_host_tensors():
    q, w, keys, nv, _ = _host()
    with pytest.raises(ValueError):
        hb.hisa_pool_blocks(keys, 4)
    with pytest.raises(ValueError):
        hb.hisa_pool_blocks_range(keys, 4, 0, 1, torch.zeros((1, 2, 64), dtype=torch.bfloat16))
