"""The host-buffer entry point (hisa_indexer_from_host, through
HisaIndexer.from_host and directly through ctypes) against the device entry
points on the same inputs: piecewise copies, incremental pooling and chunked
stages must give the same index sets as one whole-tensor call."""
import ctypes

import numpy as np
import pytest
import torch

from hierarchical_top_key_b200 import synthetic

pytestmark = pytest.mark.gpu


def _want(hb, wl, dev, fp8=False):
    ix = hb.HisaIndexer(wl.block_size, wl.top_m, wl.top_k)
    idx, _ = ix(dev["q"], dev["w"], dev["k"], dev["n_visible"], q_scale=dev["q_scale"], k_scale=dev["k_scale"])
    return ix, idx


@pytest.mark.parametrize("case,chunks", [
    (dict(num_keys=1000, heads=64, head_dim=128, block_size=64, top_m=5, top_k=100, dtype="bf16", needles=6,
          name="host_causal"), 5),
    (dict(batch=3, num_keys=2000, num_queries=40, first_query_pos=1960, heads=64, head_dim=128, block_size=128,
          top_m=4, top_k=256, dtype="bf16", needles=8, name="host_batch"), 2),
    (dict(num_keys=700, heads=4, head_dim=64, block_size=64, top_m=3, top_k=50, dtype="f32", needles=4,
          name="host_f32"), 3),
    # decode-like pieces of whole sequences: each piece takes the split refinement
    (dict(batch=8, num_keys=3000, num_queries=1, first_query_pos=2999, heads=64, head_dim=128, block_size=64,
          top_m=8, top_k=128, dtype="bf16", needles=4, name="host_decode"), 4),
])
def test_from_host_matches_device_entry_points(lib, case, chunks):
    from hierarchical_top_key_b200 import binding as hb
    wl = synthetic.small_case(**case)
    inp = synthetic.generate(wl)
    dev = hb.to_device_inputs(inp)
    ix, want = _want(hb, wl, dev)
    hq, hw, hk, hnv = (t.cpu().pin_memory() for t in (dev["q"], dev["w"], dev["k"], dev["n_visible"]))
    out = torch.full((wl.batch, wl.num_queries, wl.top_k), -7, dtype=torch.int32).pin_memory()
    for _ in range(2):       # the second call reuses the kept workspace and the library's streams
        out.fill_(-7)
        ix.from_host(hq, hw, hk, hnv, out, chunks=chunks)
        torch.cuda.current_stream().synchronize()
        hb.get_status()
        np.testing.assert_array_equal(np.sort(out.numpy(), axis=-1), np.sort(want.cpu().numpy(), axis=-1))


def test_from_host_e4m3_through_ctypes(lib):
    """E4M3 codes and scales from pageable host memory, called through the C ABI."""
    from hierarchical_top_key_b200 import binding as hb
    wl = synthetic.small_case(num_keys=1500, heads=64, head_dim=128, block_size=64, top_m=6, top_k=128,
                              dtype="bf16", needles=6, name="host_e4m3")
    dev = hb.to_device_inputs(synthetic.generate(wl), fp8=True)
    _, want = _want(hb, wl, dev, fp8=True)
    h = {k: v.cpu().contiguous() for k, v in dev.items()}
    shape = hb.Shape(1, wl.num_keys, wl.num_queries, wl.heads, wl.head_dim, wl.block_size, wl.top_m, wl.top_k,
                     hb.HISA_E4M3)
    ws = torch.empty(hb.workspace_size(hb.OP_FROM_HOST, shape), dtype=torch.uint8, device="cuda")
    out = np.full((1, wl.num_queries, wl.top_k), -7, np.int32)
    st = lib.hisa_indexer_from_host(h["q"].data_ptr(), h["q_scale"].data_ptr(), h["w"].data_ptr(),
                                    h["k"].data_ptr(), h["k_scale"].data_ptr(), h["n_visible"].data_ptr(),
                                    ctypes.byref(shape), out.ctypes.data, 7, ws.data_ptr(), ws.numel(),
                                    torch.cuda.current_stream().cuda_stream)
    assert st == 0, lib.hisa_last_error()
    torch.cuda.current_stream().synchronize()
    hb.get_status()
    np.testing.assert_array_equal(np.sort(out, axis=-1), np.sort(want.cpu().numpy(), axis=-1))
