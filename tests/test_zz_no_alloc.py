"""The coarse stage without a caller workspace (hisa_block_score_topm_static).

Some callers cannot allocate device memory when they run the indexer: code
living inside another runtime's memory arena, or a plug-in that is handed only
its input and output pointers.  For them the library keeps the block scores in
a built-in device array.  This checks, through the C ABI, that two calls in a
row return what the workspace entry point returns, and that a shape too large
for the built-in array is refused before anything is launched.

Collected last on purpose (the file name sorts after the others), so that a run
stopping at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from hierarchical_top_key_b200 import synthetic

pytestmark = pytest.mark.gpu


def _blocks_both_ways(lib, wl):
    from hierarchical_top_key_b200 import binding as hb
    inp = synthetic.generate(wl)
    dev = hb.to_device_inputs(inp)
    kpool, kps = hb.hisa_pool_blocks(dev["k"], wl.block_size, dev["k_scale"])
    kw = dict(num_keys=dev["k"].shape[1], block_size=wl.block_size, top_m=wl.top_m, q_scale=dev["q_scale"],
              kpool_scale=kps)
    ref = hb.hisa_block_score_topm(dev["q"], dev["w"], kpool, dev["n_visible"], **kw)
    first = hb.hisa_block_score_topm_static(dev["q"], dev["w"], kpool, dev["n_visible"], **kw)
    second = hb.hisa_block_score_topm_static(dev["q"], dev["w"], kpool, dev["n_visible"], **kw)
    hb.get_status()
    return [np.sort(t.cpu().numpy(), axis=-1) for t in (ref, first, second)]


@pytest.mark.parametrize("case", [
    dict(num_keys=1000, heads=64, head_dim=128, block_size=64, top_m=5, top_k=64, dtype="bf16", name="na_bf16"),
    dict(batch=2, num_keys=900, num_queries=300, first_query_pos=600, heads=4, head_dim=64, block_size=32,
         top_m=6, top_k=40, dtype="f32", name="na_f32"),
])
def test_static_scratch_matches_workspace_entry_point(lib, case):
    ref, first, second = _blocks_both_ways(lib, synthetic.small_case(**case))
    # the same kernels on the same inputs: identical block sets, call after call
    np.testing.assert_array_equal(first, ref)
    np.testing.assert_array_equal(second, ref)


def test_static_scratch_refuses_oversized_shape(lib):
    from hierarchical_top_key_b200 import binding as hb
    # 32768 queries x 256 blocks x 4 bytes = 32 MiB > the 16 MiB built-in array;
    # refused on the host, so the placeholder pointers are never used
    s = hb.Shape(1, 32768, 32768, 64, 128, 128, 32, 2048, hb.HISA_BF16)
    st = lib.hisa_block_score_topm_static(0x1000, None, 0x2000, 0x3000, None, 0x4000, ctypes.byref(s), 0x5000,
                                          torch.cuda.current_stream().cuda_stream)
    assert st == 3
    assert b"16" in lib.hisa_last_error()
