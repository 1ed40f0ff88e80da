"""The coarse stage without a caller workspace (hisa_block_score_topm_static).

Some callers cannot allocate device memory when they run the indexer: code
living inside another runtime's memory arena, or a plug-in that is handed only
its input and output pointers.  For them the library keeps the block scores in
a built-in device array.  This checks, through the C ABI, that two calls in a
row return what the workspace entry point returns, also right after a larger
call has filled the shared array with rows of another stride.  (The refusal of
a shape too large for the array is a host-side check, tested without a GPU in
test_abi.py.)

Collected last on purpose (the file name sorts after the others), so that a run
stopping at the first failure has already run every other test.
"""
import numpy as np
import pytest

from hierarchical_top_key_b200 import synthetic

pytestmark = pytest.mark.gpu


def _device_case(wl):
    from hierarchical_top_key_b200 import binding as hb
    inp = synthetic.generate(wl)
    dev = hb.to_device_inputs(inp)
    kpool, kps = hb.hisa_pool_blocks(dev["k"], wl.block_size, dev["k_scale"])
    kw = dict(num_keys=dev["k"].shape[1], block_size=wl.block_size, top_m=wl.top_m, q_scale=dev["q_scale"],
              kpool_scale=kps)
    return dev, kpool, kw


def _static_then_workspace(dev, kpool, kw):
    """The built-in-scratch entry point, then the workspace entry point, on the
    same inputs; block sets sorted per row."""
    from hierarchical_top_key_b200 import binding as hb
    got = hb.hisa_block_score_topm_static(dev["q"], dev["w"], kpool, dev["n_visible"], **kw)
    ref = hb.hisa_block_score_topm(dev["q"], dev["w"], kpool, dev["n_visible"], **kw)
    hb.get_status()
    return [np.sort(t.cpu().numpy(), axis=-1) for t in (got, ref)]


SMALL = [
    dict(num_keys=1000, heads=64, head_dim=128, block_size=64, top_m=5, top_k=64, dtype="bf16", name="na_bf16"),
    dict(batch=2, num_keys=900, num_queries=300, first_query_pos=600, heads=4, head_dim=64, block_size=32,
         top_m=6, top_k=40, dtype="f32", name="na_f32"),
]
# more queries and a wider score row (pad4(ceil(4000/32)) = 128 floats per row,
# 4000 rows: 2 MB) than either small case, so the array holds stale rows of
# another stride when the small case runs after it
WIDE = dict(num_keys=4000, heads=64, head_dim=128, block_size=32, top_m=7, top_k=64, dtype="bf16",
            name="na_wide")


@pytest.mark.parametrize("case", SMALL, ids=lambda c: c["name"])
def test_static_scratch_matches_workspace_entry_point(lib, case):
    dev, kpool, kw = _device_case(synthetic.small_case(**case))
    for _ in range(2):
        # the same kernels on the same inputs: identical block sets, call after call
        got, ref = _static_then_workspace(dev, kpool, kw)
        np.testing.assert_array_equal(got, ref)


@pytest.mark.parametrize("case", SMALL, ids=lambda c: c["name"])
def test_static_scratch_after_a_larger_call(lib, case):
    """A larger call leaves the shared array full of its own rows (another row
    stride); the next, smaller call must not read any of them."""
    wide = _device_case(synthetic.small_case(**WIDE))
    small = _device_case(synthetic.small_case(**case))
    got, ref = _static_then_workspace(*wide)
    np.testing.assert_array_equal(got, ref)
    got, ref = _static_then_workspace(*small)
    np.testing.assert_array_equal(got, ref)
