"""The host-buffer entry point (HisaIndexer.from_host) against the device
entry points on the same inputs: piecewise copies, incremental pooling and
chunked stages must give the same index sets as one whole-tensor call."""
import numpy as np
import pytest
import torch

from hierarchical_top_key_b200 import synthetic

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("case,chunks", [
    (dict(num_keys=1000, heads=64, head_dim=128, block_size=64, top_m=5, top_k=100, dtype="bf16", needles=6,
          name="host_causal"), 5),
    (dict(batch=3, num_keys=2000, num_queries=40, first_query_pos=1960, heads=64, head_dim=128, block_size=128,
          top_m=4, top_k=256, dtype="bf16", needles=8, name="host_batch"), 2),
    (dict(num_keys=700, heads=4, head_dim=64, block_size=64, top_m=3, top_k=50, dtype="f32", needles=4,
          name="host_f32"), 3),
])
def test_from_host_matches_device_entry_points(lib, case, chunks):
    from hierarchical_top_key_b200 import binding as hb
    wl = synthetic.small_case(**case)
    inp = synthetic.generate(wl)
    dev = hb.to_device_inputs(inp)
    ix = hb.HisaIndexer(wl.block_size, wl.top_m, wl.top_k)
    want, _ = ix(dev["q"], dev["w"], dev["k"], dev["n_visible"])
    hq, hw, hk, hnv = (t.cpu().pin_memory() for t in (dev["q"], dev["w"], dev["k"], dev["n_visible"]))
    out = torch.full((wl.batch, wl.num_queries, wl.top_k), -7, dtype=torch.int32).pin_memory()
    ix.from_host(hq, hw, hk, hnv, out, chunks=chunks)
    torch.cuda.current_stream().synchronize()
    hb.get_status()
    np.testing.assert_array_equal(np.sort(out.numpy(), axis=-1), np.sort(want.cpu().numpy(), axis=-1))
