"""Failure detection on the GPU without a fault: a bounded device-side wait
that is made to run out must come back as HISA_ERR_TIMEOUT through the status
word, and the context must stay usable afterwards."""
import time

import numpy as np
import pytest
import torch

from hierarchical_top_key_b200 import synthetic

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_recovers(lib):
    from hierarchical_top_key_b200 import binding as hb
    st = torch.cuda.current_stream().cuda_stream
    assert lib.hisa_get_status(st) == 0                     # clean to begin with
    t0 = time.perf_counter()
    assert lib.hisa_selftest_wait_timeout(20_000_000, st) == 0   # 20 ms
    assert lib.hisa_get_status(st) == 5                     # HISA_ERR_TIMEOUT, read and cleared
    elapsed = time.perf_counter() - t0
    assert 0.015 < elapsed < 5.0, elapsed
    assert lib.hisa_get_status(st) == 0                     # cleared
    # the context still runs the indexer correctly
    wl = synthetic.small_case(num_keys=300, heads=64, head_dim=128, block_size=64, top_m=3, top_k=32,
                              dtype="bf16", needles=2, name="after_timeout")
    dev = hb.to_device_inputs(synthetic.generate(wl))
    idx, _ = hb.HisaIndexer(wl.block_size, wl.top_m, wl.top_k)(dev["q"], dev["w"], dev["k"], dev["n_visible"])
    hb.get_status()
    got = idx.cpu().numpy()
    assert (got[0, 299] >= 0).sum() == 32 and len(set(got[0, 299].tolist())) == 32


def test_selftest_argument_validation(lib):
    st = torch.cuda.current_stream().cuda_stream
    assert lib.hisa_selftest_wait_timeout(0, st) == 1
    assert lib.hisa_selftest_wait_timeout(20_000_000_000, st) == 1
