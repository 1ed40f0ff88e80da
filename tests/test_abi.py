"""The C ABI without a GPU: the library loads, exports every entry point
include/hisa.h declares, and validates arguments on the host (no kernel is
launched by any call here)."""
import ctypes
import os
import re

import pytest

from hierarchical_top_key_b200 import binding as hb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "hisa.h")).read()
    return re.findall(r"HISA_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)


@pytest.fixture(scope="module")
def L():
    return hb.load()


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert {"hisa_pool_blocks", "hisa_block_score_topm", "hisa_token_score_topk", "dsa_flat_indexer_topk"} <= set(names)
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/hisa.h but not exported"
    assert set(names) == set(hb.EXPORTS), "binding signatures out of step with the header"


def test_status_strings(L):
    for code in range(6):
        assert L.hisa_status_string(code).decode().startswith(hb.STATUS[code])


def _shape(**kw):
    base = dict(batch=1, num_keys=32768, num_queries=32768, heads=64, head_dim=128, block_size=128, top_m=32,
                top_k=2048, dtype=hb.HISA_BF16)
    base.update(kw)
    return hb.Shape(**base)


def test_workspace_sizes(L):
    s = _shape()
    assert hb.workspace_size(hb.OP_FLAT, s) == 32768 * (32768 * 4 + 8)
    assert hb.workspace_size(hb.OP_BLOCK, s) == 32768 * 256 * 4
    assert hb.workspace_size(hb.OP_TOKEN, s) == 0
    # few queries (a decode step): room for the per-part top-k lists of split queries
    dec = _shape(batch=64, num_queries=1, num_keys=131072, top_m=64)
    parts = hb.workspace_size(hb.OP_TOKEN, dec) // (64 * 2048 * 8)
    assert parts >= 2 and hb.workspace_size(hb.OP_TOKEN, dec) == 64 * parts * 2048 * 8
    s = _shape(num_keys=1001, num_queries=3, batch=2, block_size=64)
    assert hb.workspace_size(hb.OP_FLAT, s) == 6 * (1004 * 4 + 8)    # rows padded to 16 bytes, + row range
    assert hb.workspace_size(hb.OP_BLOCK, s) == 6 * 16 * 4           # ceil(1001/64)=16


def test_workspace_sizes_of_the_extensions(L):
    s = _shape()
    rows = s.batch * s.num_queries
    # the second level of the three-level indexer: visible-block counts + (m-1) picks per row
    assert hb.workspace_size(hb.OP_BLOCK_REFINE, s) == rows * 4 + rows * (s.top_m - 1) * 4
    # the sampled flat top-k: a sample row and a pair buffer per query instead of a score row
    sampled = hb.workspace_size(hb.OP_FLAT_SAMPLED, s)
    assert 0 < sampled < hb.workspace_size(hb.OP_FLAT, s) // 2
    # shapes it does not cover are refused before anything else
    n = ctypes.c_size_t(0)
    assert L.hisa_workspace_size(hb.OP_FLAT_SAMPLED, ctypes.byref(_shape(dtype=hb.HISA_F32)), ctypes.byref(n)) == 2
    assert L.hisa_workspace_size(hb.OP_FLAT_SAMPLED, ctypes.byref(_shape(num_keys=32760)), ctypes.byref(n)) == 2


@pytest.mark.parametrize("field,value,status", [
    ("head_dim", 96, 2), ("heads", 65, 2), ("heads", 0, 2), ("batch", 0, 1), ("top_k", 0, 1),
    ("dtype", 7, 1), ("block_size", 0, 1), ("top_m", 0, 1)])
def test_shape_validation(L, field, value, status):
    s = _shape(**{field: value})
    n = ctypes.c_size_t(0)
    assert L.hisa_workspace_size(hb.OP_BLOCK, ctypes.byref(s), ctypes.byref(n)) == status
    assert L.hisa_last_error()


def test_pointer_validation_returns_before_any_launch(L):
    s = _shape()
    # NULL inputs
    assert L.dsa_flat_indexer_topk(None, None, None, None, None, None, ctypes.byref(s), None, None, None, 0,
                                   None) == 1
    # misaligned q (never dereferenced: validation fails first)
    assert L.hisa_token_score_topk(0x1001, None, 0x2000, 0x3000, None, 0x4000, 0x5000, ctypes.byref(s), 0x6000,
                                   None, None, 0, None) == 1
    # E4M3 without scales
    s8 = _shape(dtype=hb.HISA_E4M3)
    assert L.hisa_block_score_topm(0x1000, None, 0x2000, 0x3000, None, 0x4000, ctypes.byref(s8), 0x5000, 0x6000,
                                   1 << 30, None) == 1
    # workspace too small for one row of block scores
    assert L.hisa_block_score_topm(0x1000, None, 0x2000, 0x3000, None, 0x4000, ctypes.byref(s), 0x5000, 0x6000,
                                   16, None) == 3
    # too many candidates for the on-chip refinement buffer
    big = _shape(top_m=512, block_size=128)
    assert L.hisa_token_score_topk(0x1000, None, 0x2000, 0x3000, None, 0x4000, 0x5000, ctypes.byref(big), 0x6000,
                                   None, None, 0, None) == 2
    assert L.hisa_pool_blocks(None, None, None, None, ctypes.byref(s), None) == 1
    assert L.hisa_pool_blocks_range(0x1000, None, 0x2000, None, ctypes.byref(s), -1, 1, None) == 1
    assert L.hisa_pool_blocks_range(0x1000, None, 0x2000, None, ctypes.byref(s), 0, -1, None) == 1
    # a range past the last block launches nothing (the placeholder pointers are never used)
    assert L.hisa_pool_blocks_range(0x1000, None, 0x2000, None, ctypes.byref(s), 1 << 20, 4, None) == 0
    assert L.hisa_quantize_e4m3(0x1000, hb.HISA_BF16, 10, 100, 0x2000, 0x3000, None) == 2   # cols % 16
    assert L.hisa_compress_keys(0x1000, 0x2000, 1, 100, 128, 4, hb.HISA_E4M3, None) == 2


def test_paged_entries_validate_on_the_host(L):
    s = _shape()
    P = ctypes.c_int32
    # refinement over paged keys: no page table, no pages, a page range past int32 rows
    assert L.hisa_token_score_topk_paged(0x1000, None, 0x2000, 0x3000, None, None, 8, 0x4000, 0x5000,
                                         ctypes.byref(s), 0x6000, None, None, 0, None) == 1
    assert L.hisa_token_score_topk_paged(0x1000, None, 0x2000, 0x3000, None, 0x7000, 0, 0x4000, 0x5000,
                                         ctypes.byref(s), 0x6000, None, None, 0, None) == 1
    assert L.hisa_token_score_topk_paged(0x1000, None, 0x2000, 0x3000, None, 0x7000, P(1 << 30), 0x4000, 0x5000,
                                         ctypes.byref(s), 0x6000, None, None, 0, None) == 2
    # E4M3 pages without their scales
    s8 = _shape(dtype=hb.HISA_E4M3)
    assert L.hisa_token_score_topk_paged(0x1000, 0x1100, 0x2000, 0x3000, None, 0x7000, 8, 0x4000, 0x5000,
                                         ctypes.byref(s8), 0x6000, None, None, 0, None) == 1
    # shapes the tensor-core kernel does not take have no paged path (fp32 runs on CUDA cores)
    s32 = _shape(dtype=hb.HISA_F32, heads=4, head_dim=64, block_size=64, top_m=4, top_k=128)
    assert L.hisa_token_score_topk_paged(0x1000, None, 0x2000, 0x3000, None, 0x7000, 8, 0x4000, 0x5000,
                                         ctypes.byref(s32), 0x6000, None, None, 0, None) == 2
    # pooling over paged keys
    assert L.hisa_pool_blocks_paged(0x1000, None, None, 8, 0x2000, None, ctypes.byref(s), 0, 1, None) == 1
    assert L.hisa_pool_blocks_paged(0x1000, None, 0x7000, 0, 0x2000, None, ctypes.byref(s), 0, 1, None) == 1
    assert L.hisa_pool_blocks_paged(0x1000, None, 0x7000, 8, 0x2000, None, ctypes.byref(s), -1, 1, None) == 1
    assert L.hisa_pool_blocks_paged(0x1000, None, 0x7000, 8, 0x2000, None, ctypes.byref(s8), 0, 1, None) == 1
    # an empty range launches nothing
    assert L.hisa_pool_blocks_paged(0x1000, None, 0x7000, 8, 0x2000, None, ctypes.byref(s), 1 << 20, 4, None) == 0


def test_static_scratch_refuses_oversized_shape(L):
    """hisa_block_score_topm_static keeps the block scores in a built-in 16 MiB
    array; a shape whose scores need more is refused on the host, before any
    CUDA call (without a GPU an accepted shape would fail at the first CUDA
    call instead, so the placeholder pointers are never used either way)."""
    cap = 16 << 20
    nb = 256                                   # 32768 keys in blocks of 128
    rows = 2 * cap // (nb * 4)                 # twice the array's capacity
    s = _shape(num_queries=rows, num_keys=32768, block_size=128)
    st = L.hisa_block_score_topm_static(0x1000, None, 0x2000, 0x3000, None, 0x4000, ctypes.byref(s), 0x5000, None)
    assert st == 3
    assert b"16777216" in L.hisa_last_error()


def test_scored_rows_longer_than_the_on_chip_sort_are_refused(L):
    """With a score output rows come back sorted on chip, up to 16384 per row;
    longer rows are refused before anything is launched."""
    s = _shape(top_k=16385)
    assert L.dsa_flat_indexer_topk(0x1000, None, 0x2000, 0x3000, None, 0x4000, ctypes.byref(s), 0x5000, 0x6000,
                                   0x7000, 1 << 30, None) == 2
    assert b"16384" in L.hisa_last_error()
    s = _shape(top_k=16385, top_m=4, block_size=128)
    assert L.hisa_token_score_topk(0x1000, None, 0x2000, 0x3000, None, 0x4000, 0x5000, ctypes.byref(s), 0x6000,
                                   0x7000, None, 0, None) == 2


def test_host_buffer_entry_validates_on_the_host(L):
    """hisa_indexer_from_host: argument checks and the workspace rule, before
    any stream, event or copy is made."""
    s = _shape(num_keys=4096, num_queries=4096, top_m=8)
    n = ctypes.c_size_t(0)
    assert L.hisa_workspace_size(6, ctypes.byref(s), ctypes.byref(n)) == 0
    # device copies of q (4096*64*128*2), keys, w, n_visible, pooled keys, block and token indices and scratch
    assert n.value > 4096 * 64 * 128 * 2 + 4096 * 128 * 2 + 4096 * 2048 * 4
    args = (0x1000, None, 0x2000, 0x3000, None, 0x4000, ctypes.byref(s), 0x5000)
    assert L.hisa_indexer_from_host(None, None, 0x2000, 0x3000, None, 0x4000, ctypes.byref(s), 0x5000, 0, 0x6000,
                                    n.value, None) == 1
    assert L.hisa_indexer_from_host(*args, -1, 0x6000, n.value, None) == 1            # pieces out of range
    assert L.hisa_indexer_from_host(*args, 0, 0x6000, n.value - 1, None) == 3         # workspace too small
    assert L.hisa_indexer_from_host(*args, 0, 0x6001, n.value, None) == 3             # misaligned workspace
    s8 = _shape(num_keys=4096, num_queries=4096, top_m=8, dtype=hb.HISA_E4M3)
    assert L.hisa_indexer_from_host(0x1000, None, 0x2000, 0x3000, None, 0x4000, ctypes.byref(s8), 0x5000, 0,
                                    0x6000, 1 << 40, None) == 1                       # E4M3 without scales


def test_sparse_attention_validates_on_the_host(L):
    """hisa_sparse_attention: shapes this build has no kernel for and bad
    pointers are refused before any CUDA call."""
    f = ctypes.c_float
    ok = dict(q=0x1000, kv=0x2000, idx=0x3000, batch=1, Q=4, L=100, H=128, dqk=576, dv=512, k=64, scale=f(0.07),
              o=0x4000, lse=0x5000)

    def call(**kw):
        a = dict(ok, **kw)
        return L.hisa_sparse_attention(a["q"], a["kv"], a["idx"], a["batch"], a["Q"], a["L"], a["H"], a["dqk"],
                                       a["dv"], a["k"], a["scale"], a["o"], a["lse"], None)
    assert call(H=64) == 2 and call(H=192) == 2          # heads: whole 128-head slices
    assert call(dqk=192) == 2 and call(dv=128) == 2      # latent 512 + positional 64 only
    assert call(k=0) == 2 and call(k=4097) == 2
    assert call(batch=0) == 1 and call(L=0) == 1
    assert call(scale=f(float("inf"))) == 1
    assert call(q=None) == 1 and call(lse=None) == 1
    assert call(kv=0x2008) == 1 and call(idx=0x3002) == 1
