"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.

Small cases span several tiles and ragged tails and are checked on every
query the oracle can afford; the five full-size workloads run in the launch
configuration bench.py times and are checked on sampled queries (first,
last, block boundaries and random ones).
"""
from __future__ import annotations

import functools

import numpy as np
import pytest
import torch

import parity
from oracle import hisa_oracle as ho
from oracle.run import Sequence
from hierarchical_top_key_b200 import synthetic

pytestmark = pytest.mark.gpu


@functools.lru_cache(maxsize=4)
def _inputs(key):
    name, overrides = key
    wl = synthetic.WORKLOADS[name] if name in synthetic.WORKLOADS else synthetic.small_case(**dict(overrides))
    return synthetic.generate(wl)


SMALL = {
    "ragged_bf16": dict(num_keys=1000, heads=64, head_dim=128, block_size=64, top_m=5, top_k=100, dtype="bf16",
                        needles=6, name="ragged_bf16"),
    "ragged_bf16_d64": dict(num_keys=777, heads=16, head_dim=64, block_size=32, top_m=8, top_k=64, dtype="bf16",
                            needles=4, name="ragged_bf16_d64"),
    "f32_h4": dict(num_keys=700, heads=4, head_dim=64, block_size=64, top_m=3, top_k=50, dtype="f32",
                   needles=4, name="f32_h4"),
    "batch_tail": dict(batch=3, num_keys=2000, num_queries=40, first_query_pos=1960, heads=64, head_dim=128,
                       block_size=128, top_m=4, top_k=256, dtype="bf16", needles=8, name="batch_tail"),
    # few queries: the refinement stage splits each query's blocks over several CTAs and merges
    "few_rows_split": dict(batch=4, num_keys=2000, num_queries=2, first_query_pos=1998, heads=64, head_dim=128,
                           block_size=64, top_m=8, top_k=100, dtype="bf16", needles=4, name="few_rows_split"),
    "compressed": dict(num_keys=600, compress_ratio=4, num_queries=300, first_query_pos=2100, heads=64,
                       head_dim=128, block_size=64, top_m=4, top_k=96, dtype="bf16", needles=0,
                       name="compressed"),
    # head weights of both signs: scores below zero, the sign half of the ordering keys
    "signed_w_bf16": dict(num_keys=1500, heads=64, head_dim=128, block_size=64, top_m=6, top_k=200, dtype="bf16",
                          needles=6, w_low=-1.0, name="signed_w_bf16"),
    "signed_w_f32": dict(num_keys=700, heads=4, head_dim=64, block_size=64, top_m=3, top_k=50, dtype="f32",
                         needles=4, w_low=-1.0, name="signed_w_f32"),
    "signed_w_decode": dict(batch=6, num_keys=3000, num_queries=1, first_query_pos=2999, heads=64, head_dim=128,
                            block_size=64, top_m=8, top_k=128, dtype="bf16", needles=4, w_low=-1.0,
                            name="signed_w_decode"),
}


def _sample_queries(wl, n_rand, seed=0, max_boundaries=24):
    Q = wl.num_queries
    B = wl.block_size
    if n_rand >= Q:
        return list(range(Q))
    pick = {0, 1, Q - 1, Q - 2}
    rng = np.random.default_rng(seed)
    bounds = list(range(0, Q, max(1, B)))
    if len(bounds) > max_boundaries:
        bounds = sorted(rng.choice(bounds, max_boundaries, replace=False).tolist())
    for t in bounds:
        pick.update({t, t - 1, t + 1})
    pick.update(rng.integers(0, Q, n_rand).tolist())
    return sorted(x for x in pick if 0 <= x < Q)


def _run_gpu(inp, fp8):
    from hierarchical_top_key_b200 import binding as hb
    wl = inp.workload
    dev = hb.to_device_inputs(inp, fp8=fp8)
    kpool, kps = hb.hisa_pool_blocks(dev["k"], wl.block_size, dev["k_scale"])
    blocks = hb.hisa_block_score_topm(dev["q"], dev["w"], kpool, dev["n_visible"], num_keys=dev["k"].shape[1],
                                      block_size=wl.block_size, top_m=wl.top_m, q_scale=dev["q_scale"],
                                      kpool_scale=kps)
    tok, tok_sc = hb.hisa_token_score_topk(dev["q"], dev["w"], dev["k"], dev["n_visible"], blocks,
                                           block_size=wl.block_size, top_k=wl.top_k, q_scale=dev["q_scale"],
                                           k_scale=dev["k_scale"], want_scores=True)
    flat, flat_sc = hb.dsa_flat_indexer_topk(dev["q"], dev["w"], dev["k"], dev["n_visible"], top_k=wl.top_k,
                                             q_scale=dev["q_scale"], k_scale=dev["k_scale"], want_scores=True)
    hb.get_status()
    return dev, dict(kpool=kpool, kps=kps, blocks=blocks, tok=tok, tok_sc=tok_sc, flat=flat, flat_sc=flat_sc)


def _dev_float(x):
    if x.dtype == torch.uint8:
        return x.cpu().numpy()
    return x.float().cpu().numpy().astype(np.float64)


def _check_workload(inp, fp8, queries_per_seq, seqs=None):
    """Full parity of one draw: preprocessing bit-exact, then each stage."""
    from hierarchical_top_key_b200 import binding as hb
    wl = inp.workload
    dt = "e4m3" if fp8 else wl.dtype
    rtol = parity.RTOL[dt]
    dev, out = _run_gpu(inp, fp8)
    seqs = range(wl.batch) if seqs is None else seqs
    stats = dict(queries=0, swaps_block=0, swaps_tok=0, swaps_flat=0, block_mismatch=0, iou=[], recall=[],
                 negative_scores=0)
    # token stage fed with the oracle's blocks for the sampled rows
    blocks_o = out["blocks"].clone()
    plan = {}
    for b in seqs:
        seq = Sequence(inp, b, fp8=fp8)
        # preprocessing: compressed keys, quantisation, pooling are bit-exact
        if fp8:
            np.testing.assert_array_equal(dev["k"][b].cpu().numpy(), seq.k_codes, err_msg="E4M3 key codes")
            np.testing.assert_array_equal(dev["k_scale"][b].cpu().numpy(), seq.k_scale, err_msg="key scales")
            np.testing.assert_array_equal(dev["q"][b].cpu().numpy(), seq.q_codes, err_msg="E4M3 q codes")
            np.testing.assert_array_equal(dev["q_scale"][b].cpu().numpy(), seq.q_scale, err_msg="q scales")
            np.testing.assert_array_equal(out["kpool"][b].cpu().numpy(), seq.kpool_codes, err_msg="pooled codes")
            np.testing.assert_array_equal(out["kps"][b].cpu().numpy(), seq.kpool_scale, err_msg="pooled scales")
        else:
            np.testing.assert_array_equal(_dev_float(dev["k"][b]), seq.keys, err_msg="keys after compression")
            np.testing.assert_array_equal(_dev_float(out["kpool"][b]), seq.kpool, err_msg="pooled keys")
        ts = _sample_queries(wl, queries_per_seq, seed=b)
        plan[b] = (seq, ts)
        for t in ts:
            ob = seq.blocks(t)
            row = np.full(wl.top_m, -1, np.int32)
            row[:len(ob)] = ob
            blocks_o[b, t] = torch.from_numpy(row).to(blocks_o.device)
    tok_o, tok_o_sc = hb.hisa_token_score_topk(dev["q"], dev["w"], dev["k"], dev["n_visible"], blocks_o,
                                               block_size=wl.block_size, top_k=wl.top_k, q_scale=dev["q_scale"],
                                               k_scale=dev["k_scale"], want_scores=True)
    hb.get_status()
    g = {k: v.cpu().numpy() for k, v in out.items() if k in ("blocks", "tok", "tok_sc", "flat", "flat_sc")}
    tok_o, tok_o_sc = tok_o.cpu().numpy(), tok_o_sc.cpu().numpy()
    for b, (seq, ts) in plan.items():
        for t in ts:
            nt = int(seq.n_visible[t])
            what = f"{wl.name}{'/fp8' if fp8 else ''} seq {b} query {t} (n={nt})"
            stats["queries"] += 1
            # --- coarse stage
            gb = [int(x) for x in g["blocks"][b, t] if x >= 0]
            ob = seq.blocks(t).tolist()
            c = ho.current_block(nt, wl.block_size)
            if c >= 0:
                assert c in gb, f"{what}: current block {c} missing from {gb}"
                bs = seq.block_scores(t)
                stats["swaps_block"] += parity.check_selection(
                    [x for x in gb if x != c], np.arange(c), bs, wl.top_m - 1, what + " blocks")
            else:
                assert gb == [], what
            # --- refinement stage on the oracle's blocks
            cand = ho.candidate_keys(np.asarray(ob, np.int64), nt, wl.block_size)
            cs = seq.scores(t, cand) if len(cand) else np.zeros(0)
            gi = tok_o[b, t]
            assert np.all(gi[min(wl.top_k, len(cand)):] == -1), f"{what}: padding"
            stats["swaps_tok"] += parity.check_selection(gi[gi >= 0], cand, cs, wl.top_k, what + " tokens")
            parity.check_scores(gi, tok_o_sc[b, t], lambda ix: seq.scores(t, ix), rtol, what + " token scores")
            # --- whole HISA pipeline (GPU blocks)
            hi = g["tok"][b, t]
            if sorted(gb) == sorted(ob):
                stats["swaps_tok"] += parity.check_selection(hi[hi >= 0], cand, cs, wl.top_k, what + " pipeline")
            else:
                stats["block_mismatch"] += 1
                gc = set(ho.candidate_keys(np.asarray(gb, np.int64), nt, wl.block_size).tolist())
                sel = hi[hi >= 0].tolist()
                assert set(sel) <= gc and len(set(sel)) == len(sel) == min(wl.top_k, len(gc)), what
            # --- flat
            fcand = np.arange(nt)
            fs = seq.scores(t, fcand) if nt else np.zeros(0)
            fi = g["flat"][b, t]
            assert np.all(fi[min(wl.top_k, nt):] == -1), f"{what}: flat padding"
            stats["swaps_flat"] += parity.check_selection(fi[fi >= 0], fcand, fs, wl.top_k, what + " flat")
            parity.check_scores(fi, g["flat_sc"][b, t], lambda ix: seq.scores(t, ix), rtol, what + " flat scores")
            stats["iou"].append(parity.iou(hi, fi))
            stats["recall"].append(parity.recall(hi, fi))
            stats["negative_scores"] += int(np.sum(g["flat_sc"][b, t][fi >= 0] < 0))
    stats["mean_iou"] = float(np.mean(stats["iou"])) if stats["iou"] else 1.0
    stats["mean_recall"] = float(np.mean(stats["recall"])) if stats["recall"] else 1.0
    del stats["iou"], stats["recall"]
    print(f"\n[parity] {wl.name}{'/fp8' if fp8 else ''}: {stats}")
    return stats


@pytest.mark.parametrize("name", sorted(SMALL))
def test_small_parity(lib, name):
    inp = _inputs((name, tuple(sorted(SMALL[name].items()))))
    stats = _check_workload(inp, fp8=False, queries_per_seq=120)
    if SMALL[name].get("w_low", 0.0) < 0 and SMALL[name].get("first_query_pos", 0) == 0:
        # early causal queries see fewer keys than k, so some selected scores are negative
        assert stats["negative_scores"] > 0, "signed weights should give some negative selected scores"


@pytest.mark.parametrize("name", ["ragged_bf16", "batch_tail"])
def test_small_parity_fp8(lib, name):
    inp = _inputs((name, tuple(sorted(SMALL[name].items()))))
    _check_workload(inp, fp8=True, queries_per_seq=80)


def test_tiny_workload_every_query(lib):
    """The 1x1024 fp32 workload, every query; m = all 16 blocks gives flat."""
    from hierarchical_top_key_b200 import binding as hb
    inp = _inputs(("tiny", ()))
    wl = inp.workload
    stats = _check_workload(inp, fp8=False, queries_per_seq=1024)
    assert stats["queries"] == 1024
    dev = hb.to_device_inputs(inp)
    ix = hb.HisaIndexer(wl.block_size, 16, wl.top_k)
    hi, _ = ix(dev["q"], dev["w"], dev["k"], dev["n_visible"])
    fi, _ = hb.dsa_flat_indexer_topk(dev["q"], dev["w"], dev["k"], dev["n_visible"], top_k=wl.top_k)
    hs = np.sort(hi.cpu().numpy(), axis=-1)
    fs = np.sort(fi.cpu().numpy(), axis=-1)
    np.testing.assert_array_equal(hs, fs)


FULL = ["prefill_32k", "chunk_64k", "decode_128k", "compressed_256k"]


# sampled queries per sequence at full size: first, last, around block
# boundaries and random ones (every sequence of the decode workload)
FULL_SAMPLES = {"prefill_32k": 512, "chunk_64k": 96, "decode_128k": 1, "compressed_256k": 96}


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled(lib, name):
    inp = _inputs((name, ()))
    stats = _check_workload(inp, fp8=False, queries_per_seq=FULL_SAMPLES[name])
    if inp.workload.batch > 1:
        assert stats["queries"] == inp.workload.batch


def test_full_size_fp8_chunk_64k(lib):
    inp = _inputs(("chunk_64k", ()))
    _check_workload(inp, fp8=True, queries_per_seq=6)
