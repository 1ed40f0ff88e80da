"""Benchmark of the HISA indexer (one layer) on one or more B200s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--fp8]
    python bench.py --impl reference ...     # the CPU oracle on this host's cores

A step is one pass of the HISA indexer over the workload's synthetic inputs
already resident in HBM: block pooling, coarse block scoring with top-m
selection, and the fused refinement scoring with top-k (for the compressed
workload the 4:1 key compression runs first).  The flat DSA indexer is timed
on the same inputs right after, for the HISA/flat speedup.  Rank 0 prints one
JSON line.

Multi-GPU (torchrun): every rank runs an independent replica of the workload
(its own seed); there is no data-path collective.  value = all ranks' queries
/ max-over-ranks time ("weak" scaling).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from hierarchical_top_key_b200 import synthetic  # noqa: E402

DEFAULT_WORKLOAD = "prefill_32k"
FLOP_PER_PAIR_PER_HEAD_DIM = 2          # one multiply-add per (head, feature) per (query, key) pair
L2_FLUSH_BYTES = 256 << 20               # larger than the 126 MB L2

# DRAM bytes (read + write) per launch of the refinement kernel from an ncu
# capture of the same kernel build and workload (see profiles/); a workload
# missing here reports null.  Empty: the kernel gained paged-key support after
# the last capture (796,417,792 B per launch at prefill_32k), so that figure
# no longer describes the kernel the bench times.
NCU_TRAFFIC = {}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synthetic.WORKLOADS))
    ap.add_argument("--fp8", action="store_true", help="E4M3 q/k with per-token scales")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the CPU-oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-flat", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--superblock-group", type=int, default=0,
                    help="also time the three-level indexer with super-blocks of this many blocks")
    ap.add_argument("--top-m2", type=int, default=8, help="super-blocks kept by the three-level indexer")
    return ap.parse_args()


# ------------------------------------------------------------------ helpers


def candidate_pairs(wl, n_visible: np.ndarray) -> int:
    """Sum over queries of |C_t|: keys of the retained blocks that are visible
    (m-1 full blocks before the current one, or all of them, plus the
    visible part of the current block)."""
    n = n_visible.astype(np.int64).ravel()
    B, m = wl.block_size, wl.top_m
    c = np.where(n > 0, (n - 1) // B, -1)
    full = np.minimum(c, m - 1)
    return int(np.sum(np.where(n > 0, full * B + (n - c * B), 0)))


def block_pairs(wl, n_visible: np.ndarray) -> int:
    n = n_visible.astype(np.int64).ravel()
    return int(np.sum(np.where(n > 0, (n - 1) // wl.block_size, 0)))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.5)              # let the sampler start before the timed region
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def oracle_sequence(inp, fp8: bool):
    from oracle.run import Sequence
    t0 = time.perf_counter()
    seq = Sequence(inp, 0, fp8=fp8)
    return seq, time.perf_counter() - t0


def cpu_oracle_rate(inp, fp8: bool, budget_s: float, which: str = "hisa", prepared=None):
    """Time the CPU oracle, as it stands, on a seeded random sample of the
    workload's queries until `budget_s` is spent.  Returns (queries/s, sample
    description, threads)."""
    try:
        import threadpoolctl
        threads = max((i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()), default=1)
    except Exception:
        threads = 1
    wl = inp.workload
    seq, prep = prepared if prepared is not None else oracle_sequence(inp, fp8)
    # a seeded shuffle of all queries: any prefix of it is spread over the sequence
    order = np.random.default_rng(1).permutation(wl.num_queries)
    done = 0
    t0 = time.perf_counter()
    for t in order:
        if which == "hisa":
            seq.hisa(int(t))
        else:
            seq.flat(int(t))
        done += 1
        if time.perf_counter() - t0 > budget_s and done >= 4:
            break
    el = time.perf_counter() - t0
    rate = done / el
    desc = (f"{which} oracle on {done} of {wl.num_queries} queries of sequence 0 (seeded random sample), "
            f"{el:.1f} s; key preprocessing {prep:.1f} s untimed; rate scaled to queries/s")
    return rate, desc, threads


# ------------------------------------------------------------------ reference arm


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = synthetic.WORKLOADS[args.workload]
    inp = synthetic.generate(wl, args.seed, batch=1)
    budget = max(2.0, args.cpu_seconds / max(1, args.steps + args.warmup))
    prepared = oracle_sequence(inp, args.fp8)
    rates = []
    for i in range(args.warmup + args.steps):
        r, desc, threads = cpu_oracle_rate(inp, args.fp8, budget, prepared=prepared)
        if i >= args.warmup:
            rates.append(r)
    value = float(np.mean(rates))
    line = {
        "impl": "reference", "metric": "hisa_indexer_queries_per_s", "value": value, "unit": "queries/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * wl.num_queries * wl.batch / value, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, args.fp8),
        "cpu_baseline": {"value": value, "unit": "queries/s", "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def workload_config(wl, fp8):
    return {"workload": wl.name + ("_fp8" if fp8 else ""), "batch": wl.batch, "keys": wl.num_keys,
            "raw_keys": wl.raw_keys, "queries_per_seq": wl.num_queries, "first_query_pos": wl.first_query_pos,
            "heads": wl.heads, "head_dim": wl.head_dim, "block_size": wl.block_size, "top_m": wl.top_m,
            "top_k": wl.top_k, "l2": "flushed between steps (256 MiB write, outside the timed events)"}


def graph_ms(step, steps, flush, stream):
    """Mean device time of `step` replayed from a CUDA graph (launch-bound
    decode steps: no host work between the kernels), L2 flushed between
    replays outside the timed events."""
    import torch
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()                                   # warm the allocator on the capture stream
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(g, capture_error_mode="relaxed"):
        step()
    g.replay()
    torch.cuda.synchronize()
    evs = []
    for _ in range(steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    del g
    return ms


# ------------------------------------------------------------------ ranks


def replica_seed(seed: int, rank: int) -> int:
    """Each rank runs its own independent replica of the workload."""
    return seed + rank


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest of every rank's `x` (the job is as slow as its slowest rank)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / (ms_max / 1000.0)


# ------------------------------------------------------------------ our arm


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    import torch
    import torch.distributed as dist
    from hierarchical_top_key_b200 import binding as hb

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    wl = synthetic.WORKLOADS[args.workload]
    inp = synthetic.generate(wl, replica_seed(args.seed, rank))
    hb.load()
    stream = torch.cuda.current_stream()
    fp8 = args.fp8

    # ---- resident inputs
    d = hb.to_device_inputs(inp, device=dev, fp8=False, compress=False)
    raw_k = d["k"]

    def prep_keys():
        k = hb.hisa_compress_keys(raw_k, wl.compress_ratio) if wl.compress_ratio > 1 else raw_k
        if fp8:
            return hb.hisa_quantize_e4m3(k, 2)
        return k, None

    q, qs = (hb.hisa_quantize_e4m3(d["q"], 2) if fp8 else (d["q"], None))
    w, nv = d["w"], d["n_visible"]
    k_static, ks_static = prep_keys()
    indexer = hb.HisaIndexer(wl.block_size, wl.top_m, wl.top_k)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def step(stage_events=None):
        # compressed-key workloads recompress the raw keys every step (part of the path)
        if wl.compress_ratio > 1:
            k = hb.hisa_compress_keys(raw_k, wl.compress_ratio)
            ks = None
            if fp8:
                k, ks = hb.hisa_quantize_e4m3(k, 2)
        else:
            k, ks = k_static, ks_static
        if stage_events is None:
            return indexer(q, w, k, nv, q_scale=qs, k_scale=ks)
        e = stage_events
        e[0].record(stream)
        kpool, kps = hb.hisa_pool_blocks(k, wl.block_size, ks)
        e[1].record(stream)
        blocks = hb.hisa_block_score_topm(q, w, kpool, nv, num_keys=k.shape[1], block_size=wl.block_size,
                                          top_m=wl.top_m, q_scale=qs, kpool_scale=kps, workspace=ws_block)
        e[2].record(stream)
        out = hb.hisa_token_score_topk(q, w, k, nv, blocks, block_size=wl.block_size, top_k=wl.top_k,
                                       q_scale=qs, k_scale=ks)
        e[3].record(stream)
        return out

    shape = hb.make_shape(q, k_static, wl.block_size, wl.top_m, wl.top_k)
    ws_block = torch.empty(max(16, hb.workspace_size(hb.OP_BLOCK, shape)), dtype=torch.uint8, device=dev)
    ws_flat = None if args.no_flat else torch.empty(max(16, hb.workspace_size(hb.OP_FLAT, shape)),
                                                   dtype=torch.uint8, device=dev)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
        flush.zero_()
    hb.get_status()
    barrier()

    # ---- timed region: K steps, per-step events (L2 flush between steps, outside the events)
    stage_evs = [[ev() for _ in range(4)] for _ in range(args.steps)]
    step_evs = [(ev(), ev()) for _ in range(args.steps)]
    with ClockSampler(local) as clocks:
        barrier()
        for i in range(args.steps):
            flush.zero_()
            step_evs[i][0].record(stream)
            step(stage_evs[i])
            step_evs[i][1].record(stream)
        barrier()
    hb.get_status()
    step_ms = [a.elapsed_time(b) for a, b in step_evs]
    stage_ms = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(3)] for e in stage_evs])
    ms = float(np.mean(step_ms))
    ms_max = max_over_ranks(ms, world, dev)
    queries = wl.batch * wl.num_queries
    value = job_rate(queries, world, ms_max)

    # ---- flat DSA indexer on the same inputs
    flat = None
    if not args.no_flat:
        for _ in range(max(1, args.warmup)):
            hb.dsa_flat_indexer_topk(q, w, k_static, nv, top_k=wl.top_k, q_scale=qs, k_scale=ks_static,
                                     workspace=ws_flat)
        barrier()
        fms = []
        for i in range(max(1, min(args.steps, 5))):
            flush.zero_()
            a, b = ev(), ev()
            a.record(stream)
            hb.dsa_flat_indexer_topk(q, w, k_static, nv, top_k=wl.top_k, q_scale=qs, k_scale=ks_static,
                                     workspace=ws_flat)
            b.record(stream)
            fms.append((a, b))
        barrier()
        hb.get_status()
        fm = float(np.mean([a.elapsed_time(b) for a, b in fms]))
        nvis = inp.n_visible
        flat_flops = FLOP_PER_PAIR_PER_HEAD_DIM * wl.heads * wl.head_dim * float(np.minimum(nvis, wl.num_keys).sum())
        flat = {"ms_per_layer": fm, "queries_per_s": queries / (fm / 1000.0),
                "hisa_speedup": fm / ms, "score_tflops": flat_flops / (fm / 1000.0) / 1e12}
        # the sampled-threshold flat path (same result, smaller workspace), for comparison
        try:
            ws_s = torch.empty(max(16, hb.workspace_size(hb.OP_FLAT_SAMPLED, shape)), dtype=torch.uint8, device=dev)
        except hb.HisaError:
            ws_s = None
        if ws_s is not None:
            hb.dsa_flat_indexer_topk_sampled(q, w, k_static, nv, top_k=wl.top_k, q_scale=qs, k_scale=ks_static,
                                             workspace=ws_s)
            barrier()
            sms_ = []
            for i in range(max(1, min(args.steps, 5))):
                flush.zero_()
                a, b = ev(), ev()
                a.record(stream)
                hb.dsa_flat_indexer_topk_sampled(q, w, k_static, nv, top_k=wl.top_k, q_scale=qs, k_scale=ks_static,
                                                 workspace=ws_s)
                b.record(stream)
                sms_.append((a, b))
            barrier()
            hb.get_status()
            flat["sampled_ms_per_layer"] = float(np.mean([a.elapsed_time(b) for a, b in sms_]))
            flat["sampled_workspace_bytes"] = int(ws_s.numel())
            flat["workspace_bytes"] = int(ws_flat.numel())
            del ws_s

    # ---- decode with the pooled keys kept between steps: each step pools only
    # the block its new key completes (the coarse stage scores complete blocks)
    cached = None
    if wl.num_queries == 1 and wl.compress_ratio == 1 and not fp8:
        nb = -(-wl.num_keys // wl.block_size)
        kcache, _ = hb.hisa_pool_blocks(k_static, wl.block_size)      # built by earlier steps (untimed)

        def cached_step():
            hb.hisa_pool_blocks_range(k_static, wl.block_size, nb - 1, 1, kcache)
            blocks = hb.hisa_block_score_topm(q, w, kcache, nv, num_keys=k_static.shape[1],
                                              block_size=wl.block_size, top_m=wl.top_m, workspace=ws_block)
            return hb.hisa_token_score_topk(q, w, k_static, nv, blocks, block_size=wl.block_size, top_k=wl.top_k)

        for _ in range(max(3, args.warmup)):
            cached_step()
        barrier()
        cev = []
        for i in range(args.steps):
            flush.zero_()
            a, b = ev(), ev()
            a.record(stream)
            cached_step()
            b.record(stream)
            cev.append((a, b))
        barrier()
        hb.get_status()
        cm = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in cev])), world, dev)
        cg = max_over_ranks(graph_ms(cached_step, args.steps, flush, stream), world, dev)
        cached = {"ms_per_layer": cm, "queries_per_s": job_rate(queries, world, cm),
                  "hisa_speedup": (flat["ms_per_layer"] / cm) if flat else None,
                  "graph_ms_per_layer": cg, "graph_hisa_speedup": (flat["ms_per_layer"] / cg) if flat else None,
                  "what": "pooled keys of complete blocks kept between decode steps; a step pools the one block "
                          "its new key completes, then scores blocks and refines"}
        if wl.num_keys % wl.block_size == 0:
            # the same step over paged keys: one page per block, pages shuffled
            bsz = k_static.shape[0]
            gen = torch.Generator(device="cpu").manual_seed(7)
            perm = torch.randperm(bsz * nb, generator=gen).to(torch.int32).to(k_static.device)
            table = perm.view(bsz, nb).contiguous()
            pages = torch.empty((bsz * nb, wl.block_size, wl.head_dim), dtype=k_static.dtype, device=k_static.device)
            pages[perm.long()] = k_static.view(bsz * nb, wl.block_size, wl.head_dim)
            pcache = kcache.clone()

            def paged_step():
                hb.hisa_pool_blocks_paged(pages, table, num_keys=k_static.shape[1], first_block=nb - 1,
                                          block_count=1, kpool=pcache)
                blocks = hb.hisa_block_score_topm(q, w, pcache, nv, num_keys=k_static.shape[1],
                                                  block_size=wl.block_size, top_m=wl.top_m, workspace=ws_block)
                return hb.hisa_token_score_topk_paged(q, w, pages, table, nv, blocks, num_keys=k_static.shape[1],
                                                      top_k=wl.top_k)

            for _ in range(max(3, args.warmup)):
                paged_step()
            same = bool(torch.equal(torch.sort(paged_step()[0], dim=-1)[0], torch.sort(cached_step()[0], dim=-1)[0]))
            hb.get_status()
            cached["paged_graph_ms_per_layer"] = max_over_ranks(graph_ms(paged_step, args.steps, flush, stream),
                                                                world, dev)
            cached["paged_matches_contiguous"] = same
            del pages, pcache

    # ---- three levels: pooled super-blocks -> blocks -> tokens
    three = None
    if args.superblock_group > 0 and not fp8 and wl.compress_ratio == 1:
        G3 = args.superblock_group
        ix3 = hb.HisaIndexer3(wl.block_size, G3, args.top_m2, wl.top_m, wl.top_k)
        for _ in range(max(3, args.warmup)):
            ix3(q, w, k_static, nv)
        barrier()
        tev = []
        for i in range(args.steps):
            flush.zero_()
            a, b = ev(), ev()
            a.record(stream)
            idx3 = ix3(q, w, k_static, nv)
            b.record(stream)
            tev.append((a, b))
        barrier()
        hb.get_status()
        tm = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in tev])), world, dev)
        # overlap with the two-level and the flat indices on a sample of queries
        idx2, _ = indexer(q, w, k_static, nv)
        rows = np.random.default_rng(3).choice(wl.batch * wl.num_queries, min(256, wl.batch * wl.num_queries),
                                               replace=False)
        r3 = idx3.reshape(-1, wl.top_k)[torch.as_tensor(rows, device=dev)].cpu().numpy()
        r2 = idx2.reshape(-1, wl.top_k)[torch.as_tensor(rows, device=dev)].cpu().numpy()
        iou = lambda x, y: len(set(x[x >= 0]) & set(y[y >= 0])) / max(1, len(set(x[x >= 0]) | set(y[y >= 0])))  # noqa: E731
        three = {"group": G3, "top_m2": args.top_m2, "ms_per_layer": tm, "queries_per_s": job_rate(queries, world, tm),
                 "hisa_speedup": (flat["ms_per_layer"] / tm) if flat else None,
                 "iou_vs_two_level": float(np.mean([iou(r3[i], r2[i]) for i in range(len(rows))]))}
        if not args.no_flat:
            fidx, _ = hb.dsa_flat_indexer_topk(q, w, k_static, nv, top_k=wl.top_k, workspace=ws_flat)
            rf = fidx.reshape(-1, wl.top_k)[torch.as_tensor(rows, device=dev)].cpu().numpy()
            three["iou_vs_flat"] = float(np.mean([iou(r3[i], rf[i]) for i in range(len(rows))]))
            three["two_level_iou_vs_flat"] = float(np.mean([iou(r2[i], rf[i]) for i in range(len(rows))]))
        if wl.num_queries == 1:
            # decode with both pooled levels cached: a step pools the block and the
            # super-block its new key completes
            nb = -(-wl.num_keys // wl.block_size)
            nb2 = -(-wl.num_keys // (wl.block_size * G3))
            kc, _ = hb.hisa_pool_blocks(k_static, wl.block_size)
            kc2, _ = hb.hisa_pool_blocks(k_static, wl.block_size * G3)

            def cached3():
                hb.hisa_pool_blocks_range(k_static, wl.block_size, nb - 1, 1, kc)
                hb.hisa_pool_blocks_range(k_static, wl.block_size * G3, nb2 - 1, 1, kc2)
                return ix3(q, w, k_static, nv, kpool=(kc, None), kpool2=(kc2, None))

            for _ in range(3):
                cached3()
            barrier()
            cev3 = []
            for i in range(args.steps):
                flush.zero_()
                a, b = ev(), ev()
                a.record(stream)
                cached3()
                b.record(stream)
                cev3.append((a, b))
            barrier()
            hb.get_status()
            three["cached_ms_per_layer"] = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in cev3])),
                                                          world, dev)
            three["cached_graph_ms_per_layer"] = max_over_ranks(graph_ms(cached3, args.steps, flush, stream),
                                                                world, dev)

    # ---- end to end through the public API with pinned host buffers
    e2e = None
    if not args.no_e2e:
        # the user's view: bf16/fp32 q, raw keys, w and n_visible in pinned host memory
        hq = d["q"].cpu().pin_memory()
        hk = raw_k.cpu().pin_memory()
        hw, hnv = w.cpu().pin_memory(), nv.cpu().pin_memory()
        out_host = torch.empty((wl.batch, wl.num_queries, wl.top_k), dtype=torch.int32).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hw, hnv))
        d2h = out_host.numel() * out_host.element_size()

        pipelined = wl.compress_ratio == 1 and not fp8

        def e2e_step():
            if pipelined:
                # the host-buffer entry point: copies in, kernels and copies out overlap piece by piece
                indexer.from_host(hq, hw, hk, hnv, out_host)
                return
            dq = hq.to(dev, non_blocking=True)
            dk = hk.to(dev, non_blocking=True)
            dw, dnv = hw.to(dev, non_blocking=True), hnv.to(dev, non_blocking=True)
            kk = hb.hisa_compress_keys(dk, wl.compress_ratio) if wl.compress_ratio > 1 else dk
            dqs = kks = None
            if fp8:
                dq, dqs = hb.hisa_quantize_e4m3(dq, 2)
                kk, kks = hb.hisa_quantize_e4m3(kk, 2)
            idx, _ = indexer(dq, dw, kk, dnv, q_scale=dqs, k_scale=kks)
            out_host.copy_(idx, non_blocking=True)

        e2e_step()
        barrier()
        evs = []
        for i in range(max(1, min(args.steps, 5))):
            a, b = ev(), ev()
            a.record(stream)
            e2e_step()
            b.record(stream)
            evs.append((a, b))
        barrier()
        em = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in evs])), world, dev)
        e2e = {"value": job_rate(queries, world, em), "unit": "queries/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": em,
               "api": "HisaIndexer.from_host (pipelined host buffers)" if pipelined else
                      "host copies, then the device entry points"}

    # ---- roofline of the dominant kernel (the fused refinement stage)
    peaks = load_peaks()
    pairs = candidate_pairs(wl, inp.n_visible)
    tok_ms = float(np.mean(stage_ms[:, 2]))
    tok_flops = FLOP_PER_PAIR_PER_HEAD_DIM * wl.heads * wl.head_dim * pairs
    achieved = tok_flops / (tok_ms / 1000.0) / 1e12
    peak = peaks["bf16_sustained"] * (2.0 if fp8 else 1.0)
    key = wl.name + ("_fp8" if fp8 else "")
    roofline = {"kernel": "hisa_token_stage", "bound": "tensor", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "traffic": NCU_TRAFFIC.get(key),
                "peak_source": f"{peaks['source']} bf16 sustained" + (" x2 for e4m3 (nominal ratio)" if fp8 else ""),
                "algorithmic": f"{FLOP_PER_PAIR_PER_HEAD_DIM * wl.heads * wl.head_dim} flop per candidate pair x "
                               f"{pairs} pairs per launch"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r, desc, threads = cpu_oracle_rate(inp, fp8, args.cpu_seconds)
        cpu = {"value": r, "unit": "queries/s", "cores": threads, "kind": "oracle", "sample": desc}

    if rank == 0:
        # pool + coarse scoring + coarse selection + refinement, plus compression
        # (and its E4M3 quantisation) for compressed-key workloads
        launches_per_step = 4 + (1 if wl.compress_ratio > 1 else 0) + (1 if fp8 and wl.compress_ratio > 1 else 0)
        line = {
            "metric": "hisa_indexer_queries_per_s", "value": value, "unit": "queries/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3" if fp8 else wl.dtype, "data": "synthetic",
            "config": workload_config(wl, fp8),
            "stages_ms": {"pool": float(np.mean(stage_ms[:, 0])), "block_score_topm": float(np.mean(stage_ms[:, 1])),
                          "token_score_topk": tok_ms},
            "flat": flat, "pooled_keys_cached": cached, "three_level": three, "roofline": roofline,
            "cpu_baseline": cpu, "e2e": e2e,
            "clocks": clocks.summary(), "gpu_launches": launches_per_step * args.steps,
        }
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
