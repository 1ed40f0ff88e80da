"""Benchmark of the HISA indexer (one layer) on one or more B200s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--fp8]
                    [--split sequences|queries]
    python bench.py --impl reference ...     # the CPU oracle on this host's cores

A step is one pass of the HISA indexer over the workload's synthetic inputs
already resident in HBM: block pooling, coarse block scoring with top-m
selection, and the fused refinement scoring with top-k (for the compressed
workload the 4:1 key compression runs first).  The flat DSA indexer is timed
on the same inputs right after, for the HISA/flat speedup, and the overlap of
the two index sets (mean IoU and recall against flat) is measured on sampled
queries.  With one GPU the line also carries the other long-context workloads
(`workloads`: the 64K chunk in bf16 and E4M3, the 128K decode step with
pooling and with cached pooled keys), each with its speedup and overlap.
Rank 0 prints one JSON line.

Multi-GPU (torchrun), two ways to shard a job over the ranks (no collective
inside the indexer: queries are independent once keys are present):
  --split sequences  (default, weak scaling) the job holds N times the
                     workload's sequences; each rank runs its own whole
                     sequences.
  --split queries    (strong scaling) one workload is split over the ranks by
                     causal work (query ranges of a sequence, or whole
                     sequences when there are several); the step ends with one
                     NCCL all-gather that assembles [batch, Q, top_k] on every
                     rank.
value = all ranks' queries / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import hashlib
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

from hierarchical_top_key_b200 import partition, synthetic  # noqa: E402

DEFAULT_WORKLOAD = "prefill_32k"
FLOP_PER_PAIR_PER_HEAD_DIM = 2          # one multiply-add per (head, feature) per (query, key) pair
L2_FLUSH_BYTES = 256 << 20               # larger than the 126 MB L2
OVERLAP_SAMPLE = 256                     # queries on which HISA's indices are compared with flat's
EXTRA_WORKLOADS = (("chunk_64k", False), ("chunk_64k", True), ("decode_128k", False))

# DRAM bytes (read + write) per launch of the refinement kernel, from a
# single-launch ncu capture (dram__bytes_read.sum + dram__bytes_write.sum) of
# the same command and workload; see profiles/.  `src` is the hash of the
# kernel sources it was taken on: when the sources change the figure no longer
# describes the kernel and the bench reports null.
NCU_TRAFFIC = {
    # ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum --clock-control none
    #     -k regex:token_tc -c 1 python bench.py --steps 1 --warmup 1 --no-flat --no-e2e --no-extra
    #     --no-cpu-baseline --no-attention   (558,077,696 B read + 240,869,888 B written)
    "prefill_32k": {"bytes": 798947584, "src": "1ad483dea849cdd3"},
}
KERNEL_SOURCES = ("token_tc.cuh", "sm100.cuh", "select.cuh", "common.cuh")


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synthetic.WORKLOADS))
    ap.add_argument("--fp8", action="store_true", help="E4M3 q/k with per-token scales")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--split", default="sequences", choices=["sequences", "queries"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the CPU-oracle sample")
    ap.add_argument("--ref-seconds", type=float, default=60.0, help="reference arm: CPU seconds for all its steps")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-flat", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads")
    ap.add_argument("--no-attention", action="store_true", help="skip the attention over the selected keys")
    ap.add_argument("--attention-only", type=int, default=0, metavar="Q",
                    help="time only the attention over the selected keys on Q queries x top_k random positions of "
                         "the workload's keys (a small case for profilers), print one line and exit")
    ap.add_argument("--superblock-group", type=int, default=0,
                    help="also time the three-level indexer with super-blocks of this many blocks")
    ap.add_argument("--top-m2", type=int, default=8, help="super-blocks kept by the three-level indexer")
    return ap.parse_args(argv)


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


def kernel_sources_hash() -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "hierarchical_top_key_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


def overlap_stats(hisa_rows: np.ndarray, flat_rows: np.ndarray) -> dict:
    """Mean IoU and mean recall (|HISA & flat| / |flat|) of index rows (-1 = none)."""
    ious, recs = [], []
    for h, f in zip(hisa_rows, flat_rows):
        a, b = set(int(x) for x in h if x >= 0), set(int(x) for x in f if x >= 0)
        inter = len(a & b)
        ious.append(1.0 if not (a or b) else inter / len(a | b))
        recs.append(1.0 if not b else inter / len(b))
    return {"mean_iou_vs_flat": float(np.mean(ious)), "mean_recall_vs_flat": float(np.mean(recs)),
            "min_recall_vs_flat": float(np.min(recs)), "queries_compared": len(ious)}


def sample_rows(total: int, n: int, seed: int = 3) -> np.ndarray:
    if total <= n:
        return np.arange(total)
    return np.sort(np.random.default_rng(seed).choice(total, n, replace=False))


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


def oracle_threads() -> int:
    try:
        import threadpoolctl
        return max((i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()), default=1)
    except Exception:
        return 1


def cpu_oracle_rate(inp, fp8: bool, budget_s: float, which: str = "hisa", prepared=None):
    """Time the CPU oracle, as it stands, on a seeded random sample of the
    workload's queries until `budget_s` is spent.  Returns (queries/s, sample
    description, threads)."""
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
    return rate, desc, oracle_threads()


# ------------------------------------------------------------------ reference arm


def run_reference(args):
    """The oracle as it stands, on this host's cores.  A step is the oracle's
    HISA indexer on one fixed seeded sample of the workload's queries (the
    same sample every step), sized during the warm-up so that all steps take
    about --ref-seconds; ms_per_step is the measured wall time of that step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = synthetic.WORKLOADS[args.workload]
    inp = synthetic.generate(wl, args.seed, batch=1)
    seq, prep = oracle_sequence(inp, args.fp8)
    order = np.random.default_rng(1).permutation(wl.num_queries)
    # calibrate the sample size on the first warm-up step (or a 1 s probe)
    per_step_s = max(0.5, args.ref_seconds / max(1, args.steps + args.warmup))
    t0 = time.perf_counter()
    n = 0
    while time.perf_counter() - t0 < min(1.0, per_step_s) or n < 4:
        seq.hisa(int(order[n % len(order)]))
        n += 1
    rate0 = n / (time.perf_counter() - t0)
    sample = order[:max(4, min(len(order), int(rate0 * per_step_s)))]

    def step():
        for t in sample:
            seq.hisa(int(t))

    for _ in range(args.warmup):
        step()
    times = []
    for _ in range(args.steps):
        a = time.perf_counter()
        step()
        times.append(time.perf_counter() - a)
    ms = 1000.0 * float(np.mean(times))
    value = len(sample) / (ms / 1000.0)
    threads = oracle_threads()
    desc = (f"hisa oracle (float64 numpy) on a fixed seeded sample of {len(sample)} of the {wl.num_queries} "
            f"queries of sequence 0 per step; ms_per_step is the wall time of that sample; key "
            f"preprocessing {prep:.1f} s untimed")
    line = {
        "impl": "reference", "metric": "hisa_indexer_queries_per_s", "value": value, "unit": "queries/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_config(wl, args.fp8), queries_per_step=int(len(sample))),
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


def timed(fn, steps, flush, stream):
    """Mean CUDA-event time of fn() over `steps` calls, L2 flushed before each
    call outside the events."""
    import torch
    evs = []
    for _ in range(steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    return float(np.mean([a.elapsed_time(b) for a, b in evs]))


# ------------------------------------------------------------------ ranks


def replica_seed(seed: int, rank: int) -> int:
    """With --split sequences each rank draws its own sequences of the job."""
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


def gather_shards(idx, shards, batch: int, Q: int, top_k: int, world: int):
    """Assemble the [batch, Q, top_k] index tensor from every rank's shard
    (one all-gather of equal-size padded blocks, then the shards in rank
    order).  Works on any backend with all_gather_into_tensor (NCCL, gloo)."""
    import torch
    import torch.distributed as dist
    rows = [s.rows for s in shards]
    R = max(max(rows), 1)
    mine = torch.full((R, top_k), -1, dtype=torch.int32, device=idx.device)
    mine[:idx.numel() // top_k] = idx.reshape(-1, top_k)
    allb = torch.empty((world * R, top_k), dtype=torch.int32, device=idx.device)
    if world > 1:
        dist.all_gather_into_tensor(allb, mine)
    else:
        allb.copy_(mine)
    parts = [allb[r * R:r * R + rows[r]] for r in range(world)]
    out = torch.empty((batch, Q, top_k), dtype=torch.int32, device=idx.device)
    for s, p in zip(shards, parts):
        if s.rows:
            out[s.seq0:s.seq1, s.t0:s.t1] = p.view(s.seq1 - s.seq0, s.t1 - s.t0, top_k)
    return out


# ------------------------------------------------------------------ one workload on this GPU


class Run:
    """One workload's inputs on this GPU (a shard of them with --split
    queries) and the HISA / flat steps over them."""

    def __init__(self, hb, wl, fp8, seed, dev, shard=None):
        import torch
        self.hb, self.wl, self.fp8, self.dev = hb, wl, fp8, dev
        self.inp = synthetic.generate(wl, seed)
        d = hb.to_device_inputs(self.inp, device=dev, fp8=False, compress=False)
        q, w, nv, raw_k = d["q"], d["w"], d["n_visible"], d["k"]
        nvh = self.inp.n_visible
        if shard is not None:
            q = q[shard.seq0:shard.seq1, shard.t0:shard.t1].contiguous()
            w = w[shard.seq0:shard.seq1, shard.t0:shard.t1].contiguous()
            nv = nv[shard.seq0:shard.seq1, shard.t0:shard.t1].contiguous()
            raw_k = raw_k[shard.seq0:shard.seq1].contiguous()
            nvh = nvh[shard.seq0:shard.seq1, shard.t0:shard.t1]
        self.n_visible_host = nvh
        self.queries = int(q.shape[0] * q.shape[1])
        self.q_bf = q
        self.raw_k = raw_k
        self.q, self.qs = (hb.hisa_quantize_e4m3(q, 2) if fp8 else (q, None))
        self.w, self.nv = w, nv
        self.k, self.ks = self.prep_keys()
        self.indexer = hb.HisaIndexer(wl.block_size, wl.top_m, wl.top_k)
        self.shape = hb.make_shape(self.q, self.k, wl.block_size, wl.top_m, wl.top_k)
        self.ws_block = torch.empty(max(16, hb.workspace_size(hb.OP_BLOCK, self.shape)), dtype=torch.uint8,
                                    device=dev)
        self.ws_flat = None

    def prep_keys(self):
        hb, wl = self.hb, self.wl
        k = hb.hisa_compress_keys(self.raw_k, wl.compress_ratio) if wl.compress_ratio > 1 else self.raw_k
        if self.fp8:
            return hb.hisa_quantize_e4m3(k, 2)
        return k, None

    def launches_per_step(self) -> int:
        """Kernels of libhisa one HISA step launches: pooling, coarse scoring,
        coarse selection, refinement (+ the merge of split queries), plus the
        key compression (and its quantisation) for compressed keys."""
        n = 4 + (1 if self.wl.compress_ratio > 1 else 0) + (1 if self.fp8 and self.wl.compress_ratio > 1 else 0)
        if self.hb.workspace_size(self.hb.OP_TOKEN, self.shape) > 0:
            n += 1            # merge_parts_kernel after the split refinement
        return n

    def step(self, stage_events=None, stream=None):
        hb, wl = self.hb, self.wl
        # compressed-key workloads recompress the raw keys every step (part of the path)
        if wl.compress_ratio > 1:
            k, ks = self.prep_keys()
        else:
            k, ks = self.k, self.ks
        e = stage_events
        if e:
            e[0].record(stream)
        kpool, kps = hb.hisa_pool_blocks(k, wl.block_size, ks)
        if e:
            e[1].record(stream)
        blocks = hb.hisa_block_score_topm(self.q, self.w, kpool, self.nv, num_keys=k.shape[1],
                                          block_size=wl.block_size, top_m=wl.top_m, q_scale=self.qs,
                                          kpool_scale=kps, workspace=self.ws_block)
        if e:
            e[2].record(stream)
        out = hb.hisa_token_score_topk(self.q, self.w, k, self.nv, blocks, block_size=wl.block_size,
                                       top_k=wl.top_k, q_scale=self.qs, k_scale=ks, workspace=self.ws_token())
        if e:
            e[3].record(stream)
        return out[0]

    def ws_token(self):
        import torch
        if not hasattr(self, "_ws_token"):
            n = self.hb.workspace_size(self.hb.OP_TOKEN, self.shape)
            self._ws_token = torch.empty(max(16, n), dtype=torch.uint8, device=self.dev) if n else None
        return self._ws_token

    def flat(self):
        import torch
        if self.ws_flat is None:
            self.ws_flat = torch.empty(max(16, self.hb.workspace_size(self.hb.OP_FLAT, self.shape)),
                                       dtype=torch.uint8, device=self.dev)
        return self.hb.dsa_flat_indexer_topk(self.q, self.w, self.k, self.nv, top_k=self.wl.top_k,
                                             q_scale=self.qs, k_scale=self.ks, workspace=self.ws_flat)[0]

    def overlap(self, n=OVERLAP_SAMPLE):
        """HISA against flat on a seeded sample of the queries."""
        import torch
        rows = sample_rows(self.queries, n)
        ri = torch.as_tensor(rows, device=self.dev)
        h = self.step().reshape(-1, self.wl.top_k)[ri].cpu().numpy()
        f = self.flat().reshape(-1, self.wl.top_k)[ri].cpu().numpy()
        return overlap_stats(h, f)


def measure_workload(hb, name, fp8, seed, dev, steps, warmup, flush, stream, peaks, barrier, world=1,
                     shard=None, cached_decode=True):
    """HISA and flat on one workload: times, speedup, overlap, refinement roofline."""
    import torch
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    wl = synthetic.WORKLOADS[name]
    run = Run(hb, wl, fp8, seed, dev, shard)
    for _ in range(warmup):
        run.step()
        flush.zero_()
    hb.get_status()
    barrier()
    stage_evs = [[ev() for _ in range(4)] for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        run.step(stage_evs[i], stream)
    barrier()
    hb.get_status()
    step_ms = [e[0].elapsed_time(e[3]) for e in stage_evs]
    stage_ms = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(3)] for e in stage_evs])
    ms = max_over_ranks(float(np.mean(step_ms)), world, dev)
    res = {"ms_per_layer": ms, "queries_per_s": job_rate(run.queries, world, ms),
           "stages_ms": {"pool": float(np.mean(stage_ms[:, 0])), "block_score_topm": float(np.mean(stage_ms[:, 1])),
                         "token_score_topk": float(np.mean(stage_ms[:, 2]))}}
    pairs = candidate_pairs(wl, run.n_visible_host)
    tok_ms = float(np.mean(stage_ms[:, 2]))
    achieved = FLOP_PER_PAIR_PER_HEAD_DIM * wl.heads * wl.head_dim * pairs / (tok_ms / 1000.0) / 1e12
    mult = 2.0 if fp8 else 1.0
    res["refinement"] = {"tflops": achieved, "frac_of_burst": achieved / (peaks["bf16"] * mult),
                         "frac_of_sustained": achieved / (peaks["bf16_sustained"] * mult), "pairs": pairs}
    # flat on the same inputs
    run.flat()
    torch.cuda.synchronize()
    fm = max_over_ranks(timed(run.flat, max(1, min(steps, 5)), flush, stream), world, dev)
    hb.get_status()
    res["flat_ms_per_layer"] = fm
    res["hisa_speedup"] = fm / ms
    res.update(run.overlap())
    # decode: pooled keys of complete blocks kept between steps (the serving loop)
    if cached_decode and wl.num_queries == 1 and wl.compress_ratio == 1 and not fp8:
        res["pooled_keys_cached"] = cached_decode_step(hb, run, steps, flush, stream, world, dev, fm)
        res["sparse_attention"] = measure_attention(hb, run.step(), wl.num_keys, dev, steps, flush, stream, peaks)
    res["gpu_launches_per_step"] = run.launches_per_step()
    return run, res


def measure_attention(hb, idx, num_keys, dev, steps, flush, stream, peaks, seed=0):
    """Attention over the selected keys (the consumer of the indexer), fed the
    HISA indexer's own index rows: latent q / kv of the attention dimensions
    drawn on the GPU, one launch timed per step (L2 flushed between)."""
    import torch
    b, Q, K = idx.shape
    q, kv = synthetic.attention_inputs_cuda(b, Q, num_keys, seed=seed, device=dev)

    def fn():
        return hb.hisa_sparse_attention(q, kv, idx, scale=synthetic.ATTN_SCALE)

    fn()
    torch.cuda.synchronize()
    hb.get_status()
    ms = timed(fn, max(3, steps), flush, stream)
    hb.get_status()
    sel = int((idx >= 0).sum().item())                 # the indexer's rows are sets
    H, dqk, dv = q.shape[2], synthetic.ATTN_DQK, synthetic.ATTN_DV
    flops = 2.0 * sel * H * (dqk + dv)
    gathered = float(sel) * dqk * 2
    io = float(q.numel() * 2 + b * Q * H * (dv * 2 + 4) + idx.numel() * 4)
    sec = ms / 1000.0
    out = {"ms_per_layer": ms, "queries_per_s": b * Q / sec, "heads": H, "d_qk": dqk, "d_v": dv, "top_k": K,
           "selected_keys": sel, "tflops": flops / sec / 1e12, "frac_of_burst_bf16": flops / sec / 1e12 / peaks["bf16"],
           "gathered_kv_gbs": gathered / sec / 1e9, "gathered_plus_io_gbs": (gathered + io) / sec / 1e9,
           "frac_of_hbm": (gathered + io) / sec / 1e9 / peaks["hbm"],
           "what": "hisa_sparse_attention on the HISA indices of this workload; latent q/kv (576 = 512 value + 64 "
                   "positional features, 128 heads) drawn on the GPU"}
    del q, kv
    return out


def cached_decode_step(hb, run, steps, flush, stream, world, dev, flat_ms, paged=False):
    """A decode step that pools only the block its new key completes into the
    cached pooled keys, then scores blocks and refines; timed as launched and
    replayed from a CUDA graph.  With `paged`, the same step over keys
    scattered into shuffled pages."""
    import torch
    wl = run.wl
    k = run.k
    nb = -(-wl.num_keys // wl.block_size)
    kcache, _ = hb.hisa_pool_blocks(k, wl.block_size)      # built by earlier steps (untimed)
    ws_tok = run.ws_token()

    def cached_step():
        hb.hisa_pool_blocks_range(k, wl.block_size, nb - 1, 1, kcache)
        blocks = hb.hisa_block_score_topm(run.q, run.w, kcache, run.nv, num_keys=k.shape[1],
                                          block_size=wl.block_size, top_m=wl.top_m, workspace=run.ws_block)
        return hb.hisa_token_score_topk(run.q, run.w, k, run.nv, blocks, block_size=wl.block_size,
                                        top_k=wl.top_k, workspace=ws_tok)

    for _ in range(3):
        cached_step()
    torch.cuda.synchronize()
    hb.get_status()
    cm = max_over_ranks(timed(cached_step, steps, flush, stream), world, dev)
    cg = max_over_ranks(graph_ms(cached_step, steps, flush, stream), world, dev)
    out = {"ms_per_layer": cm, "queries_per_s": job_rate(run.queries, world, cm), "hisa_speedup": flat_ms / cm,
           "graph_ms_per_layer": cg, "graph_queries_per_s": job_rate(run.queries, world, cg),
           "graph_hisa_speedup": flat_ms / cg,
           "what": "pooled keys of complete blocks kept between decode steps; a step pools the one block its new "
                   "key completes, then scores blocks and refines"}
    if paged and wl.num_keys % wl.block_size == 0:
        bsz = k.shape[0]
        gen = torch.Generator(device="cpu").manual_seed(7)
        perm = torch.randperm(bsz * nb, generator=gen).to(torch.int32).to(k.device)
        table = perm.view(bsz, nb).contiguous()
        pages = torch.empty((bsz * nb, wl.block_size, wl.head_dim), dtype=k.dtype, device=k.device)
        pages[perm.long()] = k.view(bsz * nb, wl.block_size, wl.head_dim)
        pcache = kcache.clone()

        def paged_step():
            hb.hisa_pool_blocks_paged(pages, table, num_keys=k.shape[1], first_block=nb - 1, block_count=1,
                                      kpool=pcache)
            blocks = hb.hisa_block_score_topm(run.q, run.w, pcache, run.nv, num_keys=k.shape[1],
                                              block_size=wl.block_size, top_m=wl.top_m, workspace=run.ws_block)
            return hb.hisa_token_score_topk_paged(run.q, run.w, pages, table, run.nv, blocks, num_keys=k.shape[1],
                                                  top_k=wl.top_k, workspace=ws_tok)

        for _ in range(3):
            paged_step()
        same = bool(torch.equal(torch.sort(paged_step()[0], dim=-1)[0], torch.sort(cached_step()[0], dim=-1)[0]))
        hb.get_status()
        out["paged_graph_ms_per_layer"] = max_over_ranks(graph_ms(paged_step, steps, flush, stream), world, dev)
        out["paged_matches_contiguous"] = same
        del pages, pcache
    return out


def three_level(hb, run, args, flush, stream, world, dev, flat_ms, barrier):
    """Pooled super-blocks -> blocks -> tokens on the same inputs."""
    import torch
    wl = run.wl
    G3 = args.superblock_group
    ix3 = hb.HisaIndexer3(wl.block_size, G3, args.top_m2, wl.top_m, wl.top_k)
    for _ in range(3):
        ix3(run.q, run.w, run.k, run.nv)
    barrier()
    tm = max_over_ranks(timed(lambda: ix3(run.q, run.w, run.k, run.nv), args.steps, flush, stream), world, dev)
    hb.get_status()
    rows = sample_rows(run.queries, OVERLAP_SAMPLE)
    ri = torch.as_tensor(rows, device=dev)
    r3 = ix3(run.q, run.w, run.k, run.nv).reshape(-1, wl.top_k)[ri].cpu().numpy()
    r2 = run.step().reshape(-1, wl.top_k)[ri].cpu().numpy()
    rf = run.flat().reshape(-1, wl.top_k)[ri].cpu().numpy()
    out = {"group": G3, "top_m2": args.top_m2, "ms_per_layer": tm, "queries_per_s": job_rate(run.queries, world, tm),
           "hisa_speedup": flat_ms / tm, "iou_vs_two_level": overlap_stats(r3, r2)["mean_iou_vs_flat"],
           "iou_vs_flat": overlap_stats(r3, rf)["mean_iou_vs_flat"]}
    if wl.num_queries == 1:
        # decode with both pooled levels cached: a step pools the block and the
        # super-block its new key completes
        nb = -(-wl.num_keys // wl.block_size)
        nb2 = -(-wl.num_keys // (wl.block_size * G3))
        kc, _ = hb.hisa_pool_blocks(run.k, wl.block_size)
        kc2, _ = hb.hisa_pool_blocks(run.k, wl.block_size * G3)

        def cached3():
            hb.hisa_pool_blocks_range(run.k, wl.block_size, nb - 1, 1, kc)
            hb.hisa_pool_blocks_range(run.k, wl.block_size * G3, nb2 - 1, 1, kc2)
            return ix3(run.q, run.w, run.k, run.nv, kpool=(kc, None), kpool2=(kc2, None))

        for _ in range(3):
            cached3()
        barrier()
        out["cached_ms_per_layer"] = max_over_ranks(timed(cached3, args.steps, flush, stream), world, dev)
        out["cached_graph_ms_per_layer"] = max_over_ranks(graph_ms(cached3, args.steps, flush, stream), world, dev)
    return out


def end_to_end(hb, run, steps, stream, world, dev):
    """The same metric through the public API from pinned host buffers: every
    step copies q, raw keys, w and n_visible in and the indices out."""
    import torch
    wl = run.wl
    hq = run.q_bf.cpu().pin_memory()
    hk = run.raw_k.cpu().pin_memory()
    hw, hnv = run.w.cpu().pin_memory(), run.nv.cpu().pin_memory()
    out_host = torch.empty((hq.shape[0], hq.shape[1], wl.top_k), dtype=torch.int32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hw, hnv))
    d2h = out_host.numel() * out_host.element_size()
    pipelined = wl.compress_ratio == 1 and not run.fp8

    def e2e_step():
        if pipelined:
            # the host-buffer entry point: copies in, kernels and copies out overlap piece by piece
            run.indexer.from_host(hq, hw, hk, hnv, out_host)
            return
        dq = hq.to(dev, non_blocking=True)
        dk = hk.to(dev, non_blocking=True)
        dw, dnv = hw.to(dev, non_blocking=True), hnv.to(dev, non_blocking=True)
        kk = hb.hisa_compress_keys(dk, wl.compress_ratio) if wl.compress_ratio > 1 else dk
        dqs = kks = None
        if run.fp8:
            dq, dqs = hb.hisa_quantize_e4m3(dq, 2)
            kk, kks = hb.hisa_quantize_e4m3(kk, 2)
        idx, _ = run.indexer(dq, dw, kk, dnv, q_scale=dqs, k_scale=kks)
        out_host.copy_(idx, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    evs = []
    for _ in range(max(1, min(steps, 5))):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        e2e_step()
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    em = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in evs])), world, dev)
    return {"value": job_rate(run.queries, world, em), "unit": "queries/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": em,
            "api": "hisa_indexer_from_host (C ABI; pinned host buffers, 16 pipelined pieces)" if pipelined else
                   "host copies, then the device entry points"}


# ------------------------------------------------------------------ our arm


def attention_only(args):
    """The attention over the selected keys alone: Q queries of 128 heads, top_k
    distinct random positions per query among the workload's keys (seeded),
    latent rows drawn on the GPU."""
    import torch
    from hierarchical_top_key_b200 import binding as hb
    wl = synthetic.WORKLOADS[args.workload]
    Q, L, K = args.attention_only, wl.num_keys, wl.top_k
    q, kv = synthetic.attention_inputs_cuda(1, Q, L, seed=args.seed)
    g = torch.Generator(device="cuda").manual_seed(args.seed + 1)
    idx = torch.argsort(torch.rand((Q, L), generator=g, device="cuda"), dim=1)[:, :K].to(torch.int32)
    idx = idx.view(1, Q, K).contiguous()
    fn = lambda: hb.hisa_sparse_attention(q, kv, idx, scale=synthetic.ATTN_SCALE)  # noqa: E731
    for _ in range(max(1, args.warmup)):
        fn()
    torch.cuda.synchronize()
    hb.get_status()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    ms = timed(fn, max(1, args.steps), flush, torch.cuda.current_stream())
    hb.get_status()
    flops = 2.0 * Q * K * q.shape[2] * (synthetic.ATTN_DQK + synthetic.ATTN_DV)
    print(json.dumps({"attention_only": {"queries": Q, "keys": L, "top_k": K, "ms": ms,
                                         "tflops": flops / (ms / 1000.0) / 1e12}}))
    return 0


def main(argv=None):
    args = parse(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.attention_only:
        return attention_only(args)
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
    hb.load()
    stream = torch.cuda.current_stream()
    fp8 = args.fp8
    peaks = load_peaks()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # ---- the job's share of this rank
    shards = None
    if args.split == "queries":
        seed = args.seed                                   # one job, split over the ranks
        shards = partition.shard_job(synthetic.visible_keys(
            wl.first_query_pos + np.arange(wl.num_queries)[None].repeat(wl.batch, 0), wl.compress_ratio),
            wl.block_size, wl.top_m, world)
        shard = shards[rank]
    else:
        seed = replica_seed(args.seed, rank)               # this rank's own sequences of the job
        shard = None
    run = Run(hb, wl, fp8, seed, dev, shard)

    def step(stage_events=None):
        idx = run.step(stage_events, stream)
        if shards is not None:
            idx = gather_shards(idx, shards, wl.batch, wl.num_queries, wl.top_k, world)
        return idx

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
    job_queries = run.queries * world if shards is None else wl.batch * wl.num_queries
    value = job_queries / (ms_max / 1000.0)

    # ---- flat DSA indexer on the same inputs, and the overlap of the two index sets
    flat = None
    if not args.no_flat:
        run.flat()
        barrier()
        fm = max_over_ranks(timed(run.flat, max(1, min(args.steps, 5)), flush, stream), world, dev)
        hb.get_status()
        nvis = run.n_visible_host
        flat_flops = FLOP_PER_PAIR_PER_HEAD_DIM * wl.heads * wl.head_dim * float(np.minimum(nvis, wl.num_keys).sum())
        flat = {"ms_per_layer": fm, "queries_per_s": job_queries / (fm / 1000.0), "hisa_speedup": fm / ms_max,
                "score_tflops": flat_flops / (fm / 1000.0) / 1e12}
        flat.update(run.overlap())
        # the sampled-threshold flat path (same result, smaller workspace), for comparison
        try:
            ws_s = torch.empty(max(16, hb.workspace_size(hb.OP_FLAT_SAMPLED, run.shape)), dtype=torch.uint8,
                               device=dev)
        except hb.HisaError:
            ws_s = None
        if ws_s is not None:
            def sampled():
                hb.dsa_flat_indexer_topk_sampled(run.q, run.w, run.k, run.nv, top_k=wl.top_k, q_scale=run.qs,
                                                 k_scale=run.ks, workspace=ws_s)
            sampled()
            barrier()
            flat["sampled_ms_per_layer"] = max_over_ranks(timed(sampled, max(1, min(args.steps, 5)), flush, stream),
                                                          world, dev)
            hb.get_status()
            flat["sampled_workspace_bytes"] = int(ws_s.numel())
            flat["workspace_bytes"] = int(run.ws_flat.numel())
            del ws_s

    cached = None
    if wl.num_queries == 1 and wl.compress_ratio == 1 and not fp8:
        cached = cached_decode_step(hb, run, args.steps, flush, stream, world, dev,
                                    flat["ms_per_layer"] if flat else float("nan"), paged=True)

    three = None
    if args.superblock_group > 0 and not fp8 and wl.compress_ratio == 1:
        three = three_level(hb, run, args, flush, stream, world, dev,
                            flat["ms_per_layer"] if flat else float("nan"), barrier)

    e2e = None if args.no_e2e else end_to_end(hb, run, args.steps, stream, world, dev)

    attention = None
    if not args.no_attention and world == 1:
        attention = measure_attention(hb, run.step(), wl.num_keys, dev, args.steps, flush, stream, peaks)

    # ---- roofline of the dominant kernel (the fused refinement stage)
    pairs = candidate_pairs(wl, run.n_visible_host)
    tok_ms = float(np.mean(stage_ms[:, 2]))
    tok_flops = FLOP_PER_PAIR_PER_HEAD_DIM * wl.heads * wl.head_dim * pairs
    achieved = tok_flops / (tok_ms / 1000.0) / 1e12
    mult = 2.0 if fp8 else 1.0
    peak = peaks["bf16"] * mult
    key = wl.name + ("_fp8" if fp8 else "")
    tr = NCU_TRAFFIC.get(key)
    traffic = tr["bytes"] if tr and tr.get("src") == kernel_sources_hash() else None
    roofline = {"kernel": "token_tc_kernel (HISA refinement: gather, scoring, top-k)", "bound": "tensor",
                "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                "peak_source": f"{peaks['source']} bf16 burst (a kernel of a few ms, clocks at max)"
                               + (" x2 for e4m3 (nominal ratio)" if fp8 else ""),
                "frac_of_sustained": achieved / (peaks["bf16_sustained"] * mult),
                "algorithmic": f"{FLOP_PER_PAIR_PER_HEAD_DIM * wl.heads * wl.head_dim} flop per candidate pair x "
                               f"{pairs} pairs per launch",
                "gathered_key_bytes_per_launch": pairs * wl.head_dim * (1 if fp8 else 2)}
    launches = run.launches_per_step()
    inp0 = run.inp
    del run
    torch.cuda.empty_cache()

    # ---- the other long-context workloads (one GPU only)
    extra = None
    if world == 1 and not args.no_extra:
        extra = {}
        for name, x8 in EXTRA_WORKLOADS:
            if name == wl.name and x8 == fp8:
                continue
            r, res = measure_workload(hb, name, x8, args.seed, dev, min(args.steps, 20), max(3, args.warmup),
                                      flush, stream, peaks, barrier)
            extra[name + ("_fp8" if x8 else "")] = res
            del r
            torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r, desc, threads = cpu_oracle_rate(inp0, fp8, args.cpu_seconds)
        cpu = {"value": r, "unit": "queries/s", "cores": threads, "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": "hisa_indexer_queries_per_s", "value": value, "unit": "queries/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
            "scaling": "weak" if shards is None else "strong", "vs_baseline": None,
            "dtype": "e4m3" if fp8 else wl.dtype, "data": "synthetic",
            "config": dict(workload_config(wl, fp8), split=args.split,
                           parallelism=f"{world} rank(s), " + ("whole sequences per rank" if shards is None else
                                                               "queries split by causal work + all-gather")),
            "stages_ms": {"pool": float(np.mean(stage_ms[:, 0])), "block_score_topm": float(np.mean(stage_ms[:, 1])),
                          "token_score_topk": tok_ms},
            "flat": flat, "pooled_keys_cached": cached, "three_level": three, "workloads": extra,
            "sparse_attention": attention,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "clocks": clocks.summary(), "gpu_launches": launches * args.steps,
        }
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
