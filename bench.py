#!/usr/bin/env python
"""Throughput of the MISA routed indexer on B200: scored (query, prefix-token) pairs per second.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ours|reference]

One step is one pass of the hot path over one batch of synthetic input:
pool keys -> route heads -> routed token scoring + top-k (config 4 adds the
MISA-dagger re-rank).  Default workload: 128K prefill, H=32 indexer heads,
pool block 128, m=8 routed heads, top-k 2048 (every query scores its whole
causal prefix: 8.59e9 pairs per step).  Inputs are larger than L2 (q alone is
1.07 GB), so no L2 flush is needed between steps.

Multi-GPU (torchrun): every rank runs an independent problem of the same
shape on its own GPU (weak scaling, no data-path collective); the step time
is the max over ranks.  Rank 0 prints one JSON line.

--impl reference times the CPU oracle as it stands on this host's cores on a
bounded sample of the same workload (the oracle is the only reference: the
pages publish no code).
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "scored query x prefix-token pairs/sec (MISA routed indexer)"
UNIT = "pairs/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-blocks", action="store_true",
                    help="skip the routed-heads x block-pruning comparison (decode workloads)")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only the --config workload (no per_config object)")
    ap.add_argument("--shard", choices=["none", "queries"], default="none",
                    help="queries: the N ranks split ONE problem's query rows (K replicated, "
                         "results all-gathered; strong scaling) instead of each running its own")
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    ap.add_argument("--max-queries", type=int, default=0,
                    help="keep only the last N queries (small captures for ncu)")
    ap.add_argument("--k-cand", type=int, default=-1,
                    help="MISA-dagger candidate count k' (default: the workload's own; 0 = off)")
    ap.add_argument("--graph", choices=["auto", "on", "off"], default="auto",
                    help="replay each step as one CUDA graph (auto: decode workloads)")
    return ap.parse_args()


# ------------------------------------------------------------------ helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=d["hbm_gbs"], bf16=d["bf16_tflops"],
                    bf16_sustained=d["bf16_tflops_sustained"], source="measured")
    return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


def score_src_sha(kernel: str = "score_stream"):
    """Hash of the sources that one scoring kernel is compiled from."""
    main = "score_stream.cu" if kernel == "score_stream" else "score.cu"
    h = hashlib.sha256()
    for f in (main, "common.cuh", "internal.h"):
        with open(os.path.join(ROOT, "long_context_sparse_misa_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profile_traffic(kernel: str, workload: str):
    """DRAM traffic of one kernel from a committed ncu summary whose kernel
    source hash matches the current source: ("pair", bytes per scored pair)
    or ("query", bytes per query row); None when no summary matches."""
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None
    sha = score_src_sha(kernel)
    for fn in sorted(os.listdir(pdir)):
        if not fn.endswith(".md"):
            continue
        with open(os.path.join(pdir, fn)) as f:
            text = f.read()
        m_k = re.search(r"^kernel:\s*(\S+)", text, re.M)
        m_w = re.search(r"^workload:\s*(\S+)", text, re.M)
        m_s = re.search(r"^source_sha:\s*(\S+)", text, re.M)
        m_t = re.search(r"^dram_bytes_per_(pair|query):\s*([0-9.eE+-]+)", text, re.M)
        if m_k and m_w and m_s and m_t and m_k.group(1) == kernel and \
                m_w.group(1) == workload and m_s.group(1) == sha:
            return m_t.group(1), float(m_t.group(2))
    return None


class Clocks:
    """Samples nvidia-smi every 20 ms; the summary covers the samples taken
    between begin() and end() (the timed region)."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_MS = 20

    def __init__(self, uuid):
        self.uuid, self.proc, self.lines = uuid, None, []
        self.i0 = self.i1 = 0

    def start(self):
        """Starts the sampler and waits (up to 10 s) for its first sample."""
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.uuid}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.PERIOD_MS)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            t0 = time.time()
            while not self.lines and time.time() - t0 < 10 and self.proc.poll() is None:
                time.sleep(0.01)
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def begin(self):
        self.i0 = len(self.lines)

    def end(self):
        self.i1 = len(self.lines)

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        note = None
        if self.i1 <= self.i0:
            # Region shorter than the sampling period: take the next sample.
            t0 = time.time()
            while len(self.lines) <= self.i1 and time.time() - t0 < 1.0:
                time.sleep(0.005)
            self.i1 = min(len(self.lines), self.i0 + 1)
            note = "timed region shorter than the sampling period: first sample after it"
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines[self.i0:self.i1]:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        out = {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
               "samples": len(sm), "period_ms": self.PERIOD_MS, "reasons": sorted(reasons)}
        if note:
            out["note"] = note
        return out


def dist_init(backend: str = "nccl"):
    """One process per GPU (torchrun's RANK / LOCAL_RANK / WORLD_SIZE).  The
    data path has no collective: each rank runs its own problem; the process
    group only carries the barriers and the max-over-ranks of the timings.
    backend "gloo" (CPU) is used by the multi-rank tests."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    elif backend == "nccl" and torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest of the ranks' values (every rank gets it)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(cfg: int, rank: int) -> int:
    """Seed of rank `rank`'s problem: every rank scores its own independent
    problem of the same shape (weak scaling)."""
    return 1000 + cfg + 100 * rank


def job_throughput(units_per_rank: int, world: int, ms_step_max: float) -> float:
    """Whole-job units per second: every rank's units over the slowest rank's time."""
    return units_per_rank * world / (ms_step_max / 1e3)


def workload_config(wl, cfg):
    from misa_synth import CONFIGS
    c = CONFIGS[cfg]
    return {"workload": c["name"], "seqs": c["S"], "prefix_len": c["L"], "queries": wl.T,
            "H": c["H"], "d": c["d"], "pool_block": c["B"], "m": c["m"], "k": c["k"],
            "k_cand": wl.k_cand or None, "pairs_per_step": wl.pairs,
            "l2": "inputs larger than L2 (126 MB): no flush" if wl.q_bits.nbytes + wl.K_bits.nbytes > 2 * 126e6
                  else "L2 flushed between steps (256 MB write, then a 256 MB read of another buffer)",
            "launch": "a ~1 ms device sleep before each timed step keeps the stream busy, "
                      "so the events bracket device time and not host launch latency"}


# ------------------------------------------------------------------ CPU oracle sample
def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def _oracle_rows(wl, budget_s, seed, Kf, Kbar, boff):
    """Oracle MISA (and re-rank) on random query rows until budget_s of work."""
    import numpy as np
    import oracle
    order = np.random.default_rng(seed).permutation(wl.T)
    pairs, rows, t_rows = 0, 0, 0.0
    for i in order:
        s = int(wl.q_seq[i])
        k0, k1 = int(wl.key_offsets[s]), int(wl.key_offsets[s + 1])
        t1 = time.perf_counter()
        res = oracle.misa_query(oracle.widen_bf16(wl.q_bits[i]), wl.w[i].astype(np.float64),
                                Kf[k0:k1], Kbar[boff[s]:boff[s + 1]], int(wl.q_pos[i]), wl.B,
                                wl.m, wl.k_cand or wl.k)
        if wl.k_cand:
            oracle.hier_rerank_query(oracle.widen_bf16(wl.q_bits[i]),
                                     wl.w[i].astype(np.float64), Kf[k0:k1], res["idx"], wl.k)
        t_rows += time.perf_counter() - t1
        pairs += int(wl.q_pos[i]) + 1
        rows += 1
        if t_rows > budget_s:
            break
    return pairs, rows, t_rows


def cpu_oracle_sample(wl, budget_s, seed=0, one_core_s=0.0):
    """The CPU oracle (numpy fp64, BLAS on all host cores) on a bounded
    random sample of the workload's query rows, pooling charged pro rata;
    with one_core_s > 0 also a shorter sample limited to one thread."""
    import oracle
    try:
        import threadpoolctl
        cores = max([i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()] or [1])
    except Exception:
        threadpoolctl, cores = None, 1
    Kf = oracle.widen_bf16(wl.K_bits)
    t0 = time.perf_counter()
    Kbar = oracle.pool_keys(Kf, wl.key_offsets, wl.B)
    t_pool = time.perf_counter() - t0
    boff = oracle.block_offsets(wl.key_offsets, wl.B)
    pairs, rows, t_rows = _oracle_rows(wl, budget_s, seed, Kf, Kbar, boff)
    # pooling is per step; charge the sample its share
    t = t_rows + t_pool * pairs / max(wl.pairs, 1)
    out = {"value": pairs / t, "unit": UNIT, "cores": cores, "kind": "oracle",
           "cpu_model": cpu_model(),
           "sample": f"{rows} of {wl.T} query rows (random, seed {seed}), {pairs} pairs, "
                     f"{t:.2f} s incl. pro-rated pooling; numpy fp64"}
    if one_core_s > 0 and threadpoolctl is not None:
        with threadpoolctl.threadpool_limits(1):
            t0 = time.perf_counter()
            oracle.pool_keys(Kf, wl.key_offsets, wl.B)
            t_pool1 = time.perf_counter() - t0
            p1, r1, t1 = _oracle_rows(wl, one_core_s, seed + 1, Kf, Kbar, boff)
        out["value_1core"] = p1 / (t1 + t_pool1 * p1 / max(wl.pairs, 1))
        out["sample_1core"] = f"{r1} query rows, {p1} pairs, {t1:.2f} s on one thread"
    return out


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from misa_synth import make_config
    wl = make_config(args.config)
    per_step = max(1.0, 60.0 / max(args.steps + args.warmup, 1))
    for s in range(args.warmup):
        cpu_oracle_sample(wl, per_step / 4, seed=100 + s)
    vals, pairs_total, t_total, last = [], 0, 0.0, None
    for s in range(args.steps):
        last = cpu_oracle_sample(wl, per_step, seed=s)
        vals.append(last["value"])
    value = statistics.median(vals)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": wl.pairs / value * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(wl, args.config), "impl": "reference",
            "cpu_baseline": {k: last[k] for k in ("kind", "cores", "sample")} | {"value": value,
                                                                               "unit": UNIT},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "note": "CPU oracle (numpy fp64) on a bounded sample per step; ms_per_step is the "
                    "pairs/s-extrapolated time of a full step"}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm
def recall_iou_rows(A, D):
    """Token recovery of selection A against the dense selection D, row by
    row, averaged over the rows where D is not empty: recall |A n D| / |D| and
    IoU |A n D| / |A u D| (index -1 = padding).  A, D: torch int32 [rows, k]
    (any device); runs as torch sorts and searches on that device."""
    import torch
    a = torch.sort(A, dim=1).values
    d = torch.sort(D, dim=1).values.contiguous()
    pos = torch.searchsorted(d, a).clamp_(max=d.shape[1] - 1)
    inter = ((torch.gather(d, 1, pos) == a) & (a >= 0)).sum(1).double()
    na, nd = (A >= 0).sum(1).double(), (D >= 0).sum(1).double()
    keep = nd > 0
    if not bool(keep.any()):
        return 1.0, 1.0
    recall = (inter[keep] / nd[keep]).mean().item()
    iou = (inter[keep] / (na[keep] + nd[keep] - inter[keep])).mean().item()
    return recall, iou


def split_prof(prof):
    """Kernel entries of a misa.profile_collect() record, and its counters
    (names starting with '#')."""
    kern = {n: v for n, v in prof.items() if not n.startswith("#")}
    cnt = {n[1:]: v[1] for n, v in prof.items() if n.startswith("#")}
    return kern, cnt


def is_streamed(kernels) -> bool:
    """Whether a step's routed scoring was the streaming prefill pass: its
    candidates are selected by the pass after it ("select"); the row-scoring
    path (decode) takes a row top-k instead.  (A MISA-dagger prefill runs both
    a selection and the re-rank's row top-k: it is streamed.)"""
    return "select" in kernels


def decode_kbytes(wl):
    """K prefix bytes the decode scorer streams: each group of 256/m queries
    of a sequence reads its longest prefix once (256 B per key)."""
    G = 256 // wl.m
    kbytes = 0
    for s_ in range(len(wl.seq_lens)):
        pos = wl.q_pos[wl.query_offsets[s_]:wl.query_offsets[s_ + 1]]
        for g0 in range(0, len(pos), G):
            kbytes += (int(pos[g0:g0 + G].max()) + 1) * 256
    return kbytes


def roofline_of(wl, prof_ms, launches_per_step, streamed, peaks, clk, workload):
    """Roofline of the dominant kernel (routed scoring) from its CUDA-event
    time per step."""
    pairs = wl.pairs
    tp = profile_traffic("score_stream" if streamed else "score", workload)
    sec = prof_ms / 1e3
    if streamed:
        # prefill: a dense contraction, 2*m*d flops per scored pair.  The
        # timed region is sub-second, so the burst bf16 peak applies.
        flops = 2.0 * wl.m * wl.d * pairs
        achieved = flops / sec / 1e12
        r = {"kernel": "score_stream_kernel (tcgen05 routed scoring, top-k candidates in the epilogue)",
             "bound": "tensor", "achieved": achieved, "peak": peaks["bf16"], "unit": "TFLOP/s",
             "frac": achieved / peaks["bf16"],
             "peak_source": f"bf16_tflops, burst ({peaks['source']})",
             "frac_of_sustained": achieved / peaks["bf16_sustained"],
             "algorithmic_flops_per_launch": flops / max(launches_per_step, 1)}
    else:
        # decode: HBM-bound; each query group streams its prefix of K once
        # (256 B per key) and writes its fp32 score rows (4 B per pair)
        abytes = decode_kbytes(wl) + 4 * pairs
        achieved = abytes / sec / 1e9
        r = {"kernel": "score_kernel (tcgen05 routed scoring, score rows)",
             "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
             "frac": achieved / peaks["hbm_gbs"], "peak_source": f"hbm_gbs ({peaks['source']})",
             "algorithmic_bytes_per_launch": abytes / max(launches_per_step, 1)}
    r |= {"launches_per_step": launches_per_step, "kernel_ms_per_step": prof_ms,
          "sm_mhz_median": clk.get("sm_mhz"),
          "traffic": None if tp is None else
              tp[1] * (pairs if tp[0] == "pair" else wl.T) / max(launches_per_step, 1)}
    return r


class Bench:
    """One workload on this rank's GPU: inputs resident in HBM, the indexer's
    buffers, and the timing helpers shared by every leg."""

    def __init__(self, cfg, args, rank, world, dev):
        import dataclasses as dc

        import numpy as np
        import torch

        import long_context_sparse_misa_b200 as misa
        from misa_synth import CONFIGS, make_config
        self.misa, self.torch, self.np = misa, torch, np
        self.cfg, self.args, self.world, self.dev = cfg, args, world, dev
        # --shard queries: every rank draws the same problem and keeps its
        # range of query rows (sharding.query_ranges); otherwise each rank
        # draws its own problem
        self.shard = getattr(args, "shard", "none") == "queries" and world > 1
        wl = make_config(cfg, seed=rank_seed(cfg, 0 if self.shard else rank))
        if args.k_cand >= 0 and cfg == args.config:
            wl = dc.replace(wl, k_cand=args.k_cand)
        if args.max_queries and args.max_queries < wl.T:
            wl = wl.subset_queries(range(wl.T - args.max_queries, wl.T))
        self.job_pairs = wl.pairs * (1 if self.shard else world)
        self.ranges = None
        if self.shard:
            from long_context_sparse_misa_b200 import sharding
            self.ranges = sharding.query_ranges(wl.q_pos, world)
            wl = wl.subset_queries(range(*self.ranges[rank]))
        self.wl = wl
        self.hier = bool(wl.k_cand)
        self.decode = CONFIGS[cfg]["queries"] != "all"
        self.workload = CONFIGS[cfg]["name"]
        self.prob = misa.Problem.from_workload(wl, device=dev)
        self.K = torch.from_numpy(wl.K_bits).to(dev)
        self.q = torch.from_numpy(wl.q_bits).to(dev)
        self.w = torch.from_numpy(wl.w).to(dev)
        self.ix = misa.Indexer(self.prob, m=wl.m, k=wl.k, k_cand=wl.k_cand, device=dev)
        self.use_graph = args.graph == "on" or (args.graph == "auto" and self.decode)
        # Decode step: the keys before this step's queries were pooled by
        # earlier steps, so only the blocks holding the new keys are re-pooled.
        self.pool_from = None
        if self.decode:
            q_per_seq = np.diff(wl.query_offsets)
            self.pool_from = torch.tensor(wl.seq_lens - q_per_seq, dtype=torch.int32, device=dev)
            misa.pool_keys(self.prob, self.K, self.ix.Kbar)
        small = wl.q_bits.nbytes + wl.K_bits.nbytes < 2 * 126e6
        self.flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if small else None
        # Read after the write: the flush's own dirty lines are written back
        # here, outside the timed step, and L2 is left holding clean lines.
        self.clean = torch.ones(64 << 20, dtype=torch.int32, device=dev) if small else None

    def l2_flush(self):
        if self.flush is not None:
            self.flush.fill_(1)
            self.clean.sum()

    def settle(self):
        """Between timed intervals: the L2 flush (small inputs only), then a
        ~1 ms device sleep so that the host has queued the whole next step
        before the device reaches it; the events then bracket device time,
        not the host's launch latency."""
        self.l2_flush()
        self.torch.cuda._sleep(2_000_000)

    def capture(self, fn):
        """One step as a CUDA graph (all of the library's launches)."""
        torch = self.torch
        side = torch.cuda.Stream(device=self.dev)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            fn()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        return g

    def timed(self, eager, steps, warmup=1, clocks=None):
        """Device time of `steps` steps (CUDA events around each, max over
        ranks), plus the per-kernel times of the same steps launched eagerly.
        A CUDA graph replays decode steps; its kernels get no events, so their
        per-kernel times come from eager steps after the timed region.
        Returns (per-step ms sorted, per-step {kernel: (ms, launches)}, counters)."""
        torch, misa = self.torch, self.misa
        for _ in range(warmup):
            self.l2_flush()
            eager()
        torch.cuda.synchronize()
        graph = self.capture(eager) if self.use_graph else None
        run = graph.replay if graph is not None else eager
        torch.cuda.synchronize()
        barrier(self.world)
        misa.profile_enable(graph is None)
        if clocks is not None:
            clocks.begin()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        step_prof = []
        for e0, e1 in evs:
            self.settle()
            e0.record()
            run()
            e1.record()
            if graph is None:
                # waits for this step's events (the next step's own events are
                # recorded after the L2 flush and the device sleep)
                step_prof.append(misa.profile_collect())
        torch.cuda.synchronize()
        if clocks is not None:
            clocks.end()
        misa.profile_enable(False)
        barrier(self.world)
        step_ms = sorted(e0.elapsed_time(e1) for e0, e1 in evs)
        if graph is not None:
            misa.profile_enable(True)
            for _ in range(steps):
                self.settle()
                eager()
                step_prof.append(misa.profile_collect())
            torch.cuda.synchronize()
            misa.profile_enable(False)
            del graph
        code, bits = misa.stream_status()
        if code != 0:
            raise RuntimeError(f"device status {code} ({bits}) in {self.workload}")
        kerns, counters = [], {}
        for sp in step_prof:
            k_, c_ = split_prof(sp)
            kerns.append(k_)
            for n, v in c_.items():
                counters[n] = counters.get(n, 0) + v
        return step_ms, kerns, counters

    def misa_step(self):
        ix = self.ix
        if self.hier:
            out = ix.hier(self.q, self.w, self.K, pool_from=self.pool_from)
        else:
            out = ix.misa(self.q, self.w, self.K, pool_from=self.pool_from)
        if self.shard:
            # every rank ends the step with the whole problem's selection
            from long_context_sparse_misa_b200 import sharding
            self.all_idx = sharding.gather_rows(ix.idx, self.ranges)
            self.all_val = sharding.gather_rows(ix.val, self.ranges)
        return out


def summarise_kernels(kerns, steps):
    def pct(vals, q):
        vals = sorted(vals)
        return vals[min(len(vals) - 1, (q * len(vals)) // 100)]

    tot = {}
    for sp in kerns:
        for n, (t, c) in sp.items():
            t0, c0 = tot.get(n, (0.0, 0))
            tot[n] = (t0 + t, c0 + c)
    all_ms = max(sum(v[0] for v in tot.values()), 1e-9)
    out = {}
    for n, (t, c) in tot.items():
        per_step = [sp.get(n, (0.0, 0))[0] for sp in kerns]
        out[n] = {"ms_per_step": t / steps, "launches_per_step": c / steps, "share": t / all_ms,
                  "p50_ms": pct(per_step, 50), "p90_ms": pct(per_step, 90)}
    return out


def measure_config(cfg, args, world, rank, dev, steps, headline, clocks=None):
    """Time one workload: the MISA step (the headline's metric), its roofline,
    the dense DSA indexer on the same inputs with recall / IoU of MISA's
    selection against it, and (decode workloads) routed heads x block pruning.
    Returns (result dict, Bench)."""
    import torch
    bn = Bench(cfg, args, rank, world, dev)
    wl, ix = bn.wl, bn.ix
    peaks = load_peaks()
    warm = max(args.warmup, 3)
    step_ms, kerns, counters = bn.timed(bn.misa_step, steps, warmup=warm, clocks=clocks)
    clk = clocks.stop() if clocks is not None else {}
    ms = max_over_ranks(sum(step_ms), world) / steps
    p50 = max_over_ranks(step_ms[len(step_ms) // 2], world)
    p90 = max_over_ranks(step_ms[min(len(step_ms) - 1, (9 * len(step_ms)) // 10)], world)
    kernels = summarise_kernels(kerns, steps)
    k = kernels.get("score", {"ms_per_step": float("nan"), "launches_per_step": 0})
    streamed = is_streamed(kernels)
    res = {"workload": bn.workload, "ms_per_step": ms, "latency_ms": ms,
           "value": bn.job_pairs / (ms / 1e3), "unit": UNIT,
           "step_ms_p50": p50, "step_ms_p90": p90, "cuda_graph": bn.use_graph,
           "roofline": roofline_of(wl, k["ms_per_step"], k["launches_per_step"], streamed, peaks,
                                   clk, bn.workload),
           "kernels": kernels,
           "gpu_launches": sum(v["launches_per_step"] for v in kernels.values()) * steps,
           "rescanned_queries_per_step": counters.get("rescan_queries", 0) / steps}
    if clk:
        res["clocks"] = clk
    misa_idx = ix.idx.clone()  # this step's selection, before the comparisons overwrite it

    if not args.no_dense:
        dsteps = max(1, min(steps, 5))
        d_ms, d_kerns, d_cnt = bn.timed(lambda: ix.dense(bn.q, bn.w, bn.K), dsteps, warmup=1)
        dms = max_over_ranks(sum(d_ms), world) / dsteps
        d_kernels = summarise_kernels(d_kerns, dsteps)
        d_k_ms = d_kernels.get("score", {"ms_per_step": float("nan")})["ms_per_step"]
        rec, iou = recall_iou_rows(misa_idx, ix.idx)
        res["dense_dsa"] = {
            "ms_per_step": dms, "value": bn.job_pairs / (dms / 1e3), "unit": UNIT,
            "misa_speedup": dms / ms,
            "kernels": {n: v["ms_per_step"] for n, v in d_kernels.items()},
            "rescanned_queries_per_step": d_cnt.get("rescan_queries", 0) / dsteps}
        if streamed:
            d_tf = 2.0 * wl.H * wl.d * wl.pairs / (d_k_ms / 1e3) / 1e12
            res["dense_dsa"] |= {"score_kernel_tflops": d_tf,
                                 "score_kernel_frac": d_tf / peaks["bf16"]}
        # row a8: token recovery of MISA's final selection against the dense
        # indexer's, every query row of the step
        res["recall_vs_dense"] = rec
        res["iou_vs_dense"] = iou
        res["recall_rows"] = wl.T
        dense_idx = ix.idx.clone()
    else:
        dense_idx = None

    # routed heads x block pruning on the same decode step: the routed heads
    # score the pooled blocks, only the best 2k/B blocks' tokens (and the
    # incomplete block) are scored
    if bn.decode and not args.no_blocks:
        import long_context_sparse_misa_b200 as misa
        nb = max(1, 2 * wl.k // wl.B)
        bx = misa.Indexer(bn.prob, m=wl.m, k=wl.k, n_blocks=nb, device=dev)
        misa.pool_keys(bn.prob, bn.K, bx.Kbar)
        bsteps = max(1, min(steps, 5))
        b_ms, b_kerns, _ = bn.timed(lambda: bx.blocks(bn.q, bn.w, bn.K, pool_from=bn.pool_from),
                                    bsteps, warmup=1)
        bms = max_over_ranks(sum(b_ms), world) / bsteps
        blk = {"n_blocks": nb, "candidates_per_query": (nb + 1) * wl.B,
               "ms_per_step": bms, "value": bn.job_pairs / (bms / 1e3), "unit": UNIT,
               "speedup_vs_misa": ms / bms,
               "recall_of_misa_selection": recall_iou_rows(bx.idx, misa_idx)[0],
               "kernels": {n: v["ms_per_step"] for n, v in summarise_kernels(b_kerns, bsteps).items()}}
        if dense_idx is not None:
            blk["speedup_vs_dense"] = res["dense_dsa"]["ms_per_step"] / bms
            blk["recall_vs_dense"], blk["iou_vs_dense"] = recall_iou_rows(bx.idx, dense_idx)
        res["block_pruned"] = blk
    torch.cuda.synchronize()
    return res, bn


def e2e_leg(bn, args, world):
    """End to end through the public API with host buffers.  Every step copies
    its inputs from pinned host memory and reads its results back; the copies
    run on their own stream, double buffered, so step i+1's upload and step
    i's download overlap step i's compute (as a serving loop would pipeline
    them)."""
    import torch
    wl, ix, dev = bn.wl, bn.ix, bn.dev
    pin = lambda a: torch.from_numpy(a).pin_memory()
    K_h, q_h, w_h = pin(wl.K_bits), pin(wl.q_bits), pin(wl.w)
    e2e_steps = max(2, min(args.steps, 6))
    ins = [(bn.K, bn.q, bn.w),
           (torch.empty_like(bn.K), torch.empty_like(bn.q), torch.empty_like(bn.w))]
    stage = [(torch.empty_like(ix.idx), torch.empty_like(ix.val)) for _ in range(2)]
    outs_h = [(torch.empty(tuple(ix.idx.shape), dtype=torch.int32).pin_memory(),
               torch.empty(tuple(ix.val.shape), dtype=torch.float32).pin_memory())
              for _ in range(2)]
    comp = torch.cuda.current_stream()
    xfer = torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    api = ix.hier if bn.hier else ix.misa

    def h2d(b):
        with torch.cuda.stream(xfer):
            Kd, qd, wd = ins[b]
            Kd.copy_(K_h, non_blocking=True)
            qd.copy_(q_h, non_blocking=True)
            wd.copy_(w_h, non_blocking=True)
            ev_in[b].record(xfer)

    def compute(b):
        comp.wait_event(ev_in[b])
        Kd, qd, wd = ins[b]
        api(qd, wd, Kd, pool_from=bn.pool_from)  # the public API calls, one by one
        stage[b][0].copy_(ix.idx)
        stage[b][1].copy_(ix.val)
        ev_done[b].record(comp)

    def d2h(b):
        with torch.cuda.stream(xfer):
            xfer.wait_event(ev_done[b])
            outs_h[b][0].copy_(stage[b][0], non_blocking=True)
            outs_h[b][1].copy_(stage[b][1], non_blocking=True)

    def pipeline(nsteps, e0=None, e1=None):
        if e0 is not None:
            e0.record(xfer)
        h2d(0)
        if nsteps > 1:
            h2d(1)
        for i in range(nsteps):
            compute(i % 2)
            d2h(i % 2)
            if i + 2 < nsteps:
                h2d(i % 2)  # ordered after this buffer's compute and download
        if e1 is not None:
            e1.record(xfer)

    pipeline(2)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pipeline(e2e_steps, e0, e1)
    torch.cuda.synchronize()
    ems = max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps
    return {"value": bn.job_pairs / (ems / 1e3), "unit": UNIT, "ms_per_step": ems,
            "h2d_bytes_per_step": K_h.nbytes + q_h.nbytes + w_h.nbytes,
            "d2h_bytes_per_step": outs_h[0][0].nbytes + outs_h[0][1].nbytes,
            "pipelined": "uploads and downloads on a copy stream, double buffered"}


# The other configurations, each timed like the headline (decode steps as
# CUDA graphs) with its dense comparison; parity tests cover all five.
PER_CONFIG = (0, 1, 2, 4)


def run_ours(args):
    import gc

    import torch

    world, rank, local = dist_init()
    dev = torch.device("cuda", torch.cuda.current_device())
    props = torch.cuda.get_device_properties(dev)
    clocks = Clocks(f"GPU-{props.uuid}" if hasattr(props, "uuid") else str(local))
    clocks.start()
    res, bn = measure_config(args.config, args, world, rank, dev, args.steps, True, clocks)
    wl = bn.wl
    line = {"metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
            "higher_is_better": True, "scaling": "strong" if bn.shard else "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1)/sqrt(d) bf16 q,k with 1% planted needles; "
                    "w ~ N(0,1)/sqrt(H) fp32)",
            "config": workload_config(wl, args.config) | {
                "parallelism": (f"query shards of one problem x{world} (K replicated, idx/val "
                                "all-gathered every step)") if bn.shard
                               else f"independent problem per GPU x{world}"}}
    if bn.decode:
        line["config"]["decode_step"] = "pooled keys of earlier blocks kept; blocks with new keys re-pooled"
    line |= {k_: v for k_, v in res.items() if k_ not in ("value", "unit", "ms_per_step", "workload")}
    if not args.no_e2e:
        line["e2e"] = e2e_leg(bn, args, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_sample(wl, args.cpu_budget_s,
                                                   one_core_s=args.cpu_budget_s / 4)
    del bn
    gc.collect()
    torch.cuda.empty_cache()
    if world == 1 and not args.no_per_config:
        per = {}
        for c in PER_CONFIG:
            if c == args.config:
                continue
            r, b = measure_config(c, args, world, rank, dev, min(args.steps, 10), False)
            per[r.pop("workload")] = r
            del b
            gc.collect()
            torch.cuda.empty_cache()
        line["per_config"] = per
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
