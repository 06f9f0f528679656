"""Benchmark of UNO's per-cycle sampling and verification step on B200.

One step = one decode cycle of the linear 8/1/8 workload at 64 requests per
GPU (the UNO PR page's batch-64 linear configuration, vocabulary 151,936,
bf16, T = 1, top-k 50, top-p 0.95): uno_linear_cycle, which filters the 512
draft marginal rows (with the proposal draws) and the 576 target rows in one
launch and then decides every request.  Inputs are seeded synthetic logits
resident in HBM (330.6 MB per step, larger than the 126 MB L2).  The cycle is
captured once in a CUDA graph and replayed; CUDA events bracket each replay.
Beside it: the same cycle as two calls, the tree workloads and the linear
stress workload, each replayed from a graph.

Ranks (torchrun, one per GPU) each process their own 64 requests (global
request indices rank*64 ..), with no collective on the data path; timing is
the maximum over ranks.

--impl reference times the oracle (oracle/uno_ref.c) on the host cores on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import numpy as np  # noqa: E402

WORKLOAD_INDEX = 1
METRIC = "verified draft blocks/sec and logits HBM GB/s (fraction of B200 peak)"
UNIT = "blocks/s"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0
BAD_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", type=int, default=WORKLOAD_INDEX, help="index into inputs.WORKLOADS (linear only)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-tree", action="store_true", help="skip the other workloads' timings")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle time budget of the cpu_baseline")
    ap.add_argument("--only", choices=["suffix_attention"], default=None,
                    help="run one side measurement alone and print its JSON")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def init_dist(world, backend="nccl"):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def shard(rank, per_rank):
    """This rank's requests: per_rank consecutive global indices.  The global
    index is also the request word of the random-number counter, so a rank's
    draws equal those of the same requests in one big batch."""
    first = rank * per_rank
    return first, range(first, first + per_rank)


def max_over_ranks(values, world, device):
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def barrier(world, device):
    import torch
    torch.cuda.synchronize(device)
    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[device.index])
    torch.cuda.synchronize(device)


# ---------------------------------------------------------------------------
# clocks (NVML) sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index, period=0.005):
        self.index, self.period = index, period
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # pragma: no cover - NVML missing
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                try:
                    mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except Exception:
                    mask = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()
        return False

    def summary(self):
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# peaks and committed profile figures
# ---------------------------------------------------------------------------
def hbm_peak():
    p = ROOT / "MEASURED_PEAKS.json"
    try:
        d = json.loads(p.read_text())
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _code_only(text):
    """C/CUDA source without its comments and blank lines (a comment edit
    leaves the kernels, and so their counters, unchanged)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def kernel_source_hash():
    """Hash of the row kernels' code (comments and blank lines left out)."""
    h = hashlib.sha256()
    for rel in ("speculative_decoding_verification_filter_b200/csrc/uno_filter.cu",
                "speculative_decoding_verification_filter_b200/csrc/uno_device.cuh"):
        h.update(_code_only((ROOT / rel).read_text()).encode())
    return h.hexdigest()[:16]


def committed_traffic():
    """DRAM bytes (read + write) per launch of the cycle's row kernel from the
    committed ncu summary, if it was taken on the current kernel source."""
    p = ROOT / "profiles" / "traffic.json"
    try:
        d = json.loads(p.read_text())
    except Exception:
        return None
    if d.get("kernel_source_sha") != kernel_source_hash():
        return None
    return d.get("cycle_dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# the oracle on the host (cpu_baseline and --impl reference)
# ---------------------------------------------------------------------------
def oracle_requests(w, reqs, cycle=0):
    """Run the oracle over the given requests one by one; returns seconds."""
    import oracle
    from speculative_decoding_verification_filter_b200.inputs import linear_draft, linear_target
    total = 0.0
    for r in reqs:
        q = linear_draft(w, [r])
        p = linear_target(w, [r])
        t0 = time.perf_counter()
        rq = oracle.filter_softmax(q, w.dtype, w.temperature, w.top_k, w.top_p, rows_per_request=w.B,
                                   rng=(w.seed, cycle, r))
        oracle.linear_verify(p, w.dtype, 1, w.B, w.temperature, w.top_k, w.top_p, rq["sample"].reshape(1, w.B),
                             rq["ids"], rq["probs"], rq["count"], rng=(w.seed, cycle, r))
        total += time.perf_counter() - t0
    return total


def cpu_baseline(w, budget_s):
    import oracle
    oracle.build()
    done, spent = 0, 0.0
    while done < w.R and spent < budget_s:
        spent += oracle_requests(w, [done])
        done += 1
    return {"value": done / spent, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{done} of {w.R} requests ({done * (2 * w.B + 1)} logit rows), single-threaded C oracle, "
                      f"{spent:.1f} s of CPU work"}


def run_reference(args, w):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    oracle.build()
    t_req = oracle_requests(w, [0])
    budget = 150.0
    steps = max(1, min(args.steps, int(budget / max(t_req, 1e-3))))
    # at least three warm-up steps, at most about 30 s of them
    warm = max(3, min(args.warmup, int(30.0 / max(t_req, 1e-3))))
    oracle_requests(w, [1 % w.R] * warm)
    secs = oracle_requests(w, [(2 + i) % w.R for i in range(steps)])
    value = steps / secs
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": steps,
        "warmup": warm, "ms_per_step": 1e3 * secs / steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, 1),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"one request (its {2 * w.B + 1} logit rows) per step, {steps} steps "
                                   f"(capped at ~{budget:.0f} s), single-threaded C oracle"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(w, world):
    return {"workload": f"{w.name}: R={w.R} requests/GPU, B={w.B}, vocab {w.vocab}, {w.dtype} logits, "
                        f"T={w.temperature}, top-k {w.top_k}, top-p {w.top_p}",
            "global_batch": w.R * world, "requests_per_gpu": w.R, "vocab": w.vocab, "B": w.B,
            "logit_bytes_per_step_per_gpu": w.logit_bytes,
            "l2": "inputs larger than L2 (no flush): %.1f MB of logits per step vs 126 MB L2" % (w.logit_bytes / 1e6),
            "parallelism": f"requests sharded over {world} GPU(s), no collective on the data path"}


# ---------------------------------------------------------------------------
# timing helpers
# ---------------------------------------------------------------------------
def graph_of(fn, stream):
    """Capture fn(stream) in a CUDA graph (after warm-up calls)."""
    import torch
    with torch.cuda.stream(stream):
        for _ in range(3):
            fn(stream)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
    stream.synchronize()
    return g


def replay_ms(g, stream, reps, flush=None):
    """Mean CUDA-event time of a graph replay on `stream` (events on the same
    stream); `flush` (a callable) runs between replays, outside the events."""
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    with torch.cuda.stream(stream):
        for a, b in ev:
            if flush is not None:
                flush()
            a.record(stream)
            g.replay()
            b.record(stream)
    stream.synchronize()
    return statistics.fmean(a.elapsed_time(b) for a, b in ev)


def eager_ms(fn, stream, reps, flush=None):
    """Mean CUDA-event time of fn(stream) issued from Python on `stream`;
    `flush` runs between calls, outside the events."""
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    with torch.cuda.stream(stream):
        for _ in range(3):
            fn(stream)
        for a, b in ev:
            if flush is not None:
                flush()
            a.record(stream)
            fn(stream)
            b.record(stream)
    stream.synchronize()
    return statistics.fmean(a.elapsed_time(b) for a, b in ev)


def oracle_rate(fn, budget_s):
    """Requests per second of fn(i) (one request each) over about budget_s."""
    done, spent = 0, 0.0
    while spent < budget_s or done == 0:
        t0 = time.perf_counter()
        fn(done)
        spent += time.perf_counter() - t0
        done += 1
    return done / spent, done, spent


# ---------------------------------------------------------------------------
# the other named workloads (reported beside the headline)
# ---------------------------------------------------------------------------
def tree_leg(index, device, first, stream, peak, reps, cpu_budget):
    """A tree cycle (filter of the R*B draft rows, top-K extraction and
    best-first expansion, target-only verification of the node rows) replayed
    from one CUDA graph.  The small batch-1 workload fits in L2, so a 256 MB
    buffer is rewritten between replays (outside the events)."""
    import torch
    from speculative_decoding_verification_filter_b200 import (uno_filter_softmax, uno_tree_topk_expand,
                                                              uno_tree_verify)
    from speculative_decoding_verification_filter_b200.inputs import WORKLOADS, tree_draft, tree_target
    w = WORKLOADS[index]
    reqs = range(first, first + w.R)
    sp = dict(temperature=w.temperature, top_k=w.top_k, top_p=w.top_p)

    def dev(a):
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)

    q_np = tree_draft(w, reqs)
    q = dev(q_np)
    with torch.cuda.stream(stream):
        fo = uno_filter_softmax(q, rows_per_request=w.B, **sp)
        to = uno_tree_topk_expand(fo["ids"], fo["probs"], fo["count"], R=w.R, B=w.B, K=w.K, V=w.V)
    stream.synchronize()
    depth, nn = to["node_depth"].cpu().numpy(), to["num_nodes"].cpu().numpy()
    p_np = tree_target(w, depth, nn, reqs)
    p = dev(p_np)
    # the cycle word lives on the device: every replay of the graph draws the
    # next cycle's uniforms (the graph ends by advancing it)
    cyc = torch.zeros(1, dtype=torch.int32, device=device)
    rng = (w.seed, cyc, first)

    def cycle(st):
        f = uno_filter_softmax(q, rows_per_request=w.B, **sp)
        t = uno_tree_topk_expand(f["ids"], f["probs"], f["count"], R=w.R, B=w.B, K=w.K, V=w.V)
        v = uno_tree_verify(p, t["node_token"], t["node_parent"], t["num_nodes"], R=w.R, B=w.B, V=w.V, rng=rng,
                            **sp)
        cyc.add_(1)
        return v

    g = graph_of(cycle, stream)
    flush = None
    if w.logit_bytes < 256e6:
        junk = torch.empty(256 << 20, dtype=torch.uint8, device=device)
        flush = lambda: junk.fill_(1)  # noqa: E731
    ms = replay_ms(g, stream, reps, flush)
    calls = eager_ms(cycle, stream, reps, flush)
    nbytes = (w.R * w.B + int(nn.sum())) * w.vocab * w.elem_bytes

    import oracle

    def one(i):
        r = i % w.R
        rq = oracle.filter_softmax(q_np[r * w.B:(r + 1) * w.B], w.dtype, w.temperature, w.top_k, w.top_p,
                                   rows_per_request=w.B)
        rt = oracle.tree_topk_expand(rq["ids"], rq["probs"], rq["count"], 1, w.B, w.K, w.V)
        oracle.tree_verify(p_np[r * w.V:(r + 1) * w.V], w.dtype, 1, w.B, w.V, w.temperature, w.top_k, w.top_p,
                           rt["node_token"], rt["node_parent"], rt["num_nodes"], rng=(w.seed, 0, first + r))
    rate, done, spent = oracle_rate(one, cpu_budget)
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"workload": f"{w.name}: R={w.R}, B={w.B}, K={w.K}, V={w.V}, vocab {w.vocab}, {w.dtype}",
            "value": w.R / (ms / 1e3), "unit": UNIT, "ms_per_cycle": ms,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "bytes_per_cycle": nbytes},
            "l2": "256 MB buffer rewritten between replays" if flush else "inputs larger than L2",
            "timing": f"CUDA events around {reps} replays of one graph (filter, expand, verify: 4 kernels, "
                      "then the cycle word advanced on the device)",
            "calls": {"ms_per_cycle": calls, "value": w.R / (calls / 1e3),
                      "note": "the same cycle as three Python calls per cycle (no graph), CUDA events around each"},
            "cpu_baseline": {"value": rate, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"{done} requests, {spent:.1f} s, single-threaded C oracle"}}


def params_leg(q, p, w, first, stream, peak, reps):
    """uno_linear_cycle_params over the headline batch: per-request arrays
    (each request's own entries, here the workload's values), in the
    top-k-first and in the joint filter order, one graph replay per cycle."""
    import torch
    from speculative_decoding_verification_filter_b200 import uno_linear_cycle_params
    dev = q.device
    T = torch.full((w.R,), w.temperature, dtype=torch.float32, device=dev)
    K = torch.full((w.R,), w.top_k, dtype=torch.int32, device=dev)
    P = torch.full((w.R,), w.top_p, dtype=torch.float32, device=dev)
    nbytes = (q.shape[0] + p.shape[0]) * w.vocab * w.elem_bytes
    out = {}
    for order in ("topk_first", "joint"):
        g = graph_of(lambda st, order=order: uno_linear_cycle_params(
            q, p, R=w.R, B=w.B, temperature=T, top_k=K, top_p=P, rng=(w.seed, 0, first), order=order,
            top_k_max=w.top_k), stream)
        ms = replay_ms(g, stream, reps)
        del g
        gbs = nbytes / (ms / 1e3) / 1e9
        out[order] = {"ms_per_cycle": ms, "value": w.R / (ms / 1e3), "unit": UNIT,
                      "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                                   "bytes_per_cycle": nbytes}}
    out["note"] = ("uno_linear_cycle_params, CUDA events around graph replays; the joint order also forms every "
                   "row's sum of exp over the full vocabulary while it reads the row")
    return out


def suffix_attention_leg(device, stream, peak, reps=50):
    """uno_tree_suffix_attention_merge at the attention shape of an 8B model
    (32 query heads over 8 key/value heads, head dim 128, a 32-node binary
    tree, bf16 q/k/v, f32 prefix state), 1 and 64 requests; each launch timed
    alone with CUDA events, the L2 rewritten (256 MB) before it."""
    import torch
    from speculative_decoding_verification_filter_b200 import uno_tree_suffix_attention_merge
    V, H, Hkv, d = 32, 32, 8, 128
    junk = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    out = {}
    for R in (1, 64):
        g = torch.Generator(device=device)
        g.manual_seed(1000 + R)
        q = torch.randn((R, V, H, d), generator=g, device=device).to(torch.bfloat16)
        k = torch.randn((R, V, Hkv, d), generator=g, device=device).to(torch.bfloat16)
        v = torch.randn((R, V, Hkv, d), generator=g, device=device).to(torch.bfloat16)
        par = torch.tensor([-1] + [j // 2 for j in range(1, V)], dtype=torch.int32, device=device).repeat(R, 1)
        nn = torch.full((R,), V, dtype=torch.int32, device=device)
        op = torch.randn((R, V, H, d), generator=g, device=device)
        lp = torch.randn((R, V, H), generator=g, device=device)
        nbytes = q.numel() * 2 + 2 * k.numel() * 2 + 2 * (op.numel() + lp.numel()) * 4
        ts = []
        with torch.cuda.stream(stream):
            for i in range(reps + 3):
                junk.fill_(1)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                uno_tree_suffix_attention_merge(q, k, v, par, nn, op, lp, scale=d ** -0.5)
                b.record(stream)
                if i >= 3:
                    ts.append((a, b))
        stream.synchronize()
        us = statistics.median(a.elapsed_time(b) for a, b in ts) * 1e3
        gbs = nbytes / us / 1e3
        out[f"requests_{R}"] = {"us": us, "bytes": nbytes,
                                "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                                             "frac": gbs / peak}}
    out["note"] = ("tcgen05 tensor-core kernel (bf16 rows, d a multiple of 16); bound by latency at these sizes; "
                   "median of one-launch CUDA-event times, L2 rewritten before each launch")
    return out


def stress_leg(device, first, stream, peak, reps, cpu_budget):
    """The linear stress workload (512 requests, B = 16, fp32, T = 0.7): one
    uno_linear_cycle per replay.  Its 10.3 GB of logits are drawn on the GPU
    (torch's Philox generator, seed 123) with the recipe's distributions:
    base rows N(0, 1.5^2), targets = base + N(0, 1.0^2), the bonus row fresh."""
    import torch
    from speculative_decoding_verification_filter_b200 import uno_linear_cycle
    from speculative_decoding_verification_filter_b200.inputs import WORKLOADS, linear_draft, linear_target
    w = WORKLOADS[4]
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    base = torch.randn((w.R, w.B + 1, w.vocab), generator=gen, device=device) * w.sigma
    q = base[:, :w.B].contiguous()
    p = base
    p.add_(torch.randn(p.shape, generator=gen, device=device), alpha=w.noise)
    sp = dict(temperature=w.temperature, top_k=w.top_k, top_p=w.top_p)
    g = graph_of(lambda st: uno_linear_cycle(q, p, R=w.R, B=w.B, rng=(w.seed, 0, first), **sp), stream)
    ms = replay_ms(g, stream, reps)
    del g, q, p, base
    torch.cuda.empty_cache()
    import oracle

    def one(i):
        qn, pn = linear_draft(w, [i]), linear_target(w, [i])
        rq = oracle.filter_softmax(qn, w.dtype, w.temperature, w.top_k, w.top_p, rows_per_request=w.B,
                                   rng=(w.seed, 0, i))
        oracle.linear_verify(pn, w.dtype, 1, w.B, w.temperature, w.top_k, w.top_p, rq["sample"].reshape(1, w.B),
                             rq["ids"], rq["probs"], rq["count"], rng=(w.seed, 0, i))
    rate, done, spent = oracle_rate(one, cpu_budget)
    gbs = w.logit_bytes / (ms / 1e3) / 1e9
    return {"workload": f"{w.name}: R={w.R}, B={w.B}, vocab {w.vocab}, {w.dtype}, T={w.temperature}",
            "value": w.R / (ms / 1e3), "unit": UNIT, "ms_per_cycle": ms,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "bytes_per_cycle": w.logit_bytes},
            "l2": "inputs larger than L2",
            "data": "drawn on the GPU with the recipe's distributions (torch Philox, seed 123)",
            "timing": f"CUDA events around {reps} replays of one uno_linear_cycle graph",
            "cpu_baseline": {"value": rate, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"{done} requests (inputs.py rows), {spent:.1f} s, single-threaded C oracle"}}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args, w):
    import ctypes

    import torch
    from speculative_decoding_verification_filter_b200 import _binding as b
    from speculative_decoding_verification_filter_b200.inputs import linear_draft, linear_target

    rank, world, local = dist_env()
    init_dist(world)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    lib = b.load_library()
    first, reqs = shard(rank, w.R)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def dev(a):
        t = torch.from_numpy(a.view(np.int16) if w.dtype == "bf16" else a)
        return t.to(device).view(tdt)

    q_np = linear_draft(w, reqs)
    p_np = linear_target(w, reqs)
    q, p = dev(q_np), dev(p_np)
    nq, npr, V = w.q_rows, w.p_rows, w.vocab
    k = min(w.top_k, V)
    i32 = dict(dtype=torch.int32, device=device)
    toks, nacc = torch.empty((w.R, w.B + 1), **i32), torch.empty(w.R, **i32)
    ntok, rflags, drafts = torch.empty(w.R, **i32), torch.empty(w.R, **i32), torch.empty((w.R, w.B), **i32)
    ws = torch.zeros(lib.uno_linear_cycle_workspace_bytes(w.R, w.B, V, w.top_k, b.LAYOUT_GENERIC),
                     dtype=torch.uint8, device=device)
    sp = b._Params(w.temperature, w.top_k, w.top_p)
    dcode = b.UNO_BF16 if w.dtype == "bf16" else b.UNO_F32
    P = ctypes.c_void_p

    def cycle_step(stream):
        # one decode cycle: every draft and target row of the batch in one launch, then the decisions
        st = lib.uno_linear_cycle(P(q.data_ptr()), P(p.data_ptr()), dcode, w.R, w.B, V, b.LAYOUT_GENERIC, sp,
                                  b._Rng(w.seed, 0, first), P(toks.data_ptr()), P(nacc.data_ptr()),
                                  P(ntok.data_ptr()), P(rflags.data_ptr()), P(drafts.data_ptr()),
                                  P(ws.data_ptr()), ws.numel(), P(stream.cuda_stream))
        assert st == 0, b.STATUS.get(st, st)

    # the same cycle as two calls (filter + draws, then verification), for comparison
    q_ids, q_probs = torch.empty((nq, k), **i32), torch.empty((nq, k), dtype=torch.float32, device=device)
    q_count, q_flags, drafts2 = torch.empty(nq, **i32), torch.empty(nq, **i32), torch.empty(nq, **i32)
    toks2, acc2, ntok2, rflags2 = (torch.empty((w.R, w.B + 1), **i32), torch.empty(w.R, **i32),
                                   torch.empty(w.R, **i32), torch.empty(w.R, **i32))
    ws_q = torch.zeros(lib.uno_filter_softmax_workspace_bytes(nq, V, w.top_k), dtype=torch.uint8, device=device)
    ws_p = torch.zeros(lib.uno_linear_verify_workspace_bytes(w.R, w.B, V, w.top_k), dtype=torch.uint8,
                       device=device)

    def calls_step(stream):
        rng = b._Rng(w.seed, 0, first)
        st = lib.uno_filter_softmax(P(q.data_ptr()), dcode, nq, V, V, w.B, sp, k, P(q_ids.data_ptr()),
                                    P(q_probs.data_ptr()), P(q_count.data_ptr()), None, ctypes.byref(rng),
                                    P(drafts2.data_ptr()), P(q_flags.data_ptr()), P(ws_q.data_ptr()), ws_q.numel(),
                                    P(stream.cuda_stream))
        assert st == 0, b.STATUS.get(st, st)
        st = lib.uno_linear_verify(P(p.data_ptr()), dcode, w.R, w.B, V, sp, P(drafts2.data_ptr()),
                                   P(q_ids.data_ptr()), P(q_probs.data_ptr()), P(q_count.data_ptr()), k, rng,
                                   P(toks2.data_ptr()), P(acc2.data_ptr()), P(ntok2.data_ptr()),
                                   P(rflags2.data_ptr()), P(ws_p.data_ptr()), ws_p.numel(), P(stream.cuda_stream))
        assert st == 0, b.STATUS.get(st, st)

    stream = torch.cuda.Stream(device)
    for _ in range(max(3, args.warmup)):
        with torch.cuda.stream(stream):
            cycle_step(stream)
    stream.synchronize()
    g_cycle = graph_of(cycle_step, stream)
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            g_cycle.replay()
    torch.cuda.synchronize(device)

    K = args.steps

    def timed():
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world, device)
        with ClockSampler(device.index, period=0.001) as clk, torch.cuda.stream(stream):
            t0.record(stream)
            for a, bb in ev:
                a.record(stream)
                g_cycle.replay()
                bb.record(stream)
            t1.record(stream)
            stream.synchronize()
            # the clock record continues over 100 ms more of the same replays (untimed),
            # so that a short timed region still has a meaningful record
            t_end = time.perf_counter() + 0.1
            while time.perf_counter() < t_end:
                for _ in range(50):
                    g_cycle.replay()
                stream.synchronize()
        barrier(world, device)
        return t0.elapsed_time(t1), statistics.fmean(a.elapsed_time(bb) for a, bb in ev), clk.summary()

    total_ms, cyc_ms, clocks = timed()
    if any(r in clocks["reasons"] for r in BAD_REASONS):
        total_ms, cyc_ms, clocks = timed()  # re-measured once
    total_ms, cyc_ms = max_over_ranks([total_ms, cyc_ms], world, device)
    ms_step = total_ms / K
    value = w.R * world / (ms_step / 1e3)

    # the two-call form of the same cycle
    g_calls = graph_of(calls_step, stream)
    calls_ms = replay_ms(g_calls, stream, max(10, min(K, 200)))
    del g_calls

    # end to end through the public API from pinned host buffers
    from speculative_decoding_verification_filter_b200 import uno_linear_cycle
    q_host = torch.from_numpy(q_np.view(np.int16) if w.dtype == "bf16" else q_np).view(tdt).pin_memory()
    p_host = torch.from_numpy(p_np.view(np.int16) if w.dtype == "bf16" else p_np).view(tdt).pin_memory()
    sp_kw = dict(temperature=w.temperature, top_k=w.top_k, top_p=w.top_p)
    K_e2e = max(3, min(K, 20))

    def e2e_step(c):
        return uno_linear_cycle(q_host, p_host, R=w.R, B=w.B, rng=(w.seed, c, first), **sp_kw)

    for c in range(2):
        e2e_step(c)
    barrier(world, device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for c in range(K_e2e):
        out = e2e_step(c)
    e1.record()
    torch.cuda.synchronize(device)
    (e2e_ms,) = max_over_ranks([e0.elapsed_time(e1) / K_e2e], world, device)
    h2d = (q_host.numel() + p_host.numel()) * q_host.element_size()
    d2h = sum(t.numel() * t.element_size() for t in out.values())

    peak, peak_kind = hbm_peak()
    cycle_bytes = (npr + nq) * V * w.elem_bytes
    # the dominant kernel: the cycle's row kernel over all 1,088 rows; the CUDA
    # events bracket the graph, which also holds the short request-tail kernel,
    # so this understates the row kernel's own rate a little
    achieved = cycle_bytes / (cyc_ms / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic", "config": workload_config(w, world),
        "logits_gbs_per_gpu": cycle_bytes / (ms_step / 1e3) / 1e9,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": committed_traffic(),
                     "kernel": "pipe_kernel<bf16, cycle> + tail_kernel (uno_linear_cycle, 512 draft + 576 target "
                               "rows), CUDA events around each graph replay",
                     "bytes_per_launch": cycle_bytes,
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                     else "fallback (6,650 GB/s)", "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                     "cycle_ms": cyc_ms},
        "calls": {"note": "the same cycle as uno_filter_softmax then uno_linear_verify (3 kernels)",
                  "ms_per_cycle": calls_ms, "value": w.R / (calls_ms / 1e3)},
        "e2e": {"value": w.R * world / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h)},
        # uno_linear_cycle launches two kernels (rows, then request decisions)
        "gpu_launches": 2 * K,
        "clocks": dict(clocks, note="NVML every 1 ms over the timed steps and 100 ms more of the same replays"),
    }
    if not args.no_tree:
        line["per_request"] = params_leg(q, p, w, first, stream, peak, max(10, min(K, 100)))
        line["tree_16_32_32"] = tree_leg(2, device, first, stream, peak, 200, 3.0)
        line["tree_8_16_8"] = tree_leg(3, device, rank * 64, stream, peak, 100, 3.0)
        line["stress"] = stress_leg(device, first, stream, peak, 10, 4.0)
        line["suffix_attention_8b"] = suffix_attention_leg(device, stream, peak)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g_cycle
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    args = parse()
    if args.only == "suffix_attention":
        import torch
        device = torch.device("cuda", 0)
        peak, _ = hbm_peak()
        print(json.dumps(suffix_attention_leg(device, torch.cuda.Stream(device), peak, reps=10)), flush=True)
        return
    from speculative_decoding_verification_filter_b200.inputs import WORKLOADS
    w = WORKLOADS[args.workload]
    if w.mode != "linear":
        raise SystemExit("bench.py times the linear workloads")
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
