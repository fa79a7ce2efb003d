#!/usr/bin/env python
"""Throughput of the B200 speculative-decoding verifier.

One step = one verify call over one batch of B requests (B*(k+1) logit rows
of V entries), inputs already resident in HBM.  The headline workload
(`value`) is greedy verification at the Llama-3 vocabulary, B=64, k=5,
V=128256, bf16; the default run then times the other four verify
configurations the same way and reports each under `workloads`: the tiny
fp32 greedy batch, rejection sampling at the Qwen vocabulary, the large
batch with per-position top-8, and the 64-node draft trees.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--also A,B,...] [--intervals I] [--impl ours|reference]

Prints one JSON line.  Every workload is timed as I regions of exactly K
calls (a synchronize on both sides of each; a barrier too with N > 1); the
median region gives the figure and the min and max are reported beside it.
Multi-GPU: one rank per GPU (started here under torch.distributed.run when
--gpus N > 1 is given without a launcher); every rank verifies its own
batch (requests are independent; no collective on the data path) and each
time is the max over ranks.

The timed steps replay a CUDA graph of the C-ABI calls over a rotation of
input sets whose total exceeds 4x the L2 cache, so every step streams its
logits from HBM.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import gen  # noqa: E402

METRIC = "verified rows/s and achieved HBM GB/s (% of B200 peak) for B×(k+1)×V verify"
KERNEL_SOURCES = ["speculative_decoding_draft_decode_b200/csrc/verify_pass1.cuh",
                  "speculative_decoding_draft_decode_b200/csrc/verify_resample.cuh",
                  "speculative_decoding_draft_decode_b200/csrc/verify_common.cuh",
                  "speculative_decoding_draft_decode_b200/csrc/device_utils.cuh",
                  "speculative_decoding_draft_decode_b200/csrc/specdec_api.cu",
                  "speculative_decoding_draft_decode_b200/csrc/geometry.h",
                  "speculative_decoding_draft_decode_b200/csrc/philox.cuh"]
FALLBACK_HBM_GBS = 6650.0


def kernel_hash():
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def recorded_traffic(workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d.get(workload)
        if e and e.get("kernel_hash") == kernel_hash():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ---------------------------------------------------------------------------
# Workloads
# ---------------------------------------------------------------------------
def make_workload(name, seed_offset=0):
    base = {"greedy_llama3": (gen.greedy_llama3, 1), "greedy_tiny": (gen.greedy_tiny, 0),
            "greedy_large_batch": (gen.greedy_large_batch, 3), "tree_medusa": (gen.tree_medusa, 4),
            "rejection_qwen": (gen.rejection_qwen, 2), "greedy_ragged_tiers": (gen.greedy_ragged_tiers, 6),
            "rejection_qwen_adasd": (gen.rejection_qwen, 2)}
    fn, seed = base[name]
    inp = fn(seed=seed + 1000 * seed_offset)
    if name == "rejection_qwen_adasd":
        inp.stats = True
    return inp


def describe(inp):
    if isinstance(inp, gen.RaggedInputs):
        kb = np.diff(inp.offsets)
        return {"B": inp.B, "max_k": inp.max_k, "V": inp.V, "rows": inp.rows, "drafts": int(inp.offsets[-1]),
                "k_per_request": "tiers %s, mean %.2f" % (sorted(set(kb.tolist())), kb.mean()),
                "layout": "packed (draft offsets)", "counters": True}
    if isinstance(inp, gen.TreeInputs):
        return {"B": inp.B, "N": inp.N, "V": inp.V, "rows": inp.B * (inp.N + 1), "max_depth": inp.max_depth}
    d = {"B": inp.B, "k": inp.k, "V": inp.V, "rows": inp.B * (inp.k + 1)}
    if isinstance(inp, gen.GreedyInputs) and inp.topk:
        d["topk"] = inp.topk
    if isinstance(inp, gen.RejectionInputs):
        d["temperature"] = inp.temperature
        if inp.stats:
            d["adasd_stats"] = "draft entropy and Jensen-Shannon distance per draft position"
    return d


L2_POLICY = "inputs rotate over device copies totalling more than 4x the L2 cache, so every call reads HBM"


def line_config(name, inp, world):
    """The `config` of a JSON line: the workload and its shape.  Both arms
    (ours and the reference) emit the same dict for the same workload."""
    return dict(workload=name, **describe(inp), l2=L2_POLICY,
                parallelism="dp%d (requests per rank, no collective)" % world)


def rows_of(inp, req=None):
    """Logit rows of the first `req` requests (all by default)."""
    req = inp.B if req is None else req
    if isinstance(inp, gen.RaggedInputs):
        return int(inp.offsets[req]) + req
    return req * ((inp.N + 1) if isinstance(inp, gen.TreeInputs) else (inp.k + 1))


# ---------------------------------------------------------------------------
# Device side
# ---------------------------------------------------------------------------
def host_tensors(inp):
    """The workload's arrays as CPU torch tensors (bf16 logits keep their bits)."""
    import torch

    def logits_t(a, dt):
        if dt == gen.BF16:
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))

    def i32(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32))

    if isinstance(inp, gen.TreeInputs):
        return {"logits": logits_t(inp.logits, inp.dtype), "parents": i32(inp.parents),
                "node_tokens": i32(inp.node_tokens)}
    if isinstance(inp, gen.RejectionInputs):
        return {"target": logits_t(inp.target, inp.dtype),
                "q": torch.from_numpy(np.ascontiguousarray(inp.q, dtype=np.float32)), "drafts": i32(inp.drafts)}
    if isinstance(inp, gen.RaggedInputs):
        return {"logits": logits_t(inp.logits, inp.dtype), "drafts": i32(inp.drafts), "offsets": i32(inp.offsets)}
    return {"logits": logits_t(inp.logits, inp.dtype), "drafts": i32(inp.drafts)}


def host_pinned(inp):
    return {k: v.pin_memory() for k, v in host_tensors(inp).items()}


class DeviceSets:
    """`n` input sets on the device: set 0 from the generator, set i > 0 the
    same batch rolled by i*97 positions along the vocabulary (draft and node
    tokens rolled with it), so every set has the workload's structure but
    its own memory."""

    def __init__(self, inp, n, device):
        import torch
        self.inp = inp
        self.sets = []
        base = {k: v.to(device) for k, v in host_tensors(inp).items()}
        V = inp.V
        for i in range(n):
            s = (i * 97) % V
            if s == 0:
                self.sets.append(base)
                continue
            d = {}
            for key, t in base.items():
                if key in ("logits", "target", "q"):
                    d[key] = torch.roll(t, shifts=s, dims=-1).contiguous()
                elif key in ("drafts", "node_tokens"):
                    d[key] = torch.where(t >= 0, (t + s) % V, t)
                else:
                    d[key] = t
            self.sets.append(d)


def resample_bytes(inp, outs):
    """Rejection mode re-reads row h of every valid request (and q_h when
    h < k) to draw the correction or bonus token; the accepted lengths of the
    rotated input sets are those of the base set."""
    if not isinstance(inp, gen.RejectionInputs):
        return 0
    es = 2 if inp.dtype == gen.BF16 else 4
    al = outs[0].cpu().numpy()
    ok = al >= 0
    extra = 0
    if inp.stats:  # AdaSD statistics: target rows 0..k-1 and their q rows once more, 16 B out per position
        extra = int(ok.sum()) * inp.k * (inp.V * (es + 4) + 16)
    return int(inp.V * (es * ok.sum() + 4 * (ok & (al < inp.k)).sum())) + extra


SMALL_REQUEST_BYTES = 32768  # greedy requests up to this many logit bytes verify in one launch (no top-k)


def greedy_launches(inp):
    """Kernels one greedy call launches: one for requests of at most 32 KB of
    logits without top-k (a CTA per request), else the streaming pass and the
    request epilogue."""
    es = 2 if inp.dtype == gen.BF16 else 4
    k = inp.max_k if isinstance(inp, gen.RaggedInputs) else inp.k
    return 1 if inp.topk == 0 and (k + 1) * inp.V * es <= SMALL_REQUEST_BYTES else 2


def setup_calls(inp, sets, ver, device):
    """Static outputs and a list of per-set call closures (each one C-ABI
    call on the current stream)."""
    import torch
    import speculative_decoding_draft_decode_b200 as sd
    B = inp.B
    calls = []
    if isinstance(inp, gen.TreeInputs):
        al = torch.empty(B, dtype=torch.int32, device=device)
        nodes = torch.empty(B, inp.max_depth, dtype=torch.int32, device=device)
        ot = torch.empty(B, inp.max_depth + 1, dtype=torch.int32, device=device)
        outs = (al, nodes, ot)
        for s in sets:
            calls.append(lambda s=s: ver.tree(s["logits"], s["parents"], s["node_tokens"], inp.max_depth, out=outs))
        kernels = 2  # streaming pass + request epilogue
    elif isinstance(inp, gen.RejectionInputs):
        al = torch.empty(B, dtype=torch.int32, device=device)
        ot = torch.empty(B, inp.k + 1, dtype=torch.int32, device=device)
        pd = torch.empty(B, max(inp.k, 1), dtype=torch.float32, device=device)
        outs = (al, ot, pd)
        if inp.stats:
            outs = outs + (torch.empty(B, max(inp.k, 1), dtype=torch.float64, device=device),
                           torch.empty(B, max(inp.k, 1), dtype=torch.float64, device=device))
        for s in sets:
            calls.append(lambda s=s: ver.rejection(s["target"], s["q"], s["drafts"], inp.temperature, inp.seed,
                                                   inp.offset, out=outs, stats=inp.stats))
        kernels = 4  # softmax pass, request epilogue, chunk masses, token search
        if inp.stats:
            kernels += 2  # statistics chunks, statistics per position
    elif isinstance(inp, gen.RaggedInputs):
        R, T = inp.rows, int(inp.offsets[-1])
        al = torch.empty(B, dtype=torch.int32, device=device)
        ot = torch.empty(R, dtype=torch.int32, device=device)
        ids = torch.empty(R, max(inp.topk, 1), dtype=torch.int32, device=device)
        vals = torch.empty(R, max(inp.topk, 1), dtype=torch.float32, device=device)
        ctr = torch.zeros(3 + inp.max_k, dtype=torch.int64, device=device)
        outs = (al, ot, ids, vals, ctr)
        for s in sets:
            calls.append(lambda s=s: ver.greedy_ragged(s["logits"], s["drafts"], s["offsets"], T, inp.max_k,
                                                       topk=inp.topk, counters=ctr, out=outs[:4]))
        kernels = greedy_launches(inp)  # streaming pass + request epilogue (acceptance counters fused)
    else:
        k1 = inp.k + 1
        al = torch.empty(B, dtype=torch.int32, device=device)
        ot = torch.empty(B, k1, dtype=torch.int32, device=device)
        ids = torch.empty(B, k1, max(inp.topk, 1), dtype=torch.int32, device=device)
        vals = torch.empty(B, k1, max(inp.topk, 1), dtype=torch.float32, device=device)
        outs = (al, ot, ids, vals)
        for s in sets:
            calls.append(lambda s=s: ver.greedy(s["logits"], s["drafts"], topk=inp.topk, out=outs))
        kernels = greedy_launches(inp)  # streaming pass + request epilogue, or one launch for small requests
    return calls, outs, kernels


class ClockSampler:
    """nvidia-smi samples (200 ms) while the GPU runs the workload."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index, log_dir=None):
        import tempfile
        self.index = index
        self.proc = None
        self.path = os.path.join(log_dir or tempfile.gettempdir(), "specdec_clocks_rank%d.csv" % index)

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.QUERY,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) < 9:
                    continue
                try:
                    sm.append(float(p[1]))
                    mx = float(p[2])
                except ValueError:
                    continue
                for n, v in zip(names, p[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def dist_max(values, device, world):
    """Element-wise max over ranks of a list of floats (the list itself at one rank)."""
    if world == 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def measure(name, args, world, rank, local, device, cpu_seconds):
    """Times one workload on this rank's GPU and returns its entry of the JSON
    line: `intervals` timed regions of exactly `steps` calls each (a barrier
    and a synchronize on both sides of each), their median as the figure, the
    min and max beside it, all maxed over ranks."""
    import torch
    import torch.distributed as dist
    import speculative_decoding_draft_decode_b200 as sd

    inp = make_workload(name, seed_offset=rank)
    set_bytes = gen.algorithmic_bytes(inp)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    n_sets = max(2, math.ceil(4 * l2 / set_bytes) + 1) if args.sets is None else args.sets
    sets = DeviceSets(inp, n_sets, device).sets
    ver = sd.Verifier(device)
    sd.specdec_set_prefetch_inputs(False)
    calls, outs, kpl = setup_calls(inp, sets, ver, device)
    # The input sets and outputs were made on the default stream (the rolled
    # sets by kernels still queued there, and the outputs may reuse blocks of
    # its freed temporaries); the calls run on a stream of their own.
    torch.cuda.synchronize(device)
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for c in calls:  # allocates the workspace, loads the kernels
            c()
    stream.synchronize()
    per_replay = len(calls)
    graphs = {}

    def graph_of(n):
        # a graph of the first n calls, captured once (outside any timed region)
        if n not in graphs:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for c in calls[:n]:
                    c()
            graphs[n] = g
        return graphs[n]

    def capture_all():
        graphs.clear()  # the prefetch setting is baked into captured kernels
        graph_of(per_replay)
        for n in (args.warmup, args.steps):
            if n % per_replay:
                graph_of(n % per_replay)

    def run_steps(n):
        # exactly n calls, all from captured graphs
        full, rest = divmod(n, per_replay)
        for _ in range(full):
            graph_of(per_replay).replay()
        if rest:
            graph_of(rest).replay()

    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)

    def timed_intervals():
        with torch.cuda.stream(stream):
            run_steps(args.warmup)
        stream.synchronize()
        ms = []
        for _ in range(args.intervals):
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize(device)
            with torch.cuda.stream(stream):
                ev0.record(stream)
                run_steps(args.steps)
                ev1.record(stream)
            torch.cuda.synchronize(device)
            ms.append(ev0.elapsed_time(ev1))
        if world > 1:
            dist.barrier()
        med, lo, hi = dist_max([statistics.median(ms), min(ms), max(ms)], device, world)
        return med / args.steps, lo / args.steps, hi / args.steps

    capture_all()
    # clocks: sampled across a short untimed burst of the same steps and the timed region
    sampler = ClockSampler(local, args.clock_log_dir)
    sampler.start()
    t_probe = time.time()
    with torch.cuda.stream(stream):
        while time.time() - t_probe < args.clock_probe_seconds:
            run_steps(per_replay * 50)
            stream.synchronize()
    ms_step, ms_lo, ms_hi = timed_intervals()
    clocks = sampler.stop()

    # The same steps with the opt-in early loads of the streaming pass
    # (specdec_set_prefetch_inputs), reported beside the default: safe here,
    # the inputs were written by torch before any timed region.
    prefetch = None
    if not args.no_prefetch_leg:
        sd.specdec_set_prefetch_inputs(True)
        capture_all()
        prefetch = timed_intervals()
        sd.specdec_set_prefetch_inputs(False)

    # end to end: inputs from pinned host memory, H2D + verify + D2H each step
    e2e = run_e2e(inp, ver, device, stream, args.e2e_steps) if args.e2e_steps > 0 else None
    if e2e is not None:
        e2e["ms_per_step"] = dist_max([e2e["ms_per_step"]], device, world)[0]

    rows = rows_of(inp)
    peak, peak_kind = measured_peak()
    alg_bytes = set_bytes + resample_bytes(inp, outs)
    achieved = alg_bytes / (ms_step / 1e3) / 1e9
    res = {
        "value": rows * world / (ms_step / 1e3),
        "unit": "rows/s",
        "ms_per_step": ms_step,
        "us_per_call": ms_step * 1e3,
        "requests_per_s": inp.B * world / (ms_step / 1e3),
        "intervals": {"n": args.intervals, "steps_each": args.steps, "ms_per_step_median": ms_step,
                      "ms_per_step_min": ms_lo, "ms_per_step_max": ms_hi},
        "dtype": inp.dtype,
        "config": line_config(name, inp, world),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": "%s copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                     % peak_kind if peak_kind == "measured" else "fallback 6.65 TB/s",
                     "algorithmic_bytes_per_launch": alg_bytes, "traffic": recorded_traffic(name),
                     "duration_us": ms_step * 1e3, "kernels_per_step": kpl,
                     "note": "one call of every kernel of the step; duration = median timed region / steps "
                             "(launch gaps included)"},
        "timing": {"input_sets": n_sets, "input_bytes": n_sets * set_bytes, "l2_bytes": l2,
                   "launch": "CUDA graph of %d C-ABI calls, replayed" % per_replay},
        "gpu_launches": args.intervals * args.steps * kpl,
        "clocks": clocks,
    }
    if inp.B * (getattr(inp, "k", 0) + 1) * inp.V < 4_000_000:
        res["roofline"]["note"] += "; latency-bound at this size (report the time per call)"
    if prefetch is not None:
        pa = alg_bytes / (prefetch[0] / 1e3) / 1e9
        res["prefetch_inputs"] = {
            "note": "same steps with specdec_set_prefetch_inputs(1): the streaming pass loads its rows before the "
                    "previous kernel ends (opt-in; the library default is off and gives `value`)",
            "ms_per_step": prefetch[0], "ms_per_step_min": prefetch[1], "ms_per_step_max": prefetch[2],
            "value": rows * world / (prefetch[0] / 1e3), "achieved_gbs": pa, "frac": pa / peak}
    if e2e is not None:
        res["e2e"] = {"value": rows * world / (e2e["ms_per_step"] / 1e3), "unit": "rows/s",
                      "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                      "ms_per_step": e2e["ms_per_step"]}
    if rank == 0 and cpu_seconds > 0:
        res["cpu_baseline"] = cpu_baseline(inp, cpu_seconds)
    graphs.clear()
    del sets, calls, outs, ver
    torch.cuda.synchronize(device)
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    import torch
    import torch.distributed as dist
    from speculative_decoding_draft_decode_b200 import build as sd_build

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if rank == 0 or world == 1:
        sd_build.build()
    if world > 1:
        dist.barrier()

    head = measure(args.workload, args, world, rank, local, device, args.cpu_baseline_seconds)
    others = {}
    for name in args.also:
        if name != args.workload:
            others[name] = measure(name, args, world, rank, local, device, args.cpu_baseline_seconds / 3)
    line = {
        "metric": METRIC,
        "value": head["value"],
        "unit": "rows/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": head["dtype"],
        "data": "synthetic",
        "config": head["config"],
    }
    for key in ("requests_per_s", "intervals", "roofline", "gpu_launches", "clocks", "timing", "prefetch_inputs",
                "e2e", "cpu_baseline"):
        if key in head:
            line[key] = head[key]
    if others:
        line["workloads"] = others
        line["gpu_launches_all_workloads"] = head["gpu_launches"] + sum(o["gpu_launches"] for o in others.values())
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_vocab_shard(args):
    """Vocabulary-sharded greedy verification (Arctic page, "Speculator
    optimisation": each GPU holds a column slice of every logit row, takes its
    TopK, the results are all-gathered and the global TopK taken from them):
    one step = this rank's streaming pass over its columns, the all-gather of
    the row keys (NCCL over NVLink), and the combine with the accept scan.
    Every step verifies the one batch across all ranks (strong scaling).
    The rank-local kernels are also timed alone, replayed from CUDA graphs."""
    import datetime
    import torch
    import torch.distributed as dist
    import speculative_decoding_draft_decode_b200 as sd
    from speculative_decoding_draft_decode_b200 import build as sd_build
    from speculative_decoding_draft_decode_b200.sharding import vocab_range

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    if rank == 0 or world == 1:
        sd_build.build()
    if world > 1:
        dist.barrier()
    inp = make_workload(args.workload)  # the same batch on every rank
    if not isinstance(inp, gen.GreedyInputs):
        raise SystemExit("--shard vocab times greedy workloads only")
    B, k, V, topk = inp.B, inp.k, inp.V, inp.topk
    R = B * (k + 1)
    v0, v1 = vocab_range(V, world, rank)
    full = host_tensors(inp)
    shard = full["logits"][:, :, v0:v1].contiguous()
    es = shard.element_size()
    shard_bytes = shard.numel() * es
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    n_sets = max(2, math.ceil(4 * l2 / shard_bytes) + 1) if args.sets is None else args.sets
    sets = [shard.to(device) for _ in range(n_sets)]  # same values, separate memory
    drafts = full["drafts"].to(device)
    ver = sd.Verifier(device)
    kk = 8 if topk else 1
    keys = torch.empty(R, kk, dtype=torch.int64, device=device)
    vals = torch.empty(R, 8, dtype=torch.float32, device=device) if topk else None
    gk = torch.empty(world, R, kk, dtype=torch.int64, device=device)
    gv = torch.empty(world, R, 8, dtype=torch.float32, device=device) if topk else None
    outs = (torch.empty(B, dtype=torch.int32, device=device), torch.empty(B, k + 1, dtype=torch.int32, device=device),
            torch.empty(B, k + 1, max(topk, 1), dtype=torch.int32, device=device),
            torch.empty(B, k + 1, max(topk, 1), dtype=torch.float32, device=device))
    torch.cuda.synchronize(device)

    def step(i, exchange=True):
        ver.shard_greedy_rows(sets[i % n_sets], v0, topk, out=(keys, vals))
        if exchange and world > 1:
            dist.all_gather_into_tensor(gk, keys)
            if topk:
                dist.all_gather_into_tensor(gv, vals)
        else:
            gk[rank].copy_(keys)
            if topk:
                gv[rank].copy_(vals)
        ver.shard_greedy_combine(gk, gv, drafts, V, topk, out=outs)

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream = torch.cuda.Stream(device)
    graphs = {}

    def graph_of(exchange):
        # the rank-local steps (and, on one rank, the whole step) as one CUDA
        # graph of n_sets calls, so host launch time does not enter the timing
        if exchange not in graphs:
            with torch.cuda.stream(stream):
                for i in range(n_sets):
                    step(i, exchange)
            stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(n_sets):
                    step(i, exchange)
            graphs[exchange] = g
        return graphs[exchange]

    def run(n, exchange):
        if exchange and world > 1:  # the all-gather runs eagerly between the kernels
            for i in range(n):
                step(i, True)
            return
        full, rest = divmod(n, n_sets)
        for _ in range(full):
            graph_of(exchange).replay()
        for i in range(rest):
            step(i, exchange)

    def timed(exchange):
        with torch.cuda.stream(stream):
            run(args.warmup, exchange)
        ms = []
        for _ in range(args.intervals):
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize(device)
            with torch.cuda.stream(stream):
                ev0.record(stream)
                run(args.steps, exchange)
                ev1.record(stream)
            torch.cuda.synchronize(device)
            ms.append(ev0.elapsed_time(ev1))
        med, lo, hi = dist_max([statistics.median(ms), min(ms), max(ms)], device, world)
        return med / args.steps, lo / args.steps, hi / args.steps

    sampler = ClockSampler(local, args.clock_log_dir)
    sampler.start()
    ms_step, ms_lo, ms_hi = timed(True)
    clocks = sampler.stop()
    local_ms = timed(False)
    peak, peak_kind = measured_peak()
    alg_local = shard_bytes + R * kk * 8 + (R * 32 if topk else 0)  # this rank's columns, its row keys and values
    achieved_local = alg_local / (local_ms[0] / 1e3) / 1e9
    xbytes = (world - 1) * R * (kk * 8 + (32 if topk else 0))  # what one rank receives per step
    line = {
        "metric": METRIC, "value": R / (ms_step / 1e3), "unit": "rows/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": inp.dtype, "data": "synthetic",
        "config": dict(workload=args.workload, **describe(inp), l2=L2_POLICY,
                       parallelism="vocabulary split over %d ranks (one all-gather of row keys per step)" % world),
        "intervals": {"n": args.intervals, "steps_each": args.steps, "ms_per_step_median": ms_step,
                      "ms_per_step_min": ms_lo, "ms_per_step_max": ms_hi},
        "rank_local": {"ms_per_step": local_ms[0], "ms_per_step_min": local_ms[1], "ms_per_step_max": local_ms[2],
                       "note": "streaming pass over this rank's columns, row keys and combine, without the all-gather",
                       "achieved_gbs": achieved_local, "frac": achieved_local / peak,
                       "algorithmic_bytes_per_rank": alg_local},
        "exchange": {"bytes_received_per_rank_per_step": xbytes,
                     "ms_per_step": max(0.0, ms_step - local_ms[0]),
                     "note": "all-gather time = step time minus rank-local time"},
        "roofline": {"bound": "hbm", "achieved": achieved_local, "peak": peak, "unit": "GB/s",
                     "frac": achieved_local / peak, "traffic": None,
                     "peak_source": "%s copy bandwidth (MEASURED_PEAKS.json hbm_gbs)" % peak_kind,
                     "note": "rank-local kernels: this rank's column bytes over their time"},
        "gpu_launches": args.intervals * args.steps * 3, "clocks": clocks,
        "timing": {"input_sets": n_sets,
                   "launch": "rank-local kernels replayed from CUDA graphs; with more than one rank the step's "
                             "all-gather runs eagerly between eager kernel launches"},
    }
    graphs.clear()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_e2e(inp, ver, device, stream, steps):
    """Public API end to end: pinned host inputs -> device, verify, result -> host."""
    import torch
    h = host_pinned(inp)
    d = {k: torch.empty_like(v, device=device) for k, v in h.items()}
    calls, outs, _ = setup_calls(inp, [d], ver, device)
    res_h = [torch.empty_like(o, device="cpu").pin_memory() for o in outs[:2]]
    stream.wait_stream(torch.cuda.current_stream(device))  # buffers made on the default stream
    h2d = sum(v.numel() * v.element_size() for v in h.values())
    d2h = sum(o.numel() * o.element_size() for o in res_h)

    def step():
        for key, v in h.items():
            d[key].copy_(v, non_blocking=True)
        calls[0]()
        for o, r in zip(outs[:2], res_h):
            r.copy_(o, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(3):
            step()
    stream.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(steps):
            step()
        ev1.record(stream)
    stream.synchronize()
    return {"ms_per_step": ev0.elapsed_time(ev1) / steps, "h2d": h2d, "d2h": d2h}


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline leg and the reference arm)
# ---------------------------------------------------------------------------
def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_call(inp, req, threads=1):
    """The oracle on requests [0, req) of the workload (`threads` > 1: the
    oracle's request-parallel driver over the same per-request code)."""
    import oracle
    if isinstance(inp, gen.TreeInputs):
        return oracle.verify_tree(inp.logits[:req], inp.dtype, inp.parents[:req], inp.node_tokens[:req],
                                  inp.max_depth, threads=threads)
    if isinstance(inp, gen.RejectionInputs):
        res = oracle.verify_rejection(inp.target[:req], inp.dtype, inp.q[:req], inp.drafts[:req],
                                      inp.temperature, inp.seed, inp.offset, threads=threads)
        if inp.stats:
            res = res + oracle.draft_stats(inp.target[:req], inp.dtype, inp.q[:req], inp.temperature)
        return res
    if isinstance(inp, gen.RaggedInputs):
        t = int(inp.offsets[req])
        return oracle.verify_greedy_ragged(inp.logits[:t + req], inp.dtype, inp.drafts[:t], inp.offsets[:req + 1],
                                           inp.max_k, topk=inp.topk)
    return oracle.verify_greedy(inp.logits[:req], inp.dtype, inp.drafts[:req], topk=inp.topk, threads=threads)


def oracle_threads(inp, threads):
    """Threads the oracle can use on this workload (the packed layout has no
    parallel driver)."""
    return 1 if isinstance(inp, gen.RaggedInputs) else max(1, threads)


def time_oracle(inp, seconds, threads=1):
    threads = oracle_threads(inp, threads)
    t0 = time.perf_counter()
    oracle_call(inp, 1)
    one = max(time.perf_counter() - t0, 1e-6)
    req = int(max(min(threads, inp.B), min(inp.B, threads * seconds / 4 / one)))
    rows, el = 0, 0.0
    while el < seconds:
        t0 = time.perf_counter()
        oracle_call(inp, req, threads)
        el += time.perf_counter() - t0
        rows += rows_of(inp, req)
    return rows / el, req, rows, threads


def cpu_baseline(inp, seconds):
    """The oracle on the host: all cores (request-parallel driver) for 2/3 of
    the budget, one core for the rest."""
    v, req, rows, th = time_oracle(inp, seconds * 2 / 3, host_cores())
    v1, req1, rows1, _ = time_oracle(inp, seconds / 3, 1)
    return {"value": v, "unit": "rows/s", "cores": th, "kind": "oracle",
            "sample": "first %d requests of the workload, repeated for %.0f s (%d rows) on %d threads of the "
                      "fp64 C++ oracle (request-parallel driver over its per-request code)"
                      % (req, seconds * 2 / 3, rows, th),
            "single_thread": {"value": v1, "cores": 1,
                              "sample": "first %d requests, %.0f s (%d rows)" % (req1, seconds / 3, rows1)}}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    inp = make_workload(args.workload)
    budget = 120.0
    # each step verifies a bounded sample of requests so the run fits the budget
    v1, req1, _, th = time_oracle(inp, 2.0, host_cores())
    rpr = rows_of(inp) / inp.B
    step_budget = budget / max(1, args.steps + args.warmup)
    req = int(max(1, min(inp.B, step_budget * v1 / rpr)))
    for _ in range(args.warmup):
        oracle_call(inp, req, th)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_call(inp, req, th)
    el = time.perf_counter() - t0
    value = rows_of(inp, req) * args.steps / el
    sample = "first %d of %d requests per step, fp64 C++ oracle on %d threads" % (req, inp.B, th)
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus or 1)))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "rows/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": inp.dtype,
            "data": "synthetic", "config": line_config(args.workload, inp, world),
            "cpu_baseline": {"value": value, "unit": "rows/s", "cores": th, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "rows/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


SUITE = ("greedy_llama3", "greedy_tiny", "rejection_qwen", "greedy_large_batch", "tree_medusa")
WORKLOADS = SUITE + ("greedy_ragged_tiers", "rejection_qwen_adasd")


def relaunch_under_torchrun(args):
    """`--gpus N` (N > 1) without a torch.distributed launcher: start N ranks
    here, one per GPU, and return their exit status."""
    import signal
    import socket
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=%d" % args.gpus,
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
    proc = subprocess.Popen(cmd, start_new_session=True)
    try:
        return proc.wait(timeout=args.launch_timeout)
    except subprocess.TimeoutExpired:
        os.killpg(proc.pid, signal.SIGTERM)
        try:
            proc.wait(timeout=60)
        except subprocess.TimeoutExpired:
            os.killpg(proc.pid, signal.SIGKILL)
        print("bench: the %d ranks did not finish within %d s" % (args.gpus, args.launch_timeout), file=sys.stderr)
        return 1


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=None,
                    help="GPUs (one rank each); without a torch.distributed launcher N > 1 starts the ranks itself")
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--clock-log-dir", default=None,
                    help="directory for the raw nvidia-smi clock samples (default: the system temp directory)")
    ap.add_argument("--workload", default="greedy_llama3", choices=WORKLOADS,
                    help="the headline workload (`value` of the line)")
    ap.add_argument("--also", default=",".join(w for w in SUITE if w != "greedy_llama3"),
                    help="comma-separated workloads timed after the headline one and reported under `workloads` "
                         "(default: the rest of the five verify configurations; '' for none)")
    ap.add_argument("--intervals", type=int, default=30, help="timed regions of exactly --steps calls per workload")
    ap.add_argument("--sets", type=int, default=None, help="input sets in the rotation (default: > 4x L2)")
    ap.add_argument("--no-prefetch-leg", action="store_true",
                    help="skip timing the opt-in early-load mode beside the default")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-baseline-seconds", type=float, default=12.0,
                    help="oracle time for the headline workload's CPU baseline (a third of it for each other one)")
    ap.add_argument("--clock-probe-seconds", type=float, default=1.0,
                    help="untimed burst of the same steps while nvidia-smi samples clocks")
    ap.add_argument("--launch-timeout", type=int, default=1800, help="seconds for ranks started by --gpus N")
    ap.add_argument("--shard", choices=["requests", "vocab"], default="requests",
                    help="requests: every rank verifies its own batch (default); vocab: one batch with its "
                         "vocabulary split over the ranks (greedy workloads)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.steps < 1 or args.intervals < 1:
        ap.error("--steps and --intervals must be positive")
    args.also = [w for w in args.also.split(",") if w]
    bad = [w for w in args.also if w not in WORKLOADS]
    if bad:
        ap.error("unknown workloads in --also: %s" % ", ".join(bad))
    env_world = os.environ.get("WORLD_SIZE")
    if env_world is not None and args.gpus is not None and int(env_world) != args.gpus:
        ap.error("--gpus %d but the launcher started WORLD_SIZE=%s ranks" % (args.gpus, env_world))
    return args


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
        return 0
    if os.environ.get("WORLD_SIZE") is None and (args.gpus or 1) > 1:
        return relaunch_under_torchrun(args)
    if args.shard == "vocab":
        run_vocab_shard(args)
    else:
        run_ours(args)
    return 0


if __name__ == "__main__":
    sys.exit(main())
