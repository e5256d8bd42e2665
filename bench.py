#!/usr/bin/env python
"""Benchmark of the exact-load expert rebalancing hot path on B200.

One step = one layer instance through the whole path on the device:
gate top-k -> exact histogram -> replication plan -> reroute -> permute ->
gate-weighted combine (identity experts: the combine reads the dispatch
buffer). The default workload is the largest layer that fits one GPU, the
EP40 prefill layer (R=40 simulated EP ranks x 8192 tokens, E=160, K=8, S=1,
d=5120, 2.6 M pairs) with synthetic per-source-rank Zipf skew; --workload
selects another (the Qwen3-235B-shaped layer, the DeepSeek-V3-shaped layer,
the small R=8 layer).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ue|reference]

Prints one JSON line (rank 0). ``value`` is routed token-expert pairs per
second over all GPUs, device-timed with CUDA events (max over ranks).
With N > 1 (torchrun) every GPU runs its own layer instance (a different
microbatch): weak scaling, no data-path collective.
``--impl reference`` times the CPU oracle on a bounded sample of the same
workload on the host cores (rank 0 only).
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = ("routed token-expert pairs/s and µs/layer (gate→plan→permute), "
          "% of HBM roofline")
UNIT = "pairs/s"
DEFAULT_WORKLOAD = "prefill_ep40_e160"
KERNELS = ("gate_count", "plan", "reroute", "permute", "combine")
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal: the roofline is also reported against it

# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) of
# each workload's kernels, from one ncu capture of the same workload at a
# fraction of its tokens per rank, scaled up by the token ratio (the traffic
# of every kernel but the plan grows in proportion to the tokens; the
# plan's, a few KB of loads and outputs, does not and is taken as measured),
# with the SHA-256 prefix of the kernel source it was taken on; a kernel
# changed since then reports null.
TRAFFIC = {
    # ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum at 1024 tokens
    # per rank (6 launches each), times 8
    "prefill_ep40_e160": {
        "permute": {"bytes_per_launch": 29715613013, "source_sha": "07222823ab0e9db7"},
        "combine": {"bytes_per_launch": 33329068032, "source_sha": "c0631738399ffc37"},
    },
    # ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum at 512 tokens
    # per rank (8 launches each), times 4
    "dsv3_layer_r64_e256": {
        "permute": {"bytes_per_launch": 16669049472, "source_sha": "07222823ab0e9db7"},
        "combine": {"bytes_per_launch": 18684903552, "source_sha": "c0631738399ffc37"},
    },
    # ncu --set full at 512 tokens per rank, times 8
    "qwen3_layer_r64_e128": {
        "permute": {"bytes_per_launch": 18890168000, "source_sha": "07222823ab0e9db7"},
        "combine": {"bytes_per_launch": 21242032000, "source_sha": "c0631738399ffc37"},
    },
}

def sha_of(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


KERNEL_SRC = {
    "gate_count": "k_gate.cu", "plan": "k_plan.cu",
    "reroute": "k_reroute.cu", "permute": "k_permute.cu", "combine": "k_combine.cu",
}


def algorithmic_bytes(w):
    """Bytes each step must move per kernel (reads + writes of its operands).
    The histogram is taken inside the gate kernel (gate_count), so it adds no
    bytes there; "count" is the separate count kernel's, for reference."""
    N, E, K, d, Q = w.N, w.E, w.K, w.d, w.Q
    return {
        "gate_count": 4 * N * E + 8 * Q,         # logits in; idx + w out (counts are tiny)
        "count": 4 * Q,                          # idx in (the separate kernel)
        "plan": 0,                               # latency bound: reported in us
        "reroute": 4 * Q + 8 * Q,                # idx in; phys_slot + dest_row out
        "permute": 2 * N * d + 2 * Q * d,        # each row read once, written K times
        "combine": 2 * Q * d + 8 * Q + 4 * N * d,  # K rows + dest/w in; fp32 row out
    }


def row_bytes(N=0, K=0, d=0, used=0, replicated=0, bytes_per_expert=0, numel=0):
    """Bytes each row beside the path must move (reads + writes of its operands).
    combine backward: dout fp32 and the K bf16 rows y in, dest + w in, the K
    bf16 rows dy and the fp32 dw out; permute backward: the K bf16 rows and
    dest in, one fp32 row out; weight sync: every used slot's expert read and
    written once; gradient reduction: each replicated master read and written,
    each used replica slot read (fp32)."""
    Q = N * K
    return {
        "combine_backward": 4 * N * d + 2 * Q * d + 8 * Q + 2 * Q * d + 4 * Q,
        "permute_backward": 2 * Q * d + 4 * Q + 4 * N * d,
        "weight_sync": 2 * used * bytes_per_expert,
        "grad_reduce": 4 * numel * (2 * replicated + used),
    }


def kernels_per_step(w, num_sms=148):
    """Kernel launches of one step: the gate with the count fused in (K = 8, E
    a multiple of 32 from 64 to 256, each gate CTA's rows within four source
    ranks), else the gate kernel plus the count kernel; then plan, reroute,
    permute and combine. Mirrors the library's gate launch shape."""
    fused = w.K == 8 and w.E % 32 == 0 and 64 <= w.E <= 256
    if fused:
        target = num_sms * 4
        rpc = max(4, ((w.N + target - 1) // target + 3) // 4 * 4)
        fused = (rpc + w.T - 1) // w.T + 1 <= 4
    return 5 if fused else 6


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------- clocks ----
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the bench runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix="ue_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        pw = [num(r[3]) for r in rows if num(r[3]) is not None]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        # samples under load: power above the midpoint of what was seen
        if pw and len(pw) == len(sm):
            cut = (min(pw) + max(pw)) / 2
            loaded = [s for s, p in zip(sm, pw) if p >= cut] or sm
        else:
            loaded = sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(pw) if pw else None}


# ----------------------------------------------------------- distributed ----
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if n_gpus > 1 and world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} needs torchrun with {n_gpus} processes "
                         f"(WORLD_SIZE={world})")
    return world, rank, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Largest value over all ranks (the slowest rank sets the time)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------- oracle -----
def oracle_slices(w, logits, hidden, tokens_per_rank, budget_s, max_slices):
    """Run the CPU oracle over slices of the workload (every rank's tokens
    [j*t, (j+1)*t)), each as one layer instance: gate -> count -> plan ->
    reroute -> permute -> combine. Stops after budget_s seconds or
    max_slices slices. Returns (pairs, seconds, slices)."""
    import oracle
    t = tokens_per_rank
    pairs, elapsed, done = 0, 0.0, 0
    nsl = max(1, w.T // t)
    lg3 = logits.reshape(w.R, w.T, w.E)
    hd3 = hidden.reshape(w.R, w.T, w.d)
    for j in range(min(nsl, max_slices)):
        lg = lg3[:, j * t:(j + 1) * t].reshape(-1, w.E).copy()
        hd = hd3[:, j * t:(j + 1) * t].reshape(-1, w.d).copy()
        t0 = time.perf_counter()
        o = oracle.run_path(lg, w.R, t, w.S, w.K)
        disp = oracle.permute(hd, w.K, o["dest_row"])
        oracle.combine(disp, w.R * t, w.K, o["dest_row"], o["w"])
        elapsed += time.perf_counter() - t0
        pairs += w.R * t * w.K
        done += 1
        del disp
        if elapsed >= budget_s:
            break
    return pairs, elapsed, done


def host_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def threaded_oracle_slice(w, lg, hd, t, threads, bufs=None):
    """One slice (t tokens per rank, every rank) through the oracle's own C
    functions with the data-parallel steps split over host threads by token
    range: top-k and the weights, the counts (by source-rank range), the
    permute (by dispatch-row range) and the combine (by token range); the
    plan and the reroute stay sequential. The oracle's C calls release the
    interpreter lock, so the ranges run in parallel. bufs: optional
    preallocated (dispatch uint16 [Q][d], out float64 [N][d]), reused across
    slices so that first-touch page faults stay out of the timing. Returns
    the outputs."""
    from concurrent.futures import ThreadPoolExecutor

    import numpy as np

    import oracle
    R, E, K, d = w.R, w.E, w.K, w.d
    N, Q = R * t, R * t * K
    nt = max(1, threads)

    def ranges(n, parts):
        b = np.linspace(0, n, min(parts, n) + 1).astype(np.int64)
        return [(int(b[j]), int(b[j + 1])) for j in range(len(b) - 1) if b[j + 1] > b[j]]

    idx = np.empty((N, K), dtype=np.int32)
    wts = np.empty((N, K), dtype=np.float64)
    load_re = np.empty((R, E), dtype=np.int32)
    if bufs is None:
        dispatch = np.empty((Q, d), dtype=np.uint16)
        out = np.empty((N, d), dtype=np.float64)
    else:
        dispatch, out = bufs
    with ThreadPoolExecutor(nt) as ex:
        def gate(ab):
            a, b = ab
            idx[a:b], wts[a:b] = oracle.gate_topk(lg[a:b], K)
        list(ex.map(gate, ranges(N, nt)))

        def count(rr):
            r0, r1 = rr
            load_re[r0:r1], _ = oracle.count(idx[r0 * t:r1 * t], r1 - r0, t, E)
        list(ex.map(count, ranges(R, nt)))
        load_e = load_re.sum(axis=0, dtype=np.int64).astype(np.int32)
        pl = oracle.plan(load_e, R, w.S)
        phys, dest = oracle.reroute(idx, R, E, w.S, pl)

        def permute(ab):
            a, b = ab
            oracle.permute_rows(hd, K, dest, np.arange(a, b, dtype=np.int64), out=dispatch[a:b])
        list(ex.map(permute, ranges(Q, nt)))

        def combine(ab):
            a, b = ab
            oracle.combine(dispatch, N, K, dest, wts, tokens=np.arange(a, b, dtype=np.int64),
                           out=out[a:b])
        list(ex.map(combine, ranges(N, nt)))
    return dict(idx=idx, w=wts, load_re=load_re, load_e=load_e, plan=pl, phys_slot=phys,
                dest_row=dest, dispatch=dispatch, out=out)


def check_threaded_slice(w, lg, hd, t, res):
    """The threaded slice's outputs against the single-threaded oracle's on
    the same slice: every array equal (the same C functions on the same
    data; only the split differs)."""
    import numpy as np

    import oracle
    o = oracle.run_path(lg, w.R, t, w.S, w.K)
    for k in ("idx", "w", "load_re", "load_e", "phys_slot", "dest_row"):
        if not np.array_equal(res[k], o[k]):
            raise SystemExit(f"threaded CPU baseline differs from the oracle in {k}")
    for f in ("slot_expert", "n_copies", "slot_quota", "slot_offset", "rank_load", "stats"):
        if not np.array_equal(getattr(res["plan"], f), getattr(o["plan"], f)):
            raise SystemExit(f"threaded CPU baseline differs from the oracle in the plan ({f})")
    disp = oracle.permute(hd, w.K, o["dest_row"])
    if not np.array_equal(res["dispatch"], disp):
        raise SystemExit("threaded CPU baseline differs from the oracle in the dispatch rows")
    out = oracle.combine(disp, w.R * t, w.K, o["dest_row"], o["w"])
    if not np.array_equal(res["out"], out):
        raise SystemExit("threaded CPU baseline differs from the oracle in the combine")


def threaded_oracle_slices(w, logits, hidden, tokens_per_rank, budget_s, max_slices,
                           threads):
    """oracle_slices with the threaded split (threaded_oracle_slice). Before
    the timing, the threaded split is checked against the single-threaded
    oracle on a 64-token-per-rank slice of the same workload. Returns
    (pairs, seconds, slices)."""
    import numpy as np
    t = tokens_per_rank
    pairs, elapsed, done = 0, 0.0, 0
    nsl = max(1, w.T // t)
    lg3 = logits.reshape(w.R, w.T, w.E)
    hd3 = hidden.reshape(w.R, w.T, w.d)
    tc = min(64, w.T)
    lgc = lg3[:, :tc].reshape(-1, w.E).copy()
    hdc = hd3[:, :tc].reshape(-1, w.d).copy()
    check_threaded_slice(w, lgc, hdc, tc, threaded_oracle_slice(w, lgc, hdc, tc, threads))
    bufs = (np.empty((w.R * t * w.K, w.d), dtype=np.uint16),
            np.empty((w.R * t, w.d), dtype=np.float64))
    for b in bufs:
        b.fill(0)  # touch every page before the timing
    for j in range(min(nsl, max_slices)):
        lg = lg3[:, j * t:(j + 1) * t].reshape(-1, w.E).copy()
        hd = hd3[:, j * t:(j + 1) * t].reshape(-1, w.d).copy()
        t0 = time.perf_counter()
        res = threaded_oracle_slice(w, lg, hd, t, threads, bufs)
        elapsed += time.perf_counter() - t0
        pairs += w.R * t * w.K
        done += 1
        del res
        if elapsed >= budget_s:
            break
    return pairs, elapsed, done


def run_reference(args, w):
    world, rank, _ = dist_setup(args.gpus)
    if rank != 0:
        return
    import synth
    logits = synth.logits(w, mb=0)
    hidden = synth.hidden(w)
    # size each step so that warm-up + timed steps take about two minutes
    per_step_s = max(0.05, 120.0 / max(1, args.steps + args.warmup))
    t = 512
    while t > 8 and 2.2 * (t / 512) > per_step_s:
        t //= 2
    for _ in range(args.warmup):
        oracle_slices(w, logits, hidden, t, 0.0, 1)
    pairs, secs, n = 0, 0.0, 0
    for _ in range(args.steps):
        p, s, _k = oracle_slices(w, logits, hidden, t, 0.0, 1)
        pairs += p
        secs += s
        n += 1
    value = pairs / secs
    sample = (f"{t} tokens per rank x {w.R} ranks ({w.R * t * w.K} pairs) per step, the first "
              f"slice of the {w.name} workload, whole path incl. permute and combine")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / max(1, n), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


ROUTING_TEXT = {
    "small_r8_e64": "Zipf(s=1.2) log-weight bias in a seeded expert permutation",
    "qwen3_layer_r64_e128": "Zipf(s=1.0) log-weight bias scaled so that the masters-only "
                            "max/mean rank load is 2.5",
    "dsv3_layer_r64_e256": "Zipf(s=1.3) log-weight bias plus two seeded hotspot experts "
                           "boosted to draw 8% of pairs each",
    "prefill_ep40_e160": "per-source-rank Zipf bias, s_r ~ U[0.8, 1.5] for each rank over one "
                         "shared expert permutation (skew differs by source rank)",
    "pages_ep64_e256_t8k": "Zipf(s=1.0) log-weight bias scaled to the pages' runtime-test "
                           "imbalance 2.01",
}
L2_BYTES = 126 * 2 ** 20


def workload_config(w):
    base = w.name.split("_t")[0] if w.name not in ROUTING_TEXT else w.name
    routing = ("logits N(0,1) + " + ROUTING_TEXT.get(base, f"{w.recipe} bias")
               + ", seed 0 (microbatch = rank)")
    lb, hb, db = 4 * w.N * w.E, 2 * w.N * w.d, 2 * w.Q * w.d
    def size(b):
        return f"{b / 1e9:.2f} GB" if b >= 1e9 else f"{b / 1e6:.1f} MB"

    sizes = f"logits {size(lb)}, hidden {size(hb)}, dispatch {size(db)}"
    l2 = (f"inputs larger than L2 ({sizes}); no flush needed" if db > 2 * L2_BYTES
          else f"inputs L2-resident ({sizes}); not flushed between steps")
    return {"workload": w.name, "R": w.R, "T": w.T, "N": w.N, "E": w.E, "K": w.K, "S": w.S,
            "d": w.d, "pairs_per_step": w.Q, "routing": routing, "l2": l2,
            "experts": "identity (combine reads the dispatch buffer)"}


# ----------------------------------------------------------------- sweep ----
def run_sweep(args):
    """All 48 x 8 instances of the non-stationary sweep through one CUDA graph
    of the whole path. Each instance's logits are staged into the input
    buffer outside the timed region; each replay is timed with CUDA events.
    Reports the distribution of us per layer and of the imbalance. --planner
    bisect plans with the capacity planner at the pages' defaults instead of
    the greedy rule."""
    import numpy as np
    import torch

    import synth
    import token_rerouting_b200 as ue
    from token_rerouting_b200 import build as ue_build

    ue_build.build()
    w = synth.WORKLOADS["sweep_48x8_r64_e128"]
    dev = torch.device("cuda", 0)
    L = ue.Layer(w.R, w.T, w.E, w.K, w.S, w.d, device=0)
    L.hidden.copy_(torch.from_numpy(synth.hidden(w).view(np.int16)).to(dev).view(torch.bfloat16))
    L.logits.copy_(torch.from_numpy(synth.logits(w, 0, 0)))
    opts = ue.plan_opts(ue.UE_SOLVER_BISECT) if args.planner == "bisect" else None

    def run_once(st):
        L.gate_count(st)
        if opts is None:
            L.plan_reroute(st)
        else:
            L.plan_ex(opts, st)
            L.reroute(st)
        L.permute(st)
        L.combine(stream=st)

    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        for _ in range(max(3, args.warmup)):
            run_once(s)
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        run_once(s)
    torch.cuda.synchronize(dev)
    stage = torch.empty(L.logits.shape, dtype=torch.float32).pin_memory()
    times, before, after, copies = [], [], [], []
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(0)
    clocks.start()
    for layer in range(w.layers):
        for mb in range(w.microbatches):
            stage.copy_(torch.from_numpy(synth.logits(w, layer, mb)))
            L.logits.copy_(stage, non_blocking=True)
            torch.cuda.synchronize(dev)
            a.record()
            graph.replay()
            b.record()
            torch.cuda.synchronize(dev)
            times.append(a.elapsed_time(b) * 1e3)
            st = L.stats.cpu().numpy()
            before.append(float(st[1]) / (w.Q / w.R))
            after.append(float(st[2]) / (w.Q / w.R))
            copies.append(int((L.slot_expert[: w.G] >= 0).sum().item()))
    clk = clocks.stop()
    rc = L.error()
    L.close()
    if rc != 0:
        raise SystemExit(f"device error in the sweep: {ue.STATUS.get(rc, rc)}")

    def dist(x):
        x = np.asarray(x, dtype=np.float64)
        return {"min": float(x.min()), "median": float(np.median(x)), "max": float(x.max())}

    total_s = sum(times) / 1e6
    line = {
        "metric": METRIC, "value": len(times) * w.Q / total_s, "unit": UNIT, "n_gpus": 1,
        "steps": len(times), "warmup": max(3, args.warmup),
        "ms_per_step": 1e3 * total_s / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "R": w.R, "T": w.T, "E": w.E, "K": w.K, "S": w.S,
                   "d": w.d, "instances": len(times), "pairs_per_instance": w.Q,
                   "graph": "whole path captured once, replayed per instance",
                   "planner": args.planner + ("" if opts is None else
                                              " (capacity planner: eps 0.01, early stop 1.0, "
                                              "minimum 1024 pairs per replica)"),
                   "l2": "inputs larger than L2"},
        "us_per_layer": dist(times), "max_over_mean_before": dist(before),
        "max_over_mean_after": dist(after), "copies": dist(copies), "clocks": clk,
        "gpu_launches": kernels_per_step(w) * len(times),
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- rows ----
EXPERT_NUMEL = 2 * 4096 * 1536 + 4096 * 1536  # Qwen3-235B expert: fc1 2hf + fc2 hf


def expert_numel(args):
    return args.expert_numel or EXPERT_NUMEL


def run_row(args, w):
    """Backward of combine / permute, weight sync or gradient reduction on the
    Qwen3-shaped layer (expert tensors of Qwen3-235B size), device-timed."""
    import numpy as np
    import torch

    import token_rerouting_b200 as ue
    from token_rerouting_b200 import build as ue_build

    ue_build.build()
    dev = torch.device("cuda", 0)
    gen = torch.Generator(device=dev).manual_seed(0)
    rows_d = w.d if args.row in ("backward", "layouts") else 8
    L = ue.Layer(w.R, w.T, w.E, w.K, w.S, rows_d, device=0,
                 with_rows=args.row == "layouts")
    L.logits.copy_(torch.from_numpy(synth_logits(w)))
    L.run_routing()
    torch.cuda.synchronize(dev)
    peak, peak_kind = load_peaks()
    st = torch.cuda.current_stream(dev)

    def timed(fn):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        for _ in range(args.steps):
            fn()
        b.record(st)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / args.steps / 1e3

    kernels = {}
    if args.row == "backward":
        N, K, d, Q = w.N, w.K, w.d, w.Q
        dout = torch.randn((N, d), dtype=torch.float32, device=dev, generator=gen)
        y = torch.randn((Q, d), dtype=torch.float32, device=dev, generator=gen).to(torch.bfloat16)
        dy = torch.empty_like(y)
        dw = torch.empty((N, K), dtype=torch.float32, device=dev)
        dh = torch.empty((N, d), dtype=torch.float32, device=dev)
        t1 = timed(lambda: ue.ue_combine_backward(L.ctx, dout, y, L.dest_row, L.w, dy, dw, st))
        t2 = timed(lambda: ue.ue_permute_backward(L.ctx, y, L.dest_row, dh, st))
        rb = row_bytes(N=N, K=K, d=d)
        kernels["combine_backward"] = (t1, rb["combine_backward"])
        kernels["permute_backward"] = (t2, rb["permute_backward"])
        workload = dict(workload=w.name, N=N, K=K, d=d, pairs=Q)
    elif args.row == "layouts":
        # the permute's traffic (2Nd read, 2Qd written) under three row
        # layouts, beside write-only and 1:1-copy traffic of torch's own
        # kernels: where the routed layout stands between the best and the
        # worst placement of the same bytes
        N, K, d, Q = w.N, w.K, w.d, w.Q
        L.hidden.copy_(torch.randint(-30000, 30000, (N, d), dtype=torch.int16, device=dev,
                                     generator=gen).view(torch.bfloat16))
        ident = torch.arange(Q, dtype=torch.int32, device=dev).view(N, K)
        rand = torch.randperm(Q, device=dev, generator=gen).to(torch.int32).view(N, K)
        pbytes = 2 * N * d + 2 * Q * d + 4 * Q
        kernels["permute_routed"] = (timed(lambda: L.permute(st)), pbytes)
        kernels["permute_contiguous_rows"] = (
            timed(lambda: ue.ue_permute(L.ctx, L.hidden, ident, L.dispatch, st)), pbytes)
        kernels["permute_random_rows"] = (
            timed(lambda: ue.ue_permute(L.ctx, L.hidden, rand, L.dispatch, st)), pbytes)
        flat = L.dispatch.view(-1)
        half = flat.numel() // 2
        flat64 = flat[:flat.numel() // 4 * 4].view(torch.int64)
        kernels["torch_fill_write_only"] = (timed(lambda: flat64.fill_(0x3F803F803F803F80)),
                                            8 * flat64.numel())
        kernels["torch_copy_1to1"] = (timed(lambda: flat[half:2 * half].copy_(flat[:half])),
                                      4 * half)
        # the combine's gather (2Qd read, 4Nd written) under the same layouts,
        # reading the dispatch buffer as the expert outputs, beside torch's
        # read-only sum of the same 17.2 GB
        cbytes = 2 * Q * d + 8 * Q + 4 * N * d
        kernels["combine_routed"] = (timed(lambda: L.combine(stream=st)), cbytes)
        kernels["combine_contiguous_rows"] = (
            timed(lambda: ue.ue_combine(L.ctx, L.dispatch, ident, L.w, L.out, st)), cbytes)
        kernels["combine_random_rows"] = (
            timed(lambda: ue.ue_combine(L.ctx, L.dispatch, rand, L.w, L.out, st)), cbytes)
        acc = torch.empty((), dtype=torch.int64, device=dev)
        kernels["torch_sum_read_only"] = (timed(lambda: torch.sum(flat64, dim=0, out=acc)),
                                          8 * flat64.numel())
        del ident, rand
        workload = dict(workload=w.name, N=N, K=K, d=d, pairs=Q,
                        routed=("dest_row of the path's reroute: per-slot runs, 4*P regions "
                                "written at once"),
                        contiguous="dest_row = n*K + k", random="a random permutation of [0, Q)")
    else:
        plan = L.plan_arrays()
        se = plan["slot_expert"]
        used = int((se >= 0).sum())
        cnt = np.bincount(se[se >= 0], minlength=w.E)
        numel = expert_numel(args)
        if args.row == "weight_sync":
            bpe = numel * 2
            master = torch.randint(-30000, 30000, (w.E, numel), dtype=torch.int16,
                                   device=dev, generator=gen)
            reps = torch.empty((w.G, numel), dtype=torch.int16, device=dev)
            t = timed(lambda: ue.ue_weight_sync(L.ctx, L.plan, master, reps, bpe, st))
            kernels["weight_sync"] = (t, row_bytes(used=used, bytes_per_expert=bpe)["weight_sync"])
        else:
            master = torch.randn((w.E, numel), dtype=torch.float32, device=dev, generator=gen)
            reps = torch.randn((w.G, numel), dtype=torch.float32, device=dev, generator=gen)
            t = timed(lambda: ue.ue_grad_reduce(L.ctx, L.plan, reps, master, numel, st))
            nrep = int((cnt > 0).sum())
            kernels["grad_reduce"] = (t, row_bytes(used=used, replicated=nrep,
                                                   numel=numel)["grad_reduce"])
        workload = dict(workload=w.name, expert_numel=numel, replicas=used,
                        replicated_experts=int((cnt > 0).sum()),
                        expert_shape=("Qwen3-235B expert: fc1 2*4096*1536 + fc2 4096*1536"
                                      if numel == EXPERT_NUMEL else "reduced (profiling)"))
    rc = L.error()
    se_host = L.plan_arrays()["slot_expert"]
    L.close()
    if rc != 0:
        raise SystemExit(f"device error: {rc}")
    out = {}
    for k, (t, by) in kernels.items():
        gbs = by / t / 1e9
        out[k] = {"us": t * 1e6, "algorithmic_bytes": by, "gbs": gbs, "frac_of_peak": gbs / peak}
    dom = ("permute_routed" if args.row == "layouts"
           else max(out, key=lambda k: out[k]["us"]))
    line = {"row": args.row, "config": workload, "steps": args.steps, "kernels": out,
            "roofline": {"bound": "hbm", "kernel": dom, "achieved": out[dom]["gbs"], "peak": peak,
                         "unit": "GB/s", "frac": out[dom]["frac_of_peak"],
                         "peak_kind": f"of {peak_kind}", "nominal_peak": NOMINAL_HBM_GBS,
                         "frac_of_nominal": out[dom]["gbs"] / NOMINAL_HBM_GBS}}
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = row_oracle_baseline(args, w, se_host)
    print(json.dumps(line), flush=True)


def row_oracle_baseline(args, w, slot_expert):
    """The oracle (single-threaded C, fp64 where the row computes in floating
    point) on a bounded sample of the same row, reported in the row's units
    (algorithmic GB/s of the sample over the oracle's time)."""
    import numpy as np

    import oracle
    import synth
    if args.row == "backward":
        n, K, d = 4096, w.K, w.d
        dest = np.arange(n * K, dtype=np.int32).reshape(n, K)
        wts = np.random.default_rng(0).random((n, K)).astype(np.float32)
        dout = synth.normal_f32(n * d, 0, 61).reshape(n, d)
        y = synth.bf16_normal(n * K, d, 0, 62)
        t0 = time.perf_counter()
        oracle.combine_backward(dout, y, K, dest, wts)
        oracle.permute_backward(y, n, K, dest)
        secs = time.perf_counter() - t0
        by = (4 * n * d + 2 * n * K * d + 8 * n * K + 2 * n * K * d + 4 * n * K) + \
             (2 * n * K * d + 4 * n * K + 4 * n * d)
        sample = f"{n} tokens x K={K} x d={d}: combine backward + permute backward"
    elif args.row == "layouts":
        n, K, d = 8192, w.K, w.d
        dest = np.random.default_rng(0).permutation(n * K).astype(np.int32).reshape(n, K)
        hidden = synth.bf16_normal(n, d, 0, 63)
        t0 = time.perf_counter()
        oracle.permute(hidden, K, dest)
        secs = time.perf_counter() - t0
        by = 2 * n * d + 2 * n * K * d + 4 * n * K
        sample = f"{n} tokens x K={K} x d={d}: permute with random rows"
    else:
        numel = expert_numel(args)
        used = [g for g in range(len(slot_expert)) if slot_expert[g] >= 0][:8]
        experts = sorted({int(slot_expert[g]) for g in used})
        remap = {e: i for i, e in enumerate(experts)}
        se = np.array([remap[int(slot_expert[g])] for g in used], dtype=np.int32)
        rng = np.random.default_rng(0)
        if args.row == "weight_sync":
            bpe = numel * 2
            master = rng.integers(0, 256, size=(len(experts), bpe), dtype=np.uint8)
            reps = np.zeros((len(used), bpe), dtype=np.uint8)
            t0 = time.perf_counter()
            oracle.weight_sync(se, master, reps)
            secs = time.perf_counter() - t0
            by = 2 * len(used) * bpe
        else:
            master = rng.standard_normal((len(experts), numel), dtype=np.float32)
            reps = rng.standard_normal((len(used), numel), dtype=np.float32)
            t0 = time.perf_counter()
            oracle.grad_reduce(se, reps, master)
            secs = time.perf_counter() - t0
            by = 4 * numel * (2 * len(experts) + len(used))
        sample = (f"{len(used)} replica slots of {len(experts)} experts, "
                  f"{numel} elements per expert")
    gbs = by / secs / 1e9
    return {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample,
            "seconds": secs}


def run_planner(args, w):
    """Planner variants ("UltraEP" README, "Performance Tuning / Replication
    planning") on the pages' runtime-test layer (EP64, 256 experts, 4 master +
    2 redundant per rank, top-8, 8k tokens per rank) at its three initial
    imbalances, or on one given workload: balance reached, replicas, and the
    device time of every plan and reroute variant. One JSON line per layer
    instance. The pages' own numbers (one GPU of 64, the load all-gather
    included) are quoted beside ours for context only: here one GPU plans and
    reroutes for all 64 ranks."""
    import numpy as np
    import torch

    import synth
    import token_rerouting_b200 as ue
    from token_rerouting_b200 import build as ue_build

    ue_build.build()
    dev = torch.device("cuda", 0)
    st = torch.cuda.current_stream(dev)
    pages = {1.51: dict(final=1.01, replicas="4 / 38", update_placement_ms=0.067, reroute_ms=0.039),
             2.01: dict(final=1.01, replicas="5 / 46", update_placement_ms=0.072, reroute_ms=0.037),
             3.03: dict(final=1.01, replicas="6 / 51", update_placement_ms=0.078, reroute_ms=0.036)}
    if w.name.startswith("pages_"):
        instances = [(t, synth.ALPHA_PAGES[i]) for i, t in enumerate((1.51, 2.01, 3.03))]
    else:
        instances = [(None, None)]
    L = ue.Layer(w.R, w.T, w.E, w.K, w.S, 8, device=0, with_rows=False)

    def timed(fn):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        for _ in range(args.steps):
            fn()
        b.record(st)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / args.steps * 1e3  # us

    M, S = w.M, w.S
    host_of_slot = np.arange(w.P) // (M + S)
    src_of_pair = np.arange(w.Q) // (w.T * w.K)
    mean = w.Q / w.R

    def summary(plan):
        se = plan["slot_expert"]
        nc = plan["n_copies"]
        return dict(max_over_mean=float(plan["rank_load"].max() / mean),
                    replicas=int((se >= 0).sum()), max_replicas_per_expert=int(nc.max() - 1),
                    stats=plan["stats"].tolist())

    solvers = {"greedy": ue.plan_opts(ue.UE_SOLVER_GREEDY),
               "greedy_min1024": ue.plan_opts(ue.UE_SOLVER_GREEDY, min_tokens=1024),
               "bisect": ue.plan_opts(ue.UE_SOLVER_BISECT)}
    for target, alpha in instances:
        L.logits.copy_(torch.from_numpy(synth.logits(w, alpha=alpha)))
        L.gate_count()
        torch.cuda.synchronize(dev)
        load_e = L.load_e.cpu().numpy()
        before = float(load_e.reshape(w.R, M).sum(axis=1).max() / mean)
        res = {}
        for name, opts in solvers.items():
            us = timed(lambda: L.plan_ex(opts, st))
            res[name] = dict(plan_us=us, **summary(L.plan_arrays()))
            # reroutes under this plan
            res[name]["reroute_us"] = timed(lambda: L.reroute(st))
            torch.cuda.synchronize(dev)
            phys = L.phys_slot.cpu().numpy().ravel()
            res[name]["remote_pairs_prefix"] = int((host_of_slot[phys] != src_of_pair).sum())
            res[name]["reroute_interleave_us"] = timed(lambda: L.reroute_ex(ue.UE_ORDER_INTERLEAVE, st))
            res[name]["locality_split_us"] = timed(lambda: L.locality_split(st))
            res[name]["reroute_local_us"] = timed(lambda: L.reroute_local(st))
            torch.cuda.synchronize(dev)
            sq = L.src_quota.cpu().numpy()
            res[name]["remote_pairs_local"] = int(sum(sq[r, host_of_slot != r].sum()
                                                     for r in range(w.R)))
        rc = L.error()
        if rc != 0:
            raise SystemExit(f"device error: {rc}")
        line = {"row": "planner", "config": dict(workload=w.name, R=w.R, T=w.T, E=w.E, K=w.K,
                                                   S=w.S, pairs=w.Q, alpha=alpha,
                                                   target_imbalance=target),
                "steps": args.steps, "imbalance_before": before, "solvers": res}
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = planner_oracle_baseline(w, synth.logits(w, alpha=alpha))
        if target is not None:
            line["pages_context"] = pages[target]
        print(json.dumps(line), flush=True)
    L.close()


def planner_oracle_baseline(w, logits):
    """The oracle's planner variants on the same layer instance (its own
    top-k and counts), single-threaded: microseconds per call."""
    import oracle
    idx, _ = oracle.gate_topk(logits, w.K)
    load_re, load_e = oracle.count(idx, w.R, w.T, w.E)
    us = {}

    def timed(name, fn):
        t0 = time.perf_counter()
        r = fn()
        us[name] = (time.perf_counter() - t0) * 1e6
        return r

    timed("plan_greedy", lambda: oracle.plan(load_e, w.R, w.S))
    pl = timed("plan_bisect", lambda: oracle.plan_bisect(load_e, w.R, w.S))
    timed("reroute_prefix", lambda: oracle.reroute(idx, w.R, w.E, w.S, pl))
    timed("reroute_interleave", lambda: oracle.reroute_interleave(idx, w.R, w.T, w.E, w.S, pl))
    sq, so = timed("locality_split", lambda: oracle.locality_split(load_re, w.S, pl))
    timed("reroute_local", lambda: oracle.reroute_local(idx, w.R, w.T, w.E, w.S, pl, sq, so))
    return {"unit": "us per call", "us": us, "cores": 1, "kind": "oracle",
            "sample": "the whole layer instance (the oracle's own top-k and counts; the capacity "
                      "plan feeds the reroutes)"}


def run_routing_row(args, w):
    """The routing half alone (gate with the count fused in, plan, reroute) on
    one layer instance without row buffers (logits and routing arrays only:
    a small device footprint, for kernel captures). Each call timed alone as
    replays of a CUDA graph of back-to-back launches, CUDA events on the
    replay stream. The separate count call (ue_count, the same counts from
    idx) is timed beside them but not part of the routing total. Also timed
    the same way: the plan and the reroute overlapped (ue_plan_reroute), and
    the whole routing chain as launched, with and without that overlap."""
    import torch

    import token_rerouting_b200 as ue
    from token_rerouting_b200 import build as ue_build

    ue_build.build()
    dev = torch.device("cuda", 0)
    L = ue.Layer(w.R, w.T, w.E, w.K, w.S, w.d, device=0, with_rows=False)
    L.logits.copy_(torch.from_numpy(synth_logits(w)))
    for _ in range(max(3, args.warmup)):
        L.run_routing()
    torch.cuda.synchronize(dev)
    s = torch.cuda.Stream(dev)
    us = {}
    def chain(stream):
        L.gate_count(stream)
        L.plan_step(stream)
        L.reroute(stream)

    def chain_overlap(stream):
        L.gate_count(stream)
        L.plan_reroute(stream)

    for name, f in (("gate_count", L.gate_count), ("plan", L.plan_step), ("reroute", L.reroute),
                    ("count", L.count), ("plan_reroute", L.plan_reroute), ("chain", chain),
                    ("chain_overlap", chain_overlap)):
        with torch.cuda.stream(s):
            f(stream=s)
            torch.cuda.synchronize(dev)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                for _ in range(args.steps):
                    f(stream=s)
            g.replay()
            torch.cuda.synchronize(dev)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(s)
            g.replay()
            b.record(s)
        torch.cuda.synchronize(dev)
        us[name] = a.elapsed_time(b) * 1e3 / args.steps
        del g
    rc = L.error()
    plan = L.plan_arrays()
    L.close()
    if rc != 0:
        raise SystemExit(f"device error: {ue.STATUS.get(rc, rc)}")
    ab = algorithmic_bytes(w)
    peak, peak_kind = load_peaks()
    line = {"row": "routing", "config": dict(workload=w.name, R=w.R, T=w.T, E=w.E, K=w.K, S=w.S,
                                              pairs=w.Q),
            "steps": args.steps, "us": us,
            "frac_of_peak": {k: ab[k] / (us[k] / 1e6) / 1e9 / peak for k in ("gate_count",
                                                                              "reroute")},
            "peak_kind": f"of {peak_kind}",
            "us_routing_total": us["gate_count"] + us["plan"] + us["reroute"],
            # one routing pass as launched: gate, plan and reroute back to back
            # (separate calls), and with plan and reroute overlapped
            "us_routing_chain": us["chain"],
            "us_routing_chain_overlap": us["chain_overlap"],
            "plan": {"iterations": int(plan["stats"][0]),
                     "max_over_mean_before": float(plan["stats"][1]) / (w.Q / w.R),
                     "max_over_mean_after": float(plan["stats"][2]) / (w.Q / w.R)}}
    print(json.dumps(line), flush=True)


def synth_logits(w):
    import synth
    return synth.logits(w)


# ------------------------------------------------------------------ main ----
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ue", "reference"), default="ue")
    ap.add_argument("--workload", default=None,
                    help=f"default {DEFAULT_WORKLOAD} (pages_ep64_e256_t8k for --row planner)")
    ap.add_argument("--tokens-per-rank", type=int, default=0,
                    help="shrink T (profiling runs on a small case)")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--expert-numel", type=int, default=0,
                    help="expert size for --row weight_sync / grad_reduce (profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--sweep", action="store_true",
                    help="the 48 x 8 non-stationary sweep, CUDA-graph captured")
    ap.add_argument("--planner", choices=("greedy", "bisect"), default="greedy",
                    help="planner of the sweep (greedy: the path's rule)")
    ap.add_argument("--row", choices=("backward", "weight_sync", "grad_reduce", "planner",
                                      "layouts", "routing"),
                    default=None, help="measure one of the rows beside the forward path "
                    "(planner: the planner variants, on pages_ep64_e256_t8k by default; "
                    "routing: the routing half alone, without row buffers)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    import dataclasses

    import synth
    if args.workload is None:
        args.workload = "pages_ep64_e256_t8k" if args.row == "planner" else DEFAULT_WORKLOAD
    w = synth.WORKLOADS[args.workload]
    if args.tokens_per_rank:
        w = dataclasses.replace(w, T=args.tokens_per_rank, name=f"{w.name}_t{args.tokens_per_rank}")
    if args.impl == "reference":
        run_reference(args, w)
        return
    if args.sweep:
        run_sweep(args)
        return
    if args.row == "planner":
        run_planner(args, w)
        return
    if args.row == "routing":
        run_routing_row(args, w)
        return
    if args.row:
        run_row(args, w)
        return

    world, rank, local = dist_setup(args.gpus)
    import numpy as np
    import torch

    import token_rerouting_b200 as ue
    from token_rerouting_b200 import build as ue_build

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    if rank == 0:
        ue_build.build()
    if world > 1:
        dist.barrier()
    ue.load_library()

    # inputs: each rank is a different microbatch of the same layer
    logits_h = synth.logits(w, mb=rank)
    hidden_h = synth.hidden(w, seed=rank)
    L = ue.Layer(w.R, w.T, w.E, w.K, w.S, w.d, device=local)
    L.logits.copy_(torch.from_numpy(logits_h))
    L.hidden.copy_(torch.from_numpy(hidden_h.view(np.int16)).to(dev).view(torch.bfloat16))
    # a second layer instance (the next microbatch): the timed steps alternate
    # between the two, so that one instance's routing runs while the other
    # permutes and combines
    LB = ue.Layer(w.R, w.T, w.E, w.K, w.S, w.d, device=local)
    LB.logits.copy_(torch.from_numpy(synth.logits(w, mb=rank + world)))
    LB.hidden.copy_(L.hidden)
    stream = torch.cuda.current_stream(dev)

    # plan and reroute in one call: the reroute kernel starts while the plan
    # runs (programmatic dependent launch) and reads the plan once it is done
    steps_fn = [L.gate_count, L.plan_reroute, L.permute, L.combine]

    def step():
        for f in steps_fn:
            f(stream=stream)

    # Pipelined steps: step i runs on instance i % 2. Its routing (gate,
    # count, plan, reroute) goes on a side stream once step i-2's combine has
    # released the instance; its permute and combine go on the main stream
    # once its routing is done. So step i+1's routing overlaps step i's
    # permute and combine, as the pages' asynchronous update_placement and
    # reroute (events, current_stream_wait) allow; the first step's routing
    # overlaps nothing.
    insts = [L, LB]
    # the routing's stream has the higher priority: its few CTAs are placed
    # ahead of the permute's pending ones, so it holds SM slots for a shorter
    # time (measured: 6.353 against 6.375 ms per step at equal priority)
    side = torch.cuda.Stream(dev, priority=-5)
    ev_routed = [torch.cuda.Event() for _ in insts]
    ev_done = [torch.cuda.Event() for _ in insts]

    def pipelined_steps(n):
        for x in range(2):
            ev_done[x].record(stream)
        for i in range(n):
            x = i % 2
            I = insts[x]
            side.wait_event(ev_done[x])
            for f in (I.gate_count, I.plan_reroute):
                f(stream=side)
            ev_routed[x].record(side)
            stream.wait_event(ev_routed[x])
            I.permute(stream=stream)
            I.combine(stream=stream)
            ev_done[x].record(stream)

    for _ in range(args.warmup):
        step()
    pipelined_steps(max(4, args.warmup))
    torch.cuda.synchronize(dev)
    rc = L.error(stream) or LB.error(stream)
    if rc != 0:
        raise SystemExit(f"device error after warm-up: {ue.STATUS.get(rc, rc)}")
    step()
    torch.cuda.synchronize(dev)
    plan0 = L.plan_arrays()

    # the step as one CUDA graph of the path's kernels (captured once, outside
    # the timed region), so that the timed steps carry no launch gaps
    gstream = torch.cuda.Stream(dev)
    gstream.wait_stream(stream)
    with torch.cuda.stream(gstream):
        for f in steps_fn:
            f(stream=gstream)
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=gstream):
        for f in steps_fn:
            f(stream=gstream)
    torch.cuda.synchronize(dev)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize(dev)

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.2)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    pipelined_steps(args.steps)
    end.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    total_ms = start.elapsed_time(end)
    rc = L.error(stream) or LB.error(stream)
    if rc != 0:
        raise SystemExit(f"device error in the timed region: {ue.STATUS.get(rc, rc)}")

    # the same steps one after another, each one graph replay of the path's
    # kernels on one instance (reported beside the value)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    sa, sb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sa.record(stream)
    for _ in range(args.steps):
        graph.replay()
    sb.record(stream)
    torch.cuda.synchronize(dev)
    serial_ms = max_over_ranks(sa.elapsed_time(sb) / args.steps, world, dev)
    rc = L.error(stream)
    if rc != 0:
        raise SystemExit(f"device error in the serial steps: {ue.STATUS.get(rc, rc)}")

    # per-kernel breakdown (not part of the value): each kernel alone, as
    # replays of a CUDA graph of back-to-back launches on gstream (every
    # kernel is idempotent on the instance's current buffers), timed with
    # CUDA events on gstream; per launch = elapsed / launches
    kernel_fns = dict(zip(KERNELS, (L.gate_count, L.plan_step, L.reroute, L.permute, L.combine)))

    def routing_chain(stream):
        L.gate_count(stream=stream)
        L.plan_reroute(stream=stream)

    per_kernel_ms = {}
    for name, f in list(kernel_fns.items()) + [("routing_chain", routing_chain)]:
        reps = 4 if name in ("permute", "combine") else 20
        gstream.wait_stream(stream)
        with torch.cuda.stream(gstream):
            f(stream=gstream)
        torch.cuda.synchronize(dev)
        kg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(kg, stream=gstream):
            for _ in range(reps):
                f(stream=gstream)
        with torch.cuda.stream(gstream):
            for _ in range(2):
                kg.replay()
        torch.cuda.synchronize(dev)
        nrep = 3
        ka, kb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(gstream):  # replay() launches on the current stream
            ka.record(gstream)
            for _ in range(nrep):
                kg.replay()
            kb.record(gstream)
        torch.cuda.synchronize(dev)
        per_kernel_ms[name] = ka.elapsed_time(kb) / (nrep * reps)
        del kg
    clk = clocks.stop()
    chain_ms = per_kernel_ms.pop("routing_chain")
    rc = L.error(stream)
    if rc != 0:
        raise SystemExit(f"device error in the breakdown steps: {ue.STATUS.get(rc, rc)}")
    del graph

    ms_step_local = total_ms / args.steps
    ms_step = max_over_ranks(ms_step_local, world, dev)
    value = world * w.Q / (ms_step / 1e3)

    # dominant kernel and its roofline
    abytes = algorithmic_bytes(w)
    dom = max(("permute", "combine", "gate_count", "reroute"), key=lambda k: per_kernel_ms[k])
    peak, peak_kind = load_peaks()
    achieved = abytes[dom] / (per_kernel_ms[dom] / 1e3) / 1e9
    tr = TRAFFIC.get(w.name, {}).get(dom)
    src = os.path.join(ROOT, "token_rerouting_b200", "csrc", KERNEL_SRC[dom])
    traffic = (tr["bytes_per_launch"] if tr and tr.get("source_sha") == sha_of(src) else None)
    roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak,
                "unit": "GB/s", "frac": achieved / peak, "peak_kind": f"of {peak_kind}",
                "traffic": traffic, "algorithmic_bytes": abytes[dom],
                "nominal_peak": NOMINAL_HBM_GBS, "frac_of_nominal": achieved / NOMINAL_HBM_GBS}
    kernels = {}
    for k in KERNELS:
        ms = per_kernel_ms[k]
        kernels[k] = {"us": 1e3 * ms, "share": ms / sum(per_kernel_ms.values())}
        if abytes[k]:
            gbs = abytes[k] / (ms / 1e3) / 1e9
            kernels[k].update(gbs=gbs, frac_of_peak=gbs / peak)

    cfg = workload_config(w)
    gate_to_permute = sum(per_kernel_ms[k] for k in KERNELS[:4])
    cfg.update(us_per_layer_gate_to_permute=1e3 * gate_to_permute,
               us_per_layer_incl_combine=1e3 * sum(per_kernel_ms.values()),
               us_routing_chain=1e3 * chain_ms,
               timing="exactly `steps` steps, each the path's five kernels in four calls (gate "
                      "with the count fused; plan and reroute, the reroute launched as the "
                      "plan's programmatic dependent; permute; combine) over one batch; two layer "
                      "instances alternate, and step i+1's routing (gate and count, plan, reroute) "
                      "runs on a second stream during step i's permute and combine (events "
                      "order each instance's uses); per-kernel times: each kernel alone as CUDA "
                      "graph replays of back-to-back launches (20, or 4 for permute and "
                      "combine), CUDA events on the replay stream",
               ms_per_step_serial=serial_ms,
               serial="the same steps one after another, one CUDA graph replay each",
               parallelism=f"replicas: {world} independent layer instance(s), one per GPU")

    # end to end through the public API with host buffers. Every step copies
    # its inputs in from pinned host memory and its result (combine output and
    # plan stats) back out. Consecutive steps are pipelined over two buffer
    # sets and three streams, so step s+1's upload, step s's kernels and step
    # s-1's readback overlap (PCIe is full duplex): a step may start its
    # kernels once its inputs are in and its buffer set's previous result has
    # been read out.
    e2e = None
    if not args.no_e2e:
        lg_pin = torch.from_numpy(logits_h).pin_memory()
        hd_pin = torch.from_numpy(hidden_h.view(np.int16)).pin_memory()
        L2 = LB
        bufs = [L, L2]
        outs = [torch.empty(L.out.shape, dtype=torch.float32).pin_memory() for _ in bufs]
        stats_pin = [torch.empty(4 + w.R, dtype=torch.int32).pin_memory() for _ in bufs]
        s_in, s_run, s_out = (torch.cuda.Stream(dev), torch.cuda.Stream(dev),
                              torch.cuda.Stream(dev))
        ev_in = [torch.cuda.Event() for _ in bufs]
        ev_run = [torch.cuda.Event() for _ in bufs]
        ev_out = [torch.cuda.Event() for _ in bufs]
        for b in range(2):  # nothing to wait for on the first use of a set
            ev_run[b].record(s_run)
            ev_out[b].record(s_out)

        def e2e_step(i):
            b = i % 2
            Lb = bufs[b]
            s_in.wait_event(ev_run[b])          # the set's last kernels are done with its inputs
            with torch.cuda.stream(s_in):
                Lb.logits.copy_(lg_pin, non_blocking=True)
                Lb.hidden.view(torch.int16).copy_(hd_pin, non_blocking=True)
            ev_in[b].record(s_in)
            s_run.wait_event(ev_in[b])
            s_run.wait_event(ev_out[b])          # its previous result has been read out
            for f in [Lb.gate_count, Lb.plan_reroute, Lb.permute, Lb.combine]:
                f(stream=s_run)
            ev_run[b].record(s_run)
            s_out.wait_event(ev_run[b])
            with torch.cuda.stream(s_out):
                outs[b].copy_(Lb.out, non_blocking=True)
                stats_pin[b][:4].copy_(Lb.stats, non_blocking=True)
                stats_pin[b][4:].copy_(Lb.rank_load, non_blocking=True)
            ev_out[b].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s_in)
        for i in range(args.e2e_steps):
            e2e_step(i)
        b_.record(s_out)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(a.elapsed_time(b_) / args.e2e_steps, world, dev)
        rc2 = L2.error(s_run) or L.error(s_run)
        if rc2 != 0:
            raise SystemExit(f"device error in the end-to-end steps: {ue.STATUS.get(rc2, rc2)}")
        h2d = lg_pin.numel() * 4 + hd_pin.numel() * 2
        d2h = outs[0].numel() * 4 + stats_pin[0].numel() * 4
        e2e = {"value": world * w.Q / (e2e_ms / 1e3), "unit": UNIT, "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "what": "every step: pinned host logits + hidden -> device, the path's kernels, "
                       "fp32 combine output + plan stats -> pinned host; consecutive steps "
                       "pipelined over two buffer sets and three streams (upload, kernels, "
                       "readback overlap)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        pairs, secs, nsl = oracle_slices(w, logits_h, hidden_h, 512, 10.0, 8)
        cpu = {"value": pairs / secs, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"{nsl} slice(s) of 512 tokens per rank x {w.R} ranks "
                         f"({pairs} pairs, {secs:.1f} s), each a whole layer instance "
                         f"through the single-threaded C oracle incl. permute and combine"}
        nthr = host_threads()
        tp, ts, tn = threaded_oracle_slices(w, logits_h, hidden_h, 512, 10.0, 16, nthr)
        cpu["threaded"] = {
            "value": tp / ts, "unit": UNIT, "cores": nthr,
            "kind": "oracle split over host threads by token range (top-k, counts, permute, "
                    "combine); plan and reroute sequential",
            "sample": f"{tn} slice(s) of 512 tokens per rank x {w.R} ranks ({tp} pairs, "
                      f"{ts:.1f} s)",
            "checked": "outputs on a 64-token-per-rank slice equal to the single-threaded oracle's"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic", "config": cfg,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": kernels_per_step(w) * args.steps,
            "clocks": clk, "kernels": kernels,
            "imbalance": {"max_over_mean_before": float(plan0["stats"][1]) / (w.Q / w.R),
                          "max_over_mean_after": float(plan0["stats"][2]) / (w.Q / w.R),
                          "copies": int(plan0["stats"][0]),
                          "colocated_copies": int(plan0["stats"][3])},
        }
        print(json.dumps(line), flush=True)
    L.close()
    LB.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
