"""Benchmark of the W1.58A16 ternary linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--quick]
                    [--profile gemv|gemv16|gemv_elem|gemm|gemm_elem|rotate]

A step is one decode pass (M = 1) over the 252 ternarized linear tensors of a 36-layer
Qwen3-8B-shaped stack (q, k, v, o, gate, up, down per layer; 15% of rows carry a residual
plane): per layer four tern_linear_group launches, one per input the projections share (q+k+v,
o, gate+up, down), 144 per step, replayed from a CUDA graph. Weights come from a pool of 8
distinct layers (about 470 MB of packed planes, several times the 126 MB L2), assigned to the 36
layer slots round-robin, so every call streams its weights from HBM.

value     : packed-weight GB/s = (2-bit planes + fp16 scales + slot map) bytes per step / time.
roofline  : the dominant launch (gate + up at M = 1), algorithmic bytes (packed weights +
            activations) per launch / its average launch time, against the measured HBM copy
            bandwidth; traffic = the DRAM bytes of one such launch from an ncu capture.
e2e       : the same metric through the Python API with the step's inputs copied from pinned
            host memory and its outputs copied back, every step.
cpu_baseline / --impl reference: the CPU oracle (numpy float64) on a bounded sample.
extra     : per-projection, per-group and per-M decode figures, the M = 2048 prefill GEMM in
            TFLOP/s, the offset, element-plane, rotation and fit measurements, packing throughput,
            bit accounting, and dense fp16 cuBLAS on the same shapes.

For --gpus N > 1 (torchrun) every rank runs the same workload on its own GPU (replicas; the
path has no data exchange), the timed region is bracketed by barriers, and the time is the
max over ranks.
"""

from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))

# DRAM bytes (read + write) of one launch of the dominant kernel (the gate + up launch), from one
# ncu capture of the `--profile gemv` case (summary and command under profiles/), keyed by a hash of the sources the
# kernel is built from: when they change, the number no longer describes the kernel and the
# bench reports null until it is captured again.
KERNEL_TRAFFIC = {
    "gemv": {"sources": ["ternary_weight_only_tern_b200/csrc/tern_decode1.cu",
                         "ternary_weight_only_tern_b200/csrc/tern_device.cuh",
                         "ternary_weight_only_tern_b200/csrc/tern_stream.cuh"],
             "sha256": "45639663d5e346da78ff1653b6cb8d1c2dd802c6cc8bfa78cc8171310daecdb6",
             "bytes": 30926848},
}


def measured_traffic(kernel: str):
    t = KERNEL_TRAFFIC[kernel]
    if t["sha256"] is None:
        return None
    h = hashlib.sha256()
    for rel in t["sources"]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return t["bytes"] if h.hexdigest() == t["sha256"] else None
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "W1.58A16 GEMV packed-weight GB/s (% of HBM peak); GEMM TFLOP/s at M=2048"
WORKLOAD = "qwen3-8b-decode-stack-m1"
RES_PCT = 15
POOL_LAYERS = 8
LAYERS = 36
# projections that read the same activation run as one tern_linear_group launch
GROUPS = [("qkv", ("q", "k", "v")), ("o", ("o",)), ("gateup", ("gate", "up")), ("down", ("down",))]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        time.sleep(0.15)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        time.sleep(0.1)
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[4:]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        mx = max(r[1] for r in rows)
        load = [r for r in rows] or rows
        sm = float(np.median([r[0] for r in load]))
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in load for i, v in enumerate(r[2]) if v.lower().startswith("active")})
        return {"sm_mhz": sm, "sm_max_mhz": mx, "reasons": reasons, "samples": len(rows)}


def gpu_uuid(torch, dev):
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev.index or 0)


# ------------------------------------------------------------------------------ replicas
def max_over_ranks_of(dist, v: float, device=None) -> float:
    """The largest of every rank's v (all ranks call it, in the same order); v itself on one rank."""
    if dist is None:
        return v
    import torch
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_value(world: int, units_per_rank: float, max_secs: float) -> float:
    """Whole-job throughput of `world` replicas that each processed `units_per_rank` units,
    timed as the slowest rank."""
    return world * units_per_rank / max_secs


# ------------------------------------------------------------------------------ workload
def draw_layer_on_device(torch, api, shapes, dev, seed, elem_frac=None, res_pct=None, uniform=False):
    """One layer's projections, drawn on the device with a seeded torch generator (same
    distributions as the host recipe: P(0) = 0.4, P(+-1) = 0.3, or 1/3 each with uniform;
    s1 ~ U[0.005, 0.02]; s2 ~ U[0.001, 0.005]; res_pct (default 15) % residual rows uniformly
    without replacement) and packed with tern_pack_exec. With elem_frac, the second plane is
    element-level instead: each weight is masked with probability elem_frac and a masked weight
    draws a trit like the main plane, with s2e ~ U[0.001, 0.005] per (row, group)."""
    res_pct = RES_PCT if res_pct is None else res_pct
    from ternary_weight_only_tern_b200.synth import residual_count
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    out = {}
    for name, N, K in shapes:
        G = K // 128

        def trits(rows):
            if uniform:
                return torch.randint(0, 3, (rows, K), dtype=torch.int8, generator=g, device=dev) - 1
            u = torch.randint(0, 10, (rows, K), dtype=torch.uint8, generator=g, device=dev)
            return (u >= 7).to(torch.int8) - (u < 3).to(torch.int8)

        T1 = trits(N)
        s1 = (torch.rand((N, G), generator=g, device=dev) * 0.015 + 0.005).half()
        if elem_frac is not None:
            mask = torch.rand((N, K), generator=g, device=dev) < elem_frac
            T2e = trits(N) * mask.to(torch.int8)
            s2e = (torch.rand((N, G), generator=g, device=dev) * 0.004 + 0.001).half()
            w = api.TernWeight.from_trits(T1, s1, T2e=T2e, s2e=s2e)
            w.static = True
            out[name] = w
            del T1, T2e, mask
            continue
        r = residual_count(N, res_pct)
        rows = torch.randperm(N, generator=g, device=dev)[:r].sort().values.to(torch.int32)
        T2 = trits(r)
        s2 = (torch.rand((r, G), generator=g, device=dev) * 0.004 + 0.001).half()
        w = api.TernWeight.from_trits(T1, s1, rows, T2, s2)
        w.static = True            # model weights: nothing queued before a call writes them
        out[name] = w
        del T1, T2
    return out


def packed_bytes(w) -> int:
    return w.nbytes()


COLD_BYTES = 384e6        # > 3x the 126 MB L2: a pool this large cycles every call's weight out of L2


def cold_pool(torch, api, dev, shapes, seed, res_pct, uniform=False, max_copies=512):
    """Distinct copies of one group of projections (shapes [(name, N, K)]), enough of them that
    their packed bytes exceed COLD_BYTES, so that calls taken in turn each stream from HBM."""
    first = draw_layer_on_device(torch, api, shapes, dev, seed, res_pct=res_pct, uniform=uniform)
    per = sum(w.nbytes() for w in first.values())
    n = int(min(max_copies, max(8, -(-COLD_BYTES // per))))
    return [first] + [draw_layer_on_device(torch, api, shapes, dev, seed + i, res_pct=res_pct, uniform=uniform)
                      for i in range(1, n)]


def time_cold_calls(torch, api, dev, stream, pool, members, M, capture, time_graph, reps=5):
    """Seconds per call of api.linear_group over the weights `members` of every pool entry in
    turn (one launch each), replayed from a CUDA graph; and the algorithmic bytes per call."""
    K = pool[0][members[0]].K
    x = torch.randn((M, K), device=dev).half()
    ys = [torch.empty((M, pool[0][n].N), dtype=torch.float16, device=dev) for n in members]

    def fn():
        for layer in pool:
            api.linear_group(x, [layer[n] for n in members], outs=ys)
    g = capture(torch, fn, stream)
    t = time_graph(torch, g, reps, stream) / (reps * len(pool))
    del g
    wb = sum(pool[0][n].nbytes() for n in members)
    ab = 2 * M * (K + sum(pool[0][n].N for n in members))
    return t, wb, ab


def workload_extras(torch, api, synth, dev, stream, peaks, capture, time_graph):
    """The other workloads of the layer, each call on a cold weight: the single 4096 x 2560 GEMV
    (trits 1/3 each, no residual rows), one Qwen3-4B layer's 7 projections, the 36-layer
    Qwen3-4B stack at M = 1, 4 and 16 (four grouped launches per layer, like the 8B step), and
    the Qwen3-8B projections one by one at M = 1, 4, 8 and 16."""
    hbm = peaks["hbm_gbs"]
    out = {}

    def entry(t, wb, ab):
        return {"us": t * 1e6, "packed_gbs": wb / t / 1e9, "frac": (wb + ab) / t / 1e9 / hbm,
                "frac_of_8000": (wb + ab) / t / 1e9 / 8000.0}

    # config 1
    pool = cold_pool(torch, api, dev, [("single", 4096, 2560)], 5000, res_pct=0, uniform=True)
    t, wb, ab = time_cold_calls(torch, api, dev, stream, pool, ["single"], 1, capture, time_graph)
    out["single_gemv_4096x2560_m1"] = dict(entry(t, wb, ab), distinct_weights=len(pool))
    del pool
    # config 2: one launch per projection
    shapes4 = [(n, N, K) for n, (N, K) in synth.QWEN3_4B.items()]
    per = {}
    for n, N, K in shapes4:
        pool = cold_pool(torch, api, dev, [(n, N, K)], 6000, res_pct=10)
        t, wb, ab = time_cold_calls(torch, api, dev, stream, pool, [n], 1, capture, time_graph)
        per[n] = dict(entry(t, wb, ab), distinct_weights=len(pool))
        del pool
    out["qwen3_4b_layer_m1"] = {"per_projection": per,
                                "layer_us": sum(v["us"] for v in per.values()),
                                "note": "7 launches, one per projection, 10% residual rows"}
    # config 3: the 36-layer stack, grouped launches, weights from an 8-layer pool (237 MB)
    pool = [draw_layer_on_device(torch, api, shapes4, dev, seed=7000 + i, res_pct=10) for i in range(POOL_LAYERS)]
    kd = {n: K for n, _, K in shapes4}
    nd = {n: N for n, N, _ in shapes4}
    stack = {}
    for M in (1, 4, 16):
        xs = {g: torch.randn((M, kd[m[0]]), device=dev).half() for g, m in GROUPS}
        flat = torch.empty(LAYERS * M * sum(nd.values()), dtype=torch.float16, device=dev)
        ys, off = [], 0
        for _ in range(LAYERS):
            d = {}
            for n in nd:
                d[n] = flat[off:off + M * nd[n]].view(M, nd[n])
                off += M * nd[n]
            ys.append(d)

        def fn(xs=xs, ys=ys):
            for layer in range(LAYERS):
                for g, members in GROUPS:
                    api.linear_group(xs[g], [pool[layer % POOL_LAYERS][n] for n in members],
                                     outs=[ys[layer][n] for n in members])
        g = capture(torch, fn, stream)
        t = time_graph(torch, g, 20, stream) / 20
        del g
        wb = LAYERS * sum(pool[0][n].nbytes() for n in nd)
        ab = LAYERS * sum(2 * M * (kd[m[0]] + sum(nd[n] for n in m)) for _, m in GROUPS)
        stack[str(M)] = {"us_per_step": t * 1e6, "packed_gbs": wb / t / 1e9, "frac": (wb + ab) / t / 1e9 / hbm,
                         "launches": LAYERS * len(GROUPS)}
        del xs, ys, flat
    out["qwen3_4b_stack"] = dict(stack, pool_mb=sum(w.nbytes() for L in pool for w in L.values()) / 1e6)
    del pool
    # config 4: the 8B projections, one launch each, at every M
    per = {}
    for n, (N, K) in synth.QWEN3_8B.items():
        pool = cold_pool(torch, api, dev, [(n, N, K)], 8000, res_pct=15)
        per[n] = {}
        for M in (1, 4, 8, 16):
            t, wb, ab = time_cold_calls(torch, api, dev, stream, pool, [n], M, capture, time_graph)
            per[n][str(M)] = entry(t, wb, ab)
        del pool
    out["qwen3_8b_projections"] = per
    return out


def oracle_configs():
    """The oracle on the host cores for each workload: one call per projection (config 3: one
    layer, times 36, stated)."""
    import oracle
    from ternary_weight_only_tern_b200 import synth
    out = {}

    def timed(ts, M):
        t0 = time.perf_counter()
        nb = 0
        for t in ts:
            oracle.linear(t.x[:M], t.T1, t.s1, t.res_rows, t.T2, t.s2)
            nb += (t.N + t.r) * t.K // 4 + 2 * (t.N + t.r) * (t.K // 128) + 4 * t.N
        return time.perf_counter() - t0, nb

    s, nb = timed(list(synth.draw_workload(synth.WORKLOADS[1])), 1)
    out["single_gemv_4096x2560_m1"] = {"s": s, "packed_gbs": nb / s / 1e9}
    layer = list(synth.draw_workload(synth.WORKLOADS[2]))
    s, nb = timed(layer, 1)
    out["qwen3_4b_layer_m1"] = {"s": s, "packed_gbs": nb / s / 1e9}
    out["qwen3_4b_stack_m1"] = {"s": 36 * s, "packed_gbs": nb / s / 1e9, "note": "one layer timed, times 36"}
    t8 = list(synth.draw_workload(synth.WORKLOADS[4]))
    s, nb = timed(t8, 16)
    out["qwen3_8b_projections_m16"] = {"s": s, "packed_gbs": nb / s / 1e9}
    return out


def time_graph(torch, graph, reps, stream):
    """Seconds for `reps` replays; the graph is launched on `stream` (replay() uses the current
    stream), bracketed by events on that same stream."""
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        s.record(stream)
        for _ in range(reps):
            graph.replay()
        e.record(stream)
    e.synchronize()
    return s.elapsed_time(e) / 1e3


def capture(torch, fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        fn()                     # eager warm-up of this exact sequence
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=stream):
        fn()
    torch.cuda.synchronize()
    return g


# ------------------------------------------------------------------------------ CPU oracle
def oracle_sample(seconds_budget=12.0):
    """The oracle on one 8B-shaped decoder layer's 7 projections at M = 1 (numpy inputs drawn
    with the host recipe). Returns (packed bytes, seconds, threads, description)."""
    import oracle
    from ternary_weight_only_tern_b200 import synth
    try:
        from threadpoolctl import threadpool_info
        threads = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    except Exception:
        threads = 1
    tensors = list(synth.draw_workload(synth.WORKLOADS[4]))
    nbytes, secs, calls = 0, 0.0, 0
    while secs < seconds_budget:
        t = tensors[calls % len(tensors)]
        t0 = time.perf_counter()
        oracle.linear(t.x[:1], t.T1, t.s1, t.res_rows, t.T2, t.s2)
        secs += time.perf_counter() - t0
        nbytes += (t.N + t.r) * t.K // 4 + 2 * (t.N + t.r) * (t.K // 128) + 4 * t.N
        calls += 1
    return nbytes, secs, threads, f"oracle.linear (numpy float64 dequant + matmul) cycling the 7 projections of " \
                                  f"one Qwen3-8B-shaped layer at M=1, 15% residual rows ({calls} calls, " \
                                  f"{secs:.1f} s)"


def run_reference(args, rank, world):
    """--impl reference: the CPU oracle as it stands, on rank 0 only."""
    if rank != 0:
        return
    import oracle
    from ternary_weight_only_tern_b200 import synth
    try:
        from threadpoolctl import threadpool_info
        threads = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    except Exception:
        threads = 1
    tensors = list(synth.draw_workload(synth.WORKLOADS[4]))

    def step(i):
        t = tensors[i % len(tensors)]
        oracle.linear(t.x[:1], t.T1, t.s1, t.res_rows, t.T2, t.s2)
        return (t.N + t.r) * t.K // 4 + 2 * (t.N + t.r) * (t.K // 128) + 4 * t.N

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    nbytes = sum(step(args.warmup + i) for i in range(args.steps))
    secs = time.perf_counter() - t0
    val = nbytes / secs / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / max(1, args.steps) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (numpy PCG64, seed 3: the 8B projection recipe)",
        "config": {"workload": WORKLOAD, "sample": "one 8B projection per step, cycling q,k,v,o,gate,up,down",
                   "M": 1, "residual_pct": RES_PCT},
        "cpu_baseline": {"value": val, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": "one Qwen3-8B-shaped projection per step at M=1 (cycling the 7)"},
        "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------ main arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--quick", action="store_true", help="skip the extra measurements")
    ap.add_argument("--prefetch-depth", type=int, default=0, choices=[0, 1, 2],
                    help="how many following launches' weights each launch brings into L2 (with grouped "
                         "launches 0 measured best: at M = 1 1643 us per step against 1670 for 1 and 1683 for 2, "
                         "at M = 16 4569 against 4575 and 4598)")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU baseline")
    ap.add_argument("--profile", choices=["gemv", "gemv16", "gemv_elem", "gemm", "gemm_elem", "rotate"], default=None,
                    help="run a few calls of one op on one pool layer and exit (for ncu captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist
    from datetime import timedelta

    from ternary_weight_only_tern_b200 import _lib, api, synth

    _lib.load()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v: float) -> float:
        return max_over_ranks_of(dist if world > 1 else None, v, dev)

    peaks, peak_kind = load_peaks()
    shapes = list(synth.WORKLOADS[4].shapes)
    if args.profile:
        return profile_case(torch, api, shapes, dev, args.profile)
    pool = [draw_layer_on_device(torch, api, shapes, dev, seed=1000 + i) for i in range(POOL_LAYERS)]
    torch.cuda.synchronize()
    names = [s[0] for s in shapes]
    Kmax = max(K for _, _, K in shapes)
    ws = torch.empty(max(api.workspace_bytes(pool[0][n], 16) for n in names) + 256, dtype=torch.uint8, device=dev)
    launches_per_call = 1
    stream = torch.cuda.Stream(device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(7)

    flat_out = {}

    kdim = {n: K for n, _, K in shapes}
    ndim = {n: N for n, N, _ in shapes}

    def make_io(M):
        # one input per group of projections that share it; the 252 outputs of a step are views of
        # one buffer, so a step's results leave the device in one copy
        xs = {gname: torch.randn((M, kdim[members[0]]), generator=gen, device=dev).half() for gname, members in GROUPS}
        flat = torch.empty(LAYERS * M * sum(N for _, N, _ in shapes), dtype=torch.float16, device=dev)
        ys, off = [], 0
        for _ in range(LAYERS):
            d = {}
            for n, N, _ in shapes:
                d[n] = flat[off:off + M * N].view(M, N)
                off += M * N
            ys.append(d)
        flat_out[M] = flat
        return xs, ys

    def calls_of(only=None, grouped=True):
        # (layer, input, projections) of a step in order: a group per call, or (grouped=False)
        # one projection per call; `only` keeps one group or one projection
        out = []
        for layer in range(LAYERS):
            for gname, members in GROUPS:
                if grouped:
                    if only is None or only == gname:
                        out.append((layer, gname, members))
                else:
                    out += [(layer, gname, (n,)) for n in members if only is None or only == n]
        return out

    def step_fn(M, xs, ys, only=None, weights=None, grouped=True, rot=None):
        # the calls of a step in order; each also starts bringing the next call's weights into L2.
        # rot: per layer {input: (R, buffer)}: each call's input is first rotated (tern_rotate)
        calls = calls_of(only, grouped)
        wp = weights or pool

        def fn():
            for i, (layer, gname, members) in enumerate(calls):
                pf = []
                for d in range(1, args.prefetch_depth + 1):
                    nl, _, nm = calls[(i + d) % len(calls)]
                    pf += [wp[nl % POOL_LAYERS][n] for n in nm]
                x_in = xs[gname]
                if rot is not None:
                    x_in = api.rotate(x_in, rot[layer][gname][0], out=rot[layer][gname][1])
                api.linear_group(x_in, [wp[layer % POOL_LAYERS][n] for n in members],
                                 outs=[ys[layer][n] for n in members], workspace=ws, prefetch=pf[:4])
        return fn

    def step_bytes(M, only=None, weights=None, grouped=True):
        # weights streamed, and activations: each call reads its input once and writes its outputs
        wp = weights or pool
        calls = calls_of(only, grouped)
        wb = sum(packed_bytes(wp[layer % POOL_LAYERS][n]) for layer, _, members in calls for n in members)
        ab = sum(2 * M * (kdim[members[0]] + sum(ndim[n] for n in members)) for _, _, members in calls)
        return wb, ab

    # ---------------- the timed region: K graph replays of the full M = 1 step
    xs1, ys1 = make_io(1)
    flat1 = flat_out[1]                 # the buffer behind ys1
    g_step = capture(torch, step_fn(1, xs1, ys1), stream)
    launches_per_step = len(calls_of()) * launches_per_call
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            g_step.replay()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(gpu_uuid(torch, dev)) as clk:
        secs = time_graph(torch, g_step, args.steps, stream)
    torch.cuda.synchronize()
    barrier()
    secs = max_over_ranks(secs)
    wb, ab = step_bytes(1)
    value = replica_value(world, wb * args.steps, secs) / 1e9
    ms_per_step = secs / args.steps * 1e3

    # ---------------- the dominant op: the gate + up launch (tern_linear_group) at M = 1
    g_gate = capture(torch, step_fn(1, xs1, ys1, only="gateup"), stream)
    with torch.cuda.stream(stream):
        for _ in range(5):
            g_gate.replay()
    reps = max(20, min(400, args.steps // 10))
    t_gate = time_graph(torch, g_gate, reps, stream) / (reps * LAYERS)
    gw, ga = step_bytes(1, only="gateup")
    gate_bytes = (gw + ga) / LAYERS
    achieved = gate_bytes / t_gate / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": measured_traffic("gemv"),
                "op": "tern_linear_group gate+up 2 x 12288x4096 (+1843 residual rows each) M=1",
                "us_per_call": t_gate * 1e6, "bytes_per_call": gate_bytes, "peak_kind": peak_kind,
                "frac_of_8000": achieved / 8000.0}

    extra = {}
    if not args.quick and world == 1:
        extra = extras(torch, api, synth, pool, shapes, names, stream, dev, ws, step_fn, step_bytes, make_io, peaks,
                       time_graph, capture)
        extra["workloads"] = workload_extras(torch, api, synth, dev, stream, peaks, capture, time_graph)

    # ---------------- e2e through the Python API with host buffers
    e2e_steps = 100         # ~0.15 s of wall clock per mode: a single slow step moves the mean little
    xh = {gname: torch.randn((1, kdim[members[0]])).half().pin_memory() for gname, members in GROUPS}
    yh = torch.empty(flat1.numel(), dtype=torch.float16).pin_memory()
    h2d = sum(2 * kdim[members[0]] for _, members in GROUPS)
    d2h = LAYERS * sum(2 * N for _, N, _ in shapes)

    def copies_and_calls():
        for gname, _ in GROUPS:
            xs1[gname].copy_(xh[gname], non_blocking=True)
        step_fn(1, xs1, ys1)()
        yh.copy_(flat1, non_blocking=True)

    # the step as a serving loop runs it: the API calls and the host <-> device copies captured once
    # into a CUDA graph and replayed; the wall clock spans the replay and the host synchronisation
    g_e2e = capture(torch, copies_and_calls, stream)

    def e2e_step():
        with torch.cuda.stream(stream):
            g_e2e.replay()
        stream.synchronize()

    def e2e_step_eager():
        with torch.cuda.stream(stream):
            copies_and_calls()
        stream.synchronize()

    for _ in range(3):
        e2e_step()
    barrier()
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        e2e_step()
    e2e_secs = max_over_ranks(time.perf_counter() - t0)
    for _ in range(3):
        e2e_step_eager()
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        e2e_step_eager()
    eager_secs = max_over_ranks(time.perf_counter() - t0)
    del g_e2e
    e2e = {"value": world * wb * e2e_steps / eager_secs / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "steps": e2e_steps,
           "graph_value": world * wb * e2e_steps / e2e_secs / 1e9,
           "note": "value: every step issues the 144 api.linear_group calls (q+k+v, o, gate+up, down per layer) "
                   "from Python through the C ABI, with the step's 4 inputs copied in from pinned host memory "
                   "and all 252 outputs (one buffer) copied back; wall clock around the step and its stream "
                   "synchronize. graph_value: the same calls and copies captured once into a CUDA graph and "
                   "replayed each step"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        nb, cs, threads, desc = oracle_sample()
        cpu = {"value": nb / cs / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": desc,
               "seconds": cs}
        if not args.quick:
            cpu["per_workload"] = oracle_configs()

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16",
        "data": "synthetic: trits P(0)=0.4, P(+-1)=0.3, fp16 group-128 scales, seeded torch generator per pool layer",
        "config": {"workload": WORKLOAD, "layers": LAYERS, "projections": names, "M": 1, "residual_pct": RES_PCT,
                   "l2_prefetch_depth": args.prefetch_depth,
                   "launches_per_layer": "q+k+v, o, gate+up, down (tern_linear_group on a shared input)",
                   "pool_layers": POOL_LAYERS, "packed_bytes_per_step": wb, "activation_bytes_per_step": ab,
                   "l2": f"inputs larger than L2: {POOL_LAYERS}-layer weight pool of "
                         f"{sum(packed_bytes(w) for L in pool for w in L.values()) / 1e6:.0f} MB rotated through",
                   "parallelism": f"replicas x{world}", "frac_of_measured_hbm": value / peaks["hbm_gbs"],
                   "frac_of_8000": value / 8000.0},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps, "clocks": clk.summary(), "extra": extra,
    }
    print(json.dumps(line), flush=True)


def profile_case(torch, api, shapes, dev, which):
    """A minimal run for ncu, three repetitions over two layers: at M = 1 (gemv) or M = 16 (gemv16) the
    bench's four launches per layer (q+k+v, o, gate+up, down), or (gemv_elem) the same with element planes
    (3.6 % masked) in place of residual rows; at M = 2048 (gemm, gemm_elem) gate, up and down."""
    if which == "rotate":
        # tern_rotate on K = 4096 at M = 1 and M = 2048, three times
        R = (torch.randn((32, 128, 128), device=dev) / 11.3).half()
        xs = [torch.randn((M, 4096), device=dev).half() for M in (1, 2048)]
        ys = [torch.empty_like(x) for x in xs]
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_push("tern_calls")
        for _ in range(3):
            for x, y in zip(xs, ys):
                api.rotate(x, R, out=y)
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
        print(json.dumps({"profile": which, "calls": 6}))
        return
    elem = 0.036 if which in ("gemv_elem", "gemm_elem") else None
    pool = [draw_layer_on_device(torch, api, shapes, dev, seed=1000 + i, elem_frac=elem) for i in range(2)]
    kdim = {n: K for n, _, K in shapes}
    prefill = which in ("gemm", "gemm_elem")
    groups = GROUPS if not prefill else [("gate", ("gate",)), ("up", ("up",)), ("down", ("down",))]
    M = 2048 if prefill else (16 if which == "gemv16" else 1)
    xs = {g: torch.randn((M, kdim[m[0]]), device=dev).half() for g, m in groups}
    ys = {n: torch.empty((M, N), dtype=torch.float16, device=dev) for n, N, _ in shapes}
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("tern_calls")   # ncu --nvtx --nvtx-include "tern_calls/" lists these only
    for _ in range(3):
        for layer in pool:
            for g, members in groups:
                api.linear_group(xs[g], [layer[n] for n in members], outs=[ys[n] for n in members])
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    print(json.dumps({"profile": which, "calls": 3 * len(pool) * len(groups)}))


def extras(torch, api, synth, pool, shapes, names, stream, dev, ws, step_fn, step_bytes, make_io, peaks,
           time_graph, capture):
    out = {}
    kdim_of = {n: K for n, _, K in shapes}.__getitem__
    hbm = peaks["hbm_gbs"]
    # per group at M = 1 (one launch per group), each call on a cold weight (a pool of distinct
    # copies larger than three L2s)
    xs1, ys1 = make_io(1)
    per = {}
    for gi, (gname, members) in enumerate(GROUPS):
        cp = cold_pool(torch, api, dev, [s_ for s_ in shapes if s_[0] in members], 9000 + 1000 * gi, res_pct=RES_PCT)
        t, wb, ab = time_cold_calls(torch, api, dev, stream, cp, list(members), 1, capture, time_graph)
        per[gname] = {"us": t * 1e6, "packed_gbs": wb / t / 1e9, "frac": (wb + ab) / t / 1e9 / hbm,
                      "distinct_weights": len(cp)}
        del cp
    out["per_group_m1"] = per
    # the whole stack with one launch per projection (252 per step), for comparison
    g = capture(torch, step_fn(1, xs1, ys1, grouped=False), stream)
    t = time_graph(torch, g, 30, stream) / 30
    wb, ab = step_bytes(1, grouped=False)
    out["stack_m1_one_launch_per_projection"] = {"us_per_step": t * 1e6, "packed_gbs": wb / t / 1e9,
                                                 "frac": (wb + ab) / t / 1e9 / hbm}
    del g
    # per M over the whole stack
    perm = {}
    for M in (1, 4, 8, 16):
        xs, ys = make_io(M)
        g = capture(torch, step_fn(M, xs, ys), stream)
        t = time_graph(torch, g, 30, stream) / 30
        wb, ab = step_bytes(M)
        perm[str(M)] = {"us_per_step": t * 1e6, "packed_gbs": wb / t / 1e9, "frac": (wb + ab) / t / 1e9 / hbm}
        del g, xs, ys
    out["per_M_stack"] = perm
    # prefill GEMM at M = 2048 on the gate/up/down shapes
    gemm = {}
    for n in ("gate", "up", "down"):
        N, K = [(s[1], s[2]) for s in shapes if s[0] == n][0]
        x = torch.randn((2048, K), device=dev).half()
        y = torch.empty((2048, N), dtype=torch.float16, device=dev)
        wsg = torch.empty(api.workspace_bytes(pool[0][n], 2048) + 256, dtype=torch.uint8, device=dev)

        def fn(n=n, x=x, y=y, wsg=wsg):
            for i in range(4):
                api.linear(x, pool[i][n], out=y, workspace=wsg)
        g = capture(torch, fn, stream)
        t = time_graph(torch, g, 5, stream) / 20
        fl = 2.0 * 2048 * N * K
        gemm[n] = {"us": t * 1e6, "tflops": fl / t / 1e12, "frac_burst": fl / t / 1e12 / peaks["bf16_tflops"],
                   "frac_sustained": fl / t / 1e12 / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])}
        del g, x, y, wsg
    out["gemm_m2048"] = gemm
    # the activation-side rotation (tern_rotate, one 128 x 128 fp16 block per group): alone at M = 1
    # and M = 2048 on K = 4096 and 12288, and the M = 1 stack with a rotation before every launch
    # (its own blocks for each input of each of the 36 layers: 216 MB, more than L2)
    rot = {}
    for K in (4096, 12288):
        R = (torch.randn((K // 128, 128, 128), device=dev) / 11.3).half()
        for M in (1, 2048):
            x = torch.randn((M, K), device=dev).half()
            y = torch.empty_like(x)

            def fn_rot(x=x, R=R, y=y):
                for _ in range(20):
                    api.rotate(x, R, out=y)
            g = capture(torch, fn_rot, stream)
            t = time_graph(torch, g, 20, stream) / 400
            nbytes = R.numel() * 2 + 2 * x.numel() * 2
            rot[f"K{K}_M{M}"] = {"us": t * 1e6, "gbs": nbytes / t / 1e9, "frac_hbm": nbytes / t / 1e9 / hbm,
                                 "tflops": 2.0 * M * K * 128 / t / 1e12}
            del g, x, y
    xs, ys = make_io(1)
    bufs = {gname: torch.empty_like(xs[gname]) for gname, _ in GROUPS}
    rots = [{gname: ((torch.randn((kdim_of(members[0]) // 128, 128, 128), device=dev) / 11.3).half(), bufs[gname])
             for gname, members in GROUPS} for _ in range(LAYERS)]
    g = capture(torch, step_fn(1, xs, ys, rot=rots), stream)
    t = time_graph(torch, g, 30, stream) / 30
    wb, ab = step_bytes(1)
    rb = sum(r.numel() * 2 for L in rots for r, _ in L.values())
    rot["stack_m1_with_rotation"] = {"us_per_step": t * 1e6, "packed_gbs": wb / t / 1e9,
                                     "bytes_gbs": (wb + rb) / t / 1e9, "rotation_bytes_per_step": rb}
    out["rotation"] = rot
    del g, xs, ys, rots
    # the per-group offset mu (W = mu + s1 T1 + s2 T2): the same pool with an fp16 offset per
    # (row, group) drawn U[-0.01, 0.01], the M = 1 stack and the gate GEMM at M = 2048
    gm = torch.Generator(device=dev)
    gm.manual_seed(17)
    mpool = [{n: dataclasses.replace(L[n], mu=(torch.rand((L[n].N, L[n].K // 128), generator=gm, device=dev) * 0.02
                                               - 0.01).half()) for n in names} for L in pool]
    xs, ys = make_io(1)
    g = capture(torch, step_fn(1, xs, ys, weights=mpool), stream)
    t = time_graph(torch, g, 30, stream) / 30
    wb, ab = step_bytes(1, weights=mpool)
    off = {"stack_m1": {"us_per_step": t * 1e6, "packed_gbs": wb / t / 1e9, "frac": (wb + ab) / t / 1e9 / hbm,
                        "packed_bytes_per_step": wb}}
    del g, xs, ys
    g = capture(torch, step_fn(1, xs1, ys1, only="gateup", weights=mpool), stream)
    t = time_graph(torch, g, 50, stream) / (50 * LAYERS)
    wb, ab = step_bytes(1, only="gateup", weights=mpool)
    off["gateup_m1"] = {"us": t * 1e6, "frac": (wb + ab) / LAYERS / t / 1e9 / hbm}
    del g
    x = torch.randn((2048, 4096), device=dev).half()
    y = torch.empty((2048, 12288), dtype=torch.float16, device=dev)

    def fn_mu():
        for i in range(4):
            api.linear(x, mpool[i]["gate"], out=y)
    g = capture(torch, fn_mu, stream)
    t = time_graph(torch, g, 5, stream) / 20
    fl = 2.0 * 2048 * 12288 * 4096
    off["gate_m2048"] = {"us": t * 1e6, "tflops": fl / t / 1e12, "frac_burst": fl / t / 1e12 / peaks["bf16_tflops"]}
    out["offset_mu"] = off
    del g, x, y, mpool
    # the element-level second plane: 3.6 % of the weights masked (the pages' two most salient
    # masks) instead of 15 % of the rows, the M = 1 stack and the gate GEMM at M = 2048
    epool = [draw_layer_on_device(torch, api, shapes, dev, seed=2000 + i, elem_frac=0.036) for i in range(POOL_LAYERS)]
    torch.cuda.synchronize()
    xs, ys = make_io(1)
    g = capture(torch, step_fn(1, xs, ys, weights=epool), stream)
    t = time_graph(torch, g, 30, stream) / 30
    wb, ab = step_bytes(1, weights=epool)
    el = {"stack_m1": {"us_per_step": t * 1e6, "packed_gbs": wb / t / 1e9, "frac": (wb + ab) / t / 1e9 / hbm,
                       "packed_bytes_per_step": wb,
                       "nnz2_per_weight": float(np.mean([L[n].elem.nnz2 / (L[n].N * L[n].K) for L in epool
                                                          for n in names]))}}
    del g, xs, ys
    g = capture(torch, step_fn(1, xs1, ys1, only="gateup", weights=epool), stream)
    t = time_graph(torch, g, 50, stream) / (50 * LAYERS)
    wb, ab = step_bytes(1, only="gateup", weights=epool)
    el["gateup_m1"] = {"us": t * 1e6, "frac": (wb + ab) / LAYERS / t / 1e9 / hbm}
    del g
    x = torch.randn((2048, 4096), device=dev).half()
    y = torch.empty((2048, 12288), dtype=torch.float16, device=dev)

    def fn_elem():
        for i in range(4):
            api.linear(x, epool[i]["gate"], out=y)
    g = capture(torch, fn_elem, stream)
    t = time_graph(torch, g, 5, stream) / 20
    el["gate_m2048"] = {"us": t * 1e6, "tflops": fl / t / 1e12, "frac_burst": fl / t / 1e12 / peaks["bf16_tflops"]}
    out["elem_plane"] = el
    del g, x, y, epool
    # the ternarization fit on the gate shape (12288 x 4096 fp16, 15 % residual rows, offset, 15 rounds)
    Wd = (torch.randn((12288, 4096), device=dev) * 0.02).half()
    frows = torch.randperm(12288, device=dev)[:1843].sort().values.to(torch.int32)
    api.fit(Wd, frows)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(3):
        T1f, s1f, muf, T2f, s2f = api.fit(Wd, frows)
    torch.cuda.synchronize()
    dt = (time.perf_counter() - t0) / 3
    What = (s1f.float().repeat_interleave(128, 1) * T1f.float() + muf.float().repeat_interleave(128, 1))
    What[frows.long()] += s2f.float().repeat_interleave(128, 1) * T2f.float()
    rel = float(((What - Wd.float()).norm() / Wd.float().norm()).item())
    out["fit_gate"] = {"ms": dt * 1e3, "w_gbs": Wd.numel() * 2 / dt / 1e9, "groups_per_s": 12288 * 32 / dt,
                       "relative_frobenius_error": rel,
                       "note": "tern_fit, float64 sums; wall clock of 3 calls after a warm-up"}
    del Wd, frows, T1f, s1f, muf, T2f, s2f, What
    # packing throughput on the gate shape
    u = torch.randint(0, 3, (12288, 4096), dtype=torch.int8, device=dev) - 1
    for fn_name, fn in (("pack_exec", api.pack_exec), ("pack_store", api.pack_store)):
        fn(u)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for _ in range(5):
            r = fn(u)
        dt = (time.perf_counter() - t0) / 5
        out[fn_name] = {"ms": dt * 1e3, "in_gbs": u.numel() / dt / 1e9, "out_bytes": r.numel() * r.element_size(),
                        "note": "synchronous call incl. status read-back"}
    del u
    # bit accounting of the 252-tensor 8B stack
    tot = {"weights": 0, "store_bits": 0, "exec_bits": 0, "plane_trits": 0}
    for (n, N, K) in shapes:
        b = api.bits(N, K, synth.residual_count(N, RES_PCT))
        for k in tot:
            tot[k] += LAYERS * b[k]
    out["bits_8b_stack"] = {"bpw_info": 1.584962500721156 * tot["plane_trits"] / tot["weights"],
                            "bpw_store": tot["store_bits"] / tot["weights"],
                            "bpw_exec": tot["exec_bits"] / tot["weights"],
                            "store_gib": tot["store_bits"] / 8 / 2 ** 30}
    # the same stack with the element-level second plane at the pages' 3.6 % (P(t2 != 0) = 0.6 of it)
    tot = {"weights": 0, "store_bits": 0, "exec_bits": 0, "plane_trits": 0}
    for (n, N, K) in shapes:
        masked = round(0.036 * N * K)
        b = api.bits_elem(N, K, masked, round(0.6 * masked))
        for k in tot:
            tot[k] += LAYERS * b[k]
    out["bits_8b_stack_elem"] = {"bpw_info": 1.584962500721156 * tot["plane_trits"] / tot["weights"],
                                 "bpw_store": tot["store_bits"] / tot["weights"],
                                 "bpw_exec": tot["exec_bits"] / tot["weights"],
                                 "store_gib": tot["store_bits"] / 8 / 2 ** 30}
    # dense fp16 cuBLAS on the gate shape (context, as in the pages' comparison)
    Wd = [torch.randn((12288, 4096), device=dev).half() for _ in range(4)]
    x1 = torch.randn((1, 4096), device=dev).half()
    xb = torch.randn((2048, 4096), device=dev).half()

    def dense1():
        for w in Wd:
            torch.matmul(x1, w.t())

    def dense2():
        for w in Wd:
            torch.matmul(xb, w.t())
    g1 = capture(torch, dense1, stream)
    t1 = time_graph(torch, g1, 50, stream) / 200
    g2 = capture(torch, dense2, stream)
    t2 = time_graph(torch, g2, 5, stream) / 20
    out["context_fp16_cublas_gate"] = {"m1_us": t1 * 1e6, "m1_gbs": 12288 * 4096 * 2 / t1 / 1e9,
                                       "m2048_us": t2 * 1e6, "m2048_tflops": 2 * 2048 * 12288 * 4096 / t2 / 1e12}
    return out


if __name__ == "__main__":
    main()
