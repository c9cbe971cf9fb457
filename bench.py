#!/usr/bin/env python
"""Benchmark of the CSA2 decode hot path on B200.

One step = one call of the 20-layer decoder stack (csa2_layer_stack) over one
batch of seeded synthetic inputs of the `stack20_128k` workload: 16 sequences x
131072 cached positions, layers [Full, Reuse, Reuse, Reindex] x 5, pool 8192,
top-k 2048, SWA 512, 16 heads x 128, indexer 8 x 64 int8. Inputs are resident in
HBM; L2 is flushed (a 256 MB write) before every timed step, outside its events.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs its own replica (its own sequences; the path
shards by sequence with no collective) and rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA2 decode queries/s at 128K ctx (1 B200); achieved HBM GB/s vs peak"
UNIT = "queries/s"
DEFAULT_WORKLOAD = "stack20_128k"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--kernel-launches", type=int, default=50)
    ap.add_argument("--eager", action="store_true", help="launch directly instead of replaying a CUDA graph")
    ap.add_argument("--phase-trace", action="store_true",
                    help="load the phase-trace build and print per-phase CTA times and the step's launch timeline "
                         "instead of the JSON line")
    ap.add_argument("--override", default="",
                    help="replace workload fields, e.g. Tq=1024,N=33792 (a smaller case of the same shape, for profiling)")
    args = ap.parse_args()
    if args.phase_trace:
        os.environ["CSA2_LIBRARY"] = "trace"   # before the library is loaded
    args.overrides = {}
    for kv in filter(None, args.override.split(",")):
        k, v = kv.split("=")
        args.overrides[k.strip()] = int(v)
    return args


# ------------------------------------------------------------------ accounting
def unit_bytes(spec):
    """Algorithmic bytes one query moves through the whole stack (each distinct row
    once per kernel call): index keys scanned or gathered, pool/list indices, FP4
    rows gathered (D/2 + D/16 bytes), local K+V rows, queries and outputs."""
    D, Di, Hi, Hq = spec.D, spec.Di, spec.Hi, spec.Hq
    t = spec.n_pos - 1
    total = 0
    k_cur, pool_P = 0, 0
    for L in spec.layers:
        if L.mode == "FULL":
            total += entries_read(spec, t) * Di + Hi * Di + (L.P + L.k) * 4
            k_cur = L.k
            pool_P = L.P or pool_P
        elif L.mode == "REINDEX":
            total += pool_P * (Di + 4) + Hi * Di + L.k * 4
            k_cur = L.k
        total += k_cur * (D // 2 + D // 16 + 4) + min(spec.W, t + 1) * 2 * D * 2 + 2 * Hq * D * 2
    return total


def entries_read(spec, t):
    """Global entries the query at position t reads (compression rate m: complete groups)."""
    return (t + 1) // spec.m if spec.m > 1 else t + 1


def full_launch_bytes(spec, q_pos):
    """Algorithmic bytes of the first layer's Full indexer call: every sequence's keys
    up to its last query position once, then per query its index query and lists."""
    L = spec.layers[0]
    keys = sum(entries_read(spec, int(q_pos[b].max())) for b in range(spec.B)) * spec.Di
    return keys + spec.B * spec.Tq * (spec.Hi * spec.Di + (L.P + L.k) * 4)


def _window_rows(lo, hi):
    """Rows in the union of the closed intervals [lo_i, hi_i] (empty when hi < lo)."""
    rows, cur_lo, cur_hi = 0, None, None
    for a, b in sorted((int(x), int(y)) for x, y in zip(lo, hi) if y >= x):
        if cur_hi is None or a > cur_hi + 1:
            if cur_hi is not None:
                rows += cur_hi - cur_lo + 1
            cur_lo, cur_hi = a, b
        else:
            cur_hi = max(cur_hi, b)
    if cur_hi is not None:
        rows += cur_hi - cur_lo + 1
    return rows


def list_bytes(spec, q_pos, local_base, pools, topks):
    """Algorithmic bytes of one stack call, each distinct row once per kernel call,
    counted from the index lists the call produced (host arrays): keys scanned by a
    Full layer (up to the sequence's last query), pool key rows gathered by a Reindex
    layer, FP4 rows in the union of a sequence's lists, local K+V rows in the union of
    its windows, and per query its queries, lists and outputs. With one query per
    sequence this is the per-query sum of unit_bytes."""
    import numpy as np
    D, Di, Hi, Hq, W, B, Tq = spec.D, spec.Di, spec.Hi, spec.Hq, spec.W, spec.B, spec.Tq
    total, cur, pool, P_in = 0, None, None, 0
    for li, L in enumerate(spec.layers):
        if L.mode == "FULL":
            total += sum(entries_read(spec, int(q_pos[b].max())) for b in range(B)) * Di
            total += B * Tq * (Hi * Di + (L.P + L.k) * 4)
            cur = topks[li]
            if L.P:
                pool, P_in = pools[li], L.P
        elif L.mode == "REINDEX":
            total += sum(len(np.unique(pool[b][pool[b] >= 0])) for b in range(B)) * Di
            total += B * Tq * (P_in * 4 + Hi * Di + L.k * 4)
            cur = topks[li]
        total += sum(len(np.unique(cur[b][cur[b] >= 0])) for b in range(B)) * (D // 2 + D // 16)
        if W > 0:
            for b in range(B):
                t = q_pos[b].astype(np.int64)
                lo = np.maximum(np.maximum(t - W + 1, int(local_base[b])), 0)
                total += _window_rows(lo, t) * 2 * D * 2
        total += B * Tq * (cur.shape[-1] * 4 + 2 * Hq * D * 2)
    return total


def launches_per_step(spec):
    """Kernels one stack call launches: an indexer per Full/Reindex layer (two for a Full
    layer whose queries share keys: Tq >= 4 over N >= 8192, Hi <= 8, Di in {32, 64, 128},
    which is scored first) and an attention launch per layer."""
    mq = spec.Tq >= 4 and spec.N >= 8192 and spec.Hi <= 8 and spec.Di in (32, 64, 128)
    n = 0
    for L in spec.layers:
        if L.mode != "REUSE":
            n += 2 if (L.mode == "FULL" and mq) else 1
        n += 1
    return n


def metric_of(spec):
    return METRIC if spec.name == DEFAULT_WORKLOAD else f"CSA2 queries/s, {spec.name}; achieved HBM GB/s vs peak"


def workload_config(spec, units):
    """The workload fields of the JSON line's config (the same for both arms)."""
    return {"workload": spec.name, "B": spec.B, "N": spec.N, "Tq": spec.Tq, "layers": spec.L,
            "schedule": schedule_str(spec), "Hq": spec.Hq, "D": spec.D, "Hi": spec.Hi, "Di": spec.Di,
            "pool": spec.layers[0].P, "k": spec.layers[0].k, "W": spec.W, "per_gpu_queries": units}


def schedule_str(spec):
    """The layer modes, with a repeated period written once: [F,U,U,RI]x5."""
    ab = [{"FULL": "F", "REINDEX": "RI", "REUSE": "U"}[L.mode] for L in spec.layers]
    n = len(ab)
    for per in range(1, n // 2 + 1):
        if n % per == 0 and ab == ab[:per] * (n // per):
            return "[" + ",".join(ab[:per]) + "]x" + str(n // per)
    return ",".join(ab)


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:  # noqa: BLE001
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:  # noqa: BLE001
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "samples": len(sm),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------------ our arm
def capture_graph(torch, fn):
    """Capture fn(stream_ptr) into a CUDA graph; None if capture is not possible."""
    try:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            rc = fn(int(side.cuda_stream))            # one eager call to settle lazy init
            if rc:
                return None
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            rc = fn(int(torch.cuda.current_stream().cuda_stream))
        if rc:
            return None
        torch.cuda.synchronize()
        return g
    except Exception as e:  # noqa: BLE001
        print(f"graph capture failed, timing eager launches: {e}", file=sys.stderr)
        torch.cuda.synchronize()
        return None


def build_device_stack(wl, torch, ops, np):
    s = wl.spec

    def dev(a, dtype=None):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return (t.view(dtype) if dtype is not None else t).cuda()

    q_pos, base = dev(wl.q_pos()), dev(wl.local_base_arr())
    kv = dev(wl.kv_f32())
    codes, scales = ops.fp4_compress(kv.view(-1, s.D), s.m) if s.m > 1 else ops.fp4_quantize(kv.view(-1, s.D))
    del kv
    wl.drop("kv")
    codes, scales = codes.view(s.B, s.N, -1), scales.view(s.B, s.N, -1)
    keys = {}
    layers = []
    for li, L in enumerate(s.layers):
        d = {"mode": L.mode, "q": dev(wl.q(li).view(np.int16), torch.bfloat16),
             "kl": dev(wl.kl(li).view(np.int16), torch.bfloat16),
             "vl": dev(wl.vl(li).view(np.int16), torch.bfloat16), "W": s.W}
        if L.mode != "REUSE":
            if L.key_set not in keys:
                keys[L.key_set] = dev(wl.ki(L.key_set))
                wl.drop(("ki", L.key_set))
            d.update(qi=dev(wl.qi(li)), w=wl.w(li), ki=keys[L.key_set], k=L.k, P=L.P)
        layers.append(d)
    stack = ops.LayerStack(layers, q_pos, codes, scales, base, m=s.m)
    return stack, layers, q_pos, codes, scales, base


def job_rate(dist, torch, total_ms_local: float, units_per_rank: int, world: int, steps: int, device):
    """Whole-job queries/s: every rank timed `steps` steps of `units_per_rank` queries;
    the job's time is the slowest rank's (max over ranks, on the device clock)."""
    t = torch.tensor([float(total_ms_local)], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_ms = float(t.item())
    return total_ms, units_per_rank * world * steps / (total_ms / 1e3)


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch

    import synth
    from sparse_attention_shared_b200 import capi, ops

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    wl = synth.make_workload(args.workload, seed=rank, **args.overrides)
    s = wl.spec
    units = s.B * s.Tq
    stack, layers, q_pos, codes, scales, base = build_device_stack(wl, torch, ops, np)
    ws, st = ops.Workspace(), ops.Status()
    buf = ws.get(stack.ws_bytes)
    stream = torch.cuda.current_stream()
    sptr = int(stream.cuda_stream)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def call(stream_ptr):
        return stack.run_raw(int(buf.data_ptr()), buf.numel(), st.ptr, stream_ptr)

    graph = None if args.eager else capture_graph(torch, call)

    def step():
        if graph is not None:
            graph.replay()
            return 0
        return call(sptr)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        capi.check(step(), "warmup")
    st.check("warmup")

    K = args.steps
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    clocks = ClockSampler(local_rank)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks.start()
    time.sleep(0.3)
    for i in range(K):
        flush.zero_()
        ev0[i].record(stream)
        rc = step()
        ev1[i].record(stream)
        if rc:
            capi.check(rc, "timed step")
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clk = clocks.stop()
    st.check("timed region")
    step_ms = [a.elapsed_time(b) for a, b in zip(ev0, ev1)]
    total_ms, value = job_rate(dist, torch, sum(step_ms), units, world, K, "cuda")
    ms_per_step = total_ms / K
    n_launch = launches_per_step(s)

    # every kernel class of the step, each alone on the same stream with L2 flushed;
    # the roofline names the kernel with the largest share of the step
    qp_host = q_pos.cpu().numpy()
    base_host = base.cpu().numpy()
    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:  # noqa: BLE001
        pass
    hbm_peak = float(peaks.get("hbm_gbs", 6650.0))
    bf16_peak = float(peaks.get("bf16_tflops", 1590.0))
    int8_peak = 2.0 * bf16_peak   # the nominal dense int8 : bf16 ratio (4.5 : 2.25 PFLOP/s) times the measured bf16
    kernels = kernel_breakdown(args, torch, np, ops, capi, s, layers, q_pos, codes, scales, base, qp_host, base_host,
                               ws, st, flush, stream, hbm_peak, bf16_peak, int8_peak)
    traffic_db = {}
    try:
        traffic_db = json.load(open(os.path.join(ROOT, "profiles", "traffic.json"))).get(args.workload, {})
    except Exception:  # noqa: BLE001
        pass
    for kc in kernels:
        kc["traffic"] = traffic_db.get(kc["class"], {}).get("bytes_per_launch")
    # the dominant kernel: classes that run the same kernel (attention of Full, Reuse and
    # Reindex layers) are one kernel; its figures are per launch over all of its launches
    groups = {}
    for kc in kernels:
        groups.setdefault(kc["kernel"], []).append(kc)
    tops = []
    for name, g in groups.items():
        n = sum(kc["launches_per_step"] for kc in g)
        ms_l = sum(kc["ms"] * kc["launches_per_step"] for kc in g) / n
        bytes_l = sum(kc["algorithmic_bytes"] * kc["launches_per_step"] for kc in g) / n
        e = {"kernel": name, "class": "+".join(kc["class"] for kc in g), "launches_per_step": n, "ms": round(ms_l, 5),
             "algorithmic_bytes": int(bytes_l), "share": round(sum(kc["share"] for kc in g), 4),
             "traffic": next((kc["traffic"] for kc in g if kc["traffic"] is not None), None)}
        e["gbs"] = round(bytes_l / (ms_l * 1e-3) / 1e9, 1)
        e["frac"] = round(e["gbs"] / hbm_peak, 4)
        if all("tensor_ops" in kc for kc in g):
            ops_l = sum(kc["tensor_ops"] * kc["launches_per_step"] for kc in g) / n
            e.update({"tensor_ops": int(ops_l), "tensor_kind": g[0]["tensor_kind"],
                      "tensor_peak_tops": g[0]["tensor_peak_tops"]})
            e["tensor_tops"] = round(ops_l / (ms_l * 1e-3) / 1e12, 2)
            e["tensor_frac"] = round(e["tensor_tops"] / e["tensor_peak_tops"], 4)
        tops.append(e)
    top = max(tops, key=lambda e: e["share"])
    if top.get("tensor_frac", 0.0) > top["frac"]:   # the tensor pipe is the tighter bound
        roofline = {"bound": "tensor", "achieved": top["tensor_tops"], "peak": top["tensor_peak_tops"],
                    "unit": "TFLOP/s" if top["tensor_kind"] == "bf16" else "TOPS (int8)", "frac": top["tensor_frac"],
                    "traffic": top["traffic"], "kernel": top["kernel"], "class": top["class"], "kernel_ms": top["ms"],
                    "launches_per_step": top["launches_per_step"], "algorithmic_ops": top["tensor_ops"],
                    "share": top["share"],
                    "peak_source": ("MEASURED_PEAKS.json bf16_tflops (measured)" if peaks else "fallback 1590 TFLOP/s")
                    + (" x 2 (nominal int8 : bf16 dense ratio)" if top["tensor_kind"] == "int8" else "")}
    else:
        roofline = {"bound": "hbm", "achieved": top["gbs"], "peak": hbm_peak, "unit": "GB/s", "frac": top["frac"],
                    "traffic": top["traffic"], "kernel": top["kernel"], "class": top["class"],
                    "kernel_ms": top["ms"], "launches_per_step": top["launches_per_step"],
                    "algorithmic_bytes": top["algorithmic_bytes"], "share": top["share"],
                    "peak_source": "MEASURED_PEAKS.json hbm_gbs (measured)" if peaks else "fallback 6650 GB/s"}
    # the lists of the last timed step (the same inputs every step)
    host = lambda ts: [t.cpu().numpy() if t is not None else None for t in ts]
    step_bytes = list_bytes(s, qp_host, base.cpu().numpy(), host(stack.pools), host(stack.topks))
    step_gbs = step_bytes / (ms_per_step * 1e-3) / 1e9

    # end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, torch, np, ops, capi, stack, layers, q_pos, s, flush, stream, st, graph,
                      (codes, scales, base))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.workload, args.cpu_seconds, args.overrides)

    res = {
        "metric": metric_of(s),
        "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8+f16+bf16", "data": "synthetic",
        "config": {**workload_config(s, units), "parallelism": f"replicas x{world}",
                   "l2": "flushed (256 MB write) before every timed step, outside its events",
                   "launch": "CUDA graph of one csa2_layer_stack call" if graph is not None else "eager"},
        "step_hbm_gbs": round(step_gbs, 1), "step_frac_of_peak": round(step_gbs / hbm_peak, 4),
        "algorithmic_bytes_per_step": step_bytes,
        "roofline": roofline, "kernels": kernels, "e2e": e2e, "cpu_baseline": cpu,
        "gpu_launches": n_launch * K, "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(res), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def time_alone(args, torch, fn, flush, stream, n):
    """Mean device time (ms) of fn(stream_ptr) over n calls, each after an L2 flush,
    timed with CUDA events on `stream` (a CUDA graph of one call unless --eager)."""
    g = None if args.eager else capture_graph(torch, fn)
    sptr = int(stream.cuda_stream)
    evs = []
    for i in range(n + 3):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        if g is not None:
            g.replay()
        else:
            rc = fn(sptr)
            if rc:
                raise RuntimeError(f"kernel timing call failed: {rc}")
        b.record(stream)
        if i >= 3:
            evs.append((a, b))
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in evs)


def unique_rows(lists):
    """Distinct valid entries per sequence of a [B, Tq, n] list array, summed over sequences."""
    import numpy as np
    return sum(len(np.unique(l[l >= 0])) for l in lists)


def attn_call_bytes(spec, q_pos, local_base, topk):
    """Algorithmic bytes of one attention call: FP4 rows of the union of each sequence's
    lists, local K+V rows of the union of its windows, and per query its query, list
    and output."""
    import numpy as np
    D, Hq, W, B, Tq = spec.D, spec.Hq, spec.W, spec.B, spec.Tq
    total = unique_rows(topk) * (D // 2 + D // 16)
    if W > 0:
        for b in range(B):
            t = q_pos[b].astype(np.int64)
            lo = np.maximum(np.maximum(t - W + 1, int(local_base[b])), 0)
            total += _window_rows(lo, t) * 2 * D * 2
    return total + B * Tq * (topk.shape[-1] * 4 + 2 * Hq * D * 2)


def reindex_call_bytes(spec, pool, k):
    """Algorithmic bytes of one Reindex call: the key rows of each sequence's pool
    union, and per query its pool, index query and list."""
    return unique_rows(pool) * spec.Di + spec.B * spec.Tq * (pool.shape[-1] * 4 + spec.Hi * spec.Di + k * 4)


def kernel_breakdown(args, torch, np, ops, capi, s, layers, q_pos, codes, scales, base, qp_host, base_host, ws, st,
                     flush, stream, hbm_peak, bf16_peak, int8_peak):
    """Each kernel class of one step, timed alone through the public calls on the
    step's own tensors: the Full-mode indexer, the Reindex indexer, and attention for
    a Full, a Reuse and a Reindex layer. Per class: ms per launch, launches per step,
    share of the serial sum, algorithmic bytes per launch and GB/s against peak."""
    modes = [L.mode for L in s.layers]
    n_launch = {"FULL": modes.count("FULL"), "REINDEX": modes.count("REINDEX"), "REUSE": modes.count("REUSE")}
    li_f = modes.index("FULL")
    Lf = s.layers[li_f]
    d0 = layers[li_f]
    n = args.kernel_launches
    out = []

    def entry(cls, kernel, ms, count, nbytes, ops=0, ops_peak=None, ops_kind=None):
        gbs = nbytes / (ms * 1e-3) / 1e9
        e = {"class": cls, "kernel": kernel, "ms": round(ms, 5), "launches_per_step": count,
             "algorithmic_bytes": int(nbytes), "gbs": round(gbs, 1), "frac": round(gbs / hbm_peak, 4)}
        if ops and ops_peak:
            tops = ops / (ms * 1e-3) / 1e12
            e.update({"tensor_ops": int(ops), "tensor_kind": ops_kind, "tensor_tops": round(tops, 2),
                      "tensor_peak_tops": round(ops_peak, 1), "tensor_frac": round(tops / ops_peak, 4)})
        out.append(e)

    w_host = np.ascontiguousarray(np.asarray(d0["w"], dtype=np.int32))
    pool_t = torch.empty((s.B, s.Tq, max(Lf.P, 1)), dtype=torch.int32, device="cuda")
    topk_t = torch.empty((s.B, s.Tq, Lf.k), dtype=torch.int32, device="cuda")
    ia = ops.make_index_args(capi.CSA2_FULL, q_pos, d0["qi"], w_host, d0["ki"], Lf.k, Lf.P, None,
                             pool_t if Lf.P else None, topk_t, s.m)
    buf = ws.get(capi.csa2_workspace_bytes(0, ia))
    fcall = lambda sp: capi.csa2_index_topk(ia, int(buf.data_ptr()), buf.numel(), st.ptr, sp)
    ms = time_alone(args, torch, fcall, flush, stream, n)
    st.check("Full indexer timing")
    kname = index_kernel_name(s, "FULL")
    # the contraction the scan performs, counted over the causal pairs only: 2 * Hi * Di per (query, key)
    int8_ops = 2 * s.Hi * s.Di * sum(entries_read(s, int(t)) for t in qp_host.reshape(-1))
    entry("full_index", kname, ms, n_launch["FULL"], full_launch_bytes(s, qp_host), int8_ops, int8_peak, "int8")
    topk_h = topk_t.cpu().numpy()

    def attn_entry(cls, li, topk_dev, topk_host, count):
        d = layers[li]
        o = torch.empty_like(d["q"])
        lse = torch.empty(d["q"].shape[:-1], dtype=torch.float32, device="cuda")
        aa = ops.make_attn_args(q_pos, d["q"], codes, scales, topk_dev, d["kl"], d["vl"], base, s.W, o, lse, s.m)
        abuf = ws.get(capi.csa2_workspace_bytes(1, aa))
        acall = lambda sp: capi.csa2_sparse_attn(aa, int(abuf.data_ptr()), abuf.numel(), st.ptr, sp)
        t = time_alone(args, torch, acall, flush, stream, n)
        st.check(f"attention timing ({cls})")
        HQP = 16 if s.Hq <= 16 else 32
        # S = K Q^T and O = P V over the query's union: 4 * Hq * D flops per (query, entry)
        n_ent = int((topk_host >= 0).sum())
        if s.W > 0:
            t_all = qp_host.reshape(-1).astype(np.int64)
            lo = np.maximum(np.maximum(t_all - s.W + 1, np.repeat(base_host.astype(np.int64), s.Tq)), 0)
            n_ent += int(np.maximum(t_all - lo + 1, 0).sum())
        flops = 4 * s.Hq * s.D * n_ent
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        entry(cls, attn_kernel_name(s, HQP, int(topk_dev.shape[-1]), sms), t, count,
              attn_call_bytes(s, qp_host, base_host, topk_host),
              flops, bf16_peak, "bf16")

    attn_entry("attn_full", li_f, topk_t, topk_h, n_launch["FULL"])
    if n_launch["REUSE"]:
        attn_entry("attn_reuse", modes.index("REUSE"), topk_t, topk_h, n_launch["REUSE"])
    if n_launch["REINDEX"]:
        li_r = modes.index("REINDEX")
        d = layers[li_r]
        Lr = s.layers[li_r]
        wr = np.ascontiguousarray(np.asarray(d["w"], dtype=np.int32))
        topk_r = torch.empty((s.B, s.Tq, Lr.k), dtype=torch.int32, device="cuda")
        ra = ops.make_index_args(capi.CSA2_REINDEX, q_pos, d["qi"], wr, d["ki"], Lr.k, 0, pool_t, None, topk_r, s.m)
        rbuf = ws.get(capi.csa2_workspace_bytes(0, ra))
        rcall = lambda sp: capi.csa2_index_topk(ra, int(rbuf.data_ptr()), rbuf.numel(), st.ptr, sp)
        ms = time_alone(args, torch, rcall, flush, stream, n)
        st.check("Reindex timing")
        entry("reindex_index", index_kernel_name(s, "REINDEX"), ms, n_launch["REINDEX"], reindex_call_bytes(s, pool_t.cpu().numpy(), Lr.k))
        attn_entry("attn_reindex", li_r, topk_r, topk_r.cpu().numpy(), n_launch["REINDEX"])
    tot = sum(kc["ms"] * kc["launches_per_step"] for kc in out)
    for kc in out:
        kc["share"] = round(kc["ms"] * kc["launches_per_step"] / tot, 4) if tot > 0 else 0.0
    return out


def index_kernel_name(s, mode):
    """The kernel(s) csa2_index_topk launches for this workload's shapes (the library's
    dispatch rules, restated for the report)."""
    if mode == "FULL":
        if s.Tq >= 4 and s.N >= 8192 and s.Hi <= 8 and s.Di in (32, 64, 128):
            return (f"index_mq_score_kernel<{s.Di}> (sample, mark) + index_mq_estimate_kernel + "
                    f"index_mq_select_kernel<{s.Di}> + index_full_tc_kernel<{s.Di}> (queries left over)")
        if s.Di in (32, 64, 128):
            return f"index_full_tc_kernel<{s.Di}>"
    if s.Hi <= 8 and s.Di == 64:
        return "index_dp4a_kernel<8,64>"
    if s.Hi <= 4 and s.Di == 32:
        return "index_dp4a_kernel<4,32>"
    return "index_dp4a_kernel<0,0>"


def attn_kernel_name(s, HQP, k, sms):
    """The kernel csa2_sparse_attn launches (the library's dispatch rule, restated): one CTA
    per query over all of its tiles for calls of at least two queries per SM; else the
    cluster kernel while its cluster (one CTA per 256 list entries, one per 128 window rows)
    holds at most 16 CTAs and, at 16 heads, the call's clusters hold at most 4 CTAs per SM;
    else the ticket kernel."""
    if s.B * s.Tq >= 2 * sms:
        return f"sparse_attn_seq_kernel<{HQP},{s.D}>"
    cs = -(-k // 256) + -(-s.W // 128)
    many = s.Hq <= 16 and s.B * s.Tq * cs > 4 * sms
    if 1 <= cs <= 16 and s.B * s.Tq <= 65535 and not many:
        return f"sparse_attn_cl_kernel<{HQP},{s.D}>"
    return f"sparse_attn_kernel<{HQP},{s.D}>"


def run_e2e(args, torch, np, ops, capi, stack, layers, q_pos, s, flush, stream, st, graph, cache):
    """Per step: copy the step's per-query inputs (main queries of every layer, index
    queries of Full/Reindex layers, query positions) from pinned host memory, run the
    stack, and copy every layer's output and lse back to pinned host memory. The
    inputs sit in one device buffer and the outputs in another, as a caller would lay
    out a decode step, so each direction is one copy."""
    codes, scales, base = cache
    src = [q_pos] + [d["q"] for d in layers] + [d["qi"] for d in layers if d["mode"] != "REUSE"]
    din, views = ops.packed_views([(tuple(t.shape), t.dtype) for t in src], q_pos.device)
    for v, t in zip(views, src):
        v.copy_(t)
    it = iter(views[1:])
    layers2 = [dict(d) for d in layers]
    for d in layers2:
        d["q"] = next(it)
    for d in layers2:
        if d["mode"] != "REUSE":
            d["qi"] = next(it)
    stack2 = ops.LayerStack(layers2, views[0], codes, scales, base, packed_outputs=True, m=s.m)
    host_in = din.cpu().pin_memory()
    host_out = torch.empty_like(stack2.out_buf, device="cpu").pin_memory()
    h2d = din.numel()                 # bytes of the one input copy (tensors + alignment gaps)
    d2h = stack2.out_buf.numel()      # bytes of the one output copy
    dev_in, host_in, dev_out, host_out = [din], [host_in], [stack2.out_buf], [host_out]
    ws = ops.Workspace()
    buf = ws.get(stack2.ws_bytes)
    sptr = int(stream.cuda_stream)

    def call(stream_ptr):
        return stack2.run_raw(int(buf.data_ptr()), buf.numel(), st.ptr, stream_ptr)

    g2 = None if graph is None else capture_graph(torch, call)
    K = max(10, args.steps // 5)
    evs = []
    for i in range(K + 3):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for d, h in zip(dev_in, host_in):
            d.copy_(h, non_blocking=True)
        if g2 is not None:
            g2.replay()
        else:
            capi.check(call(sptr), "e2e step")
        for h, d in zip(host_out, dev_out):
            h.copy_(d, non_blocking=True)
        b.record(stream)
        if i >= 3:
            evs.append((a, b))
    torch.cuda.synchronize()
    st.check("e2e")
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    units = s.B * s.Tq
    return {"value": round(units / (ms * 1e-3), 1), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 5), "steps": K}


# ------------------------------------------------------------------ CPU oracle
def cpu_baseline(workload: str, seconds: float, overrides=None):
    """The C++ oracle, as it stands, with std::threads over (sequence, query) units on
    the host's cores: batches of every sequence's queries through all layers of the
    workload (index and attention), until `seconds` have run (at least one batch).
    Also a one-thread figure on one decode_full query (one Full layer)."""
    import synth
    from oracle import cpp as C

    wl = synth.make_workload(workload, **(overrides or {}))
    s = wl.spec
    threads = C.host_threads()
    codes, scales = C.fp4_quantize(wl.kv_f32() if s.m <= 1 else C.compress_entries(wl.kv_f32(), s.m))     # quantising the cache is setup, not a decode step
    wl.drop("kv")
    for li in range(s.L):                             # draw every input before the clock starts
        wl.q(li), wl.kl(li), wl.vl(li)
        if s.layers[li].mode != "REUSE":
            wl.qi(li), wl.ki(s.layers[li].key_set)
    done, batches, t0 = 0, 0, time.perf_counter()
    while True:
        st = C.StackState(wl)
        for li in range(s.L):
            C.run_layer(st, li, codes, scales, threads)
        done += s.B * s.Tq
        batches += 1
        if time.perf_counter() - t0 >= seconds:
            break
    el = time.perf_counter() - t0
    # one thread, one decode_full query (B = 1): its Full layer's index and attention
    w1 = synth.make_workload("decode_full", B=1)
    c1, s1 = C.fp4_quantize(w1.kv_f32())
    w1.q(0), w1.kl(0), w1.vl(0), w1.qi(0), w1.ki(0)
    reps, t1 = 0, time.perf_counter()
    while True:
        C.run_layer(C.StackState(w1), 0, c1, s1, threads=1)
        reps += 1
        if time.perf_counter() - t1 >= 2.0:
            break
    el1 = time.perf_counter() - t1
    return {"value": round(done / el, 4), "unit": UNIT, "cores": min(threads, s.B * s.Tq), "host_cores": threads,
            "kind": "oracle",
            "sample": f"{batches} batch(es) of all {s.B * s.Tq} queries through all {s.L} layers, index and attention "
                      f"(C++ oracle, {min(threads, s.B * s.Tq)} threads, {el:.1f} s)",
            "single_thread_decode_full_b1": {"value": round(reps / el1, 4), "unit": "queries/s", "cores": 1,
                                             "sample": f"{reps} query(ies) of decode_full B=1, one Full layer "
                                                       f"({el1:.1f} s)"}}


def run_reference(args, rank, world):
    """The oracle as the reference arm: the C++ oracle on the host's cores, each step
    one layer of the workload for every query (threads over the queries), cycling
    through the layer schedule; reported as whole-stack queries/s."""
    if rank != 0:
        return
    import synth
    from oracle import cpp as C

    wl = synth.make_workload(args.workload, **args.overrides)
    s = wl.spec
    threads = C.host_threads()
    codes, scales = C.fp4_quantize(wl.kv_f32() if s.m <= 1 else C.compress_entries(wl.kv_f32(), s.m))
    wl.drop("kv")
    state = {"st": C.StackState(wl)}

    def layer_step(i):
        li = i % s.L
        if li == 0:
            state["st"] = C.StackState(wl)
        C.run_layer(state["st"], li, codes, scales, threads)

    for i in range(args.warmup):
        layer_step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        layer_step(args.warmup + i)
    el = time.perf_counter() - t0
    value = args.steps / s.L * s.B * s.Tq / el
    cores = min(threads, s.B * s.Tq)
    res = {"metric": metric_of(s), "value": round(value, 4), "unit": UNIT, "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "int64+f64", "data": "synthetic", "impl": "reference",
           "config": {**workload_config(s, s.B * s.Tq), "parallelism": "CPU oracle on rank 0"},
           "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": cores, "host_cores": threads,
                            "kind": "oracle",
                            "sample": f"{args.steps} layer-steps, each one layer for all {s.B * s.Tq} queries "
                                      f"(C++ oracle, {cores} threads)"},
           "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


# ------------------------------------------------------------------ phase trace
PHASES = {
    "full_index": {1: "dependency wait", 2: "scan done", 22: "candidates listed (shared-key cut)",
                   23: "candidates scored (shared-key cut)", 24: "threshold (shared-key cut)",
                   25: "lists written (shared-key cut)",
                   3: "histograms exchanged", 4: "threshold bins",
                   5: "ordered lists", 7: "candidates exchanged", 8: "finalise", 12: "candidates loaded",
                   13: "thresholds, counts", 9: "write", 10: "lists written", 11: "end"},
    "reindex_index": {1: "dependency wait", 2: "scores done", 3: "scores published", 4: "all scores loaded",
                      5: "candidates", 6: "threshold", 7: "offsets", 11: "end"},
    "attention": {1: "dependency wait", 2: "positions", 3: "rows staged", 4: "tile ready", 5: "S done",
                  6: "softmax done", 7: "O done", 8: "partials exchanged", 9: "end"},
    "attention_seq": {1: "first tile staged", 2: "first S done", 3: "first softmax done", 4: "first O done",
                      5: "first tile done", 6: "last tile staged", 7: "last S done", 8: "last softmax done",
                      9: "last O done", 10: "last tile done", 11: "end"},
}
KINDS = {1: "index_full_tc_kernel", 2: "index_dp4a_kernel", 3: "sparse_attn_cl_kernel", 4: "sparse_attn_kernel",
         5: "index_mq_score_kernel", 6: "sparse_attn_seq_kernel", 7: "index_mq_select_kernel"}


def run_phase_trace(args):
    """The phase-trace build: per kernel class, one launch alone after an L2 flush with the
    median and 90th percentile over CTAs of the SM-clock time from the CTA's start to each
    phase boundary; then every launch of one CUDA-graph replay of the whole stack with its
    first CTA start, last CTA end and the gap to the launch before (global timer)."""
    import numpy as np
    import torch

    import synth
    from sparse_attention_shared_b200 import capi, ops

    assert capi.trace_library()
    L = capi.lib()
    wl = synth.make_workload(args.workload, **args.overrides)
    s = wl.spec
    stack, layers, q_pos, codes, scales, base = build_device_stack(wl, torch, ops, np)
    ws, st = ops.Workspace(), ops.Status()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    ncta, cap = 1 << 16, 1 << 17
    slots = torch.zeros((ncta, 32), dtype=torch.int64, device="cuda")
    tl = torch.zeros((cap, 4), dtype=torch.int64, device="cuda")
    ctr = torch.zeros((4,), dtype=torch.int32, device="cuda")
    sp = int(torch.cuda.current_stream().cuda_stream)
    clock_ghz = 1.965   # SM clocks are converted at the B200's boost clock (the bench line records the clocks seen)

    def set_all(on_slots, on_tl):
        for f in (L.csa2_trace_set_idx, L.csa2_trace_set_attn):
            capi.check(f(slots.data_ptr(), ncta, 1 if on_slots else 0, tl.data_ptr() if on_tl else None,
                         ctr.data_ptr(), cap), "trace buffers")

    modes = [x.mode for x in s.layers]
    li_f = modes.index("FULL")
    d0, Lf = layers[li_f], s.layers[li_f]
    pool_t = torch.empty((s.B, s.Tq, max(Lf.P, 1)), dtype=torch.int32, device="cuda")
    topk_t = torch.empty((s.B, s.Tq, Lf.k), dtype=torch.int32, device="cuda")
    ia = ops.make_index_args(capi.CSA2_FULL, q_pos, d0["qi"], np.ascontiguousarray(np.asarray(d0["w"], np.int32)),
                             d0["ki"], Lf.k, Lf.P, None, pool_t if Lf.P else None, topk_t, s.m)
    ibuf = ws.get(capi.csa2_workspace_bytes(0, ia))
    calls = [("full_index", lambda: capi.csa2_index_topk(ia, ibuf.data_ptr(), ibuf.numel(), st.ptr, sp))]
    if "REINDEX" in modes:
        li_r = modes.index("REINDEX")
        dr, Lr = layers[li_r], s.layers[li_r]
        topk_r = torch.empty((s.B, s.Tq, Lr.k), dtype=torch.int32, device="cuda")
        ra = ops.make_index_args(capi.CSA2_REINDEX, q_pos, dr["qi"], np.ascontiguousarray(np.asarray(dr["w"], np.int32)),
                                 dr["ki"], Lr.k, 0, pool_t, None, topk_r, s.m)
        rbuf = ws.get(capi.csa2_workspace_bytes(0, ra))
        calls.append(("reindex_index", lambda: capi.csa2_index_topk(ra, rbuf.data_ptr(), rbuf.numel(), st.ptr, sp)))
    da = layers[modes.index("REUSE") if "REUSE" in modes else li_f]
    o = torch.empty_like(da["q"])
    lse = torch.empty(da["q"].shape[:-1], dtype=torch.float32, device="cuda")
    aa = ops.make_attn_args(q_pos, da["q"], codes, scales, topk_t, da["kl"], da["vl"], base, s.W, o, lse, s.m)
    abuf = ws.get(capi.csa2_workspace_bytes(1, aa))
    calls.append(("attention", lambda: capi.csa2_sparse_attn(aa, abuf.data_ptr(), abuf.numel(), st.ptr, sp)))

    print(f"phase trace, workload {s.name} (B={s.B}, N={s.N}, Tq={s.Tq}); times in us from each CTA's start")
    for name, fn in calls:
        for _ in range(3):
            capi.check(fn(), name)
        torch.cuda.synchronize()
        slots.zero_()
        ctr.zero_()
        set_all(True, True)
        flush.zero_()
        torch.cuda.synchronize()
        capi.check(fn(), name)
        torch.cuda.synchronize()
        set_all(False, False)
        h = slots.cpu().numpy()
        n = min(int(ctr[0].item()), cap)
        t = tl[:n].cpu().numpy()
        used = np.nonzero(h[:, 31])[0]
        span = (t[:, 3].max() - t[:, 2].min()) / 1e3 if n else 0.0
        print(f"{name}: {len(used)} CTAs traced, launch span {span:.1f} us")
        table = PHASES[name]
        if name == "attention" and s.B * s.Tq >= 2 * torch.cuda.get_device_properties(0).multi_processor_count:
            table = PHASES["attention_seq"]
        for k, label in sorted(table.items(),
                               key=lambda kv: np.median(h[used, kv[0]]) if len(used) else 0):
            v = h[used, k]
            v = v[v > 0]
            if len(v):
                print(f"  {label:22s} median {np.median(v) / clock_ghz / 1e3:8.2f}  p90 {np.percentile(v, 90) / clock_ghz / 1e3:8.2f}")
        for k in (16, 17):
            v = h[used, k]
            v = v[v > 0]
            if len(v):
                print(f"  candidates (track {k - 16}) median {int(np.median(v))}")
    st.check("phase trace")

    wsb = ws.get(stack.ws_bytes)
    g = capture_graph(torch, lambda sp2: stack.run_raw(int(wsb.data_ptr()), wsb.numel(), st.ptr, sp2))
    for _ in range(5):
        flush.zero_()
        g.replay()
    torch.cuda.synchronize()
    ctr.zero_()
    set_all(False, True)
    flush.zero_()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    set_all(False, False)
    n = min(int(ctr[0].item()), cap)
    t = tl[:n].cpu().numpy()
    t = t[np.argsort(t[:, 2], kind="stable")]
    t0 = t[:, 2].min()
    launches = []
    for kind in np.unique(t[:, 0]):
        cur, seen = [], set()
        for r in t[t[:, 0] == kind]:   # a launch ends where a CTA index repeats
            if int(r[1]) in seen:
                launches.append(np.array(cur))
                cur, seen = [], set()
            cur.append(r)
            seen.add(int(r[1]))
        if cur:
            launches.append(np.array(cur))
    launches.sort(key=lambda a: a[:, 2].min())
    print(f"step timeline (one graph replay, {len(launches)} launches)")
    prev = None
    for a in launches:
        st0, en = (a[:, 2].min() - t0) / 1e3, (a[:, 3].max() - t0) / 1e3
        gap = "" if prev is None else f"  end - previous end {en - prev:6.1f}"
        print(f"  {KINDS.get(int(a[0, 0]), a[0, 0]):22s} CTAs {len(a):5d} start {st0:8.1f} end {en:8.1f}{gap}")
        prev = en
    st.check("phase trace timeline")


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.phase_trace:
        run_phase_trace(args)
        return
    run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
