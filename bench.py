"""Benchmark of the decode-time KV-cache eviction round.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload random_serving|beacon_serving|long_trace|ragged_c2|...]
                    [--extras beacon_serving,long_trace,ragged_c2] [--extra-steps K2]
                    [--requests R] [--layers L] [--no-cpu-baseline] [--no-cpu-pool] [--no-e2e]

A step is one eviction round (kvc_update_beacons + kvc_compress for the
beacon selector, kvc_compress for the random ones) over every (request,
layer, KV head) segment of the workload, with the cache already resident in
HBM.  Between steps the serving loop appends the next 64-token trigger window
to every request (untimed), so each round sees the steady state of the
Random Attention article's serving setup ("发现四": K=2048, 1k-token prompt,
128 requests, compression every 64 tokens).

Printed (rank 0, one JSON line): head-positions compressed per second over the
K timed rounds (device time, CUDA events on the library's stream; max over
ranks for N > 1), the roofline of the dominant kernel and of every kernel of
the round, the CPU oracle timed on bounded samples on one host core
(cpu_baseline) and on all of them (cpu_baseline_all_cores), an end-to-end
figure through the C ABI with the trigger window's K/V (and queries) read
from page-locked host memory every step, and the clocks sampled during the
timed region.  The headline workload is the random serving round; the
BeaconKV serving round, the long-trace compression and the ragged sweep's
2x slice follow with fewer rounds each, under extra_workloads, each with its
own phases, rooflines, clocks and CPU baselines.

Multi-GPU: one process per GPU (torchrun), each rank an independent replica
with its own requests (the round has no exchange step: weak scaling, no
collective on the data path; the barrier and the max-reduction of the timing
are the only collectives).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KV head-positions compressed/s per eviction round"
UNIT = "head-positions/s"
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="random_serving")
    ap.add_argument("--selector", default=None, help="override the workload's selector")
    ap.add_argument("--requests", type=int, default=None)
    ap.add_argument("--layers", type=int, default=None)
    ap.add_argument("--beacons", type=int, default=None, help="override the workload's beacon count")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-cpu-pool", action="store_true",
                    help="skip timing the oracle over all host cores (one spawned process per core)")
    ap.add_argument("--extras", default="beacon_serving,long_trace,ragged_c2",
                    help="comma-separated workloads also timed (fewer rounds) after the headline one and "
                         "reported under extra_workloads; '' for none")
    ap.add_argument("--extra-steps", type=int, default=8, help="timed rounds of each extra workload")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--score-impl", type=int, default=0, help="beacon score kernel: 0 auto, 1 SIMT, 2 tcgen05")
    ap.add_argument("--compaction", default="ordered", choices=["ordered", "hole_fill"],
                    help="round option: order-preserving or hole-filling compaction")
    ap.add_argument("--block", type=int, default=1, help="round option: positions per Philox draw")
    ap.add_argument("--sinks", type=int, default=None, help="round option: protect only this many sinks")
    ap.add_argument("--phase", default="round", choices=["round", "attention"],
                    help="round: the eviction round; attention: one decode step of attention over the "
                         "compacted cache (all layers)")
    ap.add_argument("--q-heads", type=int, default=32, help="query heads for --phase attention")
    return ap.parse_args()


def load_workloads():
    """The seeded workload generators (workloads.py), loaded by path so that the
    reference arm does not load libkvc.so."""
    import importlib.util
    path = os.path.join(ROOT, "decode_kv_cache_paged_b200", "workloads.py")
    spec = importlib.util.spec_from_file_location("kvc_workloads", path)
    mod = importlib.util.module_from_spec(spec)
    sys.modules["kvc_workloads"] = mod
    spec.loader.exec_module(mod)
    return mod


def make_workload(args):
    wl = load_workloads()
    name = args.workload
    if name == "random_serving":
        w = wl.random_serving()
    elif name == "beacon_serving":
        w = wl.beacon_serving()
    elif name == "long_trace":
        w = wl.long_trace()
    elif name.startswith("ragged_c"):
        w = wl.scaled(wl.ragged(int(name[len("ragged_c"):])), num_layers=12)
    else:
        raise SystemExit(f"unknown workload {name}")
    kw = {}
    if args.requests:
        kw["num_requests"] = args.requests
    if args.layers:
        kw["num_layers"] = args.layers
    if getattr(args, "beacons", None):
        kw["num_beacons"] = args.beacons
    if kw:
        w = wl.scaled(w, **kw)
    sel = args.selector or w.selectors[0]
    if sel not in ("beacon", "beacon_trigger") and w.num_beacons:
        w = wl.scaled(w, num_beacons=0, query_window=0, num_q_heads=w.num_kv_heads)
    return w, sel


# ---------------------------------------------------------------- clocks --

class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 50 ms."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_id: str):
        self.rows = []
        self.proc = None
        self.idx = device_id

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([x.strip() for x in line.split(",")])

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in self.rows:
            try:
                sm.append(float(r[0]))
                mx = float(r[1])
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, r[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- roofline --

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "decode_kv_cache_paged_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str, units: float):
    """DRAM bytes per launch from the committed ncu summary, scaled to `units`
    (moved rows or keys); None if the kernel changed since the capture."""
    if not os.path.exists(PROFILE_TRAFFIC):
        return None
    with open(PROFILE_TRAFFIC) as f:
        d = json.load(f)
    e = d.get(kernel, {}).get(workload)
    if not e or e.get("source_hash") != kernel_source_hash(e["sources"]):
        return None
    return e["dram_bytes_per_unit"] * units


def score_roofline(flops: float, nbytes: float, ms: float, peaks: dict, tensor_cores: bool,
                   recompute_flops: float = 0.0) -> dict:
    """Roofline entry of the beacon score kernel.

    flops is the method's work: one product of 2*d flops per (beacon, cached
    key) pair.  The two-pass log-sum-exp computes the candidates' products a
    second time; those recompute_flops are reported beside it but are not
    algorithmic work, so they show up as a lower fraction.  The kernel is timed
    on its own by CUDA events around its launch, so the tensor peak is the
    burst figure.  The tcgen05 kernel is HBM-bound when its flops per
    algorithmic byte fall below the ridge (tensor peak / HBM peak),
    tensor-bound otherwise.  The SIMT kernel is held against the fp32 pipe:
    148 SMs x 128 lanes x 2 flop x the max SM clock."""
    sec = ms / 1e3
    extra = {"algorithmic_flops_per_launch": flops, "recompute_flops_per_launch": recompute_flops,
             "executed_tflops": (flops + recompute_flops) / sec / 1e12, "flop_per_byte": flops / nbytes,
             "algorithmic_bytes_per_launch": nbytes, "launch_ms": ms}
    if tensor_cores:
        tpeak = peaks.get("bf16_tflops")
        ridge = tpeak * 1e12 / (peaks["hbm_gbs"] * 1e9)
        hbm = {"hbm_gbs": nbytes / sec / 1e9, "hbm_frac": nbytes / sec / 1e9 / peaks["hbm_gbs"]}
        ten = {"tflops": flops / sec / 1e12, "tensor_frac": flops / sec / 1e12 / tpeak, "tensor_peak": tpeak,
               "peak_kind": "burst", "ridge_flop_per_byte": ridge}
        if flops / nbytes < ridge:
            out = {"kernel": "beacon_score_tc", "bound": "hbm", "achieved": nbytes / sec / 1e9,
                   "peak": peaks["hbm_gbs"], "unit": "GB/s"}
        else:
            out = {"kernel": "beacon_score_tc", "bound": "tensor", "achieved": flops / sec / 1e12, "peak": tpeak,
                   "unit": "TFLOP/s"}
        out.update(hbm)
        out.update(ten)
    else:
        simt_peak = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
        out = {"kernel": "beacon_score_simt", "bound": "alu", "achieved": flops / sec / 1e12, "peak": simt_peak,
               "unit": "TFLOP/s", "hbm_gbs": nbytes / sec / 1e9}
    out.update(extra)
    return out


def update_roofline(w, ms: float, peaks: dict, tensor_cores: bool) -> dict:
    """Roofline entry of the beacon update: per segment the window's points
    (W steps x G query heads x d) are read once, and the fp32 beacons are read
    and written, their scoring copy written and the counts and trigger shares
    read and written once.  HBM-bound by its bytes (a few flops per byte)."""
    es = 2 if w.dtype == "bf16" else 4
    B, d = w.num_beacons, w.head_dim
    per_seg = w.query_window * w.G * d * es + B * d * (4 + 4 + es) + B * (4 + 4 + 4)
    nbytes = w.segments * per_seg
    sec = ms / 1e3
    return {"kernel": "beacon_update_tc" if tensor_cores else "beacon_update_simt", "bound": "hbm",
            "achieved": nbytes / sec / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": nbytes / sec / 1e9 / peaks["hbm_gbs"], "algorithmic_bytes_per_launch": nbytes,
            "launch_ms": ms, "traffic": None}


# ------------------------------------------------------------ our arm ---

def aggregate(local_ms: float, units_per_rank: float, steps: int, world: int, dist, device=None):
    """Whole-job throughput: units all ranks processed / the slowest rank's time."""
    total_ms = local_ms
    if dist is not None and world > 1:
        import torch
        t = torch.tensor([local_ms], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    return world * units_per_rank * steps / (total_ms / 1e3), total_ms


class Refill:
    """Brings every request back to its pre-round length between rounds
    (untimed): the next 64-token trigger window for the serving workloads
    (drawn once and reused), freshly drawn tokens for the others."""

    def __init__(self, ctx, w, gen):
        import numpy as np
        self.ctx, self.w, self.gen = ctx, w, gen
        self.np = np
        self.window = None
        if len(set(w.length.tolist())) == 1 and len(set(w.budget.tolist())) == 1 and \
                int(w.length[0]) - max(int(w.budget[0]), int(w.prompt[0])) == w.trigger:
            R = w.num_requests
            k, v = gen.kv(R, w.trigger)
            q = gen.queries(R, w.trigger) if w.query_window else None
            self.window = (np.arange(R, dtype=np.int32), k, v, q)

    def __call__(self):
        np, w, ctx = self.np, self.w, self.ctx
        if self.window is not None:
            ln, _ = ctx.lengths()
            if np.all(ln + w.trigger == w.length):
                ctx.append(*self.window)
                return
        ln, _ = ctx.lengths()
        need = w.length - ln
        groups = {}
        for r in range(w.num_requests):
            if need[r] > 0:
                groups.setdefault(int(need[r]), []).append(r)
        for T_all, reqs in groups.items():
            ids = np.array(reqs, np.int32)
            done = 0
            q_from = T_all - min(w.query_window, T_all) if w.query_window else T_all
            while done < T_all:
                T = min(256 if done < q_from else 16, (q_from if done < q_from else T_all) - done)
                k, v = self.gen.kv(len(ids), T)
                q = self.gen.queries(len(ids), T) if done >= q_from else None
                ctx.append(ids, k, v, q)
                done += T

def round_rooflines(w, sel, stats, upd_ms, peaks, args) -> dict:
    """Roofline entries of every kernel of the round, from the timed rounds'
    own counters: select_compact always, the score and update kernels under
    the beacon selectors."""
    beacon = sel in ("beacon", "beacon_trigger")
    variant = [] if args.compaction == "ordered" else [args.compaction]
    variant += [f"block{args.block}"] if args.block != 1 else []
    variant += [f"sinks{args.sinks}"] if args.sinks is not None else []
    traffic_key = "/".join([w.name] + variant)
    sc_ms = statistics.mean(s["ms_select_compact"] for s in stats)
    moved = statistics.mean(s["moved_rows"] for s in stats)
    cands = statistics.mean(s["candidates"] for s in stats)
    es = 2 if w.dtype == "bf16" else 4
    rb = w.head_dim * es
    # select+compact: K and V rows read and written once per moved row, the moved
    # position entries read and written, every candidate's 4-byte key source read
    sc_bytes = moved * (4 * rb + 8) + cands * 4
    peak_src = "MEASURED_PEAKS.json" if peaks.get("_kind") == "measured" else "recipe fallback"
    out = {"select_compact": {
        "kernel": "select_compact", "bound": "hbm", "achieved": sc_bytes / (sc_ms / 1e3) / 1e9,
        "peak": peaks["hbm_gbs"], "unit": "GB/s", "traffic": profiled_traffic("select_compact", traffic_key, moved),
        "algorithmic_bytes_per_launch": sc_bytes, "launch_ms": sc_ms, "moved_rows": moved, "candidates": cands}}
    if beacon:
        score_ms = statistics.mean(s["ms_score"] for s in stats)
        key_bytes = statistics.mean(s["key_bytes_scored"] for s in stats)
        keys = key_bytes / rb
        B = w.num_beacons
        flops = 2.0 * B * w.head_dim * keys          # one product per (beacon, cached key) pair
        recompute = 2.0 * B * w.head_dim * cands     # pass 2 recomputes the candidates' products
        score_bytes = key_bytes + cands * 4 + w.segments * B * rb
        tc = stats[-1].get("score_kernel", 0) == 2
        roof = score_roofline(flops, score_bytes, score_ms, peaks, tc, recompute)
        roof["traffic"] = profiled_traffic(roof["kernel"], w.name, keys)
        out["score"] = roof
        upd = statistics.mean(upd_ms)
        out["update"] = update_roofline(w, upd, peaks, w.dtype == "bf16" and w.head_dim == 128)
    for r in out.values():
        r["frac"] = r["achieved"] / r["peak"] if r.get("peak") else None
        r["peak_source"] = f"{peaks.get('_kind')} ({peak_src})"
    return out


def run_ours(args, rank, world, dist, with_e2e=True):
    """One workload: fill, W warm-up rounds, K timed rounds (device time of
    kvc_update_beacons + kvc_compress on the library's stream), the rooflines
    of the round's kernels and, for the serving workloads, the end-to-end
    figure.  Returns (JSON dict, workload, selector)."""
    import numpy as np
    import torch

    from decode_kv_cache_paged_b200 import workloads as wl
    from decode_kv_cache_paged_b200 import Context, ContextSpec

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w, sel = make_workload(args)
    w.data_seed += 7 * rank  # independent replicas
    headroom = max(0, int(max(w.budget.max(), w.prompt.max()) + w.trigger - w.length.max()))
    spec = ContextSpec(num_requests=w.num_requests, num_layers=w.num_layers, num_kv_heads=w.num_kv_heads,
                       head_dim=w.head_dim, max_seq_len=w.max_seq_len(headroom),
                       num_pages=w.pages_needed(headroom) + w.num_requests,
                       num_q_heads=w.num_q_heads or w.num_kv_heads, num_beacons=w.num_beacons,
                       query_window=w.query_window)
    ctx = Context(spec, dtype=wl.torch_dtype(w.dtype), device=dev)
    if sel in ("beacon", "beacon_trigger") and args.score_impl:
        ctx.set_option(0, args.score_impl)
    gen = wl.Generator(w, dev)
    wl.fill(ctx, w, gen)
    budgets = w.budget.astype(np.int32)
    R = w.num_requests
    ids = np.arange(R, dtype=np.int32)
    beacon = sel in ("beacon", "beacon_trigger")
    T = w.trigger
    refill = Refill(ctx, w, gen)

    opts = {"sink_tokens": args.sinks, "block": args.block, "compaction": args.compaction}

    def one_round(seed, timed):
        ev0 = torch.cuda.Event(enable_timing=True)
        ev_mid = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        ev0.record(ctx.stream)
        if beacon:
            ctx.update_beacons()
        ev_mid.record(ctx.stream)
        st = ctx.compress(sel, budgets, seed, stats=timed, **opts)
        ev1.record(ctx.stream)
        return ev0, ev_mid, ev1, st

    # the first compress brings the cache from its filled length to the budget;
    # from then on every round sees L = K + trigger
    for i in range(args.warmup):
        if beacon:
            ctx.update_beacons()
        ctx.compress(sel, budgets, w.philox_seed, **opts)
        refill()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    clock = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    clock.start()
    torch.cuda.synchronize()
    t_wall = time.perf_counter()
    rounds = []
    for i in range(args.steps):
        rounds.append(one_round(w.philox_seed, True))
        refill()  # untimed: back to the pre-round lengths
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    wall = time.perf_counter() - t_wall
    clocks = clock.stop()
    ms = [a.elapsed_time(c) for a, _, c, _ in rounds]
    upd = [a.elapsed_time(b) for a, b, _, _ in rounds]
    stats = [s for _, _, _, s in rounds]
    head_pos = stats[-1]["head_positions"]
    value, total_ms = aggregate(sum(ms), head_pos, args.steps, world, dist, dev)

    # rooflines of the round's kernels; the dominant (longest) one is the line's roofline
    peaks, peak_kind = measured_peaks()
    peaks = dict(peaks, _kind=peak_kind)
    roofs = round_rooflines(w, sel, stats, upd, peaks, args)
    dominant = max(roofs, key=lambda k: roofs[k]["launch_ms"])
    roof = dict(roofs[dominant])

    # end to end through the public API, every step: the next trigger window's
    # K/V (and queries) copied H2D from page-locked host memory on a second
    # stream while the round runs, the round, the new lengths read back, then
    # the window appended from device memory once both are done
    e2e = None
    if with_e2e and not args.no_e2e and refill.window is not None:
        _, k_win, v_win, q_win = refill.window
        k_h = k_win.cpu().pin_memory()
        v_h = v_win.cpu().pin_memory()
        q_h = q_win.cpu().pin_memory() if q_win is not None else None
        k_d, v_d = torch.empty_like(k_win), torch.empty_like(v_win)
        q_d = torch.empty_like(q_win) if q_win is not None else None
        len_h = torch.empty(R, dtype=torch.int32).pin_memory()
        lens_dev = ctx.state_tensors()["lengths"]
        side = torch.cuda.Stream(dev)
        h2d = k_h.numel() * k_h.element_size() * 2 + (q_h.numel() * q_h.element_size() if q_h is not None else 0)
        times = []
        for i in range(args.e2e_steps + 1):
            torch.cuda.synchronize()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            copied = torch.cuda.Event()
            a.record(ctx.stream)
            side.wait_event(a)
            with torch.cuda.stream(side):
                k_d.copy_(k_h, non_blocking=True)
                v_d.copy_(v_h, non_blocking=True)
                if q_h is not None:
                    q_d.copy_(q_h, non_blocking=True)
                copied.record(side)
            if beacon:
                ctx.update_beacons()
            ctx.compress(sel, budgets, w.philox_seed, **opts)
            with torch.cuda.stream(ctx.stream):
                len_h.copy_(lens_dev, non_blocking=True)
            ctx.stream.wait_event(copied)
            ctx.append(ids, k_d, v_d, q_d)
            b.record(ctx.stream)
            b.synchronize()
            if i > 0:
                times.append(a.elapsed_time(b))
        e2e_value, e2e_ms = aggregate(statistics.mean(times), head_pos, 1, world, dist, dev)
        e2e = {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(R * 4), "ms_per_step": e2e_ms,
               "what": "per step: the next trigger window's K/V(/queries) copied H2D from page-locked host "
                       "memory on a second stream, overlapped with kvc_compress (+kvc_update_beacons); the new "
                       "lengths D2H; the window appended from device memory through kvc_append"}
    ctx.sync()
    ctx.close()
    del ctx, refill, gen
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    launches = sum(s["launches"] for s in stats) + (args.steps if beacon else 0)
    ragged = len(set(w.length.tolist())) > 1
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "f32 (bf16 x bf16 scores)" if beacon else "u32",
        "data": "synthetic (seeded N(0,1) K/V with 4 outlier channels x8; vMF-mixture queries)",
        "config": {"workload": w.name, "selector": sel, "requests_per_gpu": R, "layers": w.num_layers,
                   "kv_heads": w.num_kv_heads, "head_dim": w.head_dim, "cache_dtype": w.dtype,
                   "prompt": int(w.prompt[0]) if len(set(w.prompt.tolist())) == 1 else "ragged",
                   "budget": int(w.budget[0]) if len(set(w.budget.tolist())) == 1 else "ragged",
                   "trigger": T, "beacons": w.num_beacons, "page_size": 16,
                   "compaction": args.compaction, "block": args.block,
                   "sinks": "whole prompt" if args.sinks is None else args.sinks,
                   "head_positions_per_round_per_gpu": head_pos,
                   "parallelism": f"replicas x{world} (no collective on the data path)",
                   "l2": "inputs larger than L2: the cache is tens of GB vs 126 MB L2, and each "
                         "refill between rounds writes >1 GB",
                   **({"layer_slice": f"{w.num_layers} of 36 layers (K+V of all 36 would be ~174 GB); "
                                      "segments are independent"} if ragged else {})},
        "roofline": roof,
        "rooflines": roofs,
        "moved_rows_per_round": [int(s["moved_rows"]) for s in stats],
        "phases_ms": {"update": statistics.mean(upd) if beacon else 0.0,
                      "score": statistics.mean(s["ms_score"] for s in stats),
                      "select_compact": statistics.mean(s["ms_select_compact"] for s in stats)},
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
        "wall_s_timed_region": wall,
    }
    return out, w, sel


# ---------------------------------------------------- attention phase ---

ATTN_METRIC = "cached head-positions attended/s per decode step"


def attention_workload(args):
    w, _ = make_workload(args)
    wl = load_workloads()
    if args.q_heads % w.num_kv_heads:
        raise SystemExit("--q-heads must be a multiple of the KV heads")
    return wl.scaled(w, num_beacons=0, query_window=0, num_q_heads=args.q_heads)


def run_attention(args, rank, world, dist):
    """One decode step of attention over every layer of the cache right after
    an eviction round (lengths at the budget K), per timed step."""
    import numpy as np
    import torch

    from decode_kv_cache_paged_b200 import workloads as wl
    from decode_kv_cache_paged_b200 import Context, ContextSpec

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = attention_workload(args)
    w.data_seed += 7 * rank
    spec = ContextSpec(num_requests=w.num_requests, num_layers=w.num_layers, num_kv_heads=w.num_kv_heads,
                       head_dim=w.head_dim, max_seq_len=w.max_seq_len(0),
                       num_pages=w.pages_needed(0) + w.num_requests, num_q_heads=w.num_q_heads,
                       num_beacons=0, query_window=0)
    ctx = Context(spec, dtype=wl.torch_dtype(w.dtype), device=dev)
    gen = wl.Generator(w, dev)
    wl.fill(ctx, w, gen, with_queries=False)
    ctx.compress("random", w.budget.astype(np.int32), w.philox_seed)
    lengths, _ = ctx.lengths()
    positions = int(lengths.sum()) * w.num_layers * w.num_kv_heads
    g = torch.Generator(device=dev).manual_seed(1 + rank)
    q = torch.randn((w.num_layers, w.num_requests, w.num_q_heads, w.head_dim), generator=g, device=dev)
    q = q.to(ctx.dtype)
    out = torch.empty((w.num_layers, w.num_requests, w.num_q_heads, w.head_dim), dtype=torch.float32, device=dev)
    lse = torch.empty((w.num_layers, w.num_requests, w.num_q_heads), dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        ctx.decode_attention(q, out=out, lse=lse)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    clock = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    clock.start()
    evs = []
    for _ in range(args.steps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(ctx.stream)
        ctx.decode_attention(q, out=out, lse=lse)
        b.record(ctx.stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = clock.stop()
    ms = [a.elapsed_time(b) for a, b in evs]
    value, total_ms = aggregate(sum(ms), positions, args.steps, world, dist, dev)
    peaks, peak_kind = measured_peaks()
    rb = w.head_dim * (2 if w.dtype == "bf16" else 4)
    io_bytes = q.numel() * q.element_size() + out.numel() * 4 + lse.numel() * 4
    alg_bytes = positions * rb * 2 + io_bytes
    mean_ms = statistics.mean(ms)
    roof = {"kernel": "decode_attention", "bound": "hbm", "achieved": alg_bytes / (mean_ms / 1e3) / 1e9,
            "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "traffic": profiled_traffic("decode_attention", w.name + "/decode_attention", positions),
            "peak_source": f"{peak_kind} ({'MEASURED_PEAKS.json' if peak_kind == 'measured' else 'recipe fallback'})",
            "algorithmic_bytes_per_launch": alg_bytes, "launch_ms": mean_ms}
    roof["frac"] = roof["achieved"] / roof["peak"]
    e2e = None
    if not args.no_e2e:
        # a serving pipeline over n steps, every byte inside the timed span: the
        # queries of step i+1 go H2D on one side stream and the outputs of step
        # i-1 go D2H on another while step i computes (2 buffers each)
        q_h = q.cpu().pin_memory()
        out_h = [torch.empty(out.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
        q_d = [torch.empty_like(q) for _ in range(2)]
        o_d = [torch.empty_like(out) for _ in range(2)]
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        n = max(2, args.e2e_steps)
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(ctx.stream)
        up.wait_event(a)
        landed = [torch.cuda.Event(), torch.cuda.Event()]
        done = [torch.cuda.Event(), torch.cuda.Event()]
        drained = [None, None]
        with torch.cuda.stream(up):
            q_d[0].copy_(q_h, non_blocking=True)
            landed[0].record(up)
        for i in range(n):
            cur, nxt = i % 2, (i + 1) % 2
            if i + 1 < n:
                with torch.cuda.stream(up):
                    if i >= 1:
                        up.wait_event(done[nxt])  # step i-1 has finished reading q_d[nxt]
                    q_d[nxt].copy_(q_h, non_blocking=True)
                    landed[nxt].record(up)
            ctx.stream.wait_event(landed[cur])
            if drained[cur] is not None:
                ctx.stream.wait_event(drained[cur])  # o_d[cur] has been copied out
            ctx.decode_attention(q_d[cur], out=o_d[cur], lse=lse)
            done[cur].record(ctx.stream)
            with torch.cuda.stream(down):
                down.wait_event(done[cur])
                out_h[cur].copy_(o_d[cur], non_blocking=True)
                drained[cur] = torch.cuda.Event()
                drained[cur].record(down)
        ctx.stream.wait_event(drained[(n - 1) % 2])
        b.record(ctx.stream)
        b.synchronize()
        e2e_value, e2e_ms = aggregate(a.elapsed_time(b) / n, positions, 1, world, dist, dev)
        e2e = {"value": e2e_value, "unit": "head-positions/s", "h2d_bytes_per_step": int(q_h.numel() * q_h.element_size()),
               "d2h_bytes_per_step": int(out_h[0].numel() * 4), "ms_per_step": e2e_ms,
               "what": f"{n} pipelined steps, timed from the first H2D to the last D2H: each step's queries H2D "
                       "from page-locked memory, kvc_decode_attention over all layers, outputs D2H; the copies "
                       "of neighbouring steps overlap the compute on side streams"}
    # the library's split rule: a merge kernel runs when a call splits the rows
    base = w.num_layers * w.num_requests * w.num_kv_heads
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    np_max = (int(lengths.max()) + 15) // 16
    nsplit = max(1, min(-(-4 * sms // base), 16 // w.num_layers, -(-np_max // 8))) if np_max else 1
    if nsplit > 1:
        pps = ((-(-np_max // nsplit)) + 3) & ~3
        nsplit = max(1, -(-np_max // pps))
    nsplit_launches = 2 if nsplit > 1 else 1
    ctx.sync()
    out_line = {
        "metric": ATTN_METRIC, "value": value, "unit": "head-positions/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32 (bf16 K/V and queries)" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded N(0,1) K/V with 4 outlier channels x8; N(0,1) queries)",
        "config": {"workload": w.name + "/decode_attention", "requests_per_gpu": w.num_requests,
                   "layers": w.num_layers, "kv_heads": w.num_kv_heads, "q_heads": w.num_q_heads,
                   "head_dim": w.head_dim, "cache_dtype": w.dtype, "rows_per_segment": int(lengths.max()),
                   "parallelism": f"replicas x{world} (no collective on the data path)",
                   "l2": "inputs larger than L2: every step reads all K and V rows (tens of GB)"},
        "roofline": roof, "e2e": e2e, "gpu_launches": args.steps * nsplit_launches, "clocks": clocks,
    }
    return out_line, w, lengths


def oracle_attention_rate(w, lengths, budget_s: float):
    """The oracle's decode attention on whole (layer, request) units until
    ~budget_s of oracle time; head-positions/s."""
    import numpy as np

    import oracle
    rng = np.random.default_rng(4321)
    d, H, Hq = w.head_dim, w.num_kv_heads, w.num_q_heads
    t_total, hp, n = 0.0, 0, 0
    while t_total < budget_s:
        L = int(lengths[int(rng.integers(len(lengths)))])
        k = rng.standard_normal((H, L, d))
        v = rng.standard_normal((H, L, d))
        q = rng.standard_normal((Hq, d))
        t0 = time.perf_counter()
        oracle.decode_attention_gqa(q, k, v)
        t_total += time.perf_counter() - t0
        hp += L * H
        n += 1
    return hp / t_total, (f"{n} (layer, request) units of the workload's shape ({H} KV heads, {Hq} query heads, "
                          f"rows = the post-round lengths), oracle float64, one thread, {t_total:.1f} s")


# ------------------------------------------------------- oracle timing ---

def oracle_sample_rate(w, sel, budget_s: float, rank_seed: int = 0, seg_offset: int = 0):
    """Times the oracle (single thread) on whole segments of the workload until
    ~budget_s seconds of oracle time; returns (head_positions/s, description)."""
    import numpy as np

    import oracle
    rng = np.random.default_rng(1234 + rank_seed)
    d = w.head_dim
    es = 2 if w.dtype == "bf16" else 4
    t_total = 0.0
    hp = 0
    n_seg = 0
    H, Ly = w.num_kv_heads, w.num_layers
    segs = [(r, l, h) for r in range(w.num_requests) for l in range(Ly) for h in range(H)]
    segs = segs[seg_offset % len(segs):] + segs[:seg_offset % len(segs)]
    cache = {}
    while t_total < budget_s and n_seg < len(segs):
        r, l, h = segs[n_seg]
        L, P, K = int(w.length[r]), int(w.prompt[r]), int(w.budget[r])
        key = (L, P)
        if key not in cache:
            rows_k = rng.integers(0, 255, (L, d * es), dtype=np.uint8)
            rows_v = rng.integers(0, 255, (L, d * es), dtype=np.uint8)
            keys = rng.standard_normal((L, d)) if sel.startswith("beacon") else None
            pts = rng.standard_normal((w.query_window * w.G, d)) if sel.startswith("beacon") else None
            cache[key] = (rows_k, rows_v, keys, pts)
        rows_k, rows_v, keys, pts = cache[key]
        pos = np.arange(L, dtype=np.int32)
        t0 = time.perf_counter()
        if sel == "beacon":
            c, cnt, _ = oracle.beacon_update(pts, np.zeros((w.num_beacons, d)), np.zeros(w.num_beacons), init=True)
            kept, _ = oracle.beacon_round_segment(keys, P, K, oracle.round_bf16(c) if w.dtype == "bf16" else c)
        elif sel == "beacon_trigger":
            c, cnt, _ = oracle.beacon_update(pts, np.zeros((w.num_beacons, d)), np.zeros(w.num_beacons), init=True)
            sc = oracle.beacon_trigger_score(keys, oracle.round_bf16(c) if w.dtype == "bf16" else c, cnt, P)
            kept = oracle.beacon_select_with_pos(sc.astype(np.float32), pos, P, K)
        else:
            kept, _ = oracle.random_round_segment(w.philox_seed, 0, r, l, h, sel == "random_shared", P, K, pos)
        oracle.compact_rows(rows_k, P, kept[P:])
        oracle.compact_rows(rows_v, P, kept[P:])
        t_total += time.perf_counter() - t0
        hp += L
        n_seg += 1
    desc = (f"{n_seg} whole segments (requests from 0, all layers and heads in order) of {w.name}, "
            f"selector {sel}: score + full-sort select + K/V compaction, {t_total:.1f} s of oracle time")
    return hp / t_total, desc, n_seg


def _pool_worker(job):
    """One host core of the all-cores oracle figure (run in a spawned process)."""
    name, requests, layers, beacons, selector, budget_s, offset = job
    import types
    args = types.SimpleNamespace(workload=name, requests=requests, layers=layers, beacons=beacons, selector=selector)
    w, sel = make_workload(args)
    t0 = time.perf_counter()
    rate, _, n_seg = oracle_sample_rate(w, sel, budget_s, rank_seed=offset, seg_offset=offset)
    return rate * min(budget_s, time.perf_counter() - t0), n_seg, time.perf_counter() - t0


def oracle_pool_rate(args, budget_s: float):
    """The same oracle over all host cores: one single-threaded process per
    core, each on its own run of whole segments; head-positions/s summed over
    the processes, divided by the longest process time."""
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor
    cores = len(os.sched_getaffinity(0))
    w, sel = make_workload(args)
    n_segs = w.num_requests * w.num_layers * w.num_kv_heads
    jobs = [(args.workload, args.requests, args.layers, getattr(args, "beacons", None), sel, budget_s,
             (i * n_segs) // cores)
            for i in range(cores)]
    # spawn (never fork after CUDA is initialised); a worker that dies raises
    # instead of leaving the pool waiting
    with ProcessPoolExecutor(max_workers=cores, mp_context=mp.get_context("spawn")) as ex:
        res = list(ex.map(_pool_worker, jobs, timeout=budget_s * 10 + 120))
    hp = sum(r[0] for r in res)
    wall = max(r[2] for r in res)
    return hp / wall, cores, (f"{sum(r[1] for r in res)} whole segments of {w.name} over {cores} processes "
                              f"(one per host core), each ~{budget_s:.0f} s of oracle time")


def add_cpu_baselines(out, args, w, sel, single_s: float, pool_s: float, pool: bool):
    """The oracle on one host core (cpu_baseline) and, unless disabled, on
    every host core (cpu_baseline_all_cores), on bounded samples of the same
    workload."""
    rate, desc, _ = oracle_sample_rate(w, sel, single_s)
    out["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc}
    if pool:
        xa = argparse.Namespace(**vars(args))
        xa.selector = sel
        prate, cores, pdesc = oracle_pool_rate(xa, pool_s)
        out["cpu_baseline_all_cores"] = {"value": prate, "unit": UNIT, "cores": cores, "kind": "oracle",
                                         "sample": pdesc}


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle as it stands, on the host cores."""
    if args.phase == "attention":
        import numpy as np
        w = attention_workload(args)
        lengths = np.where(w.length <= w.budget, w.length, np.maximum(w.prompt, w.budget))
        per_step = max(2.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
        oracle_attention_rate(w, lengths, per_step / 4 * args.warmup)
        rates, desc = [], ""
        for _ in range(args.steps):
            rate, desc = oracle_attention_rate(w, lengths, per_step)
            rates.append(rate)
        value = statistics.mean(rates)
        positions = int(lengths.sum()) * w.num_layers * w.num_kv_heads
        return {
            "impl": "reference", "metric": ATTN_METRIC, "value": value, "unit": "head-positions/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": positions / value * 1e3,
            "ms_per_step_kind": "extrapolated from the oracle's rate on the sampled units",
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name + "/decode_attention"},
            "cpu_baseline": {"value": value, "unit": "head-positions/s", "cores": 1, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "head-positions/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
    w, sel = make_workload(args)
    per_step = max(2.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample_rate(w, sel, per_step / 4)
    rates = []
    desc = ""
    for s in range(args.steps):
        rate, desc, _ = oracle_sample_rate(w, sel, per_step, rank_seed=s)
        rates.append(rate)
    value = statistics.mean(rates)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": w.head_positions / value * 1e3,
        "ms_per_step_kind": "extrapolated: one whole round's head-positions divided by the oracle's rate on the "
                            "sampled segments (a whole round would take this long; each timed step is a bounded "
                            "sample)",
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": w.name, "selector": sel},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return
    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    try:
        if args.phase == "attention":
            out, w, lengths = run_attention(args, rank, world, dist)
            if rank == 0:
                if not args.no_cpu_baseline:
                    rate, desc = oracle_attention_rate(w, lengths, 12.0)
                    out["cpu_baseline"] = {"value": rate, "unit": "head-positions/s", "cores": 1, "kind": "oracle",
                                           "sample": desc}
                print(json.dumps(out), flush=True)
            return
        out, w, sel = run_ours(args, rank, world, dist)
        if rank == 0 and not args.no_cpu_baseline:
            add_cpu_baselines(out, args, w, sel, 12.0, 10.0, pool=not args.no_cpu_pool)
        # the other workloads, fewer rounds each, under extra keys of the same line
        extras = [x for x in args.extras.split(",") if x and x != args.workload] if args.phase == "round" else []
        if extras:
            out["extra_workloads"] = {}
        for name in extras:
            xa = argparse.Namespace(**vars(args))
            xa.workload, xa.selector, xa.requests, xa.layers = name, None, None, None
            xa.steps, xa.warmup = max(2, args.extra_steps), max(3, min(args.warmup, 3))
            xo, xw, xsel = run_ours(xa, rank, world, dist, with_e2e=False)
            if rank == 0 and not args.no_cpu_baseline:
                add_cpu_baselines(xo, xa, xw, xsel, 6.0, 6.0, pool=not args.no_cpu_pool)
            for k in ("metric", "unit", "n_gpus", "higher_is_better", "scaling", "vs_baseline", "data", "e2e"):
                xo.pop(k, None)
            out["extra_workloads"][name] = xo
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if dist:
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
