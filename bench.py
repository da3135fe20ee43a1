"""Benchmark of the MoE-layer hot path on B200.

Workload (default): the 35B-A3B-shaped decode — 48 MoE layer positions sharing
one layer's parameters (H=2048, E=128, top-8, I=768, NVFP4 experts), a global
HBM slot pool holding 25% of the 6144 (layer, expert) blocks, the rest streamed
from pinned host memory, Zipf(1.1)-skewed routing.  A step is one decode step
of T tokens through all 48 layers: route -> LRU slot lookup -> miss streaming on
the copy engine -> FP4 expert FFN -> combine, per layer.

Printed (rank 0, one JSON line): decode tokens/s (device-timed, inputs resident);
e2e tokens/s through DecodeLayer with x uploaded from pinned host memory and y
read back every step; the decode FFN kernel's HBM roofline, measured on an
all-resident pool over the same layers; the copy engine's H2D GB/s; hit rate;
the oracle timed on a bounded sample of host cores; SM clocks during the timed
region.  `--impl reference` times the oracle alone on the same workload.
Multi-GPU: independent replicas, one per rank (the layer does not shard);
timing is the max over ranks.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synthetic import gen, workloads as W  # noqa: E402

METRIC = json.load(open(os.path.join(ROOT, "BASELINE.json")))["metric"] \
    if os.path.exists(os.path.join(ROOT, "BASELINE.json")) else "MoE decode tokens/s"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], "measured"
    return 6650.0, 1590.0, "fallback"


# ----------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index, self.proc, self.lines = index, None, []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.index)], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
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
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [v.strip() for v in ln.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx.append(float(f[1]))
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "samples": len(sm),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------------- inputs

def make_pool(m, w, n_slots, T, host_layers, experts):
    pool = m.Pool(w.H, w.I, w.E, w.k, w.L, w.fmt, n_slots, max_tokens=T, host_layers=host_layers)
    for hl in range(pool.host_layers):
        for e in range(w.E):
            pool.load_expert(hl, e, experts[e])
    return pool


def preload(torch, m, pool, w):
    """Make every (layer, expert) resident: one lookup of all E experts per layer
    (k distinct per row) and its miss streaming."""
    idx = torch.arange(w.E, dtype=torch.int32, device="cuda").view(-1, w.k)
    slot_of = torch.empty_like(idx)
    cs = torch.cuda.Stream()
    for l in range(w.L):
        res = m.slot_lookup(pool, l, idx, slot_of)
        m.stream_misses(pool, l, res, cs)
    cs.synchronize()


def ffn_roofline(torch, m, w, pool, T, x_dev, wr, bias, reps=4):
    """Time the decode FFN kernel alone: route and look up all L layers first (all
    resident, so every expert is a hit), then enqueue reps*L FFN launches back to
    back behind a device-side sleep (so the host's launch latency stays outside the
    window) between two CUDA events on the launching stream."""
    L_ = w.L
    idx = torch.empty((L_, T, w.k), dtype=torch.int32, device="cuda")
    wt = torch.empty((L_, T, w.k), dtype=torch.float32, device="cuda")
    slot_of = torch.empty((L_, T, w.k), dtype=torch.int32, device="cuda")
    y_part = torch.empty((T, w.k, w.H), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.zeros(m.route_workspace_bytes(T, w.E), dtype=torch.uint8, device="cuda")
    uniq = []
    for l in range(L_):
        m.route(x_dev[l], wr, bias, w.k, 1, idx[l], wt[l], ws)
        res = m.slot_lookup(pool, l, idx[l], slot_of[l])
        assert res.n_miss == 0, "roofline pass expects an all-resident pool"
        uniq.append(res.n_uniq)
    for l in range(L_):     # warm-up
        m.expert_ffn(pool, l, x_dev[l], idx[l], wt[l], slot_of[l], y_part, status)
    torch.cuda.synchronize()
    cur = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(20_000_000)
    e0.record(cur)
    for r in range(reps):
        for l in range(L_):
            m.expert_ffn(pool, l, x_dev[l], idx[l], wt[l], slot_of[l], y_part, status)
    e1.record(cur)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ms = e0.elapsed_time(e1) / (reps * L_)
    return ms, uniq


def expert_bytes_alg(w):
    """Algorithmic HBM bytes of one expert: FP4 codes + block scales of gate, up, down."""
    bs = W.block_elems(w.fmt)
    return 3 * (w.H * w.I // 2 + w.H * w.I // bs)


# ---------------------------------------------------------------- decode runs

def decode_run(torch, m, w, pool, T, xs_dev, wr, bias, steps, warmup, events=False, overlap=True):
    """Times `steps` decode steps (all L layers each) on the current stream."""
    lo = m.DecodeLayer(pool, T, overlap=overlap)
    cur = torch.cuda.current_stream()
    for s in range(warmup):
        for l in range(w.L):
            lo(l, xs_dev[s % xs_dev.shape[0], l], wr, bias)
    torch.cuda.synchronize()
    st0 = pool.stats()
    if events:
        lo.ffn_events, lo.copy_events = [], []
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    for s in range(steps):
        for l in range(w.L):
            lo(l, xs_dev[(warmup + s) % xs_dev.shape[0], l], wr, bias)
    e1.record(cur)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    st1 = pool.stats()
    d = {k: st1[k] - st0[k] for k in st1}
    out = dict(ms=ms, stats=d, status=int(lo.status.item()))
    if events:
        out["ffn"] = [(a.elapsed_time(b), u, mm) for (a, b), u, mm in lo.ffn_events]
        out["copy"] = [(a.elapsed_time(b), n) for (a, b), n in lo.copy_events]
    return out


def e2e_run(torch, m, w, pool, T, xs_host, wr, bias, steps, warmup, overlap=True):
    """Through DecodeLayer with x copied in from pinned host memory and every
    layer's y read back to pinned host memory, each step."""
    lo = m.DecodeLayer(pool, T, overlap=overlap)
    cur = torch.cuda.current_stream()
    nbuf = xs_host.shape[0]
    x_dev = torch.empty(xs_host.shape[1:], dtype=torch.bfloat16, device="cuda")
    y_dev = torch.empty((w.L, T, w.H), dtype=torch.bfloat16, device="cuda")
    y_host = torch.empty((w.L, T, w.H), dtype=torch.bfloat16, pin_memory=True)

    def step(s):
        x_dev.copy_(xs_host[s % nbuf], non_blocking=True)
        for l in range(w.L):
            y_dev[l].copy_(lo(l, x_dev[l], wr, bias))
        y_host.copy_(y_dev, non_blocking=True)

    for s in range(warmup):
        step(s)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    for s in range(steps):
        step(warmup + s)
    e1.record(cur)
    torch.cuda.synchronize()
    return dict(ms=e0.elapsed_time(e1), h2d=x_dev.numel() * 2, d2h=y_host.numel() * 2)


# ------------------------------------------------------------------- CPU oracle

def oracle_sample(w, T, experts, budget_s=10.0, min_layers=2):
    """The oracle (single thread) on a bounded sample of the workload: routing,
    LRU and the FFN of the chosen experts for consecutive (step, layer) pairs
    until budget_s of oracle time has passed; tokens/s extrapolated to all L
    layers (input generation is not timed)."""
    import oracle
    lru = oracle.LRU(W.n_slots(w), w.L, w.E)
    wr = gen.router_weight(w, 0)
    b = gen.router_bias(w, 0)
    busy, n = 0.0, 0
    while busy < budget_s or n < min_layers:
        s, l = divmod(n, w.L)
        x = gen.activations(w, l, s, T)
        ta = time.perf_counter()
        idx, wt, _ = oracle.route(x, wr, b, w.k, 1)
        lru.step(l, idx)
        oracle.moe_decode(w.fmt, w.H, w.I, w.E, x, idx, wt,
                          {e: experts[e] for e in set(idx.ravel().tolist())})
        busy += time.perf_counter() - ta
        n += 1
    per_layer = busy / n
    return dict(value=T / (per_layer * w.L), unit="tokens/s", cores=1, kind="oracle",
                sample=f"{n} (step, layer) evaluations of routing + LRU + FFN at T={T}, "
                       f"{busy:.1f} s on one host core, extrapolated to {w.L} layers")


def ffn_only(args, w, T):
    """The decode FFN kernel alone on `args.layers` all-resident layer positions."""
    from dataclasses import replace
    wl = replace(w, L=args.layers)
    experts = gen.expert_weights_many(wl, 0, range(wl.E))
    import torch
    import expert_offload_fp4_b200 as m
    pool = make_pool(m, wl, wl.L * wl.E, 8, 1, experts)
    preload(torch, m, pool, wl)
    xs = np.stack([gen.activations(wl, l, 0, T) for l in range(wl.L)])
    x_dev = torch.from_numpy(xs.view(np.int16)).cuda().view(torch.bfloat16)
    wr = torch.from_numpy(gen.router_weight(wl, 0).view(np.int16)).cuda().view(torch.bfloat16)
    bias = torch.from_numpy(gen.router_bias(wl, 0)).cuda()
    ms, uniq = ffn_roofline(torch, m, wl, pool, T, x_dev, wr, bias, reps=2)
    phases = None
    if args.trace:
        buf = torch.zeros((148, 8), dtype=torch.int64, device="cuda")
        m._lib.load().moe_set_ffn_trace(buf.data_ptr())
        ffn_roofline(torch, m, wl, pool, T, x_dev, wr, bias, reps=1)
        m._lib.load().moe_set_ffn_trace(None)
        tr = buf.cpu().numpy().astype(np.float64)
        t0 = tr[:, 0].min()
        rel = (tr - t0) / 1000.0
        phases = {name: [round(float(np.median(rel[:, i])), 2), round(float(rel[:, i].max()), 2)]
                  for i, name in enumerate(["start", "table", "staged", "first_data", "a_done",
                                            "b_dep", "items_done", "end"])}
    pool.close()
    per = expert_bytes_alg(wl)
    alg = sum(u * per + T * wl.H * 2 + T * wl.k * wl.H * 4 for u in uniq) / len(uniq)
    print(json.dumps({"mode": "ffn", "workload": wl.name, "layers": wl.L, "batch": T,
                      "launch_ms_avg": round(ms, 5), "alg_bytes_per_launch": int(alg),
                      "achieved_gbs": round(alg / (ms * 1e-3) / 1e9, 1),
                      "phases_us_median_max": phases}), flush=True)


# ---------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=32)
    ap.add_argument("--warmup", type=int, default=4)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--batch", type=int, default=1, help="decode tokens per step (1, 4 or 8)")
    ap.add_argument("--all-batches", action="store_true", help="also time batches 4 and 8")
    ap.add_argument("--oracle-budget", type=float, default=10.0)
    ap.add_argument("--mode", default="decode", choices=["decode", "ffn"],
                    help="ffn: only the decode FFN kernel on a small all-resident pool "
                         "(a few layers), e.g. for an ncu capture")
    ap.add_argument("--layers", type=int, default=4, help="layer positions in --mode ffn")
    ap.add_argument("--trace", action="store_true", help="--mode ffn: per-CTA phase timestamps")
    ap.add_argument("--no-overlap", action="store_true",
                    help="issue miss copies before each FFN launch (for runs under ncu, which "
                         "serialises kernels)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = W.DECODE_35B
    T = args.batch

    if args.impl == "reference":
        if rank != 0:
            return
        experts = gen.expert_weights_many(w, 0, range(w.E))
        t0 = time.perf_counter()
        cb = oracle_sample(w, T, experts, budget_s=args.oracle_budget)
        el = time.perf_counter() - t0
        line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "tokens/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1000.0 * T / cb["value"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": w.name, "layers": w.L, "batch": T, "format": w.fmt},
                "cpu_baseline": cb,
                "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0},
                "wall_s": round(el, 2)}
        print(json.dumps(line), flush=True)
        return

    if args.mode == "ffn":
        return ffn_only(args, w, T)

    # inputs first (spawned generator workers), then CUDA
    experts = gen.expert_weights_many(w, 0, range(w.E))
    import torch
    torch.cuda.set_device(local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    import expert_offload_fp4_b200 as m
    m._lib.load()

    hbm_peak, _, peak_kind = peaks()
    nbuf = 16
    xs = np.stack([np.stack([gen.activations(w, l, s, 8) for l in range(w.L)]) for s in range(nbuf)])
    wr = torch.from_numpy(gen.router_weight(w, 0).view(np.int16)).cuda().view(torch.bfloat16)
    bias = torch.from_numpy(gen.router_bias(w, 0)).cuda()

    def dev_x(Tb):
        return torch.from_numpy(np.ascontiguousarray(xs[:, :, :Tb]).view(np.int16)).cuda().view(torch.bfloat16)

    host_layers = w.L if world == 1 else 12
    pool = make_pool(m, w, W.n_slots(w), 8, host_layers, experts)
    res = {}
    batches = [T] + ([b for b in (1, 4, 8) if b != T] if args.all_batches else [])
    sampler = ClockSampler(local)
    for b in batches:
        xd = dev_x(b)
        if b == T:
            if world > 1:
                torch.distributed.barrier()
            torch.cuda.synchronize()
            sampler.start()
            r = decode_run(torch, m, w, pool, b, xd, wr, bias, args.steps, args.warmup, events=True,
                           overlap=not args.no_overlap)
            clocks = sampler.stop()
        else:
            r = decode_run(torch, m, w, pool, b, xd, wr, bias, args.steps, args.warmup,
                           overlap=not args.no_overlap)
        res[b] = r
        del xd

    # e2e through the public call with host buffers
    xs_host = torch.from_numpy(np.ascontiguousarray(xs[:, :, :T]).view(np.int16)).view(torch.bfloat16).pin_memory()
    e2e = e2e_run(torch, m, w, pool, T, xs_host, wr, bias, args.steps, args.warmup,
                  overlap=not args.no_overlap)
    pool.close()

    # all-resident pool: the FFN kernel's own HBM roofline on the same layers
    rpool = make_pool(m, w, w.L * w.E, 8, 1, experts)
    preload(torch, m, rpool, w)
    xd = dev_x(T)
    ffn_ms, ffn_u = ffn_roofline(torch, m, w, rpool, T, xd[0], wr, bias)
    rpool.close()
    per_exp = expert_bytes_alg(w)
    alg_bytes = [u * per_exp + T * w.H * 2 + T * w.k * w.H * 4 for u in ffn_u]
    alg_avg = sum(alg_bytes) / len(alg_bytes)
    achieved = alg_avg / (ffn_ms * 1e-3) / 1e9

    # reduce over ranks: max time, summed tokens
    r = res[T]
    ms = r["ms"]
    if world > 1:
        t = torch.tensor([ms, e2e["ms"]], device="cuda", dtype=torch.float64)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms, e2e_ms = float(t[0]), float(t[1])
        torch.distributed.barrier()
    else:
        e2e_ms = e2e["ms"]
    tokens = T * args.steps * world
    value = tokens / (ms * 1e-3)
    st = r["stats"]
    copy_ms = sum(t for t, _ in r["copy"])
    h2d_gbs = st["h2d_bytes"] / (copy_ms * 1e-3) / 1e9 if copy_ms > 0 else None
    traffic = None
    prof = os.path.join(ROOT, "profiles", "ffn_decode_traffic.json")
    if os.path.exists(prof):
        traffic = json.load(open(prof)).get("dram_bytes_per_launch")

    if rank == 0:
        cb = oracle_sample(w, T, experts, budget_s=args.oracle_budget) if world == 1 else None
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": w.name, "layers": w.L, "batch": T, "format": w.fmt,
                       "slot_pool": f"{W.n_slots(w)} slots (25% of {w.L * w.E})",
                       "zipf_s": w.zipf_s, "parallelism": f"replicas x{world}",
                       "l2": "inputs larger than L2: ~1 GB of expert weights per step"},
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak,
                         "unit": "GB/s", "frac": round(achieved / hbm_peak, 4), "traffic": traffic,
                         "kernel": "ffn_decode_kernel", "peak_source": peak_kind,
                         "measured_on": "all-resident pool, same layers/inputs",
                         "launch_ms_avg": round(ffn_ms, 5),
                         "alg_bytes_per_launch_avg": int(alg_avg)},
            "e2e": {"value": round(tokens / (e2e_ms * 1e-3), 3), "unit": "tokens/s",
                    "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"]},
            "gpu_launches": 4 * w.L * args.steps,
            "clocks": clocks,
            "h2d_gbs": round(h2d_gbs, 2) if h2d_gbs else None,
            "h2d_bytes_per_step": st["h2d_bytes"] // args.steps,
            "hit_rate": round(st["hits"] / max(1, st["unique"]), 4),
            "misses_per_layer": round(st["misses"] / (args.steps * w.L), 3),
            "batches": {str(b): round(b * args.steps / (res[b]["ms"] * 1e-3), 3) for b in res},
            "status": r["status"],
        }
        if cb is not None:
            line["cpu_baseline"] = cb
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
