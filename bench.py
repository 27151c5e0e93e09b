"""Benchmark of the grouped-int4 routed-expert FFN layer on B200.

One step = one moe_expert_ffn call (router, on-device row map, fused gate+up+SiLU,
down projection, weighted scatter-add) over one batch of synthetic input.  Default
workload: batched decode, 32 tokens, hidden 6144, 256 experts of intermediate 2048,
top-8, skewed routing (16 hot experts get +3 on logits of variance 2).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Prints one JSON line (rank 0).  N > 1 (under torchrun): independent replicas, one per
GPU (the layer has no exchange step), weak scaling, time = max over ranks.

The line's headline is the chosen workload (default: batched decode).  At N = 1 it also
carries a "configs" object with every other workload of the specification, each timed
the same way (CUDA-graph replay between L2 flushes, device events; an end-to-end figure
through the public API with host buffers; the roofline of its dominant kernel):
  * MoE decode, 1 token, hidden 4096, 128 experts of 1536, top-8;
  * MoE prefill, 4096 tokens, hidden 6144, 256 experts of 2048, top-8;
  * the dense gq4_matvec sweep at batch 1 (4096x4096, 14336x4096, 4096x14336,
    151936x4096);
  * the single expert: gate+up+SiLU [2048][1024] and down [1024][2048] with f32 x.
(--configs none skips them.)
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from weight_only_int4_gq4_b200 import synth  # noqa: E402

L2_FLUSH_BYTES = 256 << 20
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")


def kernel_source_hash() -> str:
    """Hash of the kernel sources' code (comments and blank space left out), tying a
    stored traffic figure to the code it was measured on."""
    import re
    h = hashlib.sha256()
    d = os.path.join(ROOT, "weight_only_int4_gq4_b200", "csrc")
    for f in sorted(os.listdir(d)):
        with open(os.path.join(d, f), encoding="utf-8") as fh:
            code = fh.read()
        code = re.sub(r"/\*.*?\*/", " ", code, flags=re.S)
        code = re.sub(r"//[^\n]*", " ", code)
        code = " ".join(code.split())
        h.update(f.encode() + code.encode())
    return h.hexdigest()[:16]


# Nominal B200 figures the metric is also quoted against: HBM3e 8 TB/s, dense bf16
# tensor throughput 2.25 PFLOP/s.
NOMINAL_HBM_GBS = 8000.0
NOMINAL_BF16_TFLOPS = 2250.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


def roofline(bound, achieved, hbm, bf16, peak_kind):
    """Roofline entry of one kernel: the fraction of the measured peak (copy bandwidth or
    cuBLAS bf16) and of the nominal one (8 TB/s or 2.25 PFLOP/s)."""
    if bound == "tensor":
        r = {"bound": "tensor", "achieved": achieved, "peak": bf16, "unit": "TFLOP/s",
             "peak_nominal": NOMINAL_BF16_TFLOPS}
    else:
        r = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "peak_nominal": NOMINAL_HBM_GBS}
    r["frac"] = achieved / r["peak"]
    r["frac_nominal"] = achieved / r["peak_nominal"]
    r["peak_kind"] = peak_kind
    return r


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, smax, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = max(smax, float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_baseline(cfg: synth.MoEConfig, budget_s: float = 12.0, max_tokens: int = 16):
    """The oracle as it stands, on host cores, over a bounded sample of the workload's
    tokens (whole MoE layer per token: gate+up+SiLU and down of its K experts)."""
    import oracle
    lg, _ = cfg.logits()
    x = cfg.x()
    st, idx, wts, _ = oracle.route(lg, cfg.K)
    order = cfg.sample_tokens() if cfg.oracle_sample else np.arange(cfg.T)
    experts = {}
    done, elapsed = 0, 0.0
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    for t in order[:max_tokens]:
        need = [int(e) for e in idx[t]]
        for e in need:
            if e not in experts:
                experts[e] = (cfg.gate(e), cfg.up(e), cfg.down(e))
        # a compact stack holding only this token's experts (oracle takes stacked arrays)
        loc = {e: i for i, e in enumerate(need)}
        pg = np.stack([experts[e][0][0] for e in need]); sg = np.stack([experts[e][0][1] for e in need])
        pu = np.stack([experts[e][1][0] for e in need]); su = np.stack([experts[e][1][1] for e in need])
        pd = np.stack([experts[e][2][0] for e in need]); sd = np.stack([experts[e][2][1] for e in need])
        idx_l = np.zeros_like(idx)
        idx_l[t] = [loc[e] for e in need]
        t0 = time.perf_counter()
        oracle.moe_tokens(pg, sg, pu, su, pd, sd, cfg.H, cfg.F, x, idx_l, wts, np.array([t]))
        elapsed += time.perf_counter() - t0
        done += 1
        if elapsed >= budget_s:
            break
    # one token on a single thread as well (the oracle's loops are otherwise spread over
    # all host cores with OpenMP)
    t = int(order[0])
    need = [int(e) for e in idx[t]]
    pg = np.stack([experts[e][0][0] for e in need]); sg = np.stack([experts[e][0][1] for e in need])
    pu = np.stack([experts[e][1][0] for e in need]); su = np.stack([experts[e][1][1] for e in need])
    pd = np.stack([experts[e][2][0] for e in need]); sd = np.stack([experts[e][2][1] for e in need])
    idx_l = np.zeros_like(idx)
    idx_l[t] = np.arange(len(need))
    prev = oracle.set_threads(1)
    t0 = time.perf_counter()
    oracle.moe_tokens(pg, sg, pu, su, pd, sd, cfg.H, cfg.F, x, idx_l, wts, np.array([t]))
    single = time.perf_counter() - t0
    oracle.set_threads(prev)
    return {"value": done / elapsed, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{done} token(s) of {cfg.name}, whole layer per token (K={cfg.K} experts), "
                      f"{elapsed:.1f} s, fp64 plain C",
            "single_thread_tokens_per_s": 1.0 / single, "cpu_model": cpu_model()}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def per_matrix_bytes(O, I):
    """Packed nibbles plus f32 group scales of one [O][I] matrix."""
    return O * (I // 2) + O * (I // 64) * 4


def split_experts(cfg, cnt):
    """The experts moe_expert_ffn sends to the tensor-core kernels (at least
    GQ4_MOE_LARGE_MIN_ROWS rows, when T and the shapes allow) and to the decode kernels."""
    from weight_only_int4_gq4_b200 import gq4
    lim = gq4.MOE_LARGE_MIN_ROWS
    tc = cfg.T >= lim and cfg.H % 128 == 0 and cfg.F % 64 == 0
    large = (cnt >= lim) if tc else np.zeros(cnt.shape, bool)
    small = (cnt > 0) & ~large
    return {"tc": tc, "n_small": int(small.sum()), "rows_small": int(cnt[small].sum()),
            "n_large": int(large.sum()), "rows_large": int(cnt[large].sum())}


STAGES = ("route_rowmap", "gate_up_small", "gate_up_large", "down_small", "down_large")


def stage_work(cfg, sp):
    """Algorithmic HBM bytes and tensor-core FLOPs of each timed stage of one step:
    weights + scales of the experts the stage serves, the activations it must read once,
    the outputs it must write.  The row gather before the tensor-core gate+up is an
    implementation choice: its time is in the stage, its bytes are not."""
    H, F, T, n = cfg.H, cfg.F, cfg.T, cfg.T * cfg.K
    rs, rl = sp["rows_small"], sp["rows_large"]
    y_rmw = 2 * T * H * 4
    fs = rs / max(rs + rl, 1)
    w = {
        "route_rowmap": (T * cfg.E * 4 + n * 20 + cfg.E * 8, 0.0),
        "gate_up_small": (sp["n_small"] * 2 * per_matrix_bytes(F, H) + (T * H * 2 if rs else 0)
                          + rs * F * 2 + T * H * 4, 0.0),
        "gate_up_large": (sp["n_large"] * 2 * per_matrix_bytes(F, H) + (T * H * 2 if rl else 0)
                          + rl * F * 2, 2.0 * rl * 2 * F * H),
        "down_small": (sp["n_small"] * per_matrix_bytes(H, F) + rs * F * 2 + fs * y_rmw, 0.0),
        "down_large": (sp["n_large"] * per_matrix_bytes(H, F) + rl * F * 2 + (1 - fs) * y_rmw,
                       2.0 * rl * H * F),
    }
    return w


def stage_kernels(cfg, sp):
    if cfg.H % 256 == 0 and cfg.F % 256 == 0:
        few = "gq4_stream_kernel"  # TMA-fed decode kernel (whole four-group stages)
    else:
        few = "gq4_band_kernel" if min(cfg.T, 23 if sp["tc"] else cfg.T) >= 3 else "gq4_skinny_kernel"
    n = cfg.T * cfg.K
    route = "gq4_route_rowmap_small_kernel" if n <= 1024 else \
        "gq4_route_kernel + gq4_rowmap_{count,scan,fill}_kernel"
    return {"route_rowmap": route, "gate_up_small": f"{few}<MoeGateUp>",
            "gate_up_large": "gq4_gather_rows_kernel + gq4_tc_kernel<GateUp>",
            "down_small": f"{few}<MoeDown>", "down_large": "gq4_tc_kernel<Down>"}


def launches_per_step(cfg, sp):
    """Kernels of this library one moe_expert_ffn call launches (the status memset is a
    runtime memset, not counted)."""
    n = cfg.T * cfg.K
    return (1 if n <= 1024 else 4) + 2 + (3 if sp["tc"] else 0)


def max_over_ranks(values, world, device):
    """Each timing as the maximum over the replicas (one all-reduce of a few scalars; the
    layer itself exchanges nothing between GPUs)."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def job_tokens_per_s(world, tokens_per_replica, ms):
    """Whole-job throughput: every replica processes its own batch in the slowest
    replica's time."""
    return world * tokens_per_replica / (ms * 1e-3)


def run_reference(args, cfg, rank):
    if rank != 0:
        return
    import oracle  # noqa: F401
    per = []
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline(cfg, budget_s=0.0, max_tokens=1)
        if i >= args.warmup:
            per.append(1.0 / cb["value"])
    sec = float(np.mean(per))
    v = 1.0 / sec
    line = {"impl": "reference", "metric": "expert-FFN tokens/s (MoE layer, 1 B200)", "value": v,
            "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "E": cfg.E, "F": cfg.F, "K": cfg.K,
                       "step": "1 sampled token through the CPU oracle"},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cb["cores"], "kind": "oracle",
                             "sample": "1 token per step, whole layer (K experts), fp64 plain C"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def moe_run(cfg, args, dev, world, local, with_cpu):
    """Time one MoE workload: device-timed graph replays, the per-stage split, the
    end-to-end figure through the public API, and the dominant kernel's roofline.
    Returns the fields of its JSON entry."""
    import torch
    from weight_only_int4_gq4_b200 import gq4

    # ---- inputs resident in HBM (weights of all E experts, logits, x)
    def stack(fn):
        parts = [fn(e) for e in range(cfg.E)]
        return np.stack([a for a, _ in parts]), np.stack([b for _, b in parts])

    Wg = gq4.upload(*stack(cfg.gate))
    Wu = gq4.upload(*stack(cfg.up))
    Wd = gq4.upload(*stack(cfg.down))
    lg_h, _ = cfg.logits()
    x_h = cfg.x()
    logits = torch.from_numpy(lg_h).to(dev)
    x = torch.from_numpy(x_h.view(np.int16)).view(torch.bfloat16).to(dev)
    y = torch.empty(cfg.T, cfg.H, dtype=torch.float32, device=dev)
    ws = gq4.MoEWorkspace(cfg.T, cfg.E, cfg.K, cfg.H, cfg.F, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    NEV = gq4.MOE_STAGE_EVENTS

    def step(ev=None):
        gq4.moe_expert_ffn(Wg, Wu, Wd, logits, x, cfg.K, y=y, ws=ws, stage_events=ev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert ws.status() == 0
    cnt = ws.routing()["cnt"].cpu().numpy()[:cfg.E]
    split = split_experts(cfg, cnt)

    # ---- device-timed steps: one moe_expert_ffn call captured in a CUDA graph and
    # replayed, so the step's kernels run without host launch gaps, timed by events on the
    # launching stream around the replay; L2 flushed between steps, outside the events.
    # The stage split comes from a second graph of the same call with its stage events
    # (event nodes inside a graph cost a few microseconds each, so they stay out of the
    # timed step).
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(NEV)]
    for e in ev:  # torch creates the CUDA event lazily, at its first record
        e.record(stream)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    graph_st = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_st):
        step(ev)
    for _ in range(args.warmup):
        graph.replay()
        graph_st.replay()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    step_ms = np.zeros(args.steps)
    ta, tb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            ta.record(stream)
            graph.replay()
            tb.record(stream)
            tb.synchronize()
            step_ms[i] = ta.elapsed_time(tb)
    if world > 1:
        dist.barrier()
    ms = float(step_ms.mean())
    stage = np.zeros((args.steps, NEV - 1))
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        graph_st.replay()
        torch.cuda.synchronize()
        stage[i] = [ev[j].elapsed_time(ev[j + 1]) for j in range(NEV - 1)]
    del graph, graph_st

    # ---- end to end through the public API, host buffers (pinned), copies timed
    x_pin = torch.from_numpy(x_h.view(np.int16)).view(torch.bfloat16).pin_memory()
    lg_pin = torch.from_numpy(lg_h).pin_memory()
    y_pin = torch.empty(cfg.T, cfg.H, dtype=torch.float32).pin_memory()
    x_d = torch.empty_like(x)
    lg_d = torch.empty_like(logits)
    e2e_ms = []
    for i in range(args.warmup + args.steps):
        flush.fill_(i & 0xFF)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        x_d.copy_(x_pin, non_blocking=True)
        lg_d.copy_(lg_pin, non_blocking=True)
        gq4.moe_expert_ffn(Wg, Wu, Wd, lg_d, x_d, cfg.K, y=y, ws=ws)
        y_pin.copy_(y, non_blocking=True)
        b.record(stream)
        b.synchronize()
        if i >= args.warmup:
            e2e_ms.append(a.elapsed_time(b))
    e2e = float(np.mean(e2e_ms))

    ms, e2e = max_over_ranks([ms, e2e], world, dev)

    hbm, bf16, peak_kind = peaks()
    work = stage_work(cfg, split)
    kern = stage_kernels(cfg, split)
    t_stage = {k: float(stage[:, i].mean()) for i, k in enumerate(STAGES)}
    busy = [k for k in STAGES[1:] if work[k][0] > 0 and (k.endswith("small") and split["n_small"] or
                                                         k.endswith("large") and split["n_large"])]
    dom = max(busy or STAGES[1:], key=lambda k: t_stage[k])
    dbytes, dflops = work[dom]
    if dflops > 0:
        roof = roofline("tensor", dflops / (t_stage[dom] * 1e-3) / 1e12, hbm, bf16, peak_kind)
        roof["alg_flops_per_launch"] = dflops
    else:
        roof = roofline("hbm", dbytes / (t_stage[dom] * 1e-3) / 1e9, hbm, bf16, peak_kind)
    roof["alg_bytes_per_launch"] = dbytes
    traffic = None
    if os.path.exists(PROFILE_TRAFFIC):
        with open(PROFILE_TRAFFIC) as f:
            tr = json.load(f)
        rec = tr.get(f"{cfg.name}:{dom}")
        if rec and rec.get("source_hash") == kernel_source_hash():
            traffic = rec["bytes_per_launch"]
    roof["traffic"] = traffic
    roof = {"kernel": kern[dom], "stage": dom, **roof}
    step_bytes = sum(b for b, _ in work.values())
    step_flops = sum(f for _, f in work.values())
    per_expert = 2 * per_matrix_bytes(cfg.F, cfg.H) + per_matrix_bytes(cfg.H, cfg.F)
    n_active = split["n_small"] + split["n_large"]
    out = {
        "value": job_tokens_per_s(world, cfg.T, ms), "unit": "tokens/s", "ms_per_step": ms,
        "ms_p10_p50_p90": [float(v) for v in np.percentile(step_ms, [10, 50, 90])],
        "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "E": cfg.E, "F": cfg.F, "K": cfg.K,
                   "gs": 64, "distinct_experts": n_active, "experts_tensor_core": split["n_large"],
                   "parallelism": f"replicas x{world}",
                   "launch": "value: CUDA-graph replay of one moe_expert_ffn call, events around the "
                             "replay; stage_ms: a second graph with the call's stage events; "
                             "e2e: direct calls",
                   "l2": f"{L2_FLUSH_BYTES >> 20} MiB flush between steps; touched weights "
                         f"{n_active * per_expert / 1e9:.2f} GB/step"},
        "hbm_gbs_step": step_bytes / (ms * 1e-3) / 1e9,
        "stage_ms": t_stage,
        "roofline": roof,
        "e2e": {"value": job_tokens_per_s(world, cfg.T, e2e), "unit": "tokens/s",
                "h2d_bytes_per_step": x_h.nbytes + lg_h.nbytes, "d2h_bytes_per_step": cfg.T * cfg.H * 4},
        "gpu_launches": launches_per_step(cfg, split) * args.steps,
        "clocks": clk.summary(),
    }
    if step_flops > 0:
        out["tflops_step"] = step_flops / (ms * 1e-3) / 1e12
    if with_cpu:
        out["cpu_baseline"] = cpu_baseline(cfg)
    del Wg, Wu, Wd, ws, flush
    torch.cuda.empty_cache()
    return out


def time_replays(fn, steps, warmup, flush):
    """Milliseconds per replay of one captured call (mean, p10/p50/p90), L2 flushed
    between replays, events on the launching stream around each replay."""
    import torch
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    for _ in range(warmup):
        g.replay()
    stream = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ts = []
    for i in range(steps):
        flush.fill_(i & 0xFF)
        a.record(stream)
        g.replay()
        b.record(stream)
        b.synchronize()
        ts.append(a.elapsed_time(b))
    del g
    return float(np.mean(ts)), [float(v) for v in np.percentile(ts, [10, 50, 90])]


def time_e2e(fn, steps, warmup, flush):
    """Milliseconds per direct call including the caller's host<->device copies (fn does
    the copies and the call), events around each step."""
    import torch
    stream = torch.cuda.current_stream()
    ts = []
    for i in range(warmup + steps):
        flush.fill_(i & 0xFF)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()
        if i >= warmup:
            ts.append(a.elapsed_time(b))
    return float(np.mean(ts))


def dense_run(args, dev):
    """The dense gq4_matvec sweep (batch 1, bf16 x): per shape the device time of the
    call, its HBM roofline (packed nibbles + scales + x read, y written) and the end-to-end
    time with x copied in from pinned host memory and y copied out."""
    import torch
    from weight_only_int4_gq4_b200 import gq4
    hbm, bf16, kind = peaks()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    res = {}
    for O, I in synth.DENSE_SHAPES:
        p, sc, xb = synth.dense_matvec(O, I)
        W = gq4.upload(p, sc)
        x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(dev)
        y = torch.empty(1, O, dtype=torch.float32, device=dev)
        ms, pct = time_replays(lambda: gq4.matvec(W, x, y), args.steps, args.warmup, flush)
        x_pin = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).pin_memory()
        y_pin = torch.empty(1, O, dtype=torch.float32).pin_memory()

        def e2e_step():
            x.copy_(x_pin, non_blocking=True)
            gq4.matvec(W, x, y)
            y_pin.copy_(y, non_blocking=True)
        e2e = time_e2e(e2e_step, args.steps, args.warmup, flush)
        nbytes = per_matrix_bytes(O, I) + I * 2 + O * 4
        res[f"{O}x{I}"] = {
            "value": 1.0 / (ms * 1e-3), "unit": "tokens/s", "us": ms * 1e3, "us_p10_p50_p90": [v * 1e3 for v in pct],
            "roofline": {"kernel": "gq4_matvec", **roofline("hbm", nbytes / (ms * 1e-3) / 1e9, hbm, bf16, kind),
                         "alg_bytes_per_launch": nbytes, "traffic": None},
            "e2e": {"value": 1.0 / (e2e * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": I * 2,
                    "d2h_bytes_per_step": O * 4}}
        del W
    del flush
    torch.cuda.empty_cache()
    return res


def single_expert_run(args, dev):
    """The single-expert layer: gate+up+SiLU ([2048][1024] each) then down ([1024][2048])
    on one f32 token, device time of the pair of calls and end to end."""
    import torch
    from weight_only_int4_gq4_b200 import gq4
    se = synth.SingleExpert()
    hbm, bf16, kind = peaks()
    Wg = gq4.upload(gq4.pack(se.qg), se.sg)
    Wu = gq4.upload(gq4.pack(se.qu), se.su)
    Wd = gq4.upload(gq4.pack(se.qd), se.sd)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    x = torch.from_numpy(se.x).to(dev)
    h = torch.empty(1, se.F, dtype=torch.float32, device=dev)
    y = torch.empty(1, se.H, dtype=torch.float32, device=dev)

    def layer():
        gq4.gate_up_silu(Wg, Wu, x, h)
        gq4.matvec(Wd, h, y)
    ms, pct = time_replays(layer, args.steps, args.warmup, flush)
    x_pin = torch.from_numpy(se.x).pin_memory()
    y_pin = torch.empty(1, se.H, dtype=torch.float32).pin_memory()

    def e2e_step():
        x.copy_(x_pin, non_blocking=True)
        layer()
        y_pin.copy_(y, non_blocking=True)
    e2e = time_e2e(e2e_step, args.steps, args.warmup, flush)
    nbytes = 2 * per_matrix_bytes(se.F, se.H) + per_matrix_bytes(se.H, se.F) + 4 * (2 * se.H + 2 * se.F)
    out = {"value": 1.0 / (ms * 1e-3), "unit": "tokens/s", "us": ms * 1e3, "us_p10_p50_p90": [v * 1e3 for v in pct],
           "roofline": {"kernel": "gq4_gate_up_silu + gq4_matvec (2 launches)",
                        **roofline("hbm", nbytes / (ms * 1e-3) / 1e9, hbm, bf16, kind),
                        "alg_bytes_per_launch": nbytes, "traffic": None,
                        "note": "3.5 MB of weights: latency-bound, far below any bandwidth roof"},
           "e2e": {"value": 1.0 / (e2e * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": se.H * 4,
                   "d2h_bytes_per_step": se.H * 4}}
    del Wg, Wu, Wd, flush
    torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=synth.MOE_BATCHED.name, choices=list(synth.MOE_CONFIGS))
    ap.add_argument("--configs", default="all", choices=["all", "none"],
                    help="also time the other workloads of the specification (N = 1 only)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    cfg = synth.MOE_CONFIGS[args.workload]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, cfg, rank)
        return

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    head = moe_run(cfg, args, dev, world, local, with_cpu=not args.no_cpu_baseline and world == 1)
    configs = None
    if args.configs == "all" and world == 1:
        configs = {}
        for c in (synth.MOE_DECODE, synth.MOE_BATCHED, synth.MOE_PREFILL):
            if c.name != cfg.name:
                configs[c.name] = moe_run(c, args, dev, world, local, with_cpu=False)
        configs["dense_matvec_t1_bf16"] = dense_run(args, dev)
        configs["single_expert_f32_1024_2048"] = single_expert_run(args, dev)

    if rank == 0:
        line = {
            "metric": "expert-FFN tokens/s (MoE layer, 1 B200)", "value": head["value"],
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": head["ms_per_step"], "ms_p10_p50_p90": head["ms_p10_p50_p90"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": head["config"],
            "hbm_gbs_step": head["hbm_gbs_step"],
            "stage_ms": head["stage_ms"],
            "roofline": head["roofline"],
            "e2e": head["e2e"],
            "gpu_launches": head["gpu_launches"],
            "clocks": head["clocks"],
        }
        if "cpu_baseline" in head:
            line["cpu_baseline"] = head["cpu_baseline"]
        if configs is not None:
            line["configs"] = configs
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
