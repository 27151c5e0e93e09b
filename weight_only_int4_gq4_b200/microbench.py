"""Timings of the library's calls outside the MoE layer step, one JSON line each.

    python -m weight_only_int4_gq4_b200.microbench [--only NAME ...] [--reps N]

Each case captures one call in a CUDA graph and replays it between L2 flushes (a 256 MiB
write), timing the replay with CUDA events on the launching stream (the median of the
replays).  Bytes are the algorithmic HBM bytes of the call (packed nibbles + f32 scales
read, activations read, outputs written); fractions are of the measured HBM copy
bandwidth (MEASURED_PEAKS.json at the repository root, else 6650 GB/s).  Inputs are
seeded synthetic data with the shapes of the workloads:
  * dense matvec sweep, batch 1, bf16 x: 4096x4096, 14336x4096, 4096x14336, 151936x4096;
  * the single-expert layer: f32 x [1][1024], gate/up [2048][1024], down [1024][2048];
  * quantisation of f32 weights (a 6144x2048 expert, a 151936x4096 matrix);
  * row gather of 512 rows of a 151936x4096 matrix to bf16 (embedding lookup);
  * matvec over 512 selected rows of that matrix;
  * general group size: a 14336x4096 matvec with gs = 128;
  * the MLA absorb projections over a 28672x512 kv_b tensor (64 heads of 192 key and
    256 value rows), 1 and 32 tokens.
"""
from __future__ import annotations

import argparse
import json
import os

import numpy as np
import torch

from . import gq4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def hbm_peak() -> float:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f).get("hbm_gbs", 6650.0))
    return 6650.0


def time_graph(fn, reps: int, flush: torch.Tensor) -> float:
    """Median milliseconds of one replay of the captured call."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    for _ in range(3):
        g.replay()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ts = []
    for i in range(reps):
        flush.fill_(i & 0xFF)
        a.record()
        g.replay()
        b.record()
        b.synchronize()
        ts.append(a.elapsed_time(b))
    del g
    return float(np.median(ts))


def rand_tensor(O, I, gs=64, seed=0):
    rng = np.random.default_rng(seed)
    p = rng.integers(0, 256, size=(O, I // 2), dtype=np.uint8)
    s = rng.uniform(0.002, 0.02, size=(O, -(-I // gs))).astype(np.float32)
    return gq4.upload(p, s, gs=gs)


def wbytes(O, I, gs=64):
    return O * (I // 2) + O * (-(-I // gs)) * 4


def report(name, ms, nbytes, peak, **extra):
    gbs = nbytes / (ms * 1e-3) / 1e9
    line = {"case": name, "us": round(ms * 1e3, 2), "bytes": int(nbytes), "gbs": round(gbs, 1),
            "frac_of_measured_hbm": round(gbs / peak, 3), **extra}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--only", nargs="*", default=None)
    ap.add_argument("--reps", type=int, default=20)
    args = ap.parse_args()
    want = lambda n: args.only is None or any(n.startswith(o) for o in args.only)  # noqa: E731
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    peak = hbm_peak()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    for O, I in [(4096, 4096), (14336, 4096), (4096, 14336), (151936, 4096)]:
        name = f"matvec_{O}x{I}_t1_bf16"
        if not want(name):
            continue
        W = rand_tensor(O, I, seed=O + I)
        x = torch.randn(1, I, device=dev).to(torch.bfloat16)
        y = torch.empty(1, O, device=dev)
        ms = time_graph(lambda: gq4.matvec(W, x, y), args.reps, flush)
        report(name, ms, wbytes(O, I) + I * 2 + O * 4, peak)
        del W

    if want("single_expert"):
        Wg, Wu, Wd = rand_tensor(2048, 1024, seed=1), rand_tensor(2048, 1024, seed=2), rand_tensor(1024, 2048, seed=3)
        x = torch.randn(1, 1024, device=dev)
        h = torch.empty(1, 2048, device=dev)
        y = torch.empty(1, 1024, device=dev)

        def layer():
            gq4.gate_up_silu(Wg, Wu, x, h)
            gq4.matvec(Wd, h, y)
        ms = time_graph(layer, args.reps, flush)
        report("single_expert_gate_up_silu_down_f32", ms, 3 * wbytes(2048, 1024) + 1024 * 4 * 2 + 2048 * 4 * 2, peak)

    for O, I in [(6144, 2048), (151936, 4096)]:
        name = f"quantize_{O}x{I}_gs64"
        if not want(name):
            continue
        w = torch.randn(O, I, device=dev)
        ms = time_graph(lambda: gq4.quantize(w, 64), args.reps, flush)
        report(name, ms, O * I * 4 + wbytes(O, I), peak)
        del w

    if want("dequant_rows") or want("matvec_rows"):
        O, I = 151936, 4096
        W = rand_tensor(O, I, seed=7)
        idx = torch.randint(0, O, (512,), dtype=torch.int32, device=dev)
        if want("dequant_rows"):
            out = torch.empty(512, I, dtype=torch.bfloat16, device=dev)
            ms = time_graph(lambda: gq4.dequant_rows(W, idx, out=out), args.reps, flush)
            report("dequant_rows_512_of_151936x4096_bf16", ms, 512 * (wbytes(1, I) + I * 2), peak)
        if want("matvec_rows"):
            x = torch.randn(1, I, device=dev).to(torch.bfloat16)
            y = torch.empty(1, 512, device=dev)
            ms = time_graph(lambda: gq4.matvec_rows(W, idx, x, y), args.reps, flush)
            report("matvec_rows_512_of_151936x4096_t1", ms, 512 * wbytes(1, I) + I * 2 + 512 * 4, peak)
        del W

    if want("matvec_gs128"):
        O, I = 14336, 4096
        W = rand_tensor(O, I, gs=128, seed=9)
        x = torch.randn(1, I, device=dev).to(torch.bfloat16)
        y = torch.empty(1, O, device=dev)
        ms = time_graph(lambda: gq4.matvec(W, x, y), args.reps, flush)
        report("matvec_gs128_14336x4096_t1", ms, wbytes(O, I, 128) + I * 2 + O * 4, peak)

    if want("mla_absorb"):
        # the pages' kv_b tensor: 28,672 rows x 512 latent inputs, read as 64 heads of
        # 192 key + 256 value rows
        nh, dn, dv, R = 64, 192, 256, 512
        W = rand_tensor(nh * (dn + dv), R, seed=31)
        for T in (1, 32):
            qn = torch.randn(T, nh, dn, device=dev).to(torch.bfloat16)
            lat = torch.randn(T, nh, R, device=dev).to(torch.bfloat16)
            ql = torch.empty(T, nh, R, device=dev)
            o = torch.empty(T, nh, dv, device=dev)
            ms = time_graph(lambda: gq4.mla_absorb_q(W, nh, dn, dv, qn, ql), args.reps, flush)
            report(f"mla_absorb_q_kvb28672x512_t{T}", ms, nh * wbytes(dn, R) + qn.numel() * 2 + ql.numel() * 4, peak)
            ms = time_graph(lambda: gq4.mla_absorb_v(W, nh, dn, dv, lat, o), args.reps, flush)
            report(f"mla_absorb_v_kvb28672x512_t{T}", ms, nh * wbytes(dv, R) + lat.numel() * 2 + o.numel() * 4, peak)


if __name__ == "__main__":
    main()
