"""Profiling cases of the KronQ library (one GPU).

    python -m post_quantization_b200.profcase stages [--tokens N]
        per-stage CUDA-event times of one LLaMA-2-7B-shaped block step (after 2 warm-up steps)
    python -m post_quantization_b200.profcase acc --d 4096 --tokens 16384
        Kronecker-factor sum of one X stream (for an ncu capture of accumulate_tc_kernel)
    python -m post_quantization_b200.profcase biip --d-out 4096 --d-in 4096
    python -m post_quantization_b200.profcase cholinv --d 4096
    python -m post_quantization_b200.profcase quantize --d-out 4096 --d-in 4096
Each case runs its call `--reps` times (default 3) after one warm-up call.
"""
from __future__ import annotations

import argparse
import json

import torch

from . import kronq as K
from . import pipeline as P
from . import synth


def ev():
    return torch.cuda.Event(enable_timing=True)


def stages(args):
    wl = synth.WORKLOADS["llama2_7b_block"]
    n = args.tokens or wl.n_tokens
    dev = torch.device("cuda")
    ws = P.Workspace(dev)
    tag = ("profcase",)
    x = {nm: synth.correlated_x(n, d, synth.seed_for(tag, nm), device=dev)
         for nm, d in wl.streams().items()}
    g = {s.name: synth.gradients(n, s.d_out, synth.seed_for(tag, s.name, "G"), device=dev)
         for s in wl.sublayers}
    w = {s.name: synth.weight(s.d_out, s.d_in, synth.seed_for(tag, s.name, "W"), device=dev)
         for s in wl.sublayers}
    si = {s.name: synth.rademacher(s.d_in, synth.seed_for(tag, s.name, "si"), device=dev)
          for s in wl.sublayers}
    so = {s.name: synth.rademacher(s.d_out, synth.seed_for(tag, s.name, "so"), device=dev)
          for s in wl.sublayers}
    hx = {nm: torch.zeros(d, d, device=dev) for nm, d in wl.streams().items()}
    hg = {s.name: torch.zeros(s.d_out, s.d_out, device=dev) for s in wl.sublayers}
    times = {}

    def timed(key, fn):
        a, b = ev(), ev()
        a.record()
        fn()
        b.record()
        times.setdefault(key, []).append((a, b))

    for it in range(3):
        times.clear()
        for nm in hx:
            hx[nm].zero_()
            timed(f"acc_x/{nm}", lambda nm=nm: P.accumulate(xq=x[nm], hx_sum=hx[nm], ws=ws))
        for s in wl.sublayers:
            hg[s.name].zero_()
            timed(f"acc_g/{s.name}", lambda s=s: P.accumulate(g=g[s.name], hg_sum=hg[s.name], ws=ws))
        res = {}
        for s in wl.sublayers:
            def f(s=s):
                res[s.name] = P.biip(w[s.name], hx[s.x_stream], hg[s.name], None, 1.0 / n,
                                     si[s.name], so[s.name], K.BIIP_FULL, ws=ws)
            timed(f"biip/{s.name}", f)
        for s in wl.sublayers:
            timed(f"cholinv/{s.name}", lambda s=s: P.cholinv(res[s.name], 0.01, ws=ws))
            timed(f"quantize/{s.name}", lambda s=s: P.quantize(res[s.name], wl.bits, ws=ws))
        torch.cuda.synchronize()
    out = {k: sum(a.elapsed_time(b) for a, b in v) for k, v in times.items()}
    groups = {}
    for k, v in out.items():
        groups[k.split("/")[0]] = groups.get(k.split("/")[0], 0.0) + v
    print(json.dumps({"tokens": n, "ms": out, "ms_by_stage": groups,
                      "total_ms": sum(out.values())}, indent=1))


def case_acc(args):
    n, d = args.tokens or 16384, args.d
    x = synth.correlated_x(n, d, synth.seed_for("profcase-acc", d), device="cuda")
    h = torch.zeros(d, d, device="cuda")
    P.accumulate(xq=x, hx_sum=h)
    torch.cuda.synchronize()
    a, b = ev(), ev()
    a.record()
    for _ in range(args.reps):
        P.accumulate(xq=x, hx_sum=h)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.reps
    print(json.dumps({"case": "acc", "d": d, "tokens": n, "ms": ms,
                      "tflops": n * d * (d + 1) / ms / 1e9}))


def case_biip(args):
    d_out, d_in, n = args.d_out, args.d_in, 4096
    x = synth.correlated_x(n, d_in, synth.seed_for("pc-b", "x"), device="cuda")
    g = synth.gradients(n, d_out, synth.seed_for("pc-b", "g"), device="cuda")
    w = synth.weight(d_out, d_in, synth.seed_for("pc-b", "w"), device="cuda")
    si = synth.rademacher(d_in, 1, device="cuda"); so = synth.rademacher(d_out, 2, device="cuda")
    hx = torch.zeros(d_in, d_in, device="cuda"); hg = torch.zeros(d_out, d_out, device="cuda")
    P.accumulate(xq=x, g=g, hx_sum=hx, hg_sum=hg)
    P.biip(w, hx, hg, None, 1.0 / n, si, so, K.BIIP_FULL)
    torch.cuda.synchronize()
    a, b = ev(), ev()
    a.record()
    for _ in range(args.reps):
        P.biip(w, hx, hg, None, 1.0 / n, si, so, K.BIIP_FULL)
    b.record()
    torch.cuda.synchronize()
    print(json.dumps({"case": "biip", "d_out": d_out, "d_in": d_in,
                      "ms": a.elapsed_time(b) / args.reps}))


def case_cholinv(args):
    d, n = args.d, 2 * args.d
    x = synth.correlated_x(n, d, synth.seed_for("pc-c", d), device="cuda")
    h = torch.zeros(d, d, device="cuda")
    P.accumulate(xq=x, hx_sum=h)
    h /= n
    info = torch.empty(1, dtype=torch.int32, device="cuda")
    k = h.clone()
    K.kronq_cholinv(k, 0.01, info, K.CHOLINV_SYNC)
    a, b = ev(), ev()
    a.record()
    for _ in range(args.reps):
        k.copy_(h)
        K.kronq_cholinv(k, 0.01, info, 0)
    b.record()
    torch.cuda.synchronize()
    print(json.dumps({"case": "cholinv", "d": d, "ms": a.elapsed_time(b) / args.reps}))


def case_quantize(args):
    d_out, d_in, n = args.d_out, args.d_in, 2 * args.d_in
    x = synth.correlated_x(n, d_in, synth.seed_for("pc-q", "x"), device="cuda")
    w = synth.weight(d_out, d_in, synth.seed_for("pc-q", "w"), device="cuda")
    si = synth.rademacher(d_in, 1, device="cuda"); so = synth.rademacher(d_out, 2, device="cuda")
    hx = torch.zeros(d_in, d_in, device="cuda")
    P.accumulate(xq=x, hx_sum=hx)
    r = P.biip(w, hx, None, None, 1.0 / n, si, so, K.BIIP_SCALE_IN | K.BIIP_ROTATE_IN | K.BIIP_ROTATE_OUT)
    P.cholinv(r, 0.01, sync=True)
    P.quantize(r, 4, group=args.group)
    torch.cuda.synchronize()
    a, b = ev(), ev()
    a.record()
    for _ in range(args.reps):
        P.quantize(r, 4, group=args.group)
    b.record()
    torch.cuda.synchronize()
    print(json.dumps({"case": "quantize", "d_out": d_out, "d_in": d_in, "group": args.group,
                      "ms": a.elapsed_time(b) / args.reps}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["stages", "acc", "biip", "cholinv", "quantize"])
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--d", type=int, default=4096)
    ap.add_argument("--d-out", type=int, default=4096)
    ap.add_argument("--d-in", type=int, default=4096)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--group", type=int, default=0, help="quantize: 0 (per row) or 128")
    args = ap.parse_args()
    K.load_library()
    K.kronq_device_check()
    {"stages": stages, "acc": case_acc, "biip": case_biip, "cholinv": case_cholinv,
     "quantize": case_quantize}[args.case](args)


if __name__ == "__main__":
    main()
