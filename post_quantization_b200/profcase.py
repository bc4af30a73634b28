"""Profiling cases of the KronQ library (one GPU).

    python -m post_quantization_b200.profcase stages [--tokens N]
        per-stage CUDA-event times of one LLaMA-2-7B-shaped block step (after 2 warm-up steps)
    python -m post_quantization_b200.profcase acc --d 4096 --tokens 16384
        Kronecker-factor sum of one X stream (for an ncu capture of accumulate_tc_kernel)
    python -m post_quantization_b200.profcase biip --d-out 4096 --d-in 4096
    python -m post_quantization_b200.profcase cholinv --d 4096
    python -m post_quantization_b200.profcase quantize --d-out 4096 --d-in 4096
    python -m post_quantization_b200.profcase twosided --d-out 1024 --d-in 1024 --bits 2
        the comparison variant with output-side feedback against the column solve
    python -m post_quantization_b200.profcase qlinear --block --bits 2 --group 128 --tokens 1
        the quantized layers at inference, per layer (graph replays) and as one block sweep
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
    ws = P.Workspace(torch.device("cuda"))
    if args.drift:
        # the drift sum D += (X - X~)^T X~ alone (X~ = X + N(0, (0.05 rms X)^2))
        xq = synth.perturbed(x, synth.seed_for("profcase-acc", d, "q"), rel_std=0.05)
        call = lambda: P.accumulate(xq=xq, xfp=x, dxx_sum=h, ws=ws)
        flops = 2.0 * n * d * d
    else:
        call = lambda: P.accumulate(xq=x, hx_sum=h, ws=ws)
        flops = float(n) * d * (d + 1)
    call()
    torch.cuda.synchronize()
    a, b = ev(), ev()
    a.record()
    for _ in range(args.reps):
        call()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.reps
    print(json.dumps({"case": "acc", "d": d, "tokens": n, "drift": args.drift, "ms": ms,
                      "tflops": flops / ms / 1e9}))


def case_twosided(args):
    """The comparison variant (output-side feedback too) against KronQ's column solve on one
    layer: time per call, update passes, and the Kronecker objective tr[H_G dW H_X dW^T] of both
    (fp64 on the device; a measurement, not part of the library)."""
    d_out, d_in, n, bits = args.d_out, args.d_in, max(2 * args.d_in, 4096), args.bits
    x = synth.correlated_x(n, d_in, synth.seed_for("pc-2s", "x"), device="cuda")
    g = synth.gradients(n, d_out, synth.seed_for("pc-2s", "g"), device="cuda")
    w = synth.weight(d_out, d_in, synth.seed_for("pc-2s", "w"), device="cuda")
    si = synth.rademacher(d_in, 1, device="cuda"); so = synth.rademacher(d_out, 2, device="cuda")
    hx = torch.zeros(d_in, d_in, device="cuda"); hg = torch.zeros(d_out, d_out, device="cuda")
    P.accumulate(xq=x, g=g, hx_sum=hx, hg_sum=hg)
    r = P.biip(w, hx, hg, None, 1.0 / n, si, so, K.BIIP_FULL | K.BIIP_WRITE_HG)
    hx_p, hg_p = r.hx.clone(), hg.clone()
    P.cholinv(r, 0.01, sync=True)
    k_out = hg.clone()
    info = torch.empty(1, dtype=torch.int32, device="cuda")
    K.kronq_cholinv(k_out, 0.01, info, K.CHOLINV_SYNC)
    out = K.kronq_quantize_layer_twosided(r.w_prime, r.hx, k_out, bits)
    P.quantize(r, bits)
    torch.cuda.synchronize()
    a, b = ev(), ev()
    a.record()
    out = K.kronq_quantize_layer_twosided(r.w_prime, r.hx, k_out, bits)
    b.record()
    torch.cuda.synchronize()
    ms2 = a.elapsed_time(b)
    a.record()
    P.quantize(r, bits)
    b.record()
    torch.cuda.synchronize()
    ms1 = a.elapsed_time(b)
    wp = r.w_prime.double()

    def obj(wh):
        dw = wp - wh.double()
        return float(torch.trace(hg_p.double() @ dw @ hx_p.double() @ dw.T))
    o1, o2 = obj(r.w_hat), obj(out[3])
    print(json.dumps({"case": "twosided", "d_out": d_out, "d_in": d_in, "bits": bits,
                      "updates": out[4], "ms_twosided": ms2, "ms_column_solve": ms1,
                      "objective_column_solve": o1, "objective_twosided": o2,
                      "objective_ratio": o2 / o1}))


def case_peaks(args):
    """torch (cuBLAS) matmul rates, 8192^3, best of 10 after 3 warm-ups: bf16, fp16, TF32 and
    fp32 (the denominators of the fp32-accurate tensor-core GEMM)."""
    n = 8192
    out = {"case": "peaks", "n": n}
    for name, dt, tf32 in (("bf16", torch.bfloat16, False), ("fp16", torch.float16, False),
                           ("tf32", torch.float32, True), ("fp32", torch.float32, False)):
        torch.backends.cuda.matmul.allow_tf32 = tf32
        a = torch.randn(n, n, device="cuda", dtype=dt)
        b = torch.randn(n, n, device="cuda", dtype=dt)
        for _ in range(3):
            a @ b
        best = 1e30
        for _ in range(10):
            e0, e1 = ev(), ev()
            e0.record()
            a @ b
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        out[name + "_tflops"] = 2.0 * n ** 3 / best / 1e9
        del a, b
    torch.backends.cuda.matmul.allow_tf32 = False
    print(json.dumps(out))


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
    n0 = K.kronq_launch_count()
    K.kronq_cholinv(k, 0.01, info, K.CHOLINV_SYNC)
    per_call = K.kronq_launch_count() - n0
    a, b = ev(), ev()
    a.record()
    for _ in range(args.reps):
        k.copy_(h)
        K.kronq_cholinv(k, 0.01, info, 0)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.reps
    # the same calls replayed from a CUDA graph: the difference is the launch gaps
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        k.copy_(h)
        K.kronq_cholinv(k, 0.01, info, 0)
    g.replay()
    torch.cuda.synchronize()
    a.record()
    for _ in range(args.reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    print(json.dumps({"case": "cholinv", "d": d, "ms": ms,
                      "graph_ms": a.elapsed_time(b) / args.reps,
                      "launches_per_call": per_call}))
    del g


def case_quantize(args):
    d_out, d_in, n = args.d_out, args.d_in, 2 * args.d_in
    x = synth.correlated_x(n, d_in, synth.seed_for("pc-q", "x"), device="cuda")
    w = synth.weight(d_out, d_in, synth.seed_for("pc-q", "w"), device="cuda")
    si = synth.rademacher(d_in, 1, device="cuda"); so = synth.rademacher(d_out, 2, device="cuda")
    hx = torch.zeros(d_in, d_in, device="cuda")
    dxx = None
    if args.drift:
        xq = synth.perturbed(x, synth.seed_for("pc-q", "xq"), rel_std=0.05)
        dxx = torch.zeros(d_in, d_in, device="cuda")
        P.accumulate(xq=xq, xfp=x, hx_sum=hx, dxx_sum=dxx)
    else:
        P.accumulate(xq=x, hx_sum=hx)
    r = P.biip(w, hx, None, dxx, 1.0 / n, si, so,
               K.BIIP_SCALE_IN | K.BIIP_ROTATE_IN | K.BIIP_ROTATE_OUT)
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
                      "drift": args.drift, "ms": a.elapsed_time(b) / args.reps}))


LLAMA3_70B_LINEARS = [("q", 8192, 8192), ("k", 1024, 8192), ("v", 1024, 8192),
                      ("o", 8192, 8192), ("gate", 28672, 8192), ("up", 28672, 8192),
                      ("down", 8192, 28672)]


def qlinear_bytes(d_out, d_in, bits, group, n_tok, x_bytes=4):
    """Algorithmic bytes of one kronq_qlinear call: packed codes, grid, x, y, scales, signs."""
    ng = (d_in + 127) // 128 if group else 1
    return (K.kronq_packed_codes_bytes(d_out, d_in, bits) + 8 * d_out * ng
            + n_tok * d_in * x_bytes + n_tok * d_out * 4 + 5 * (d_in + d_out))


def case_qlinear(args):
    """Decode through the linears of one LLaMA-3-70B-shaped block (or one --d-out x --d-in
    layer) at --bits, --group, --tokens tokens; each layer's call is captured in its own CUDA
    graph and timed by replays (the block's packed codes, 214 MB at 2 bits, exceed L2)."""
    dev = torch.device("cuda")
    n = args.tokens or 1
    bits, group = args.bits, args.group
    shapes = LLAMA3_70B_LINEARS if args.block else [("layer", args.d_out, args.d_in)]
    layers = []
    for nm, do, di in shapes:
        tag = ("qlinear-case", nm, do, di, bits)
        c = synth.codes(do, di, bits, synth.seed_for(tag, "c"), device=dev)
        packed = K.kronq_pack_codes(c, bits)
        del c
        ng = (di + 127) // 128 if group else 0
        scale, zero = synth.grid_params(do, ng, bits, synth.seed_for(tag, "g"), device=dev)
        grid = K.kronq_pack_grid(scale, zero, do, di, group)
        lay = dict(name=nm, d_out=do, d_in=di, packed=packed, grid=grid,
                   s_x=synth.positive_scales(di, synth.seed_for(tag, "sx"), device=dev),
                   s_g=synth.positive_scales(do, synth.seed_for(tag, "sg"), device=dev),
                   si=synth.rademacher(di, synth.seed_for(tag, "si"), device=dev),
                   so=synth.rademacher(do, synth.seed_for(tag, "so"), device=dev),
                   x=synth.activations(n, di, synth.seed_for(tag, "x"), device=dev),
                   y=torch.empty(n, do, device=dev))
        nb = K.kronq_qlinear_workspace_size(do, di, n)
        lay["ws"] = P.Workspace(dev).get(nb)
        layers.append(lay)

    def call(L):
        K.kronq_qlinear(L["x"], L["packed"], L["grid"], L["s_x"], L["s_g"], L["si"], L["so"],
                        K.BIIP_FULL, L["d_out"], bits, L["y"], group=group, workspace=L["ws"])

    for L in layers:
        call(L)
    torch.cuda.synchronize()

    class Eager:
        """Stands in for a graph (eager calls), for runs under a profiler."""
        def __init__(self, L):
            self.L = L

        def replay(self):
            call(self.L)

    graphs = []
    for L in layers:
        if args.no_graphs:
            graphs.append(Eager(L))
            continue
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            call(L)
        graphs.append(g)
    for _ in range(3):
        for g in graphs:
            g.replay()
    torch.cuda.synchronize()
    res = []
    tot_ms, tot_bytes = 0.0, 0
    for L, g in zip(layers, graphs):
        a, b = ev(), ev()
        # interleave the other layers between timed replays so that this layer's codes are
        # not in L2 when its replay starts
        ms = 0.0
        for _ in range(args.reps):
            for g2 in graphs:
                if g2 is not g:
                    g2.replay()
            a.record()
            g.replay()
            b.record()
            b.synchronize()
            ms += a.elapsed_time(b)
        ms /= args.reps
        nbytes = qlinear_bytes(L["d_out"], L["d_in"], bits, group, n)
        tot_ms += ms
        tot_bytes += nbytes
        res.append({"layer": L["name"], "d_out": L["d_out"], "d_in": L["d_in"], "us": ms * 1e3,
                    "GBps": nbytes / ms / 1e6})
    # the whole block as one sweep of graph replays
    a, b = ev(), ev()
    a.record()
    for _ in range(args.reps):
        for g in graphs:
            g.replay()
    b.record()
    torch.cuda.synchronize()
    sweep_ms = a.elapsed_time(b) / args.reps
    # the whole block in one graph (the layers' kernels chained back to back, as in a decode
    # step); replayed with the other copies of the codes in between so that L2 starts cold
    block_us = conc_us = None
    if not args.no_graphs:
        gb = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gb):
            for L in layers:
                call(L)
        for _ in range(3):
            gb.replay()
        torch.cuda.synchronize()
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
        tot = 0.0
        for _ in range(args.reps):
            flush.zero_()                      # 256 MB through L2
            a.record()
            gb.replay()
            b.record()
            b.synchronize()
            tot += a.elapsed_time(b)
        block_us = tot / args.reps * 1e3
        del gb
        if args.block:
            # the block's own dependency order: q, k and v read the same input and run as
            # three branches, then o, then gate and up as two branches, then down
            stages = [["q", "k", "v"], ["o"], ["gate", "up"], ["down"]]
            by_name = {L["name"]: L for L in layers}
            side = [torch.cuda.Stream() for _ in range(3)]
            gc = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gc):
                main = torch.cuda.current_stream()
                for names in stages:
                    if len(names) == 1:
                        call(by_name[names[0]])
                        continue
                    fork = torch.cuda.Event()
                    fork.record(main)
                    for st, nm in zip(side, names):
                        st.wait_event(fork)
                        with torch.cuda.stream(st):
                            call(by_name[nm])
                    for st in side[:len(names)]:
                        main.wait_stream(st)
            for _ in range(3):
                gc.replay()
            torch.cuda.synchronize()
            tot = 0.0
            for _ in range(args.reps):
                flush.zero_()
                a.record()
                gc.replay()
                b.record()
                b.synchronize()
                tot += a.elapsed_time(b)
            conc_us = tot / args.reps * 1e3
            del gc
        del flush
    print(json.dumps({"case": "qlinear", "bits": bits, "group": group, "tokens": n,
                      "layers": res, "sum_us": tot_ms * 1e3, "sweep_us": sweep_ms * 1e3,
                      "sweep_GBps": tot_bytes / sweep_ms / 1e6, "block_graph_us": block_us,
                      "block_graph_GBps": tot_bytes / block_us / 1e3 if block_us else None,
                      "block_branches_us": conc_us,
                      "block_branches_GBps": tot_bytes / conc_us / 1e3 if conc_us else None,
                      "launches": K.kronq_launch_count()}))
    del graphs


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["stages", "acc", "biip", "cholinv", "quantize", "qlinear",
                                     "peaks", "twosided"])
    ap.add_argument("--drift", action="store_true", help="acc: the drift sum D alone; "
                                                          "quantize: with D (P pre-shift)")
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--d", type=int, default=4096)
    ap.add_argument("--d-out", type=int, default=4096)
    ap.add_argument("--d-in", type=int, default=4096)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--group", type=int, default=0, help="quantize: 0 (per row) or 128")
    ap.add_argument("--bits", type=int, default=2, help="qlinear: code width")
    ap.add_argument("--block", action="store_true", help="qlinear: the LLaMA-3-70B block")
    ap.add_argument("--no-graphs", action="store_true", help="qlinear: eager calls")
    args = ap.parse_args()
    K.load_library()
    K.kronq_device_check()
    {"stages": stages, "acc": case_acc, "biip": case_biip, "cholinv": case_cholinv,
     "quantize": case_quantize, "qlinear": case_qlinear, "peaks": case_peaks,
     "twosided": case_twosided}[args.case](args)


if __name__ == "__main__":
    main()
