"""KronQ layer-path benchmark on B200.

One step = the whole hot path over one LLaMA-3-70B-shaped transformer block (7 sublayers:
q/o 8192x8192, k/v 1024x8192, gate/up 28672x8192, down 8192x28672; 262144 calibration tokens;
2-bit per-channel grid; BiIP on; X~ = X + N(0, (0.05 rms X)^2), so the drift term and the GPTAQ
pre-shift are active):
  Kronecker-factor sums (H_X and the drift sum D for the 4 distinct inputs - q/k/v share one,
  gate/up share one - and H_G for the 7 output-gradient streams) -> BiIP of every sublayer ->
  traces to the host -> scores and bit allocation -> damped inverse factor -> P pre-shift and
  column solve of every sublayer. The per-sublayer steps run side by side, one CUDA stream each.
Metric: quantized weight params/s (whole job: params of all ranks' blocks / max step time).
Each rank quantizes its own block (weak scaling, no collective on the data path).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]

--workload llama2_7b_block / llama3_8b_block select the smaller blocks; llama2_7b_stack runs
the 32-block mixed-precision stack (see run_stack).
--impl reference times the fp64 CPU oracle on a bounded sample of the same workload (see
oracle_sample) on the host cores.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "llama3_70b_block"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="kronq", choices=["kronq", "reference"])
    ap.add_argument("--tokens", type=int, default=None, help=argparse.SUPPRESS)
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=["llama2_7b_block", "llama3_8b_block", "llama3_70b_block",
                             "llama2_7b_stack"],
                    help="block shape (default: the LLaMA-3-70B block)")
    ap.add_argument("--graphs", default="auto", choices=["auto", "on", "off"],
                    help="replay the per-sublayer phases as CUDA graphs (each graph keeps its own "
                         "copies of the phase's outputs); auto: on when the block's inputs "
                         "take less than 60 GB of device memory")
    ap.add_argument("--no-graphs", action="store_true", help=argparse.SUPPRESS)
    ap.add_argument("--schedule", default="phases", choices=["phases", "overlapped"],
                    help="phases: all statistics, then every sublayer's BiIP, inverse factor and "
                         "solve; overlapped: each sublayer's chain starts when its sums are "
                         "complete, beside the remaining statistics")
    ap.add_argument("--overlap", type=int, default=0, metavar="SMS",
                    help="overlapped schedule with SMS SMs kept free of statistics for the "
                         "chains (0: no reservation)")
    ap.add_argument("--calibration", default="synthetic", choices=["synthetic", "backward"],
                    help="synthetic: seeded X and G generators; backward: X and G of every linear "
                         "from the forward and backward of a random-weight block")
    ap.add_argument("--hg-diag", action="store_true",
                    help="diagonal-only H_G: sum diag(G^T G) in one streaming pass instead of "
                         "the G^T G product (BiIP's scales and the trace need only the diagonal)")
    ap.add_argument("--no-e2e", action="store_true", help=argparse.SUPPRESS)
    ap.add_argument("--no-cpu-baseline", action="store_true", help=argparse.SUPPRESS)
    return ap.parse_args()


# ---------------------------------------------------------------------------------- oracle

PROXY_D = 2048        # proxy sublayer of the oracle sample: d_out = d_in = 2048
PROXY_TOKENS = 8192
PROXY_ROWS = 128


def _biip_flops(d_out, d_in, drift):
    """Flops of the oracle's BiIP: dense b x b Hadamard-block products on each side of W, on both
    sides of H_X (and D), and of H_G."""
    bi = d_in & -d_in
    bo = d_out & -d_out
    f = 2 * d_out * d_in * (bi + bo) + 4 * d_in * d_in * bi + 4 * d_out * d_out * bo
    return f + (4 * d_in * d_in * bi if drift else 0)


def cpu_info():
    model = ""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    from threadpoolctl import threadpool_info
    threads = max([int(i.get("num_threads", 0)) for i in threadpool_info()] or [0])
    return model, os.cpu_count() or 1, threads or (os.cpu_count() or 1)


def oracle_layer256():
    """The 256 x 256 layer (2048 tokens, 2 bits, drift term on) through the whole oracle, BiIP on
    and off: seconds per stage."""
    from oracle import kronq_oracle as O
    from post_quantization_b200 import synth
    tag = ("bench-oracle", "layer256")
    d, n = 256, 2048
    xt = synth.correlated_x(n, d, synth.seed_for(tag, "X"))
    xfp = xt.double().numpy()
    xq = synth.perturbed(xt, synth.seed_for(tag, "Xq"), abs_std=0.01).double().numpy()
    g = synth.gradients(n, d, synth.seed_for(tag, "G")).double().numpy()
    w = synth.weight(d, d, synth.seed_for(tag, "W"), dtype=__import__("torch").float32).double().numpy()
    si = synth.rademacher(d, synth.seed_for(tag, "si")).numpy()
    so = synth.rademacher(d, synth.seed_for(tag, "so")).numpy()
    out = {}
    for name, flags in (("biip_on", O.BIIP_FULL), ("biip_off", 0)):
        t = {}
        t0 = time.perf_counter()
        hx, hg, dxx = O.accumulate(xq, xfp, g)
        t["statistics"] = time.perf_counter() - t0
        t0 = time.perf_counter()
        b = O.biip(w, hx, hg, dxx, 1.0 / n, si, so, flags)
        t["biip"] = time.perf_counter() - t0
        t0 = time.perf_counter()
        k = O.cholinv(b["hx"], 0.01)
        t["cholinv"] = time.perf_counter() - t0
        t0 = time.perf_counter()
        O.quantize_layer(b["w"], k, b["dxx"], 2)
        t["solve"] = time.perf_counter() - t0
        out[name] = {key: round(v, 4) for key, v in t.items()}
    return out


def oracle_sample(wl_name: str = WORKLOAD):
    """Time the fp64 oracle, stage by stage, on a proxy sublayer and report its measured rates.

    Sample: a 2048 x 2048 sublayer (one Hadamard block per side, like the hidden-size sublayers)
    with 8192 calibration tokens: the statistics (with the drift sum when the workload has it),
    the whole BiIP, the damped inverse factor, GPTAQ's P (drift workloads), and the column solve
    of 128 output rows (rows are independent given K). Each stage gives a measured rate: GFLOP/s
    of the oracle's own arithmetic for the statistics and BiIP, seconds at d = 2048 for the
    inverse factor and P, rows/s for the solve.

    The block estimate divides the block's work in each stage by that stage's measured rate:
    statistics and BiIP by their flop counts, the inverse factor and P by d_in^3, the solve by
    d_out d_in^2. It is an estimate, labelled as one; the measured quantities are the rates.
    Returns (estimated seconds per block step, record dict, seconds spent measuring).
    """
    from oracle import kronq_oracle as O
    from post_quantization_b200 import synth

    wl = synth.WORKLOADS[wl_name]
    drift = wl.drift != "none"
    d, n_s, rows = PROXY_D, PROXY_TOKENS, PROXY_ROWS
    tag = ("bench-oracle", wl_name)
    xt = synth.correlated_x(n_s, d, synth.seed_for(tag, "X"))
    xfp = xt.double().numpy()
    xq = (synth.perturbed(xt, synth.seed_for(tag, "Xq"), rel_std=0.05).double().numpy()
          if drift else xfp)
    del xt
    g = synth.gradients(n_s, d, synth.seed_for(tag, "G")).double().numpy()
    w = synth.weight(d, d, synth.seed_for(tag, "W")).double().numpy()
    si = synth.rademacher(d, synth.seed_for(tag, "si")).numpy()
    so = synth.rademacher(d, synth.seed_for(tag, "so")).numpy()

    spent0 = time.perf_counter()
    t0 = time.perf_counter()
    hx, hg, dxx = O.accumulate(xq, xfp if drift else None, g)
    t_acc = time.perf_counter() - t0
    t0 = time.perf_counter()
    b = O.biip(w, hx, hg, dxx, 1.0 / n_s, si, so, O.BIIP_FULL)
    t_biip = time.perf_counter() - t0
    t0 = time.perf_counter()
    k = O.cholinv(b["hx"], 0.01)
    t_chol = time.perf_counter() - t0
    t_p = 0.0
    if drift:
        t0 = time.perf_counter()
        O.p_matrix(b["dxx"], k)
        t_p = time.perf_counter() - t0
    t0 = time.perf_counter()
    O.quantize_layer(b["w"][:rows], k, b["dxx"] if drift else None, wl.bits)
    t_q = time.perf_counter() - t0 - t_p         # quantize_layer forms P itself
    t_q = max(t_q, 1e-9)
    spent = time.perf_counter() - spent0

    # measured rates
    acc_fl = 2.0 * n_s * d * d * (3 if drift else 2)      # X~^T X~, G^T G (and D), full matrices
    r_acc = acc_fl / t_acc
    r_biip = _biip_flops(d, d, drift) / t_biip
    rows_per_s = rows / t_q

    # block estimate from those rates
    N = wl.n_tokens
    e_acc = sum(2.0 * N * dd * dd * (2 if drift else 1) for dd in wl.streams().values())
    e_acc += sum(2.0 * N * s.d_out * s.d_out for s in wl.sublayers)
    est = e_acc / r_acc
    est += sum(_biip_flops(s.d_out, s.d_in, drift) for s in wl.sublayers) / r_biip
    est += sum((s.d_in / d) ** 3 for s in wl.sublayers) * t_chol
    if drift:
        est += sum((s.d_in / d) ** 3 for s in wl.sublayers) * t_p
    est += sum(s.d_out * (s.d_in / d) ** 2 for s in wl.sublayers) / rows_per_s
    rec = {
        "statistics_gflops": round(r_acc / 1e9, 2),
        "biip_gflops": round(r_biip / 1e9, 2),
        f"cholinv_s_d{d}": round(t_chol, 3),
        f"p_matrix_s_d{d}": round(t_p, 3) if drift else None,
        f"solve_rows_per_s_d{d}": round(rows_per_s, 2),
        "estimated_s_per_step": round(est, 1),
    }
    return est, rec, spent


# ---------------------------------------------------------------------------------- clocks

class ClockSampler:
    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 8:
                self.samples.append(parts)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        if not self.samples:
            return None
        sm = [float(s[0]) for s in self.samples if s[0].replace(".", "").isdigit()]
        mx = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for s in self.samples:
            for nm, v in zip(names, s[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------------- GPU arm

class Block:
    """Device-resident inputs and buffers of one block; `step` runs the whole path."""

    def __init__(self, wl, rank, device, n_tokens, ws, calibration="synthetic", hg_diag=False):
        import torch

        from post_quantization_b200 import kronq as K
        from post_quantization_b200 import synth
        self.wl = wl
        self.dev = device
        self.n = n_tokens
        self.ws = ws
        tag = (wl.name, "rank", rank)
        self.drift = wl.drift != "none"
        self.hg_diag = hg_diag
        self.biip_flags = K.BIIP_FULL | (K.BIIP_HG_DIAG if hg_diag else 0)
        self.w = {s.name: synth.weight(s.d_out, s.d_in, synth.seed_for(tag, s.name, "W"),
                                       dtype=wl.w_dtype, device=device) for s in wl.sublayers}
        # X~ (the quantized model's input) in self.x; with the asymmetric term on, also X (the
        # full-precision model's input) in self.xfp, and D = (X - X~)^T X~ per stream
        if calibration == "backward":
            # X and G from the forward and backward of a random-weight block with these weights
            xs, gs = synth.block_calibration(wl, n_tokens, synth.seed_for(tag, "block"),
                                             device=device, weights=self.w)
        else:
            xs = {name: synth.correlated_x(n_tokens, d, synth.seed_for(tag, name, "X"),
                                           device=device) for name, d in wl.streams().items()}
            gs = None
        if self.drift:
            kind, amount = wl.drift[:3], float(wl.drift[3:])
            self.xfp = xs
            self.x = {name: synth.perturbed(x, synth.seed_for(tag, name, "Xq"),
                                            **({"rel_std": amount} if kind == "rel"
                                               else {"abs_std": amount}))
                      for name, x in xs.items()}
            self.dxx = {name: torch.zeros(d, d, device=device)
                        for name, d in wl.streams().items()}
        else:
            self.xfp = None
            self.x = xs
            self.dxx = None
        self.g = gs if gs is not None else {
            s.name: synth.gradients(n_tokens, s.d_out, synth.seed_for(tag, s.name, "G"),
                                    device=device) for s in wl.sublayers}
        self.si = {s.name: synth.rademacher(s.d_in, synth.seed_for(tag, s.name, "si"),
                                            device=device) for s in wl.sublayers}
        self.so = {s.name: synth.rademacher(s.d_out, synth.seed_for(tag, s.name, "so"),
                                            device=device) for s in wl.sublayers}
        self.hx = {name: torch.zeros(d, d, device=device) for name, d in wl.streams().items()}
        # H_G sums, or only their diagonals in the diagonal-only mode
        self.hg = {s.name: torch.zeros((s.d_out,) if hg_diag else (s.d_out, s.d_out),
                                       device=device) for s in wl.sublayers}
        self.results = {}
        self.acc_events = []        # (start, end, flops) of each tensor-core statistics call
        self.diag_events = []       # (start, end, bytes) of each diagonal-only H_G call
        self.bits = None
        self.streams = None         # one stream per sublayer for the per-sublayer steps
        self.use_graphs = True
        self.overlap = False        # per-sublayer chains alongside the statistics (see step)
        self.reserve = 16           # SMs kept free of statistics while overlapping

    def input_bytes(self):
        tot = 0
        xfp = list(self.xfp.values()) if self.xfp else []
        for t in list(self.x.values()) + xfp + list(self.g.values()) + list(self.w.values()):
            tot += t.numel() * t.element_size()
        return tot

    def inputs(self):
        """(kind, stream or sublayer name, device tensor) of every calibration input: X~, X (drift
        workloads) and G."""
        out = [("x", k, v) for k, v in self.x.items()]
        if self.xfp:
            out += [("xfp", k, v) for k, v in self.xfp.items()]
        out += [("g", k, v) for k, v in self.g.items()]
        return out

    def step(self, time_acc=False):
        import torch

        from post_quantization_b200 import kronq as K
        from post_quantization_b200 import pipeline as P
        wl = self.wl
        x, g = self.x, self.g
        if not self.use_graphs:
            self.results = {}       # eager phases allocate new outputs: drop the last step's
        if self.overlap:
            self._step_overlapped(time_acc=time_acc)
            return
        for name, h in self.hx.items():
            h.zero_()
            if self.drift:
                self.dxx[name].zero_()
            if time_acc:
                e0 = torch.cuda.Event(enable_timing=True); e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
            P.accumulate(xq=x[name], xfp=self.xfp[name] if self.drift else None, hx_sum=h,
                         dxx_sum=self.dxx[name] if self.drift else None, ws=self.ws)
            if time_acc:
                e1.record()
                d = h.shape[0]
                # N d(d+1) for H_X (one triangle), 2 N d^2 for D
                self.acc_events.append((e0, e1, self.n * d * (d + 1)
                                        + (2 * self.n * d * d if self.drift else 0)))
        for s in wl.sublayers:
            h = self.hg[s.name]
            h.zero_()
            self._hg_sum(time_acc, g[s.name], h)
        inv_n = 1.0 / self.n
        if self.streams is None:
            # the per-sublayer phases (BiIP; inverse factor + column solve) run side by side on
            # one stream per sublayer, each phase captured once as a CUDA graph and replayed
            # (or enqueued eagerly every step when graphs are off)
            self.streams = P.SublayerStreams(len(wl.sublayers), self.dev)
            jobs = [(self.w[s.name], self.hx[s.x_stream], self.hg[s.name],
                     self.dxx[s.x_stream] if self.drift else None, inv_n,
                     self.si[s.name], self.so[s.name], self.biip_flags) for s in wl.sublayers]
            self.biip_phase = (P.CapturedPhase(lambda: self.streams.biip(jobs))
                               if self.use_graphs else (lambda: self.streams.biip(jobs)))
            self.solve_phases = {}
            self.solve_res = None
        res = self.biip_phase()
        for s, r in zip(wl.sublayers, res):
            self.results[s.name] = r
        tr = torch.stack([self.results[s.name].tr for s in wl.sublayers]).cpu()
        choices = wl.extra.get("choices", (wl.bits,))
        avg = wl.extra.get("avg_bits", float(wl.bits))
        _, self.bits = K.kronq_score_allocate(tr[:, 0].tolist(), tr[:, 1].tolist(),
                                              [s.d_out * s.d_in for s in wl.sublayers], choices,
                                              avg)
        if self.solve_res is not res:       # a new BiIP output set: new solve graphs
            self.solve_res = res
            self.solve_phases = {}
        if not self.use_graphs:
            self.streams.solve(res, list(self.bits), 0.01)
            return
        key = tuple(self.bits)
        if key not in self.solve_phases:
            bits = list(self.bits)
            self.solve_phases[key] = P.CapturedPhase(
                lambda: self.streams.solve(res, bits, 0.01))
        self.solve_phases[key]()

    def step_streamed(self, host, copy_stream):
        """One step with the inputs in page-locked host memory, as a user with host data runs it.

        host[(kind, name)] is the host copy of the device input of the same key (see inputs()).
        Every copy goes over the host link on `copy_stream`, one tensor at a time, in the order
        the overlapped step consumes them (longest inverse-factor chain first); each statistic
        waits only for its own inputs.
        """
        import torch
        main = torch.cuda.current_stream()
        dev = {(kind, name): t for kind, name, t in self.inputs()}
        landed = {}
        copy_stream.wait_stream(main)
        for key in self._consumption_order():
            with torch.cuda.stream(copy_stream):
                dev[key].copy_(host[key], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(copy_stream)
            landed[key] = ev
        self._step_overlapped(landed=landed)

    def _chain_order(self):
        subs = self.wl.sublayers
        return sorted(range(len(subs)),
                      key=lambda i: -(subs[i].d_in ** 3 + 128 * subs[i].d_out * subs[i].d_in))

    def _consumption_order(self):
        subs = self.wl.sublayers
        seq, seen = [], set()
        for i in self._chain_order():
            if subs[i].x_stream not in seen:
                seen.add(subs[i].x_stream)
                seq.append(("x", subs[i].x_stream))
                if self.drift:
                    seq.append(("xfp", subs[i].x_stream))
            seq.append(("g", subs[i].name))
        return seq

    def _step_overlapped(self, landed=None, time_acc=False):
        """Statistics, sublayer by sublayer (longest inverse-factor chain first), on all but
        `reserve` SMs; as soon as a sublayer's sums are complete its BiIP and inverse factor
        start on its own stream (a captured graph sized to the reserved SMs), alongside the
        remaining statistics. The bit allocation needs every sublayer's traces; the column
        solves follow it on the whole GPU."""
        import torch

        from post_quantization_b200 import kronq as K
        from post_quantization_b200 import pipeline as P
        wl = self.wl
        subs = wl.sublayers
        x, g = self.x, self.g
        inv_n = 1.0 / self.n
        main = torch.cuda.current_stream()
        sms = torch.cuda.get_device_properties(self.dev).multi_processor_count
        if getattr(self, "_st", None) is None:
            self._st = {}
            st = self._st
            st["order"] = self._chain_order()
            st["streams"] = [torch.cuda.Stream(device=self.dev) for _ in subs]
            st["ws"] = [P.Workspace(self.dev) for _ in subs]

            # with one bit width the allocation is known before any trace: each sublayer's
            # solve then follows its inverse factor at once, beside the remaining statistics
            st["fixed_bits"] = wl.extra.get("choices", (wl.bits,))
            st["fixed_bits"] = st["fixed_bits"][0] if len(st["fixed_bits"]) == 1 else None

            def chain(i):
                sl = subs[i]
                r = P.biip(self.w[sl.name], self.hx[sl.x_stream], self.hg[sl.name],
                           self.dxx[sl.x_stream] if self.drift else None, inv_n,
                           self.si[sl.name], self.so[sl.name], self.biip_flags, ws=st["ws"][i])
                P.cholinv(r, 0.01, st["ws"][i])
                if st["fixed_bits"] is not None:
                    P.quantize(r, st["fixed_bits"], st["ws"][i])
                return r
            st["chain"] = [P.CapturedPhase(lambda i=i: chain(i)) if self.use_graphs
                           else (lambda i=i: chain(i)) for i in range(len(subs))]
            st["solve"] = {}
            st["solve_res"] = None
        st = self._st
        if not self.use_graphs:
            self.results = {}       # eager chains allocate new outputs: drop the last step's
        res = [None] * len(subs)
        done = set()
        acc_budget = sms - self.reserve if self.reserve > 0 else 0
        for i in st["order"]:
            sl = subs[i]
            K.kronq_set_sm_budget(acc_budget)
            if sl.x_stream not in done:
                done.add(sl.x_stream)
                if landed is not None:
                    main.wait_event(landed[("x", sl.x_stream)])
                    if self.drift:
                        main.wait_event(landed[("xfp", sl.x_stream)])
                h = self.hx[sl.x_stream]
                h.zero_()
                if self.drift:
                    self.dxx[sl.x_stream].zero_()
                self._timed_acc(time_acc, h.shape[0], self.drift, lambda: P.accumulate(
                    xq=x[sl.x_stream], xfp=self.xfp[sl.x_stream] if self.drift else None,
                    hx_sum=h, dxx_sum=self.dxx[sl.x_stream] if self.drift else None, ws=self.ws))
            if landed is not None:
                main.wait_event(landed[("g", sl.name)])
            h = self.hg[sl.name]
            h.zero_()
            self._hg_sum(time_acc, g[sl.name], h)
            s_i = st["streams"][i]
            s_i.wait_stream(main)
            K.kronq_set_sm_budget(self.reserve)
            with torch.cuda.stream(s_i):
                res[i] = st["chain"][i]()
        K.kronq_set_sm_budget(0)
        for s_i in st["streams"]:
            main.wait_stream(s_i)
        for sl, r in zip(subs, res):
            self.results[sl.name] = r
        tr = torch.stack([r.tr for r in res]).cpu()
        choices = wl.extra.get("choices", (wl.bits,))
        avg = wl.extra.get("avg_bits", float(wl.bits))
        _, self.bits = K.kronq_score_allocate(tr[:, 0].tolist(), tr[:, 1].tolist(),
                                              [sl.d_out * sl.d_in for sl in subs], choices, avg)
        bits = list(self.bits)
        if st["fixed_bits"] is not None:
            return                  # every sublayer was solved in its chain

        def solve():
            for j in st["order"]:
                s_j = st["streams"][j]
                s_j.wait_stream(torch.cuda.current_stream())
                with torch.cuda.stream(s_j):
                    P.quantize(res[j], bits[j], st["ws"][j])
            for s_j in st["streams"]:
                torch.cuda.current_stream().wait_stream(s_j)
        if not self.use_graphs:
            solve()
            return
        if st["solve_res"] != [id(r) for r in res]:     # new chain outputs: new solve graphs
            st["solve_res"] = [id(r) for r in res]
            st["solve"] = {}
        key = tuple(bits)
        if key not in st["solve"]:
            st["solve"][key] = P.CapturedPhase(solve)
        st["solve"][key]()

    def _hg_sum(self, time_acc, g, h):
        """H_G += G^T G (tensor cores), or its diagonal alone in the diagonal-only mode."""
        import torch

        from post_quantization_b200 import pipeline as P
        if self.hg_diag:
            fn = lambda: P.accumulate_diag(g, h, ws=self.ws)
        else:
            fn = lambda: P.accumulate(g=g, hg_sum=h, ws=self.ws)
        if not time_acc:
            fn()
            return
        e0 = torch.cuda.Event(enable_timing=True); e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        if self.hg_diag:
            self.diag_events.append((e0, e1, g.numel() * g.element_size()))
        else:
            d = h.shape[0]
            self.acc_events.append((e0, e1, self.n * d * (d + 1)))

    def _timed_acc(self, time_acc, d, drift, fn):
        import torch
        if not time_acc:
            fn()
            return
        e0 = torch.cuda.Event(enable_timing=True); e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        # N d(d+1) for a symmetric sum (one triangle), 2 N d^2 for D
        self.acc_events.append((e0, e1, self.n * d * (d + 1) + (2 * self.n * d * d if drift else 0)))


def describe(wl, n_tok):
    """The workload in words: shapes, tokens, grid, BiIP, asymmetric term."""
    shapes = {}
    for s in wl.sublayers:
        shapes.setdefault(f"{s.d_out}x{s.d_in}", []).append(s.name.replace("_proj", ""))
    parts = ", ".join(f"{'/'.join(v)} {k}" for k, v in shapes.items())
    drift = "drift term off" if wl.drift == "none" else \
        f"drift term on (X~ = X + noise {wl.drift})"
    name = {"llama2_7b_block": "LLaMA-2-7B", "llama3_8b_block": "LLaMA-3-8B",
            "llama3_70b_block": "LLaMA-3-70B"}.get(wl.name, wl.name)
    return (f"{name}-shaped block: {parts}; {n_tok} tokens; {wl.bits}-bit per-channel grid; "
            f"BiIP on; {drift}")


def run_gpu(args):
    import torch
    import torch.distributed as dist

    from post_quantization_b200 import build
    from post_quantization_b200 import kronq as K
    from post_quantization_b200 import pipeline as P
    from post_quantization_b200 import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=600))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    K.load_library()
    K.kronq_device_check()

    wl = synth.WORKLOADS[args.workload]
    n_tok = args.tokens or wl.n_tokens
    ws = P.Workspace(dev)
    blk = Block(wl, rank, dev, n_tok, ws, calibration=args.calibration, hg_diag=args.hg_diag)
    graphs = args.graphs
    if args.no_graphs:
        graphs = "off"
    blk.use_graphs = graphs == "on" or (graphs == "auto" and blk.input_bytes() < 60e9)
    blk.overlap = args.overlap > 0 or args.schedule == "overlapped"
    blk.reserve = args.overlap
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        blk.step()
    barrier()
    assert K.kronq_device_error() == 0

    clocks = ClockSampler(local)
    clocks.start()
    launches0 = K.kronq_launch_count() + P.replayed_launches()
    barrier()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record()
    for _ in range(args.steps):
        blk.step(time_acc=True)
    t_end.record()
    barrier()
    clk = clocks.stop()
    launches = K.kronq_launch_count() + P.replayed_launches() - launches0
    elapsed = t_start.elapsed_time(t_end) / 1e3
    acc_ms = [a.elapsed_time(b) for a, b, _ in blk.acc_events]
    acc_flops = [f for _, _, f in blk.acc_events]
    diag = None
    if blk.diag_events:
        d_s = sum(a.elapsed_time(b) for a, b, _ in blk.diag_events) / 1e3
        diag = {"kernel": "diag_partial_kernel (+ diag_finalize_kernel)",
                "achieved_gbs": sum(nb for _, _, nb in blk.diag_events) / d_s / 1e9,
                "basis": "bytes of G read / CUDA-event time of the diagonal-sum calls",
                "ms_per_step": d_s * 1e3 / args.steps}
    scores = {sl.name: float(blk.results[sl.name].tr[0] * blk.results[sl.name].tr[1])
              for sl in wl.sublayers if sl.name in blk.results}
    from post_quantization_b200 import dist as D
    elapsed_max = D.max_over_ranks(elapsed, device=dev)
    params = wl.params_per_block * world
    value = params * args.steps / elapsed_max

    # ---- end to end: host inputs (page-locked), host->device copies and the result read-back
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(blk, args, world, dist if world > 1 else None, barrier)

    result = None
    if rank == 0:
        import json as _json
        peaks = {}
        pp = os.path.join(ROOT, "MEASURED_PEAKS.json")
        if os.path.exists(pp):
            peaks = _json.load(open(pp))
        peak = peaks.get("bf16_tflops_sustained")
        peak_src = "measured (sustained bf16)"
        if not peak:
            peak = 1400.0
            peak_src = "fallback (sustained bf16)"
        acc_tflops = sum(acc_flops) / (sum(acc_ms) / 1e3) / 1e12
        # the captures cover the full-H_G step only (the diagonal mode has other launches)
        traffic = None if args.hg_diag else TRAFFIC.get((args.workload, n_tok))
        result = {
            "metric": "quantized weight params/s (BiIP+GPTAQ solve); H_X/H_G accumulate TFLOP/s",
            "value": value,
            "unit": "params/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": elapsed_max / args.steps * 1e3,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16 statistics (fp16 drift operands), fp32 solve",
            "data": "synthetic (seeded LLaMA-shaped activations, gradients and weights)",
            "config": {"workload": describe(wl, n_tok),
                       "tokens": n_tok, "params_per_block": wl.params_per_block,
                       "parallelism": f"one block per GPU x{world}",
                       "graphs": blk.use_graphs,
                       "schedule": ("overlapped" + (f", {blk.reserve} SMs reserved"
                                                    if blk.reserve else "")
                                    if blk.overlap else "phases"),
                       "calibration": ("X and G from the forward and backward of a random-weight "
                                       "block" if args.calibration == "backward" else
                                       "seeded synthetic X and G"),
                       "hg": "diagonal only" if args.hg_diag else "full G^T G",
                       "l2": f"inputs ({blk.input_bytes() / 1e9:.0f} GB) larger than L2"},
            "accumulate_tflops": acc_tflops,
            "roofline": {"bound": "tensor", "kernel": "accumulate_tc_kernel",
                         "achieved": acc_tflops, "peak": peak, "unit": "TFLOP/s",
                         "frac": acc_tflops / peak, "peak_source": peak_src,
                         "achieved_basis": "algorithmic flops of the statistics calls (N d(d+1) "
                                           "per symmetric sum, 2 N d^2 per drift sum) / their "
                                           "CUDA-event time",
                         "traffic": traffic, "traffic_unit": "bytes per launch"},
            "gpu_launches": launches,
            "clocks": clk,
            "e2e": e2e,
            "scores": scores,
        }
        if diag is not None:
            hbm = peaks.get("hbm_gbs") or 6650.0
            diag.update({"peak_gbs": hbm, "frac": diag["achieved_gbs"] / hbm})
            result["hg_diag"] = diag
        if not args.no_cpu_baseline:
            samples = [oracle_sample(args.workload) for _ in range(3)]
            est = statistics.mean(e for e, _, _ in samples)
            rec = samples[-1][1]
            spent = sum(sp for _, _, sp in samples)
            model, nproc, threads = cpu_info()
            result["cpu_baseline"] = {
                "value": wl.params_per_block / est, "unit": "params/s", "cores": threads,
                "kind": "oracle",
                "value_kind": "estimate: the block's work per stage / the oracle's measured "
                              "rate per stage (rates measured on the sample)",
                "sample": (f"fp64 oracle on a {PROXY_D}x{PROXY_D} sublayer, {PROXY_TOKENS} "
                           f"tokens: statistics, BiIP, inverse factor"
                           + (", P" if blk.drift else "") +
                           f", column solve of {PROXY_ROWS} rows; 3 samples, {spent:.1f} s"),
                "rates": rec, "cpu_model": model, "nproc": nproc,
                "layer256_full_s": oracle_layer256()}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


# DRAM bytes (read + write) per accumulate_tc_kernel launch, averaged over the launches of one
# step: bounded ncu captures of this kernel version scaled to the step's launches (commands and
# scaling in the accumulate profile summaries under profiles/); keyed by (workload, tokens)
TRAFFIC = {("llama3_70b_block", 262144): 24.7e9}


def _mem_available():
    """Host memory this process may still use: MemAvailable, capped by the container's memory
    limit (cgroup v2 memory.max - memory.current, or v1 limit - usage) when there is one."""
    avail = None
    try:
        with open("/proc/meminfo") as f:
            for line in f:
                if line.startswith("MemAvailable:"):
                    avail = int(line.split()[1]) * 1024
    except OSError:
        pass
    for lim_f, use_f in (("/sys/fs/cgroup/memory.max", "/sys/fs/cgroup/memory.current"),
                         ("/sys/fs/cgroup/memory/memory.limit_in_bytes",
                          "/sys/fs/cgroup/memory/memory.usage_in_bytes")):
        try:
            lim = open(lim_f).read().strip()
            use = int(open(use_f).read().strip())
        except (OSError, ValueError):
            continue
        if lim.isdigit() and int(lim) < (1 << 60):
            room = int(lim) - use
            avail = room if avail is None else min(avail, room)
        break
    return avail


def run_e2e(blk, args, world, dist, barrier):
    """Same step through the same API, the inputs starting in page-locked host memory every
    step: every X~, X and G tensor is copied to the device inside the timed region, and the
    codes and grid of every sublayer are read back."""
    import torch
    # the streamed step runs the overlapped phases with their own outputs and workspaces: free
    # the resident step's first (the LLaMA-3-70B block does not hold both sets)
    blk.results = {}
    blk.streams = None
    blk.biip_phase = None
    blk.solve_phases = {}
    blk.solve_res = None
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    items = blk.inputs()
    sizes = [t.numel() * t.element_size() for _, _, t in items]
    total = sum((sz + 4095) // 4096 * 4096 for sz in sizes)
    avail = _mem_available()
    # host copies of the inputs, each page-locked by registration (the pinned-tensor allocator
    # would round every tensor up to a power of two)
    if avail is not None and total > avail - 24e9:
        return {"value": None, "unit": "params/s",
                "skipped": f"needs {total / 1e9:.0f} GB of page-locked host memory, "
                           f"{avail / 1e9:.0f} GB available"}
    cudart = torch.cuda.cudart()
    registered = []
    try:
        host = {}
        for (kind, name, t), sz in zip(items, sizes):
            h = torch.empty(t.shape, dtype=t.dtype)
            rc = cudart.cudaHostRegister(h.data_ptr(), sz, 0)
            if int(rc) != 0:
                return {"value": None, "unit": "params/s",
                        "skipped": f"cudaHostRegister failed ({rc})"}
            registered.append(h)
            h.copy_(t)
            host[(kind, name)] = h
        pinned = all(h.is_pinned() for h in host.values())
        h2d = sum(sizes)
        # the device copies are written by every streamed step (same shapes, same addresses)
        copy_stream = torch.cuda.Stream(device=blk.dev)
        outs = None

        def one():
            nonlocal outs
            blk.step_streamed(host, copy_stream)
            if outs is None:
                outs = []
                for sl in blk.wl.sublayers:
                    r = blk.results[sl.name]
                    outs += [torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                             for t in (r.codes, r.scale, r.zero)]
            k = 0
            for sl in blk.wl.sublayers:
                r = blk.results[sl.name]
                for t in (r.codes, r.scale, r.zero):
                    outs[k].copy_(t, non_blocking=True)
                    k += 1
            torch.cuda.current_stream().synchronize()

        for _ in range(2):          # first step allocates and (with graphs) captures
            one()
        barrier()
        steps = max(2, min(args.steps, 10))
        e0 = torch.cuda.Event(enable_timing=True); e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            one()
        e1.record()
        barrier()
        el = e0.elapsed_time(e1) / 1e3
        d2h = sum(o.numel() * o.element_size() for o in outs)
        t = torch.tensor([el], dtype=torch.float64, device=blk.dev)
        if dist is not None:
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
        value = blk.wl.params_per_block * world * steps / float(t)
        return {"value": value, "unit": "params/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": steps,
                "ms_per_step": float(t) / steps * 1e3,
                "host_inputs": "registered (page-locked) host tensors" if pinned else
                               "registered buffer not reported page-locked: staged copies"}
    finally:
        torch.cuda.synchronize()
        for h in registered:
            cudart.cudaHostUnregister(h.data_ptr())


# ---------------------------------------------------------------------------------- stack

def run_stack(args):
    """The mixed-precision stack: 32 LLaMA-2-7B-shaped blocks (224 sublayers, 6.5B weights),
    every sublayer with its own X and G (65536 tokens; per-block G scale log-uniform on
    [1e-2, 1e1]). One step: statistics and BiIP of every sublayer, the traces of all 224 to the
    host (gathered over ranks), one {2,3,4}-bit allocation at 2.5 average bits over the whole
    stack, then the inverse factor and column solve of every sublayer with its width.

    Blocks are split over ranks (strong scaling). The stack's calibration inputs (330 GB) do not
    fit in device memory, so each sublayer's X and G are generated on the device just before its
    statistics; the timed intervals (CUDA events on the one stream that runs everything) cover
    the library calls only, and the step time is their sum.
    """
    import torch
    import torch.distributed as dist

    from post_quantization_b200 import build
    from post_quantization_b200 import dist as D
    from post_quantization_b200 import kronq as K
    from post_quantization_b200 import pipeline as P
    from post_quantization_b200 import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=600))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    K.load_library()
    K.kronq_device_check()

    wl = synth.WORKLOADS["llama2_7b_stack"]
    n = args.tokens or wl.n_tokens
    subs = wl.sublayers
    lo, hi = wl.extra["g_block_multiplier_log10"]
    blocks = D.shard(wl.n_blocks, rank, world)
    sizes = [s.d_out * s.d_in for _ in range(wl.n_blocks) for s in subs]
    owned = [b * len(subs) + j for b in blocks for j in range(len(subs))]
    w, si, so, mult = {}, {}, {}, {}
    for b in blocks:
        mult[b] = synth.block_g_multiplier(b, lo, hi, synth.seed_for(wl.name))
        for j, sl in enumerate(subs):
            tag = (wl.name, b, sl.name)
            i = b * len(subs) + j
            w[i] = synth.weight(sl.d_out, sl.d_in, synth.seed_for(tag, "W"), device=dev)
            si[i] = synth.rademacher(sl.d_in, synth.seed_for(tag, "si"), device=dev)
            so[i] = synth.rademacher(sl.d_out, synth.seed_for(tag, "so"), device=dev)
    ws = P.Workspace(dev)
    streams = P.SublayerStreams(len(subs), dev)
    state = {"bits": None}

    def step():
        timed = []
        res = {}

        def timed_call(fn):
            e0 = torch.cuda.Event(enable_timing=True); e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            out = fn()
            e1.record()
            timed.append((e0, e1))
            return out

        for b in blocks:
            for j, sl in enumerate(subs):
                i = b * len(subs) + j
                tag = (wl.name, b, sl.name)
                x = synth.correlated_x(n, sl.d_in, synth.seed_for(tag, "X"), device=dev)
                g = synth.gradients(n, sl.d_out, synth.seed_for(tag, "G"), device=dev,
                                    multiplier=mult[b])
                hx = torch.zeros(sl.d_in, sl.d_in, device=dev)
                hg = torch.zeros(sl.d_out, sl.d_out, device=dev)

                def stats_and_biip():
                    P.accumulate(xq=x, g=g, hx_sum=hx, hg_sum=hg, ws=ws)
                    return P.biip(w[i], hx, hg, None, 1.0 / n, si[i], so[i], K.BIIP_FULL,
                                  ws=ws, copy_hx=False)
                res[i] = timed_call(stats_and_biip)
                del x, g, hg

        def allocate_and_solve():
            tr = torch.stack([res[i].tr for i in owned]).cpu()
            local_tr = {i: (float(tr[k, 0]), float(tr[k, 1])) for k, i in enumerate(owned)}
            _, bits = P.allocate_global(local_tr, sizes, wl.extra["choices"],
                                        wl.extra["avg_bits"], device=dev)
            state["bits"] = bits
            for b in blocks:
                idx = [b * len(subs) + j for j in range(len(subs))]
                streams.solve([res[i] for i in idx], [bits[i] for i in idx], 0.01)
        timed_call(allocate_and_solve)
        return timed, res

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    barrier()
    assert K.kronq_device_error() == 0
    clocks = ClockSampler(local)
    clocks.start()
    launches0 = K.kronq_launch_count()
    total_s = 0.0
    for _ in range(args.steps):
        timed, res = step()
        torch.cuda.synchronize()
        total_s += sum(a.elapsed_time(b) for a, b in timed) / 1e3
        del res
    barrier()
    clk = clocks.stop()
    launches = K.kronq_launch_count() - launches0
    t_max = D.max_over_ranks(total_s, device=dev)
    params = sum(sizes)
    bits = state["bits"]
    hist = {str(b): sum(1 for v in bits if v == b) for b in sorted(set(bits))}
    avg = sum(b * s for b, s in zip(bits, sizes)) / params
    result = None
    if rank == 0:
        result = {
            "metric": "quantized weight params/s (BiIP+GPTAQ solve); H_X/H_G accumulate TFLOP/s",
            "value": params * args.steps / t_max, "unit": "params/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t_max / args.steps * 1e3, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16 statistics, fp32 solve",
            "data": "synthetic (seeded LLaMA-shaped activations, gradients and weights)",
            "config": {"workload": f"mixed-precision stack: {wl.n_blocks} LLaMA-2-7B-shaped "
                                   f"blocks, {len(sizes)} sublayers, {params} weights, own X "
                                   f"and G per sublayer, {n} tokens, {{2,3,4}} bits at "
                                   f"{wl.extra['avg_bits']} average; BiIP on; drift term off",
                       "parallelism": f"blocks split over {world} GPU(s)",
                       "timing": "sum of CUDA-event intervals around the library calls; the "
                                 "per-sublayer input generation between them is not timed",
                       "l2": "inputs larger than L2"},
            "allocation": {"bits_histogram": hist, "average_bits": avg},
            "gpu_launches": launches, "clocks": clk,
            "e2e": {"value": None, "unit": "params/s",
                    "skipped": "the stack's 330 GB of calibration inputs exceed host memory"},
        }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


# ---------------------------------------------------------------------------------- reference

def run_reference(args):
    """The oracle as it stands on the host cores, one bounded sample per step (oracle_sample):
    value = the block estimate from the measured stage rates; ms_per_step = the measured time
    of one sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    from post_quantization_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    ests, spents = [], []
    rec = {}
    for i in range(args.warmup + args.steps):
        est, rec, spent = oracle_sample(args.workload)
        if i >= args.warmup:
            ests.append(est)
            spents.append(spent)
    est = statistics.mean(ests)
    value = wl.params_per_block / est
    model, nproc, threads = cpu_info()
    sample = (f"fp64 oracle on a {PROXY_D}x{PROXY_D} sublayer, {PROXY_TOKENS} tokens: "
              f"statistics, BiIP, inverse factor" + (", P" if wl.drift != "none" else "") +
              f", column solve of {PROXY_ROWS} rows, per step")
    return {
        "impl": "reference",
        "metric": "quantized weight params/s (BiIP+GPTAQ solve); H_X/H_G accumulate TFLOP/s",
        "value": value, "unit": "params/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": statistics.mean(spents) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded LLaMA-shaped activations, gradients and weights)",
        "config": {"workload": describe(wl, wl.n_tokens)},
        "value_kind": "estimate: the block's work per stage / the oracle's measured rate per "
                      "stage; ms_per_step is the measured time of one sample",
        "estimated_s_per_block": est,
        "cpu_baseline": {"value": value, "unit": "params/s", "cores": threads, "kind": "oracle",
                         "sample": sample, "rates": rec, "cpu_model": model, "nproc": nproc},
        "e2e": {"value": value, "unit": "params/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    if args.impl == "reference":
        res = run_reference(args)
    elif args.workload == "llama2_7b_stack":
        res = run_stack(args)
    else:
        res = run_gpu(args)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
