"""Orchestration of the KronQ layer path over the C ABI (buffers and call order only).

A sublayer goes through: Kronecker-factor sums -> BiIP -> damped inverse factor -> column
solve; a block or stack adds the trace-product scores and the bit allocation in between. Every
arithmetic step is one of the five library calls; this module only allocates device buffers
with torch and sequences the calls, on the caller's stream or, for the independent sublayers of
a block, on one stream per sublayer (SublayerStreams).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import kronq as K


@dataclass
class SublayerResult:
    w_prime: torch.Tensor     # W' = U S_G W S_X V^T (fp32)
    hx: torch.Tensor          # H_X' (fp32), overwritten by K after cholinv
    s_x: torch.Tensor
    s_g: torch.Tensor
    tr: torch.Tensor          # [tr H_X', tr H_G'] fp64 on device
    dxx: torch.Tensor | None
    info: torch.Tensor
    codes: torch.Tensor | None = None
    scale: torch.Tensor | None = None
    zero: torch.Tensor | None = None
    w_hat: torch.Tensor | None = None


class Workspace:
    """One device scratch buffer, grown on demand and reused by every call on one stream."""

    def __init__(self, device):
        self.device = device
        self.buf = torch.empty(0, dtype=torch.uint8, device=device)

    def get(self, nbytes: int):
        if nbytes == 0:
            return None
        if self.buf.numel() < nbytes + 256:
            self.buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=self.device)
        off = (-self.buf.data_ptr()) % 256
        return self.buf[off:off + nbytes]


def accumulate(xq=None, xfp=None, g=None, hx_sum=None, hg_sum=None, dxx_sum=None, ws=None,
               stream=None):
    n = (xq if xq is not None else g).shape[0]
    d_in = xq.shape[1] if xq is not None else 0
    d_out = g.shape[1] if g is not None else 0
    wsz = K.kronq_accumulate_workspace_size(n, d_in, d_out, dxx_sum is not None)
    K.kronq_accumulate(xq, xfp, g, hx_sum, hg_sum, dxx_sum,
                       workspace=ws.get(wsz) if ws is not None else None, stream=stream)


def accumulate_diag(g, hg_diag_sum, ws=None, stream=None):
    """hg_diag_sum += the diagonal of g^T g (for biip with K.BIIP_HG_DIAG)."""
    wsz = K.kronq_accumulate_diag_workspace_size(g.shape[0], g.shape[1])
    K.kronq_accumulate_diag(g, hg_diag_sum, workspace=ws.get(wsz) if ws is not None else None,
                            stream=stream)


def biip(w, hx_sum, hg_sum, dxx_sum, inv_n, sign_in, sign_out, flags=K.BIIP_FULL, ws=None,
         stream=None, copy_hx=True):
    """Runs kronq_biip on copies of the sums (hx is copied unless copy_hx is False)."""
    dev = w.device
    d_out, d_in = w.shape
    hx = hx_sum.clone() if copy_hx else hx_sum
    dxx = dxx_sum.clone() if dxx_sum is not None else None
    w_out = torch.empty(d_out, d_in, dtype=torch.float32, device=dev)
    s_x = torch.empty(d_in, dtype=torch.float32, device=dev)
    s_g = torch.empty(d_out, dtype=torch.float32, device=dev)
    tr = torch.zeros(2, dtype=torch.float64, device=dev)
    wsz = K.kronq_biip_workspace_size(d_out, d_in)
    K.kronq_biip(w, w_out, hx, hg_sum, dxx, inv_n, sign_in, sign_out, flags, s_x, s_g, tr[0:1],
                 tr[1:2] if hg_sum is not None else None,
                 workspace=ws.get(wsz) if ws is not None else None, stream=stream)
    info = torch.empty(1, dtype=torch.int32, device=dev)
    return SublayerResult(w_out, hx, s_x, s_g, tr, dxx, info)


def cholinv(r: SublayerResult, damp_rel=0.01, ws=None, stream=None, sync=False):
    d = r.hx.shape[0]
    wsz = K.kronq_cholinv_workspace_size(d)
    K.kronq_cholinv(r.hx, damp_rel, r.info, K.CHOLINV_SYNC if sync else 0,
                    workspace=ws.get(wsz) if ws is not None else None, stream=stream)


def quantize(r: SublayerResult, bits: int, ws=None, stream=None, group: int = 0):
    """Column solve of r (K in r.hx). group 0: one grid per row (scale, zero: d_out); group 128:
    one grid per row and per 128 columns (scale, zero: d_out x ceil(d_in / 128))."""
    d_out, d_in = r.w_prime.shape
    dev = r.w_prime.device
    grid_shape = (d_out, (d_in + group - 1) // group) if group else (d_out,)
    if r.codes is None:
        r.codes = torch.empty(d_out, d_in, dtype=torch.uint8, device=dev)
        r.w_hat = torch.empty(d_out, d_in, dtype=torch.float32, device=dev)
    if r.scale is None or tuple(r.scale.shape) != grid_shape:
        r.scale = torch.empty(grid_shape, dtype=torch.float32, device=dev)
        r.zero = torch.empty(grid_shape, dtype=torch.float32, device=dev)
    wsz = K.kronq_quantize_layer_workspace_size(d_out, d_in, 128, r.dxx is not None)
    K.kronq_quantize_layer(r.w_prime, r.hx, r.dxx, bits, r.codes, r.scale, r.zero, r.w_hat,
                           workspace=ws.get(wsz) if ws is not None else None, stream=stream,
                           group=group)


def quantize_sublayer(w, hx_sum, hg_sum, dxx_sum, inv_n, sign_in, sign_out, bits,
                      flags=K.BIIP_FULL, damp_rel=0.01, ws=None, stream=None):
    r = biip(w, hx_sum, hg_sum, dxx_sum, inv_n, sign_in, sign_out, flags, ws, stream)
    cholinv(r, damp_rel, ws, stream)
    quantize(r, bits, ws, stream)
    return r


def allocate_global(local_traces: dict, n_params: list, choices, avg_bits: float, device=None):
    """Bit widths of every sublayer of a stack whose sublayers are spread over ranks.

    local_traces maps a global sublayer index to (tr H_X', tr H_G') for the sublayers this rank
    processed. The traces of all ranks are gathered (dist.gather_traces) and every rank runs
    kronq_score_allocate on the same full list, so every rank gets the same bits.
    Returns (scores, bits) for all len(n_params) sublayers.
    """
    from . import dist as D
    traces = D.gather_traces(local_traces, len(n_params), device=device)
    return K.kronq_score_allocate([a for a, _ in traces], [b for _, b in traces], list(n_params),
                                  choices, avg_bits)


class SublayerStreams:
    """Runs the per-sublayer steps of a block on one CUDA stream per sublayer.

    The sublayers of a block are independent once their statistics exist, and each of their
    kernel chains (BiIP passes, the recursive inverse factor, the column solve) leaves most of
    the GPU idle on its own, so they run side by side. Each stream has its own workspace. Every
    method makes its streams wait for the caller's stream first and makes the caller's stream
    wait for all of them before it returns.
    """

    def __init__(self, count: int, device):
        self.streams = [torch.cuda.Stream(device=device) for _ in range(count)]
        self.ws = [Workspace(device) for _ in range(count)]

    def _fan_out(self, jobs, fn, order=None):
        """Enqueues fn(job, workspace) per job, in `order` (longest chains first, so that they
        start while the host is still enqueueing the rest); returns results in job order."""
        main = torch.cuda.current_stream()
        out = [None] * len(jobs)
        for i in (order if order is not None else range(len(jobs))):
            s = self.streams[i % len(self.streams)]
            s.wait_stream(main)
            with torch.cuda.stream(s):
                out[i] = fn(jobs[i], self.ws[i % len(self.ws)])
        for s in self.streams:
            main.wait_stream(s)
        return out

    def biip(self, jobs):
        """jobs: (w, hx_sum, hg_sum, dxx_sum, inv_n, sign_in, sign_out, flags) per sublayer."""
        return self._fan_out(jobs, lambda j, ws: biip(*j, ws=ws))

    def solve(self, results, bits, damp_rel=0.01):
        def one(job, ws):
            r, b = job
            cholinv(r, damp_rel, ws)
            quantize(r, b, ws)
            return r
        # the inverse factor's chain grows with d_in^3, the solve's with d_out * d_in
        cost = [r.w_prime.shape[1] ** 3 + 128 * r.w_prime.shape[0] * r.w_prime.shape[1]
                for r in results]
        order = sorted(range(len(results)), key=lambda i: -cost[i])
        return self._fan_out(list(zip(results, bits)), one, order)


_replayed_launches = [0]


def replayed_launches() -> int:
    """Library kernel launches issued by CapturedPhase replays so far (the C launch counter
    sees each captured launch once, at capture time)."""
    return _replayed_launches[0]


class CapturedPhase:
    """A sequence of library calls captured as a CUDA graph and replayed.

    A block's per-sublayer phases are thousands of small launches (the inverse factor's
    recursion and the column solve's block loop); replaying them as one graph takes the host
    and the per-launch latency off the critical path. fn must only enqueue device work (no
    synchronisation) and read inputs at fixed addresses. The first call runs fn eagerly (so
    that workspaces and kernel attributes exist before any capture) and returns its result; the
    second call captures fn and replays the graph; later calls only replay. From the second
    call on, the returned tensors live in the graph's pool and every replay overwrites them.
    """

    def __init__(self, fn):
        self.fn = fn
        self.calls = 0
        self.graph = None
        self.out = None
        self.launches = 0

    def __call__(self):
        self.calls += 1
        if self.calls == 1:
            return self.fn()
        if self.graph is None:
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            n0 = K.kronq_launch_count()
            with torch.cuda.graph(g):
                self.out = self.fn()
            self.launches = K.kronq_launch_count() - n0   # counted once, here
            self.graph = g
        else:
            _replayed_launches[0] += self.launches
        self.graph.replay()
        return self.out

    def release(self):
        self.graph = None
        self.out = None
