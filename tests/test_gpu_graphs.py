"""Per-sublayer phases replayed as CUDA graphs give the same results as eager calls.

The column solve and the inverse factor are deterministic (no atomics), so a replayed solve
must reproduce an eager solve of the same BiIP outputs bit for bit; the BiIP phase (fp64
atomics in its norm sums) is compared at 1e-6.
"""
import pytest
import torch

from post_quantization_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    from post_quantization_b200 import build
    build.build()
    from post_quantization_b200 import kronq
    kronq.load_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    kronq.kronq_device_check()
    return kronq


@pytest.fixture(scope="module")
def P(K):
    from post_quantization_b200 import pipeline
    return pipeline


def _clone(P, r):
    return P.SublayerResult(r.w_prime.clone(), r.hx.clone(), r.s_x.clone(), r.s_g.clone(),
                            r.tr.clone(), None if r.dxx is None else r.dxx.clone(),
                            torch.empty_like(r.info))


def test_captured_phases_match_eager(K, P):
    # three sublayers of different shapes (one ragged, one with the drift term), 2048 tokens
    shapes = [(256, 384, False), (384, 256, True), (200, 520, False)]
    n = 2048
    dev = torch.device("cuda", 0)
    jobs = []
    for i, (d_out, d_in, drift) in enumerate(shapes):
        tag = ("graphs", i)
        x = synth.correlated_x(n, d_in, synth.seed_for(tag, "X"), device=dev)
        xq = synth.perturbed(x, synth.seed_for(tag, "Xq"), abs_std=0.01) if drift else x
        g = synth.gradients(n, d_out, synth.seed_for(tag, "G"), device=dev)
        w = synth.weight(d_out, d_in, synth.seed_for(tag, "W"), device=dev)
        si = synth.rademacher(d_in, synth.seed_for(tag, "si"), device=dev)
        so = synth.rademacher(d_out, synth.seed_for(tag, "so"), device=dev)
        hx = torch.zeros(d_in, d_in, device=dev)
        hg = torch.zeros(d_out, d_out, device=dev)
        dxx = torch.zeros(d_in, d_in, device=dev) if drift else None
        K.kronq_accumulate(xq, x if drift else None, g, hx, hg, dxx)
        jobs.append((w, hx, hg, dxx, 1.0 / n, si, so, K.BIIP_FULL))
    torch.cuda.synchronize()
    bits = [2, 4, 3]

    eager = [P.biip(*j) for j in jobs]
    streams = P.SublayerStreams(len(jobs), dev)
    biip_phase = P.CapturedPhase(lambda: streams.biip(jobs))
    res = None
    for _ in range(3):
        res = biip_phase()
    torch.cuda.synchronize()
    assert biip_phase.graph is not None and biip_phase.launches > 0
    for r, e in zip(res, eager):
        for a, b in ((r.w_prime, e.w_prime), (r.hx, e.hx), (r.s_x, e.s_x), (r.s_g, e.s_g)):
            assert torch.allclose(a, b, rtol=1e-6, atol=0)

    solve_phase = P.CapturedPhase(lambda: streams.solve(res, bits, 0.01))
    before = P.replayed_launches()
    for _ in range(3):
        biip_phase()                   # fresh H_X' for the in-place factor
        torch.cuda.synchronize()
        snap = [_clone(P, r) for r in res]
        solve_phase()
    torch.cuda.synchronize()
    assert solve_phase.launches > 0
    assert P.replayed_launches() - before == 3 * biip_phase.launches + solve_phase.launches
    for r, s, b in zip(res, snap, bits):
        P.cholinv(s, 0.01)
        P.quantize(s, b)
        torch.cuda.synchronize()
        assert int(s.info.item()) < 0
        assert torch.equal(r.hx, s.hx)
        assert torch.equal(r.codes, s.codes)
        assert torch.equal(r.scale, s.scale) and torch.equal(r.zero, s.zero)
        assert torch.equal(r.w_hat, s.w_hat)
    assert K.kronq_device_error() == 0
