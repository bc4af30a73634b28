"""The SM budget changes grids, not results.

kronq_set_sm_budget caps the CTAs of the persistent kernels. Every output tile of the
tensor-core GEMMs is computed the same way whichever CTA takes it, so the inverse factor and the
column solve must come out bit for bit the same under any budget.
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


@pytest.mark.parametrize("budget", [1, 16, 100])
def test_budget_does_not_change_results(K, P, budget):
    # a 1536 x 1280 layer: the inverse factor has tensor-core levels (halves above 256 columns)
    d_out, d_in, n = 1536, 1280, 4096
    dev = torch.device("cuda", 0)
    x = synth.correlated_x(n, d_in, synth.seed_for("budget", "X"), device=dev)
    g = synth.gradients(n, d_out, synth.seed_for("budget", "G"), device=dev)
    w = synth.weight(d_out, d_in, synth.seed_for("budget", "W"), device=dev)
    si = synth.rademacher(d_in, synth.seed_for("budget", "si"), device=dev)
    so = synth.rademacher(d_out, synth.seed_for("budget", "so"), device=dev)
    hx = torch.zeros(d_in, d_in, device=dev); hg = torch.zeros(d_out, d_out, device=dev)
    K.kronq_accumulate(x, None, g, hx, hg)
    r0 = P.biip(w, hx, hg, None, 1.0 / n, si, so, K.BIIP_FULL)
    torch.cuda.synchronize()

    def solve(b):
        r = P.SublayerResult(r0.w_prime.clone(), r0.hx.clone(), r0.s_x, r0.s_g, r0.tr, None,
                             torch.empty_like(r0.info))
        K.kronq_set_sm_budget(b)
        try:
            P.cholinv(r, 0.01)
            P.quantize(r, 3)
            torch.cuda.synchronize()
        finally:
            K.kronq_set_sm_budget(0)
        return r

    assert K.kronq_sm_budget() == 0
    full = solve(0)
    capped = solve(budget)
    assert int(full.info.item()) < 0 and int(capped.info.item()) < 0
    assert torch.equal(full.hx, capped.hx)
    assert torch.equal(full.codes, capped.codes)
    assert torch.equal(full.w_hat, capped.w_hat)
    assert K.kronq_device_error() == 0
