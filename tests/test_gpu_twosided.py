"""Comparison variant: rounding with output-side feedback too, CUDA path vs the fp64 oracle.

[YAQA notes], generalized LDLQ: the fixed point W^ = Q(W + L_O'^T D L_I' + L_O'^T D + D L_I')
with H_O = H_G' and H_I = H_X'. Bars: the oracle runs in follow mode (it adopts the GPU's code
only within 1e-3 grid units of a rounding boundary) and must then agree on every code, with
disagreements on at most 0.1% of entries; W^ within 1e-3 relative Frobenius. With a diagonal
H_O the output-side terms vanish and the codes must be those of KronQ's column solve.
"""
import numpy as np
import pytest
import torch

from oracle import kronq_oracle as O
from post_quantization_b200 import synth

pytestmark = pytest.mark.gpu

TOL = 1e-3


@pytest.fixture(scope="module")
def K():
    from post_quantization_b200 import build
    build.build()
    from post_quantization_b200 import kronq
    kronq.load_library()
    kronq.kronq_device_check()
    return kronq


def rel(a, b):
    a = np.asarray(a, dtype=np.float64); b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def h64(t):
    return t.detach().double().cpu().numpy()


def padded(t):
    """Same values in storage whose row stride is a multiple of 8 elements (16 bytes), as the
    statistics call requires of its bf16 inputs."""
    c = t.shape[1]
    if c % 8 == 0:
        return t
    base = torch.zeros(t.shape[0], (c + 7) // 8 * 8, dtype=t.dtype, device=t.device)
    base[:, :c] = t
    return base[:, :c]


def layer(K, d_out, d_in, n, tag):
    """W', H_X' and the full H_G' of a synthetic layer through the library (fp32 on device)."""
    from post_quantization_b200 import pipeline as P
    x = padded(synth.correlated_x(n, d_in, synth.seed_for(tag, "X"), device="cuda"))
    g = padded(synth.gradients(n, d_out, synth.seed_for(tag, "G"), device="cuda"))
    w = synth.weight(d_out, d_in, synth.seed_for(tag, "W"), dtype=torch.float32, device="cuda")
    si = synth.rademacher(d_in, synth.seed_for(tag, "si"), device="cuda")
    so = synth.rademacher(d_out, synth.seed_for(tag, "so"), device="cuda")
    hx = torch.zeros(d_in, d_in, device="cuda"); hg = torch.zeros(d_out, d_out, device="cuda")
    K.kronq_accumulate(x, None, g, hx, hg)
    r = P.biip(w, hx, hg, None, 1.0 / n, si, so, K.BIIP_FULL | K.BIIP_WRITE_HG)
    hx_p = r.hx.clone(); hg_p = hg.clone()          # H_X' and H_G' (hg was transformed in place)
    P.cholinv(r, 0.01, sync=True)                    # r.hx now holds K_in
    k_out = hg.clone()
    info = torch.empty(1, dtype=torch.int32, device="cuda")
    K.kronq_cholinv(k_out, 0.01, info, K.CHOLINV_SYNC)
    torch.cuda.synchronize()
    return r, hx_p, hg_p, k_out


def check_follow(gpu_codes, o, total):
    mism = int((h64(gpu_codes) != o["codes"]).sum())
    assert mism == 0, f"{mism} codes differ away from rounding boundaries"
    assert int(o["disagree"].sum()) <= 1e-3 * total


@pytest.mark.parametrize("d_out,d_in,bits", [(64, 96, 2), (130, 200, 3), (256, 256, 2),
                                              (96, 520, 4), (300, 136, 2)])
def test_twosided_matches_oracle(K, d_out, d_in, bits):
    n = 2048
    r, hx_p, hg_p, k_out = layer(K, d_out, d_in, n, ("twosided", d_out, d_in))
    codes, scale, zero, w_hat, its = K.kronq_quantize_layer_twosided(r.w_prime, r.hx, k_out, bits)
    torch.cuda.synchronize()
    o = O.yaqa_round(h64(r.w_prime), h64(hg_p), h64(hx_p), bits, follow_codes=h64(codes))
    check_follow(codes, o, d_out * d_in)
    np.testing.assert_array_equal(h64(scale), o["scale"])
    np.testing.assert_array_equal(h64(zero), o["zero"])
    assert rel(h64(w_hat), o["w_hat"]) <= TOL
    assert its <= d_out + d_in
    print(f"{d_out}x{d_in} b{bits}: {its} updates (oracle {o['iterations']}), near-ties "
          f"{int(o['near_tie'].sum())}")


def test_twosided_with_diagonal_output_side_is_the_column_solve(K):
    # H_O diagonal => L_O' = 0: the fixed point is the input-side solve, KronQ's own
    from post_quantization_b200 import pipeline as P
    d_out, d_in, n, bits = 192, 384, 2048, 3
    r, _, _, _ = layer(K, d_out, d_in, n, ("twosided-diag",))
    k_diag = torch.diag(torch.rand(d_out, device="cuda") + 0.5)
    codes, _, _, w_hat, its = K.kronq_quantize_layer_twosided(r.w_prime, r.hx, k_diag, bits)
    P.quantize(r, bits)
    torch.cuda.synchronize()
    same = float((codes == r.codes).double().mean())
    assert same >= 1 - 1e-3, same
    assert rel(h64(w_hat), h64(r.w_hat)) <= TOL


def test_twosided_lowers_the_kronecker_objective(K):
    # the measured contrast: with a strongly non-uniform H_G (four decades of gradient scale),
    # output-side feedback lowers tr[H_G dW H_X dW^T] below the input-side solve's
    from post_quantization_b200 import pipeline as P
    d_out, d_in, n, bits = 256, 256, 4096, 2
    r, hx_p, hg_p, k_out = layer(K, d_out, d_in, n, ("twosided-obj",))
    _, _, _, w_hat2, _ = K.kronq_quantize_layer_twosided(r.w_prime, r.hx, k_out, bits)
    P.quantize(r, bits)
    torch.cuda.synchronize()
    w = h64(r.w_prime)
    o1 = O.objective(w, h64(r.w_hat), h64(hx_p), h64(hg_p))
    o2 = O.objective(w, h64(w_hat2), h64(hx_p), h64(hg_p))
    print(f"objective: column solve {o1:.4g}, two-sided {o2:.4g} ({o2 / o1:.3f})")
    assert o2 < o1
