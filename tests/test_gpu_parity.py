"""CUDA path vs fp64 oracle, element by element, through the C ABI.

Bars (written in each test): relative Frobenius error <= 1e-3 for H_X, H_G, D, W', scales,
traces, K and W^; codes: the oracle runs in follow mode (it adopts the GPU's code only where its
own value lies within 1e-3 grid units of a rounding boundary) and must then agree on every code,
with near-ties <= 0.1% of entries; grid scale/zero bit-exact when both sides see the same W'.
"""
import math

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
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    kronq.kronq_device_check()
    return kronq


@pytest.fixture(scope="module")
def P(K):
    from post_quantization_b200 import pipeline
    return pipeline


def rel(a, b):
    a = np.asarray(a, dtype=np.float64); b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def h64(t):
    return t.detach().double().cpu().numpy()


def padded(t):
    """Same values in storage whose row stride is a multiple of 8 elements (16 bytes)."""
    c = t.shape[1]
    if c % 8 == 0:
        return t
    base = torch.zeros(t.shape[0], (c + 7) // 8 * 8, dtype=t.dtype, device=t.device)
    base[:, :c] = t
    return base[:, :c]


def layer_inputs(d_out, d_in, n, drift="abs0.01", w_dtype=torch.float32, tag="t", dev="cuda"):
    xfp = synth.correlated_x(n, d_in, synth.seed_for(tag, "X"), device=dev)
    if drift == "none":
        xq = xfp
    elif drift.startswith("abs"):
        xq = synth.perturbed(xfp, synth.seed_for(tag, "Xq"), abs_std=float(drift[3:]))
    else:
        xq = synth.perturbed(xfp, synth.seed_for(tag, "Xq"), rel_std=float(drift[3:]))
    g = synth.gradients(n, d_out, synth.seed_for(tag, "G"), device=dev)
    w = synth.weight(d_out, d_in, synth.seed_for(tag, "W"), dtype=w_dtype, device=dev)
    si = synth.rademacher(d_in, synth.seed_for(tag, "si"), device=dev)
    so = synth.rademacher(d_out, synth.seed_for(tag, "so"), device=dev)
    return padded(xq), padded(xfp), padded(g), w, si, so


def gpu_sums(K, xq, xfp, g, with_dxx=True):
    d_in = xq.shape[1]; d_out = g.shape[1]
    hx = torch.zeros(d_in, d_in, device="cuda"); hg = torch.zeros(d_out, d_out, device="cuda")
    dxx = torch.zeros(d_in, d_in, device="cuda") if with_dxx else None
    K.kronq_accumulate(xq, xfp if with_dxx else None, g, hx, hg, dxx)
    torch.cuda.synchronize()
    return hx, hg, dxx


# ------------------------------------------------------------------------------ accumulate

@pytest.mark.parametrize("n,d_in,d_out", [(2048, 256, 256), (1000, 200, 72), (77, 64, 136),
                                          (4100, 384, 520), (64, 8, 16)])
def test_accumulate_matches_oracle(K, n, d_in, d_out):
    xq, xfp, g, *_ = layer_inputs(d_out, d_in, n, tag=("acc", n, d_in, d_out))
    hx, hg, dxx = gpu_sums(K, xq, xfp, g)
    ohx, ohg, odxx = O.accumulate(h64(xq), h64(xfp), h64(g))
    assert rel(h64(hx), ohx) <= TOL
    assert rel(h64(hg), ohg) <= TOL
    assert rel(h64(dxx), odxx) <= TOL
    assert torch.equal(hx, hx.T) and torch.equal(hg, hg.T)
    print("rel err hx %.2e hg %.2e dxx %.2e" % (rel(h64(hx), ohx), rel(h64(hg), ohg),
                                                  rel(h64(dxx), odxx)))


def test_accumulate_is_additive_and_strided(K):
    n, d = 3000, 130
    base = torch.zeros(n, 136, dtype=torch.bfloat16, device="cuda")
    base[:, :d] = synth.correlated_x(n, d, synth.seed_for("strided"), device="cuda")
    x = base[:, :d]                                   # row stride 136, width 130
    h1 = torch.zeros(d, d, device="cuda")
    K.kronq_accumulate(x, None, None, h1)
    h2 = torch.zeros(d, d, device="cuda")
    K.kronq_accumulate(x[:1234], None, None, h2)
    K.kronq_accumulate(x[1234:], None, None, h2)
    torch.cuda.synchronize()
    o = O.accumulate(h64(x))[0]
    assert rel(h64(h1), o) <= TOL and rel(h64(h2), o) <= TOL
    # n = 0 is a no-op
    K.kronq_accumulate(x[:0], None, None, h2)
    torch.cuda.synchronize()
    assert rel(h64(h2), o) <= TOL


@pytest.mark.parametrize("d", [4096, 11008])
def test_accumulate_llama_width_sampled(K, d):
    # LLaMA-2-7B widths (hidden 4096, MLP 11008), 16384 tokens, 16 sampled 128 x 128 tiles
    n = 16384
    x = synth.correlated_x(n, d, synth.seed_for("acc-full", d), device="cuda")
    h = torch.zeros(d, d, device="cuda")
    K.kronq_accumulate(x, None, None, h)
    torch.cuda.synchronize()
    r = np.random.default_rng(d)
    xc = x.float()
    for _ in range(16):
        i0 = int(r.integers(0, d // 128)) * 128; j0 = int(r.integers(0, d // 128)) * 128
        a = xc[:, i0:i0 + 128].double().cpu().numpy(); b = xc[:, j0:j0 + 128].double().cpu().numpy()
        assert rel(h64(h[i0:i0 + 128, j0:j0 + 128]), a.T @ b) <= TOL
    tr = float(np.sum(h64(x) ** 2))
    assert abs(float(torch.trace(h.double())) - tr) <= TOL * tr


@pytest.mark.parametrize("n,d", [(5000, 4096), (3000, 200), (77, 36), (4100, 11008)])
def test_accumulate_diag_matches_oracle(K, n, d):
    # diag(G^T G) in one streaming pass: against the oracle's sums, and against the diagonal of
    # the tensor-core G^T G; "+=" onto a non-zero start; 2048-token blocks with a ragged last one,
    # widths that end part-way through a lane's 8 columns (36, 200)
    g = padded(synth.gradients(n, d, synth.seed_for("diag", n, d), device="cuda"))
    start = torch.rand(d, device="cuda")
    dg = start.clone()
    K.kronq_accumulate_diag(g, dg)
    hg = torch.zeros(d, d, device="cuda")
    K.kronq_accumulate(None, None, g, None, hg)
    torch.cuda.synchronize()
    o = O.accumulate_diag(h64(g))
    assert rel(h64(dg) - h64(start), o) <= TOL
    assert rel(h64(dg) - h64(start), h64(torch.diagonal(hg))) <= TOL
    dg2 = start.clone()
    K.kronq_accumulate_diag(g, dg2)
    torch.cuda.synchronize()
    assert torch.equal(dg, dg2)                      # fixed summation order
    assert K.kronq_device_error() == 0


# ------------------------------------------------------------------------------ biip

def run_biip(K, P, w, hx_sum, hg_sum, dxx_sum, inv_n, si, so, flags):
    r = P.biip(w, hx_sum, hg_sum, dxx_sum, inv_n, si, so, flags)
    torch.cuda.synchronize()
    return r


@pytest.mark.parametrize("flags", [0, 1 | 2, 4 | 8, 15, 15 | 16])
@pytest.mark.parametrize("shape", [(256, 256), (200, 96), (72, 520)])
@pytest.mark.parametrize("w_dtype", [torch.float32, torch.bfloat16])
def test_biip_matches_oracle(K, P, flags, shape, w_dtype):
    d_out, d_in = shape
    n = 1024
    xq, xfp, g, w, si, so = layer_inputs(d_out, d_in, n, w_dtype=w_dtype,
                                         tag=("biip", d_out, d_in))
    hx, hg, dxx = gpu_sums(K, xq, xfp, g)
    hg_in = hg.clone()
    r = run_biip(K, P, w, hx, hg_in, dxx, 1.0 / n, si, so, flags)
    o = O.biip(h64(w), h64(hx), h64(hg), h64(dxx), 1.0 / n, h64(si), h64(so), flags & 15)
    assert rel(h64(r.w_prime), o["w"]) <= TOL
    assert rel(h64(r.hx), o["hx"]) <= TOL
    assert rel(h64(r.dxx), o["dxx"]) <= TOL
    assert rel(h64(r.s_x), o["s_x"]) <= TOL and rel(h64(r.s_g), o["s_g"]) <= TOL
    assert abs(float(r.tr[0]) - o["tr_hx"]) <= TOL * abs(o["tr_hx"])
    assert abs(float(r.tr[1]) - o["tr_hg"]) <= TOL * abs(o["tr_hg"])
    if flags & 16:
        assert rel(h64(hg_in), o["hg"]) <= TOL
    else:
        assert torch.equal(hg_in, hg)          # read-only without WRITE_HG


@pytest.mark.parametrize("d_out,d_in", [(24, 96), (40, 192), (9, 640), (7, 1536), (5, 1024),
                                        (3, 6144), (33, 4096)])
@pytest.mark.parametrize("w_dtype", [torch.float32, torch.bfloat16])
def test_biip_row_block_sizes(K, P, d_out, d_in, w_dtype):
    # every input Hadamard block size of the row pass's tiled kernel (b = 32 .. 4096), with
    # matrices whose row count is not a multiple of the rows a chunk takes (4096 / b)
    n = 256
    xq, xfp, g, w, si, so = layer_inputs(d_out, d_in, n, w_dtype=w_dtype,
                                         tag=("biip-b", d_out, d_in))
    hx, hg, dxx = gpu_sums(K, xq, xfp, g)
    hg_in = hg.clone()
    r = run_biip(K, P, w, hx, hg_in, dxx, 1.0 / n, si, so, 15 | 16)
    o = O.biip(h64(w), h64(hx), h64(hg), h64(dxx), 1.0 / n, h64(si), h64(so), 15)
    assert rel(h64(r.w_prime), o["w"]) <= TOL
    assert rel(h64(r.hx), o["hx"]) <= TOL
    assert rel(h64(r.dxx), o["dxx"]) <= TOL
    assert rel(h64(hg_in), o["hg"]) <= TOL
    assert K.kronq_device_error() == 0


@pytest.mark.parametrize("d_out,d_in", [(4096, 100), (256, 36), (96, 68), (1024, 20),
                                        (2048, 44)])
def test_biip_col_pass_ragged(K, P, d_out, d_in):
    # the column pass over output Hadamard blocks of 32 .. 4096 rows (one pass up to 256, two
    # above), on W widths that end part-way through a 32-column tile; H_G written back
    n = 256
    xq, xfp, g, w, si, so = layer_inputs(d_out, d_in, n, tag=("biip-c", d_out, d_in))
    hx, hg, dxx = gpu_sums(K, xq, xfp, g)
    hg_in = hg.clone()
    r = run_biip(K, P, w, hx, hg_in, dxx, 1.0 / n, si, so, 15 | 16)
    o = O.biip(h64(w), h64(hx), h64(hg), h64(dxx), 1.0 / n, h64(si), h64(so), 15)
    assert rel(h64(r.w_prime), o["w"]) <= TOL
    assert rel(h64(r.hx), o["hx"]) <= TOL
    assert rel(h64(hg_in), o["hg"]) <= TOL
    assert abs(float(r.tr[1]) - o["tr_hg"]) <= TOL * abs(o["tr_hg"])
    assert K.kronq_device_error() == 0


@pytest.mark.parametrize("shape", [(256, 384), (11008, 256)])
def test_biip_with_diagonal_hg(K, P, shape):
    # KRONQ_BIIP_HG_DIAG: only diag(G^T G) from kronq_accumulate_diag; W', H_X', S_G and the
    # traces against the oracle run on that diagonal
    d_out, d_in = shape
    n = 1024
    xq, xfp, g, w, si, so = layer_inputs(d_out, d_in, n, w_dtype=torch.bfloat16,
                                         tag=("biip-diag", d_out, d_in))
    hx = torch.zeros(d_in, d_in, device="cuda")
    K.kronq_accumulate(xq, None, None, hx)
    hgd = torch.zeros(d_out, device="cuda")
    K.kronq_accumulate_diag(g, hgd)
    torch.cuda.synchronize()
    r = run_biip(K, P, w, hx, hgd, None, 1.0 / n, si, so, K.BIIP_FULL | K.BIIP_HG_DIAG)
    o = O.biip(h64(w), h64(hx), np.diag(h64(hgd)), None, 1.0 / n, h64(si), h64(so), 15)
    assert rel(h64(r.w_prime), o["w"]) <= TOL
    assert rel(h64(r.hx), o["hx"]) <= TOL
    assert rel(h64(r.s_g), o["s_g"]) <= TOL and rel(h64(r.s_x), o["s_x"]) <= TOL
    assert abs(float(r.tr[0]) - o["tr_hx"]) <= TOL * abs(o["tr_hx"])
    assert abs(float(r.tr[1]) - o["tr_hg"]) <= TOL * abs(o["tr_hg"])
    assert K.kronq_device_error() == 0


def test_biip_llama_gate_shape(K, P):
    # gate_proj of LLaMA-2-7B: 11008 x 4096 (output Hadamard blocks of 256, input 4096)
    d_out, d_in, n = 11008, 4096, 4096
    xq, _, g, w, si, so = layer_inputs(d_out, d_in, n, drift="none", w_dtype=torch.bfloat16,
                                       tag="biip-gate")
    hx = torch.zeros(d_in, d_in, device="cuda"); hg = torch.zeros(d_out, d_out, device="cuda")
    K.kronq_accumulate(xq, None, g, hx, hg)
    r = run_biip(K, P, w, hx, hg, None, 1.0 / n, si, so, 15)
    o = O.biip(h64(w), h64(hx), h64(hg), None, 1.0 / n, h64(si), h64(so), 15)
    assert rel(h64(r.w_prime), o["w"]) <= TOL
    assert rel(h64(r.hx), o["hx"]) <= TOL
    assert rel(h64(r.s_g), o["s_g"]) <= TOL
    assert abs(float(r.tr[1]) - o["tr_hg"]) <= TOL * o["tr_hg"]


# ------------------------------------------------------------------------------ cholinv

def spd_gpu(d, seed, cond=1e3):
    r = np.random.default_rng(seed)
    q, _ = np.linalg.qr(r.standard_normal((d, d)))
    ev = np.exp(r.uniform(0, math.log(cond), d))
    return torch.tensor((q * ev) @ q.T, dtype=torch.float32, device="cuda")


@pytest.mark.parametrize("d", [256, 200, 65, 64, 1, 513])
def test_cholinv_matches_oracle(K, d):
    h = spd_gpu(d, d)
    o = O.cholinv(h64(h), 0.01)
    k = h.clone()
    info = torch.empty(1, dtype=torch.int32, device="cuda")
    K.kronq_cholinv(k, 0.01, info, K.CHOLINV_SYNC)
    assert int(info) == -1
    assert rel(h64(k), o) <= TOL
    assert torch.all(torch.tril(k, -1) == 0)


@pytest.mark.parametrize("d", [4096, 11008])
def test_cholinv_llama_width(K, d):
    # LLaMA-2-7B widths: the whole K against the oracle's fp64 three-step factor of the same H
    n = 3 * d
    x = synth.correlated_x(n, d, synth.seed_for("chol", d), device="cuda")
    h = torch.zeros(d, d, device="cuda")
    K.kronq_accumulate(x, None, None, h)
    h /= n
    k = h.clone()
    info = torch.empty(1, dtype=torch.int32, device="cuda")
    K.kronq_cholinv(k, 0.01, info, K.CHOLINV_SYNC)
    hd = h64(h); kd = h64(k)
    ko = O.cholinv(hd, 0.01)
    err = rel(kd, ko)
    # A forward error below kappa(A) * u is out of reach for any fp32 factorization, so the bar
    # is 1e-3 or 4 kappa(A) 2^-24 where that is larger (kappa by power iteration on A and on
    # A^-1 = K^T K).
    lam = 0.01 * np.mean(np.diag(hd))
    kappa = cond_estimate(hd + lam * np.eye(d), ko)
    bar = max(TOL, 4 * kappa * 2.0 ** -24)
    print(f"d={d}: |K - K_oracle| / |K_oracle| = {err:.2e}, kappa ~ {kappa:.2e}, bar {bar:.2e}")
    assert err <= bar
    assert np.all(np.diag(kd) > 0)
    assert np.all(np.tril(kd, -1) == 0)


def cond_estimate(a, k, iters=30):
    """2-norm condition number of SPD a, with a^-1 = k^T k (power iteration on both)."""
    r = np.random.default_rng(5)
    v = r.standard_normal(a.shape[0])
    for _ in range(iters):
        v = a @ v; v /= np.linalg.norm(v)
    big = float(v @ (a @ v))
    u = r.standard_normal(a.shape[0])
    for _ in range(iters):
        u = k.T @ (k @ u); u /= np.linalg.norm(u)
    small_inv = float(u @ (k.T @ (k @ u)))
    return big * small_inv


def test_cholinv_not_positive_definite(K):
    h = torch.eye(96, device="cuda")
    h[40, 40] = -1000.0
    info = torch.empty(1, dtype=torch.int32, device="cuda")
    with pytest.raises(K.KronqError) as e:
        K.kronq_cholinv(h, 0.0, info, K.CHOLINV_SYNC)
    assert e.value.status == K.ERR_NOT_PD
    assert int(info) == 40
    # asynchronous form reports through info only
    h2 = torch.eye(96, device="cuda"); h2[5, 5] = -1.0
    K.kronq_cholinv(h2, 0.0, info, 0)
    torch.cuda.synchronize()
    assert int(info) == 5


# ------------------------------------------------------------------------------ quantize

def check_codes(gpu, oracle_res, total):
    # every code the oracle decides on its own (away from a rounding boundary) must match, and
    # the oracle's own decision may differ from the GPU's on at most 0.1% of entries, all of
    # them within 1e-3 grid units of a boundary
    mism = (h64(gpu) != oracle_res["codes"]).sum()
    assert mism == 0, f"{mism} codes differ away from rounding boundaries"
    dis = int(oracle_res["disagree"].sum())
    print(f"near-ties {int(oracle_res['near_tie'].sum())}, disagreements {dis} of {total}")
    assert dis <= 1e-3 * total


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("with_dxx", [False, True])
@pytest.mark.parametrize("shape", [(256, 256), (96, 200), (130, 384)])
def test_quantize_matches_oracle(K, P, bits, with_dxx, shape):
    d_out, d_in = shape
    n = 2048
    xq, xfp, g, w, si, so = layer_inputs(d_out, d_in, n, drift="rel0.05", tag=("q", shape))
    hx, hg, dxx = gpu_sums(K, xq, xfp, g, with_dxx=with_dxx)
    r = P.biip(w, hx, hg, dxx, 1.0 / n, si, so, 15)
    wp = r.w_prime.clone(); dxx_p = None if dxx is None else r.dxx.clone()
    P.cholinv(r, 0.01, sync=True)
    kk = r.hx.clone()
    P.quantize(r, bits)
    torch.cuda.synchronize()
    o = O.quantize_layer(h64(wp), h64(kk), None if dxx_p is None else h64(dxx_p), bits,
                         follow_codes=h64(r.codes))
    assert np.array_equal(h64(r.scale), o["scale"].astype(np.float64))
    assert np.array_equal(h64(r.zero), o["zero"].astype(np.float64))
    check_codes(r.codes, o, d_out * d_in)
    assert rel(h64(r.w_hat), o["w_hat"]) <= TOL


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("with_dxx", [False, True])
@pytest.mark.parametrize("shape", [(256, 256), (96, 200), (130, 384)])
def test_quantize_group128_matches_oracle(K, P, bits, with_dxx, shape):
    # group-wise grid, g = 128 ([KronQ-hyper] Experiments): one scale / zero per row and per
    # 128 columns, from the weights the solve is about to quantize. The oracle follows the GPU's
    # group grid only where the two agree to 1e-5 (scale) and, for the zero, only at a rounding
    # boundary of -lo / scale; then codes as for the per-row grid
    d_out, d_in = shape
    n = 2048
    xq, xfp, g, w, si, so = layer_inputs(d_out, d_in, n, drift="rel0.05", tag=("qg", shape))
    hx, hg, dxx = gpu_sums(K, xq, xfp, g, with_dxx=with_dxx)
    r = P.biip(w, hx, hg, dxx, 1.0 / n, si, so, 15)
    wp = r.w_prime.clone(); dxx_p = None if dxx is None else r.dxx.clone()
    P.cholinv(r, 0.01, sync=True)
    kk = r.hx.clone()
    P.quantize(r, bits, group=128)
    torch.cuda.synchronize()
    ng = (d_in + 127) // 128
    assert tuple(r.scale.shape) == (d_out, ng)
    o = O.quantize_layer(h64(wp), h64(kk), None if dxx_p is None else h64(dxx_p), bits,
                         follow_codes=h64(r.codes), group=128,
                         follow_grid=(h64(r.scale), h64(r.zero)))
    assert np.array_equal(h64(r.scale), o["scale"].astype(np.float64))
    assert np.array_equal(h64(r.zero), o["zero"].astype(np.float64))
    assert int(o["grid_tie"].sum()) <= 1e-2 * d_out * ng
    check_codes(r.codes, o, d_out * d_in)
    assert rel(h64(r.w_hat), o["w_hat"]) <= TOL
    if not with_dxx:
        # nothing has touched the first group yet: its grid is the min-max grid of W' over its
        # columns, bit for bit (with P the first group is taken from W' (I + P) instead)
        s0, z0 = O.grid(h64(wp)[:, :128].astype(np.float32), bits)
        assert np.array_equal(h64(r.scale)[:, 0], s0.astype(np.float64))
        assert np.array_equal(h64(r.zero)[:, 0], z0.astype(np.float64))


def test_quantize_llama_shape_sampled_rows(K, P):
    # q_proj of LLaMA-2-7B (4096 x 4096), 4 bits: 48 random rows re-run by the oracle from the
    # GPU's K and W' (rows are independent given K)
    d_out = d_in = 4096
    n = 8192
    xq, _, g, w, si, so = layer_inputs(d_out, d_in, n, drift="none", w_dtype=torch.bfloat16,
                                       tag="q-full")
    hx = torch.zeros(d_in, d_in, device="cuda"); hg = torch.zeros(d_out, d_out, device="cuda")
    K.kronq_accumulate(xq, None, g, hx, hg)
    r = P.biip(w, hx, hg, None, 1.0 / n, si, so, 15)
    wp = r.w_prime.clone()
    P.cholinv(r, 0.01, sync=True)
    P.quantize(r, 4)
    torch.cuda.synchronize()
    rows = np.random.default_rng(1).choice(d_out, 48, replace=False)
    o = O.quantize_layer(h64(wp[rows]), h64(r.hx), None, 4, follow_codes=h64(r.codes[rows]))
    check_codes(r.codes[rows], o, 48 * d_in)
    assert rel(h64(r.w_hat[rows]), o["w_hat"]) <= TOL


def test_quantize_llama_shape_with_oracle_factor(K, P):
    # The same q_proj shape, but the oracle quantizes its rows with its own fp64 factor of the
    # GPU's H_X' (not the GPU's K): codes and W^ must still meet the bars, so the fp32 factor's
    # error does not leak into the result.
    d_out = d_in = 4096
    n = 8192
    xq, _, g, w, si, so = layer_inputs(d_out, d_in, n, drift="none", w_dtype=torch.bfloat16,
                                       tag="q-full-ofac")
    hx = torch.zeros(d_in, d_in, device="cuda"); hg = torch.zeros(d_out, d_out, device="cuda")
    K.kronq_accumulate(xq, None, g, hx, hg)
    r = P.biip(w, hx, hg, None, 1.0 / n, si, so, 15)
    wp = r.w_prime.clone(); hxp = r.hx.clone()
    P.cholinv(r, 0.01, sync=True)
    P.quantize(r, 4)
    torch.cuda.synchronize()
    ko = O.cholinv(h64(hxp), 0.01)
    rows = np.random.default_rng(2).choice(d_out, 32, replace=False)
    o = O.quantize_layer(h64(wp[rows]), ko, None, 4, follow_codes=h64(r.codes[rows]))
    check_codes(r.codes[rows], o, 32 * d_in)
    assert rel(h64(r.w_hat[rows]), o["w_hat"]) <= TOL


# ------------------------------------------------------------------------------ end to end

@pytest.mark.parametrize("flags", [0, 15])
def test_layer256_end_to_end(K, P, flags):
    # single 256 x 256 layer, 2048 tokens, fp32 W, X~ = X + N(0, 0.01^2), 2 bits, damp 0.01
    d = 256; n = 2048; bits = 2
    xq, xfp, g, w, si, so = layer_inputs(d, d, n, drift="abs0.01", tag="layer256")
    hx, hg, dxx = gpu_sums(K, xq, xfp, g)
    r = P.quantize_sublayer(w, hx, hg, dxx, 1.0 / n, si, so, bits, flags=flags)
    torch.cuda.synchronize()
    ohx, ohg, odxx = O.accumulate(h64(xq), h64(xfp), h64(g))
    ob = O.biip(h64(w), ohx, ohg, odxx, 1.0 / n, h64(si), h64(so), flags)
    ok = O.cholinv(ob["hx"], 0.01)
    oq = O.quantize_layer(ob["w"], ok, ob["dxx"], bits, follow_codes=h64(r.codes))
    check_codes(r.codes, oq, d * d)
    assert rel(h64(r.w_hat), oq["w_hat"]) <= TOL
    hg_p = ob["hg"]
    j_gpu = O.objective(ob["w"], h64(r.w_hat), ob["hx"], hg_p, ob["dxx"])
    j_ora = O.objective(ob["w"], oq["w_hat"], ob["hx"], hg_p, ob["dxx"])
    assert abs(j_gpu - j_ora) <= TOL * abs(j_ora)


def test_no_device_error_recorded(K):
    assert K.kronq_device_error() == 0


# ------------------------------------------------------------------------------ other workloads

def test_drift_term_llama3_8b_width(K):
    # LLaMA-3-8B hidden width 4096, X~ = X + N(0, (0.05 rms X)^2), 16384 tokens: sampled tiles of
    # the drift sum D += (X - X~)^T X~ and of H_X against fp64 sums of the same bf16 values
    n, d = 16384, 4096
    x = synth.correlated_x(n, d, synth.seed_for("drift8b", "X"), device="cuda")
    xq = synth.perturbed(x, synth.seed_for("drift8b", "Xq"), rel_std=0.05)
    hx = torch.zeros(d, d, device="cuda"); dxx = torch.zeros(d, d, device="cuda")
    K.kronq_accumulate(xq, x, None, hx, None, dxx)
    torch.cuda.synchronize()
    r = np.random.default_rng(7)
    for _ in range(8):
        i0 = int(r.integers(0, d // 128)) * 128; j0 = int(r.integers(0, d // 128)) * 128
        xa = h64(x[:, i0:i0 + 128]); qa = h64(xq[:, i0:i0 + 128]); qb = h64(xq[:, j0:j0 + 128])
        assert rel(h64(dxx[i0:i0 + 128, j0:j0 + 128]), (xa - qa).T @ qb) <= TOL
        assert rel(h64(hx[i0:i0 + 128, j0:j0 + 128]), qa.T @ qb) <= TOL


@pytest.mark.parametrize("scale", [1.0, 2.0 ** 40, 2.0 ** -40])
def test_drift_term_across_chunks_and_magnitudes(K, scale):
    # The drift product runs in fp16 after a power-of-two rescale taken from the largest
    # magnitude over all n tokens. 70000 tokens span three conversion chunks (the largest value
    # of the whole call sets the scale of each); inputs scaled by 2^40 would overflow fp16
    # without the rescale and inputs scaled by 2^-40 would vanish in it. The width 136 is ragged (17 groups of 8, padded
    # stride). The oracle sums the same bf16 values in fp64.
    n, d = 70000, 136
    tag = ("drift-chunks", scale)
    x = padded((synth.correlated_x(n, d, synth.seed_for(tag, "X"), device="cuda").float()
                * scale).to(torch.bfloat16))
    xq = padded(synth.perturbed(x, synth.seed_for(tag, "Xq"), rel_std=0.05))
    hx = torch.zeros(d, d, device="cuda"); dxx = torch.zeros(d, d, device="cuda")
    K.kronq_accumulate(xq, x, None, hx, None, dxx)
    torch.cuda.synchronize()
    assert torch.isfinite(dxx).all()
    o_hx, _, o_dxx = O.accumulate(h64(xq), h64(x))
    assert rel(h64(dxx), o_dxx) <= TOL
    assert rel(h64(hx), o_hx) <= TOL
    # the largest value late in the tokens: the scale must come from all of them, not the
    # first chunk
    x2 = x.clone(); x2[-5, 3] = x2[-5, 3] * 64
    xq2 = xq.clone(); xq2[-7, 11] = xq2[-7, 11] * 64
    d2 = torch.zeros(d, d, device="cuda")
    K.kronq_accumulate(xq2, x2, None, None, None, d2)
    torch.cuda.synchronize()
    assert rel(h64(d2), O.accumulate(h64(xq2), h64(x2))[2]) <= TOL


@pytest.mark.parametrize("d", [8192, 28672])
def test_drift_term_llama3_70b_width_sampled(K, d):
    # LLaMA-3-70B input widths (hidden 8192; MLP 28672 for down_proj), X~ = X + N(0, (0.05 rms
    # X)^2), 8192 tokens: 12 sampled 128 x 128 tiles of D = (X - X~)^T X~ and of H_X, each against
    # fp64 sums of the same bf16 values; and the trace of H_X against its closed form.
    n = 8192
    x = synth.correlated_x(n, d, synth.seed_for("drift70b", d, "X"), device="cuda")
    xq = synth.perturbed(x, synth.seed_for("drift70b", d, "Xq"), rel_std=0.05)
    hx = torch.zeros(d, d, device="cuda"); dxx = torch.zeros(d, d, device="cuda")
    K.kronq_accumulate(xq, x, None, hx, None, dxx)
    torch.cuda.synchronize()
    r = np.random.default_rng(d + 1)
    for t in range(12):
        i0 = int(r.integers(0, d // 128)) * 128
        j0 = i0 if t == 0 else int(r.integers(0, d // 128)) * 128   # one diagonal tile
        xa = h64(x[:, i0:i0 + 128]); qa = h64(xq[:, i0:i0 + 128]); qb = h64(xq[:, j0:j0 + 128])
        assert rel(h64(dxx[i0:i0 + 128, j0:j0 + 128]), (xa - qa).T @ qb) <= TOL, (i0, j0)
        assert rel(h64(hx[i0:i0 + 128, j0:j0 + 128]), qa.T @ qb) <= TOL, (i0, j0)
    tr = float(np.sum(h64(xq) ** 2))
    assert abs(float(torch.trace(hx.double())) - tr) <= TOL * tr
    del hx, dxx


@pytest.mark.parametrize("d", [8192, 28672])
def test_accumulate_llama3_70b_bench_size_sampled(K, d):
    # The benchmark's launch configuration: 262144 tokens at the LLaMA-3-70B widths, X~ = X +
    # N(0, (0.05 rms X)^2). H_X runs as four 65536-token work units per output tile whose fp32
    # partials meet by atomic adds; D = (X - X~)^T X~ as eight 32768-token fp16 products. 8
    # sampled 128 x 128 tiles of each (one diagonal) against fp64 sums of the same bf16 values,
    # and the trace of H_X against ||X~||^2 summed in fp64.
    n = 262144
    torch.cuda.empty_cache()                 # ~40 GB below: start from released memory
    x = synth.correlated_x(n, d, synth.seed_for("acc70b-bench", d), device="cuda")
    xq = synth.perturbed(x, synth.seed_for("acc70b-bench", d, "q"), rel_std=0.05)
    hx = torch.zeros(d, d, device="cuda"); dxx = torch.zeros(d, d, device="cuda")
    K.kronq_accumulate(xq, x, None, hx, None, dxx)
    torch.cuda.synchronize()
    r = np.random.default_rng(d + 7)
    for t in range(8):
        i0 = int(r.integers(0, d // 128)) * 128
        j0 = i0 if t == 0 else int(r.integers(0, d // 128)) * 128
        qa = h64(xq[:, i0:i0 + 128]); qb = qa if j0 == i0 else h64(xq[:, j0:j0 + 128])
        assert rel(h64(hx[i0:i0 + 128, j0:j0 + 128]), qa.T @ qb) <= TOL, (i0, j0)
        xa = h64(x[:, i0:i0 + 128])
        assert rel(h64(dxx[i0:i0 + 128, j0:j0 + 128]), (xa - qa).T @ qb) <= TOL, (i0, j0)
    tr = 0.0
    for c0 in range(0, n, 16384):
        tr += float(torch.sum(xq[c0:c0 + 16384].double() ** 2))
    assert abs(float(torch.trace(hx.double())) - tr) <= TOL * tr
    del x, xq, hx, dxx
    torch.cuda.empty_cache()


@pytest.mark.parametrize("d_out,d_in", [(8192, 28672), (1024, 8192), (16384, 16384)])
def test_biip_llama3_70b_shapes(K, P, d_out, d_in):
    # LLaMA-3-70B shapes: down_proj 8192 x 28672 (input Hadamard blocks of 4096, output 8192),
    # k/v 1024 x 8192 (input blocks of 8192: the row pass's widest chunk), and 16384-wide blocks
    # on both sides. Full-size check through the inverse transforms:
    # (U^T W' V)_ij = s_g,i W_ij s_x,j and (V^T H_X' V)_ij = (S_X^-1 H_X S_X^-1 / n)_ij on sampled
    # entries, each from one b x b block; plus the oracle's scales.
    n = 2048
    tag = ("b70", d_out, d_in) if d_in != 28672 else "b70"
    x = synth.correlated_x(n, d_in, synth.seed_for(tag, "X"), device="cuda")
    g = synth.gradients(n, d_out, synth.seed_for(tag, "G"), device="cuda")
    w = synth.weight(d_out, d_in, synth.seed_for(tag, "W"), device="cuda")
    si = synth.rademacher(d_in, synth.seed_for(tag, "si"), device="cuda")
    so = synth.rademacher(d_out, synth.seed_for(tag, "so"), device="cuda")
    hx = torch.zeros(d_in, d_in, device="cuda"); hg = torch.zeros(d_out, d_out, device="cuda")
    K.kronq_accumulate(x, None, g, hx, hg)
    hx_diag = torch.diagonal(hx).clone(); hg_diag = torch.diagonal(hg).clone()
    hx_orig = hx.clone()
    r = P.biip(w, hx, hg, None, 1.0 / n, si, so, 15, copy_hx=False)
    torch.cuda.synchronize()
    w64 = h64(w)
    col_sq = (w64 ** 2).sum(0); row_sq = (w64 ** 2).sum(1)
    sx = (h64(hx_diag) / n / col_sq) ** 0.25
    sg = (h64(hg_diag) / n / row_sq) ** 0.25
    assert rel(h64(r.s_x), sx) <= TOL and rel(h64(r.s_g), sg) <= TOL
    tr_hx = float(np.sum(h64(hx_diag) / n / sx ** 2))
    assert abs(float(r.tr[0]) - tr_hx) <= TOL * tr_hx
    bi, bo = O.hadamard_block_size(d_in), O.hadamard_block_size(d_out)

    class _Cols:
        # column k of the normalised Sylvester matrix, (-1)^popcount(i & k) / sqrt(b), built
        # on demand (the b = 16384 matrix would be 2 GB in fp64)
        def __init__(self, b):
            self.b = b
            self.i = np.arange(b, dtype=np.uint32)

        def __getitem__(self, key):
            _, k = key
            par = np.bitwise_count(self.i & np.uint32(k)) & 1
            return (1.0 - 2.0 * par.astype(np.float64)) / math.sqrt(self.b)

    hb_i = _Cols(bi); hb_o = _Cols(bo)
    # the on-demand columns agree with the oracle's Sylvester matrix
    small = O.sylvester(64) / 8.0
    assert all(np.array_equal(_Cols(64)[:, k], small[:, k]) for k in range(64))
    sin = h64(si); sout = h64(so)
    rng = np.random.default_rng(70)
    got, want = [], []
    def bilinear(mat, ib, jb, b1, b2, u, v):
        # u^T mat[ib:ib+b1, jb:jb+b2] v in fp64, on the device (the blocks can be 1 GB)
        blk = mat[ib:ib + b1, jb:jb + b2].double()
        uu = torch.from_numpy(u).to(blk.device); vv = torch.from_numpy(v).to(blk.device)
        return float(uu @ (blk @ vv))

    for _ in range(24):
        i = int(rng.integers(0, d_out)); j = int(rng.integers(0, d_in))
        ib, jb = (i // bo) * bo, (j // bi) * bi
        u_i = hb_o[:, i - ib] * sout[i]          # column i of U = (1/sqrt b)(H_b) diag(sign)
        v_j = hb_i[:, j - jb] * sin[j]
        got.append(bilinear(r.w_prime, ib, jb, bo, bi, u_i, v_j))
        want.append(sg[i] * w64[i, j] * sx[j])
    assert rel(np.array(got), np.array(want)) <= TOL
    # the rotation preserves the Frobenius norm of S_G W S_X
    nrm = float(torch.linalg.vector_norm(r.w_prime.double()))
    assert abs(nrm - np.linalg.norm(sg[:, None] * w64 * sx[None, :])) <= TOL * nrm
    # H_X' through the inverse input transform, on sampled entries
    got, want = [], []
    for _ in range(16):
        i = int(rng.integers(0, d_in)); j = int(rng.integers(0, d_in))
        ib, jb = (i // bi) * bi, (j // bi) * bi
        v_i = hb_i[:, i - ib] * sin[i]
        v_j = hb_i[:, j - jb] * sin[j]
        got.append(bilinear(r.hx, ib, jb, bi, bi, v_i, v_j))
        want.append(float(hx_orig[i, j]) / n / (sx[i] * sx[j]))
    scale = float(np.max(np.abs(want)))
    assert np.max(np.abs(np.array(got) - np.array(want))) <= TOL * scale


def test_cholinv_llama3_70b_width(K):
    # H_X of the 70B down_proj input (d = 28672, 3.3 GB fp32). Backward error of the factor:
    # with R = K^-1 (an exact fp64 triangular solve of the GPU's K), R R^T v must equal
    # (H + lambda I) v to the bar, for random v. Unlike K (H + lambda I) K^T - I, this residual
    # is not multiplied by the condition number (~4e4 here), so it measures the factor's
    # accuracy rather than the fp32 rounding of its storage.
    import scipy.linalg as sla
    d = 28672
    n = 2 * d
    x = synth.correlated_x(n, d, synth.seed_for("chol70", d), device="cuda", chunk=8192)
    h = torch.zeros(d, d, device="cuda")
    K.kronq_accumulate(x, None, None, h)
    del x
    h /= n
    hd = h64(h)
    info = torch.empty(1, dtype=torch.int32, device="cuda")
    K.kronq_cholinv(h, 0.01, info, K.CHOLINV_SYNC)
    kd = h64(h)
    del h
    torch.cuda.empty_cache()
    lam = 0.01 * np.mean(np.diag(hd))
    r = np.random.default_rng(1)
    worst = 0.0
    for _ in range(3):
        v = r.standard_normal(d)
        av = hd @ v + lam * v
        y = sla.solve_triangular(kd, v, trans="T", lower=False)   # K^-T v = R^T v
        rrt = sla.solve_triangular(kd, y, lower=False)            # K^-1 K^-T v = R R^T v
        worst = max(worst, np.linalg.norm(rrt - av) / np.linalg.norm(av))
    print(f"d={d}: max |R R^T v - A v| / |A v| = {worst:.2e}")
    assert worst <= TOL
    assert np.all(np.diag(kd) > 0)
    # the bottom-right block of K depends only on the bottom-right block of A (the factorization
    # runs from the last index up): compare it with the oracle's factor of that block alone
    m = 2048
    sub = hd[-m:, -m:]
    ko = O.cholinv(sub, lam / float(np.mean(np.diag(sub))))
    assert rel(kd[-m:, -m:], ko) <= TOL


def test_quantize_with_drift_llama3_8b_kv(K, P):
    # k_proj of LLaMA-3-8B (1024 x 4096), 3 bits, drifted input so P is active: 32 rows re-run
    # by the oracle (literal column update with the P term) from the GPU's K, W' and D'
    d_out, d_in, n = 1024, 4096, 8192
    x = synth.correlated_x(n, d_in, synth.seed_for("kv8b", "X"), device="cuda")
    xq = synth.perturbed(x, synth.seed_for("kv8b", "Xq"), rel_std=0.05)
    g = synth.gradients(n, d_out, synth.seed_for("kv8b", "G"), device="cuda")
    w = synth.weight(d_out, d_in, synth.seed_for("kv8b", "W"), device="cuda")
    si = synth.rademacher(d_in, synth.seed_for("kv8b", "si"), device="cuda")
    so = synth.rademacher(d_out, synth.seed_for("kv8b", "so"), device="cuda")
    hx = torch.zeros(d_in, d_in, device="cuda"); hg = torch.zeros(d_out, d_out, device="cuda")
    dxx = torch.zeros(d_in, d_in, device="cuda")
    K.kronq_accumulate(xq, x, g, hx, hg, dxx)
    r = P.biip(w, hx, hg, dxx, 1.0 / n, si, so, 15)
    wp = r.w_prime.clone(); dp = r.dxx.clone()
    P.cholinv(r, 0.01, sync=True)
    P.quantize(r, 3)
    torch.cuda.synchronize()
    rows = np.random.default_rng(8).choice(d_out, 32, replace=False)
    o = O.quantize_layer(h64(wp[rows]), h64(r.hx), h64(dp), 3, follow_codes=h64(r.codes[rows]))
    check_codes(r.codes[rows], o, 32 * d_in)
    assert rel(h64(r.w_hat[rows]), o["w_hat"]) <= TOL


@pytest.mark.parametrize("d_out,d_in", [(8192, 28672), (28672, 8192)])
def test_quantize_llama3_70b_with_drift_sampled_rows(K, P, d_out, d_in):
    # LLaMA-3-70B down_proj (8192 x 28672: the 28672-wide inverse factor, P and pre-shift) and
    # gate_proj (28672 x 8192: 28672 output rows), 2 bits, drifted input (X~ = X + N(0, (0.05
    # rms X)^2)) so P is active. 32 rows re-run by the oracle - the literal column update with
    # the P term, P = striu(D K^T) K formed in fp64 - from the GPU's K, W' and D'.
    n = 8192
    tag = ("q70b", d_out, d_in)
    x = synth.correlated_x(n, d_in, synth.seed_for(tag, "X"), device="cuda")
    xq = synth.perturbed(x, synth.seed_for(tag, "Xq"), rel_std=0.05)
    g = synth.gradients(n, d_out, synth.seed_for(tag, "G"), device="cuda")
    w = synth.weight(d_out, d_in, synth.seed_for(tag, "W"), device="cuda")
    si = synth.rademacher(d_in, synth.seed_for(tag, "si"), device="cuda")
    so = synth.rademacher(d_out, synth.seed_for(tag, "so"), device="cuda")
    hx = torch.zeros(d_in, d_in, device="cuda"); dxx = torch.zeros(d_in, d_in, device="cuda")
    hg = torch.zeros(d_out, device="cuda")
    K.kronq_accumulate(xq, x, None, hx, None, dxx)
    K.kronq_accumulate_diag(g, hg)
    del x, xq, g
    r = P.biip(w, hx, hg, dxx, 1.0 / n, si, so, 15 | K.BIIP_HG_DIAG, copy_hx=False)
    del hx, dxx
    wp = r.w_prime.clone(); dp = r.dxx.clone()
    P.cholinv(r, 0.01, sync=True)
    P.quantize(r, 2)
    torch.cuda.synchronize()
    rows = np.random.default_rng(d_out + d_in).choice(d_out, 32, replace=False)
    o = O.quantize_layer(h64(wp[rows]), h64(r.hx), h64(dp), 2, follow_codes=h64(r.codes[rows]))
    check_codes(r.codes[rows], o, 32 * d_in)
    assert rel(h64(r.w_hat[rows]), o["w_hat"]) <= TOL


def test_quantize_group128_llama3_70b_gate_sampled_rows(K, P):
    # LLaMA-3-70B gate_proj (28672 x 8192), 2 bits, group-wise grid g = 128 ([KronQ-hyper]
    # Experiments: the 2-bit results use g = 128), drifted input so P is active. 32 rows re-run
    # by the oracle in follow mode (codes and group grids) from the GPU's K, W' and D'.
    d_out, d_in, n, bits = 28672, 8192, 8192, 2
    tag = ("qg70b",)
    x = synth.correlated_x(n, d_in, synth.seed_for(tag, "X"), device="cuda")
    xq = synth.perturbed(x, synth.seed_for(tag, "Xq"), rel_std=0.05)
    g = synth.gradients(n, d_out, synth.seed_for(tag, "G"), device="cuda")
    w = synth.weight(d_out, d_in, synth.seed_for(tag, "W"), device="cuda")
    si = synth.rademacher(d_in, synth.seed_for(tag, "si"), device="cuda")
    so = synth.rademacher(d_out, synth.seed_for(tag, "so"), device="cuda")
    hx = torch.zeros(d_in, d_in, device="cuda"); dxx = torch.zeros(d_in, d_in, device="cuda")
    hg = torch.zeros(d_out, device="cuda")
    K.kronq_accumulate(xq, x, None, hx, None, dxx)
    K.kronq_accumulate_diag(g, hg)
    del x, xq, g
    r = P.biip(w, hx, hg, dxx, 1.0 / n, si, so, 15 | K.BIIP_HG_DIAG, copy_hx=False)
    wp = r.w_prime.clone(); dp = r.dxx.clone()
    P.cholinv(r, 0.01, sync=True)
    P.quantize(r, bits, group=128)
    torch.cuda.synchronize()
    rows = np.random.default_rng(77).choice(d_out, 32, replace=False)
    o = O.quantize_layer(h64(wp[rows]), h64(r.hx), h64(dp), bits, follow_codes=h64(r.codes[rows]),
                         group=128, follow_grid=(h64(r.scale[rows]), h64(r.zero[rows])))
    assert np.array_equal(h64(r.scale[rows]), o["scale"].astype(np.float64))
    assert np.array_equal(h64(r.zero[rows]), o["zero"].astype(np.float64))
    assert int(o["grid_tie"].sum()) <= 1e-2 * 32 * (d_in // 128)
    check_codes(r.codes[rows], o, 32 * d_in)
    assert rel(h64(r.w_hat[rows]), o["w_hat"]) <= TOL


def test_stack_scores_and_allocation(K, P):
    # Two blocks of the LLaMA-2-7B mixed-precision stack (14 sublayers, each its own X and G,
    # 65536 tokens, per-block G scale log-uniform on [1e-2, 1e1]): traces after BiIP against
    # fp64 sums of the same bf16 inputs, and the {2,3,4}-bit allocation at 2.5 average bits
    # bit-exact against the oracle's greedy on the same scores.
    wl = synth.WORKLOADS["llama2_7b_stack"]
    n = wl.n_tokens
    tr_gpu, tr_ora, sizes = [], [], []
    for blk in range(2):
        mult = 10 ** np.random.default_rng(blk).uniform(-2, 1)
        for s in wl.sublayers:
            tag = ("stack", blk, s.name)
            x = synth.correlated_x(n, s.d_in, synth.seed_for(tag, "X"), device="cuda")
            g = synth.gradients(n, s.d_out, synth.seed_for(tag, "G"), device="cuda", multiplier=mult)
            w = synth.weight(s.d_out, s.d_in, synth.seed_for(tag, "W"), device="cuda")
            si = synth.rademacher(s.d_in, synth.seed_for(tag, "si"), device="cuda")
            so = synth.rademacher(s.d_out, synth.seed_for(tag, "so"), device="cuda")
            hx = torch.zeros(s.d_in, s.d_in, device="cuda")
            hg = torch.zeros(s.d_out, s.d_out, device="cuda")
            K.kronq_accumulate(x, None, g, hx, hg)
            r = P.biip(w, hx, hg, None, 1.0 / n, si, so, 15, copy_hx=False)
            torch.cuda.synchronize()
            tr_gpu.append((float(r.tr[0]), float(r.tr[1])))
            # fp64: diag sums from the inputs, norms from W, traces of S^-1 H S^-1
            dx = (x.double() ** 2).sum(0).cpu().numpy() / n
            dg = (g.double() ** 2).sum(0).cpu().numpy() / n
            w64 = h64(w)
            sx = (dx / (w64 ** 2).sum(0)) ** 0.25; sg = (dg / (w64 ** 2).sum(1)) ** 0.25
            tr_ora.append((float(np.sum(dx / sx ** 2)), float(np.sum(dg / sg ** 2))))
            sizes.append(s.d_out * s.d_in)
            del x, g, hx, hg, r
    for (a, b), (c, e) in zip(tr_gpu, tr_ora):
        assert abs(a - c) <= TOL * c and abs(b - e) <= TOL * e
    s_k, bits_k = K.kronq_score_allocate([t[0] for t in tr_gpu], [t[1] for t in tr_gpu], sizes,
                                         [2, 3, 4], 2.5)
    s_o, bits_o = O.score_allocate([t[0] for t in tr_gpu], [t[1] for t in tr_gpu], sizes,
                                   [2, 3, 4], 2.5)
    assert bits_k == bits_o and s_k == s_o
    assert sum(b * m for b, m in zip(bits_k, sizes)) <= math.floor(2.5 * sum(sizes))
    assert len(set(bits_k)) > 1
