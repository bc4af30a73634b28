"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each test ties one oracle function to a closed form, a brute-force computation on a tiny
input, a textbook special case, or a figure the KronQ pages state. They are chosen so that a
plausible slip (a dropped term, a wrong sign, a transposed operand, the wrong Kronecker order,
a wrong row of the inverse factor) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg as sla

from oracle import kronq_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rng(seed):
    return np.random.default_rng(seed)


def spd(r, d, cond=10.0):
    q, _ = np.linalg.qr(r.standard_normal((d, d)))
    ev = np.exp(r.uniform(0, math.log(cond), d))
    return (q * ev) @ q.T


# ------------------------------------------------------------------ statistics (P1)

def test_accumulate_equals_sum_of_token_outer_products():
    r = rng(1)
    n, d_in, d_out = 7, 5, 3
    xq = r.standard_normal((n, d_in))
    xfp = xq + 0.1 * r.standard_normal((n, d_in))
    g = r.standard_normal((n, d_out))
    hx, hg, dxx = O.accumulate(xq, xfp, g)
    bx = np.zeros((d_in, d_in)); bg = np.zeros((d_out, d_out)); bd = np.zeros((d_in, d_in))
    for t in range(n):
        for i in range(d_in):
            for j in range(d_in):
                bx[i, j] += xq[t, i] * xq[t, j]
                bd[i, j] += (xfp[t, i] - xq[t, i]) * xq[t, j]
        for i in range(d_out):
            for j in range(d_out):
                bg[i, j] += g[t, i] * g[t, j]
    np.testing.assert_allclose(hx, bx, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(hg, bg, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(dxx, bd, rtol=1e-13, atol=1e-13)


def test_accumulate_trace_symmetry_psd():
    r = rng(2)
    x = r.standard_normal((50, 9))
    hx, _, _ = O.accumulate(x)
    assert abs(np.trace(hx) - float((x ** 2).sum())) < 1e-11        # tr X^T X = |X|_F^2
    np.testing.assert_array_equal(hx, hx.T)
    assert np.linalg.eigvalsh(hx).min() > -1e-12


def test_accumulate_diag_closed_form():
    # G_tj = (t + 1)(j + 1)  =>  sum_t G_tj^2 = (j + 1)^2 n (n + 1)(2n + 1) / 6
    n, d = 11, 6
    t = np.arange(1, n + 1, dtype=np.float64)[:, None]
    j = np.arange(1, d + 1, dtype=np.float64)[None, :]
    got = O.accumulate_diag(t * j)
    np.testing.assert_allclose(got, (j[0] ** 2) * n * (n + 1) * (2 * n + 1) / 6, rtol=1e-15)


def test_biip_needs_only_the_diagonal_of_hg():
    # S_G = diag(H_G,ii / |W_i,:|^2)^(1/4) and tr(H_G') = sum_i H_G,ii / s_i^2 read only the
    # diagonal ([KronQ-hyper] Method: BiIP equations, sensitivity): BiIP with diag(H_G) alone
    # gives the same W', H_X', S_G and traces as with the full H_G; and the diagonal sums equal
    # the diagonal of the full (brute-force pinned) G^T G.
    r = rng(31)
    n, d_out, d_in = 40, 16, 8
    x = r.standard_normal((n, d_in)); g = r.standard_normal((n, d_out)) * r.uniform(0.1, 3, d_out)
    w = r.standard_normal((d_out, d_in))
    hx, hg, _ = O.accumulate(x, None, g)
    dg = O.accumulate_diag(g)
    np.testing.assert_allclose(dg, np.diag(hg), rtol=1e-13)
    si = np.where(r.standard_normal(d_in) > 0, 1.0, -1.0)
    so = np.where(r.standard_normal(d_out) > 0, 1.0, -1.0)
    full = O.biip(w, hx, hg, None, 1.0 / n, si, so, O.BIIP_FULL)
    diag = O.biip(w, hx, np.diag(dg), None, 1.0 / n, si, so, O.BIIP_FULL)
    for key in ("w", "hx", "s_x", "s_g"):
        np.testing.assert_allclose(diag[key], full[key], rtol=1e-12, atol=1e-14)
    assert abs(diag["tr_hg"] - full["tr_hg"]) <= 1e-12 * abs(full["tr_hg"])
    assert abs(diag["tr_hx"] - full["tr_hx"]) <= 1e-12 * abs(full["tr_hx"])
    assert not np.allclose(diag["hg"], full["hg"])          # the off-diagonal part is not there


def test_drift_term_sign_for_shrunk_input():
    # x~ = (1 - eps) x  =>  D = sum (x - x~) x~^T = eps (1 - eps) X^T X
    r = rng(3)
    x = r.standard_normal((20, 4)); eps = 0.125
    _, _, dxx = O.accumulate((1 - eps) * x, x)
    np.testing.assert_allclose(dxx, eps * (1 - eps) * x.T @ x, rtol=1e-13)


def test_fisher_is_kronecker_product_for_product_design():
    # All pairs (x_a, g_b): E[x x^T (x) g g^T] factorises exactly into H_X (x) H_G
    # ([KronQ-hyper] Method: Fisher equation and K-FAC split). Pins the Kronecker order.
    r = rng(4)
    xa = r.standard_normal((3, 3)); gb = r.standard_normal((4, 2))
    xs = np.repeat(xa, len(gb), axis=0)
    gs = np.tile(gb, (len(xa), 1))
    f = O.fisher_kron(xs, gs)
    hx, hg, _ = O.accumulate(xs, None, gs)
    n = len(xs)
    np.testing.assert_allclose(f, np.kron(hx / n, hg / n), rtol=1e-12, atol=1e-14)
    assert not np.allclose(f, np.kron(hg / n, hx / n))


# ------------------------------------------------------------------ objective (P2, P3)

def test_kronecker_objective_equals_vec_form():
    r = rng(5)
    d_out, d_in = 3, 4
    hx = spd(r, d_in); hg = spd(r, d_out)
    w = r.standard_normal((d_out, d_in)); wh = r.standard_normal((d_out, d_in))
    v = (w - wh).reshape(-1, order="F")
    brute = v @ np.kron(hx, hg) @ v
    assert abs(O.objective(w, wh, hx, hg) - brute) < 1e-11 * max(1.0, abs(brute))


def test_asymmetric_objective_equals_sample_mean():
    # (1/N) sum_n (W x_n - W^ x~_n)^T H_G (W x_n - W^ x~_n) = objective + constant(W, data)
    r = rng(6)
    n, d_out, d_in = 40, 3, 5
    x = r.standard_normal((n, d_in)); xq = x + 0.2 * r.standard_normal((n, d_in))
    hg = spd(r, d_out)
    w = r.standard_normal((d_out, d_in))
    hx, _, dxx = O.accumulate(xq, x)
    hx /= n; dxx /= n

    def sample(wh):
        tot = 0.0
        for t in range(n):
            e = w @ x[t] - wh @ xq[t]
            tot += e @ hg @ e
        return tot / n

    const = sum((w @ (x[t] - xq[t])) @ hg @ (w @ (x[t] - xq[t])) for t in range(n)) / n
    for _ in range(3):
        wh = w + 0.3 * r.standard_normal((d_out, d_in))
        assert abs(sample(wh) - (O.objective(w, wh, hx, hg, dxx) + const)) < 1e-10


# ------------------------------------------------------------------ inverse factor (P7)

@pytest.mark.parametrize("d", [1, 2, 7, 33])
def test_cholinv_factor(d):
    r = rng(10 + d)
    h = spd(r, d, cond=1e3)
    k = O.cholinv(h, 0.01)
    lam = 0.01 * np.mean(np.diag(h))
    np.testing.assert_allclose(k.T @ k @ (h + lam * np.eye(d)), np.eye(d), atol=1e-10)
    np.testing.assert_array_equal(k, np.triu(k))
    assert (np.diag(k) > 0).all()
    # reversed-order route: J(H+lam I)J = L L^T, K = (J L J)^-1 is the same matrix
    j = np.eye(d)[::-1]
    l = np.linalg.cholesky(j @ (h + lam * np.eye(d)) @ j)
    np.testing.assert_allclose(np.linalg.inv(j @ l @ j), k, atol=1e-9, rtol=1e-9)


def test_cholinv_not_pd():
    h = np.diag([1.0, 1.0, -50.0])
    with pytest.raises(O.NotPositiveDefinite):
        O.cholinv(h, 0.01)


# ------------------------------------------------------------------ Hadamard (P8)

@pytest.mark.parametrize("b", [1, 2, 4, 8, 16, 32, 64])
def test_sylvester_matches_textbook(b):
    np.testing.assert_array_equal(O.sylvester(b), sla.hadamard(b))
    np.testing.assert_array_equal(O.sylvester(b) @ O.sylvester(b).T, b * np.eye(b))


def test_block_size_of_llama_dims():
    assert O.hadamard_block_size(11008) == 256
    assert O.hadamard_block_size(14336) == 2048
    assert O.hadamard_block_size(28672) == 4096
    assert O.hadamard_block_size(4096) == 4096
    assert O.hadamard_block_size(1024) == 1024


@pytest.mark.parametrize("d", [8, 24, 96])
def test_transform_orthogonal_and_blockwise(d):
    r = rng(20 + d)
    s = r.choice([-1.0, 1.0], d)
    t = O.transform_matrix(d, s)
    np.testing.assert_allclose(t @ t.T, np.eye(d), atol=1e-14)
    m = r.standard_normal((d, 5))
    np.testing.assert_allclose(O.apply_transform(m, s, 0), t @ m, atol=1e-13)
    m2 = r.standard_normal((6, d))
    np.testing.assert_allclose(O.apply_transform(m2, s, 1), m2 @ t.T, atol=1e-13)
    # constant vector with unit signs maps to sqrt(b) e_0 in each block
    b = O.hadamard_block_size(d)
    ones = O.apply_transform(np.ones((1, d)), np.ones(d), 1)[0]
    exp = np.zeros(d); exp[::b] = math.sqrt(b)
    np.testing.assert_allclose(ones, exp, atol=1e-13)


# ------------------------------------------------------------------ BiIP (P9)

def _layer(r, d_out, d_in, n=64):
    x = r.standard_normal((n, d_in)) * r.uniform(0.2, 3.0, d_in)
    xq = x + 0.05 * r.standard_normal((n, d_in))
    g = r.standard_normal((n, d_out)) * 10 ** r.uniform(-2, 1, d_out)
    w = 0.02 * r.standard_normal((d_out, d_in))
    hx, hg, dxx = O.accumulate(xq, x, g)
    return w, hx, hg, dxx, 1.0 / n


def test_biip_scaling_formula_and_invariance():
    r = rng(30)
    d_out, d_in = 8, 16
    w, hx, hg, dxx, inv_n = _layer(r, d_out, d_in)
    si = r.choice([-1, 1], d_in); so = r.choice([-1, 1], d_out)
    out = O.biip(w, hx, hg, dxx, inv_n, si, so, O.BIIP_FULL)
    # S_X, S_G exactly as the BiIP equation states
    sx = (np.diag(hx * inv_n) / (w ** 2).sum(0)) ** 0.25
    sg = (np.diag(hg * inv_n) / (w ** 2).sum(1)) ** 0.25
    np.testing.assert_allclose(out["s_x"], sx, rtol=1e-14)
    np.testing.assert_allclose(out["s_g"], sg, rtol=1e-14)
    # W' = U S_G W S_X V^T with explicit dense U, V
    u = O.transform_matrix(d_out, so); v = O.transform_matrix(d_in, si)
    np.testing.assert_allclose(out["w"], u @ np.diag(sg) @ w @ np.diag(sx) @ v.T, atol=1e-14)
    # objective invariance: any W^' mapped back gives the same objective in original space
    wh_p = out["w"] + 0.01 * r.standard_normal((d_out, d_in))
    wh = np.diag(1 / sg) @ u.T @ wh_p @ v @ np.diag(1 / sx)
    a = O.objective(out["w"], wh_p, out["hx"], out["hg"], out["dxx"])
    b = O.objective(w, wh, hx * inv_n, hg * inv_n, dxx * inv_n)
    assert abs(a - b) <= 1e-10 * abs(b)
    # the rotation preserves traces; the traces are those of the processed H's
    sc = O.biip(w, hx, hg, dxx, inv_n, si, so, O.SCALE_IN | O.SCALE_OUT)
    assert abs(sc["tr_hx"] - out["tr_hx"]) < 1e-12 * abs(out["tr_hx"])
    assert abs(sc["tr_hg"] - out["tr_hg"]) < 1e-12 * abs(out["tr_hg"])
    assert abs(out["tr_hx"] - np.trace(out["hx"])) < 1e-12 * abs(out["tr_hx"])
    # tr(H_X (x) H_G) = tr H_X tr H_G  ([KronQ-hyper] Method: sensitivity derivation)
    assert abs(np.trace(np.kron(out["hx"], out["hg"])) - O.score(out["tr_hx"], out["tr_hg"])) \
        < 1e-10 * O.score(out["tr_hx"], out["tr_hg"])


def test_biip_off_is_identity_after_normalisation():
    r = rng(31)
    w, hx, hg, dxx, inv_n = _layer(r, 4, 8)
    out = O.biip(w, hx, hg, dxx, inv_n, np.ones(8), np.ones(4), 0)
    np.testing.assert_array_equal(out["w"], w)
    np.testing.assert_allclose(out["hx"], hx * inv_n)
    np.testing.assert_array_equal(out["s_x"], np.ones(8))


def test_biip_zero_column_gets_unit_scale():
    r = rng(32)
    w, hx, hg, dxx, inv_n = _layer(r, 4, 8)
    w[:, 3] = 0.0
    out = O.biip(w, hx, hg, dxx, inv_n, np.ones(8), np.ones(4), O.SCALE_IN | O.SCALE_OUT)
    assert out["s_x"][3] == 1.0


# ------------------------------------------------------------------ solve (P4, P5, P6)

def _gptq_ref_prop1(w, hx_damped, hg, fixed_cols, fixed_vals):
    """argmin over free columns of vec(dW)^T (H_X (x) H_G) vec(dW), explicit Kronecker system."""
    d_out, d_in = w.shape
    big = np.kron(hx_damped, hg)
    free = [j for j in range(d_in) if j not in fixed_cols]
    idx = lambda i, j: j * d_out + i               # column-stacked vec index
    fi = [idx(i, j) for j in free for i in range(d_out)]
    xi = [idx(i, j) for j in fixed_cols for i in range(d_out)]
    e_fixed = np.array([w[i, j] - fixed_vals[i, j] for j in fixed_cols for i in range(d_out)])
    e_free = -np.linalg.solve(big[np.ix_(fi, fi)], big[np.ix_(fi, xi)] @ e_fixed)
    out = w.copy()
    for n_, (j, i) in enumerate([(j, i) for j in free for i in range(d_out)]):
        out[i, j] = w[i, j] - e_free[n_]
    return out


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_obs_step_is_kronecker_optimum_and_hg_cancels(seed):
    # Before column p is rounded, the oracle's running weights equal the minimiser of the full
    # Kronecker objective over the not-yet-fixed columns, for any SPD H_G (Proposition 1: H_G
    # cancels) - pins the update's sign, the row of K it uses and the delta scaling.
    r = rng(40 + seed)
    d_out, d_in, bits = 3, 5, 2
    hx = spd(r, d_in, cond=50); w = r.standard_normal((d_out, d_in))
    k = O.cholinv(hx, 0.01)
    hxd = hx + 0.01 * np.mean(np.diag(hx)) * np.eye(d_in)
    res = O.quantize_layer(w, k, None, bits)
    for hg in (np.eye(d_out), spd(r, d_out, cond=1e3)):
        for p in range(d_in):
            opt = _gptq_ref_prop1(w, hxd, hg, list(range(p)), res["w_hat"])
            np.testing.assert_allclose(res["pre"][:, p], opt[:, p], atol=1e-10)


def test_diagonal_hessian_reduces_to_round_to_nearest():
    r = rng(50)
    w = r.standard_normal((6, 9)); hx = np.diag(r.uniform(0.5, 2.0, 9))
    res = O.quantize_layer(w, O.cholinv(hx, 0.01), None, 3)
    scale, zero = O.grid(w, 3)
    for p in range(9):
        rtn = np.clip(np.rint(w[:, p].astype(np.float32) / scale) + zero, 0, 7)
        np.testing.assert_array_equal(res["codes"][:, p], rtn)


def test_grid_textbook_values():
    # row [-1, 0, 0.5, 2] at 2 bits: scale = 3/3 = 1, zero = rint(1) = 1
    scale, zero = O.grid(np.array([[-1.0, 0.0, 0.5, 2.0], [3.0, 3.0, 3.0, 3.0]]), 2)
    assert scale[0] == 1.0 and zero[0] == 1.0
    assert scale[1] == 1.0 and zero[1] == -3.0           # hi == lo: scale := 1
    c = O.quantize_codes(np.array([-1.0, 0.5, 2.5]), np.float32(1.0), np.float32(1.0), 2)
    np.testing.assert_array_equal(c, [0.0, 1.0, 3.0])     # rint(0.5) = 0 (half to even) + 1


def test_error_feedback_energy_identity():
    # Per row, sum_p delta_p^2 = e (H + lambda I) e^T with e = W - W^  (P = 0): the OBS losses add.
    r = rng(51)
    d_out, d_in = 4, 12
    hx = spd(r, d_in, cond=100); w = r.standard_normal((d_out, d_in))
    k = O.cholinv(hx, 0.01)
    hxd = hx + 0.01 * np.mean(np.diag(hx)) * np.eye(d_in)
    res = O.quantize_layer(w, k, None, 2)
    deq = res["w_hat"]
    delta = (res["pre"] - deq) / np.diag(k)[None, :]
    e = w - deq
    for i in range(d_out):
        assert abs((delta[i] ** 2).sum() - e[i] @ hxd @ e[i]) < 1e-9 * max(1, e[i] @ hxd @ e[i])


def test_p_matrix_structure_and_drift_cancellation():
    r = rng(60)
    n, d = 200, 6
    x = r.standard_normal((n, d)) @ r.standard_normal((d, d))
    eps = 0.1
    hx, _, dxx = O.accumulate((1 - eps) * x, x)
    k = O.cholinv(hx / n, 0.0)
    p = O.p_matrix(dxx / n, k)
    np.testing.assert_array_equal(p, np.triu(p, 1))
    # untruncated pre-shift w + w (D K^T) K = w + w D H^-1 = w / (1 - eps): drift cancelled
    w = r.standard_normal((3, d))
    full = w + w @ ((dxx / n) @ k.T) @ k
    np.testing.assert_allclose(full, w / (1 - eps), rtol=1e-9)


def test_p_matrix_golden_cases():
    # [KronQ-hyper] Method, OBS update: the W_:,p [P]_p,p+1: term. P = striu(D K^T) K is the
    # reading of the undefined GPTAQ matrix (causal part of the exact shift w D (H + lambda I)^-1);
    # the cases are worked by hand in tests/golden/p_matrix_cases.json. A transposed or swapped
    # operand (K striu(D K^T), striu(K^T D) K, striu(D K) K, striu(M) K^T) or a non-strict
    # triangle changes at least one entry of these small-integer cases.
    with open(os.path.join(GOLDEN, "p_matrix_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        k = np.array(c["k"], dtype=np.float64)
        d = np.array(c["d"], dtype=np.float64)
        p = O.p_matrix(d, k)
        np.testing.assert_array_equal(p, np.array(c["p"], dtype=np.float64), err_msg=c["name"])
        w = np.array(c["w"], dtype=np.float64)
        np.testing.assert_array_equal(w @ (np.eye(3) + p), np.array(c["w_preshift"], dtype=np.float64),
                                      err_msg=c["name"])


@pytest.mark.parametrize("seed", [64, 65, 66])
def test_p_matrix_is_causal_part_of_exact_shift(seed):
    # [KronQ-hyper] Method, OBS update, with the reading of P as the causal part of the exact
    # row shift w D (H + lambda I)^-1. In the K basis (right-multiplying by K^-1) that shift is
    # w D (H + lambda I)^-1 K^-1; P K^-1 must equal its strictly upper part and vanish on and
    # below the diagonal. (H + lambda I)^-1 is taken from a plain matrix inverse here, not from
    # K, so a slip in how p_matrix combines D and K cannot cancel out.
    r = rng(seed)
    d = 7
    h = spd(r, d, cond=50.0)
    lam = O.damping(h, 0.01)
    dxx = r.standard_normal((d, d))
    k = O.cholinv(h, 0.01)
    p = O.p_matrix(dxx, k)
    kinv = np.linalg.inv(k)
    shift = dxx @ np.linalg.inv(h + lam * np.eye(d)) @ kinv
    got = p @ kinv
    np.testing.assert_allclose(got, np.triu(shift, 1), rtol=0, atol=1e-10 * np.abs(shift).max())
    # the full (untruncated) shift recovers the exact optimum w + w D (H + lambda I)^-1
    w = r.standard_normal((3, d))
    np.testing.assert_allclose(w + (w @ dxx @ k.T) @ k,
                               w + w @ dxx @ np.linalg.inv(h + lam * np.eye(d)), rtol=1e-9)


def _plain_gptq(w, k, bits):
    scale, zero = O.grid(w, bits)
    cur = w.copy(); codes = np.zeros(w.shape)
    for p in range(w.shape[1]):
        c = np.clip(np.rint(cur[:, p].astype(np.float32) / scale) + zero, 0, 2 ** bits - 1)
        dq = (scale * (c - zero)).astype(np.float32).astype(np.float64)
        err = (cur[:, p] - dq) / k[p, p]
        cur[:, p:] -= np.outer(err, k[p, p:])
        codes[:, p] = c
    return codes


def test_asymmetric_update_equals_gptq_on_preshifted_weights():
    # The P term uses the weights before any update, so its total on column j is known up
    # front: the literal update equals plain GPTQ on W (I + P) with W's own grid, and the final
    # error decomposes as e = delta K - W P.
    r = rng(61)
    n, d_out, d_in, bits = 300, 5, 10, 2
    x = r.standard_normal((n, d_in)) @ r.standard_normal((d_in, d_in))
    xq = x + 0.3 * r.standard_normal((n, d_in))
    hx, _, dxx = O.accumulate(xq, x)
    hx /= n; dxx /= n
    k = O.cholinv(hx, 0.01)
    w = r.standard_normal((d_out, d_in))
    res = O.quantize_layer(w, k, dxx, bits)
    p = O.p_matrix(dxx, k)
    # GPTQ on W(I+P) with W's grid
    scale, zero = O.grid(w, bits)
    cur = w @ (np.eye(d_in) + p); codes = np.zeros(w.shape)
    for c_ in range(d_in):
        t = cur[:, c_] / scale
        c = np.clip(np.rint(cur[:, c_].astype(np.float32) / scale) + zero, 0, 2 ** bits - 1)
        dq = (scale * (c - zero)).astype(np.float64)
        err = (cur[:, c_] - dq) / k[c_, c_]
        cur[:, c_:] -= np.outer(err, k[c_, c_:])
        codes[:, c_] = c
        assert np.all(np.abs(t - np.floor(t) - 0.5) > 1e-9)   # no near-tie in this draw
    np.testing.assert_array_equal(res["codes"], codes)
    delta = (res["pre"] - res["w_hat"]) / np.diag(k)[None, :]
    np.testing.assert_allclose(w - res["w_hat"], delta @ k - w @ p, atol=1e-10)


def test_objective_not_below_exhaustive_optimum():
    r = rng(62)
    d_in, bits = 5, 2
    hx = spd(r, d_in, cond=30); w = r.standard_normal((2, d_in))
    k = O.cholinv(hx, 0.0)
    res = O.quantize_layer(w, k, None, bits)
    scale, zero = O.grid(w, bits)
    import itertools
    for i in range(2):
        best = min(
            float((w[i] - scale[i] * (np.array(c) - zero[i])) @ hx
                  @ (w[i] - scale[i] * (np.array(c) - zero[i])))
            for c in itertools.product(range(4), repeat=d_in))
        e = w[i] - res["w_hat"][i]
        assert e @ hx @ e >= best - 1e-12


def test_follow_mode_adopts_only_near_ties():
    r = rng(63)
    w = r.standard_normal((4, 6)); hx = spd(r, 6)
    k = O.cholinv(hx, 0.01)
    base = O.quantize_layer(w, k, None, 2)
    same = O.quantize_layer(w, k, None, 2, follow_codes=base["codes"])
    np.testing.assert_array_equal(base["codes"], same["codes"])
    # other codes are never adopted away from ties
    other = (base["codes"].astype(int) + 1) % 4
    fol = O.quantize_layer(w, k, None, 2, follow_codes=other)
    assert np.array_equal(fol["codes"] != base["codes"], fol["near_tie"] & (fol["codes"] != base["codes"]))
    assert not same["disagree"].any()
    # a disagreement is recorded exactly where a different code was adopted at a near-tie
    assert np.array_equal(fol["disagree"][:, 0], fol["near_tie"][:, 0] & (other[:, 0] != base["codes"][:, 0]))


# ------------------------------------------------------------------ incoherence figure (P10)

def test_biip_makes_gradient_covariance_incoherent():
    # [KronQ-hyper] Method, incoherence figure: mu(H_G)/sqrt(d_out) is about 0.99 before BiIP and
    # below 0.10 after. Gradients with log-uniform channel scales over [1e-3, 1e1] reproduce the
    # setting. For the population covariance diag(sigma^2) (distinct eigenvalues) the figure's
    # numbers hold exactly: 1 before, 1/sqrt(256) = 0.0625 after.
    import torch
    from post_quantization_b200 import synth
    d, n = 256, 2048
    gseed = synth.seed_for("pin-mu", "G")
    sig = synth.gradient_scales(d, synth.seed_for(gseed, "sigma")).double().numpy()
    w = synth.weight(d, d, synth.seed_for("pin-mu", "W"), dtype=torch.float32).double().numpy()
    so = synth.rademacher(d, synth.seed_for("pin-mu", "so")).numpy()
    pop = O.biip(w, np.eye(d), np.diag(sig ** 2), None, 1.0, np.ones(d), so,
                 O.SCALE_OUT | O.ROTATE_OUT)
    assert O.mu_incoherence(np.diag(sig ** 2)) >= 0.9
    assert abs(O.mu_incoherence(pop["hg"]) - 1 / 16) < 1e-9
    # Sampled covariance (2048 tokens): eigenvalues of the weak channels nearly coincide and their
    # eigenvectors mix, so the floor after any rotation is the largest entry of a delocalised
    # unit vector, about sqrt(2 ln(2d)/d) = 0.2 at d = 256; the drop from ~1 is what is checked.
    g = synth.gradients(n, d, gseed).double().numpy()
    _, hg, _ = O.accumulate(np.zeros((n, 1)), None, g)
    out = O.biip(w, np.eye(d), hg, None, 1.0 / n, np.ones(d), so, O.SCALE_OUT | O.ROTATE_OUT)
    assert O.mu_incoherence(hg / n) >= 0.9
    assert O.mu_incoherence(out["hg"]) <= 0.3
    # BiIP lowers the spread of the weights' row norms (CV_out) - [KronQ-hyper] Method
    x = synth.correlated_x(n, d, synth.seed_for("pin-mu", "X")).double().numpy()
    hx, _, _ = O.accumulate(x)
    si = synth.rademacher(d, synth.seed_for("pin-mu", "si")).numpy()
    full = O.biip(w, hx, hg, None, 1.0 / n, si, so, O.BIIP_FULL)
    scaled = O.biip(w, hx, hg, None, 1.0 / n, si, so, O.SCALE_IN | O.SCALE_OUT)
    assert O.cv_norms(full["w"])[1] < O.cv_norms(scaled["w"])[1]


# ------------------------------------------------------------------ allocation (P11)

def test_allocation_golden_cases():
    with open(os.path.join(GOLDEN, "allocation_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        s, bits = O.score_allocate(c["tr_hx"], c["tr_hg"], c["n_params"], c["choices"],
                                   c["avg_bits"])
        assert bits == c["bits"], c["name"]
        total = sum(c["n_params"])
        assert sum(b * n for b, n in zip(bits, c["n_params"])) <= math.floor(c["avg_bits"] * total)


def test_allocation_shared_input_tie_broken_by_gradients():
    # [KronQ-hyper] Method: Q, K, V share H_X, so tr(H_X) ties; tr(H_G) separates them.
    s, bits = O.score_allocate([5.0, 5.0, 5.0], [1.0, 1.0, 1.0], [10, 10, 10], [2, 4], 8 / 3)
    assert bits == [4, 2, 2]                       # pure tie: index order
    s, bits = O.score_allocate([5.0, 5.0, 5.0], [0.5, 3.0, 1.0], [10, 10, 10], [2, 4], 8 / 3)
    assert bits == [2, 4, 2]


def test_allocation_rejects_nan_and_infeasible_budget():
    with pytest.raises(ValueError):
        O.score_allocate([float("nan")], [1.0], [10], [2, 3], 3)
    with pytest.raises(ValueError):
        O.score_allocate([1.0], [1.0], [10], [2, 3], 1.5)


# ------------------------------------------------------------------------------ group-wise grid
# [KronQ-hyper] Experiments quote 2-bit results with g = 128: one grid per row and per 128
# consecutive columns, taken when the solve reaches the group (from the weights it is about to
# quantize).

def test_group_covering_all_columns_is_the_per_row_grid():
    # with P = 0 and one group spanning the row, the group grid is taken at column 0 from W
    # itself: the same solve as the per-row grid
    r = rng(71)
    d_out, d_in = 6, 37
    w = 0.02 * r.standard_normal((d_out, d_in))
    a = r.standard_normal((d_in, d_in))
    k = O.cholinv(a @ a.T / d_in + 0.1 * np.eye(d_in), 0.01)
    per_row = O.quantize_layer(w, k, None, 3)
    one_group = O.quantize_layer(w, k, None, 3, group=d_in)
    assert np.array_equal(per_row["codes"], one_group["codes"])
    assert np.array_equal(per_row["w_hat"], one_group["w_hat"])
    assert np.array_equal(per_row["scale"], one_group["scale"][:, 0])
    assert np.array_equal(per_row["zero"], one_group["zero"][:, 0])


@pytest.mark.parametrize("group", [8, 16, 40])
def test_group_grid_without_feedback_is_groupwise_rtn(group):
    # diagonal H: K is diagonal, the error of a column feeds nothing forward, and the solve is
    # round-to-nearest with each group's own min-max grid (brute force per group, ragged last)
    r = rng(72 + group)
    d_out, d_in, bits = 5, 43, 2
    w = r.standard_normal((d_out, d_in))
    k = O.cholinv(np.diag(r.uniform(0.5, 2.0, d_in)), 0.01)
    assert np.count_nonzero(np.triu(k, 1)) == 0
    res = O.quantize_layer(w, k, None, bits, group=group)
    maxq = 2 ** bits - 1
    for g0 in range(0, d_in, group):
        blk = w[:, g0:g0 + group].astype(np.float32)
        for i in range(d_out):
            lo, hi = np.float32(blk[i].min()), np.float32(blk[i].max())
            s = np.float32((hi - lo) / np.float32(maxq)) if hi != lo else np.float32(1.0)
            z = np.float32(np.rint(np.float32(-lo) / s))
            assert res["scale"][i, g0 // group] == s and res["zero"][i, g0 // group] == z
            for j in range(blk.shape[1]):
                c = min(max(np.rint(np.float32(blk[i, j]) / s) + z, 0), maxq)
                assert res["codes"][i, g0 + j] == c


def test_group_grid_sees_the_pending_p_terms():
    # with K diagonal nothing but P moves a column before it is quantized, so the value of each
    # column at its turn ("pre") is exactly what the group's grid must have been taken from:
    # a dropped P term, or one from the wrong triangle, changes some group's min or max
    r = rng(75)
    n, d_out, d_in, bits, group = 400, 6, 24, 3, 8
    x = r.standard_normal((n, d_in))
    xq = x + 0.4 * r.standard_normal((n, d_in))
    _, _, dxx = O.accumulate(xq, x)
    dxx /= n
    k = O.cholinv(np.diag(r.uniform(0.5, 2.0, d_in)), 0.01)
    w = r.standard_normal((d_out, d_in))
    res = O.quantize_layer(w, k, dxx, bits, group=group)
    assert np.abs(O.p_matrix(dxx, k)).max() > 1e-3          # P is not negligible here
    for g0 in range(0, d_in, group):
        s, z = O.grid(res["pre"][:, g0:g0 + group], bits)
        # the two sides sum the same P terms in different orders (fp64): equal up to rounding
        assert np.allclose(s, res["scale"][:, g0 // group], rtol=1e-6, atol=0)
        assert np.array_equal(z, res["zero"][:, g0 // group])


def test_follow_grid_adopts_only_near_ties():
    # following another side's group grids changes nothing when that side equals this one, and
    # a scale further off than scale_rtol is never adopted
    r = rng(76)
    d_out, d_in, group = 4, 32, 16
    w = r.standard_normal((d_out, d_in))
    a = r.standard_normal((d_in, d_in))
    k = O.cholinv(a @ a.T / d_in + 0.1 * np.eye(d_in), 0.01)
    own = O.quantize_layer(w, k, None, 3, group=group)
    same = O.quantize_layer(w, k, None, 3, group=group, follow_grid=(own["scale"], own["zero"]))
    assert np.array_equal(same["codes"], own["codes"]) and not same["grid_tie"].any()
    off = O.quantize_layer(w, k, None, 3, group=group,
                           follow_grid=(own["scale"] * 1.01, own["zero"] + 1))
    assert np.array_equal(off["scale"], own["scale"]) and np.array_equal(off["zero"], own["zero"])


# ------------------------------------------------------------------ inference side

@pytest.mark.parametrize("d", [1, 2, 8, 48, 64, 192])
def test_fwht_matches_explicit_sylvester_blocks(d):
    # (I (x) H_b) along the last axis equals the product with the textbook Sylvester blocks
    r = rng(88)
    m = r.standard_normal((3, d))
    b = O.hadamard_block_size(d)
    want = (m.reshape(3, d // b, b) @ O.sylvester(b).T).reshape(3, d)
    np.testing.assert_allclose(O.fwht_last(m), want, rtol=0, atol=1e-12)
    # H_b H_b = b I
    np.testing.assert_allclose(O.fwht_last(O.fwht_last(m)), b * m, atol=1e-11)


@pytest.mark.parametrize("flags", [15, 3, 12, 5, 10, 0])
def test_qlinear_inverts_the_incoherence_processing(flags):
    # With the unquantized W' = U S_G W S_X V^T in place of W^', the layer gives back W x:
    # S_G^-1 U^T (U S_G W S_X V^T) V S_X^-1 = W. A transposed U or V, an inverted scale, or a
    # sign taken on the wrong side of the Hadamard product breaks the identity.
    r = rng(90)
    d_out, d_in = 24, 40      # Hadamard blocks of 8 on both sides, several per vector
    w, hx, hg, dxx, inv_n = _layer(r, d_out, d_in)
    si = r.choice([-1, 1], d_in); so = r.choice([-1, 1], d_out)
    out = O.biip(w, hx, hg, dxx, inv_n, si, so, flags)
    x = 3.0 * r.standard_normal((5, d_in))
    y = O.qlinear_dense(out["w"], x, out["s_x"], out["s_g"], si, so, flags)
    np.testing.assert_allclose(y, x @ w.T, rtol=0, atol=1e-12 * np.abs(x @ w.T).max())
    # the same map with explicit dense transforms
    u = O.transform_matrix(d_out, so) if flags & O.ROTATE_OUT else np.eye(d_out)
    v = O.transform_matrix(d_in, si) if flags & O.ROTATE_IN else np.eye(d_in)
    wh = r.standard_normal((d_out, d_in))
    dense = np.diag(1 / out["s_g"]) @ u.T @ wh @ v @ np.diag(1 / out["s_x"])
    np.testing.assert_allclose(O.qlinear_dense(wh, x, out["s_x"], out["s_g"], si, so, flags),
                               x @ dense.T, rtol=0, atol=1e-12 * np.abs(x @ dense.T).max())


@pytest.mark.parametrize("group", [0, 16])
def test_dequantize_matches_the_solve_and_the_rtn_bound(group):
    r = rng(91)
    d_out, d_in, bits = 6, 40, 3
    w = r.standard_normal((d_out, d_in))
    # the solve's own dequantized weights, kept in fp32 there
    res = O.quantize_layer(w, O.cholinv(spd(r, d_in), 0.01), None, bits, group=group)
    wq = O.dequantize_layer(res["codes"], res["scale"], res["zero"], group)
    np.testing.assert_allclose(wq, res["w_hat"], rtol=2.0 ** -23, atol=0)
    # diagonal H: the solve is round-to-nearest, so every element lies within half a step of
    # its own group's grid (a zero point of the wrong sign or a column mapped to the wrong
    # group's grid does not)
    k = O.cholinv(np.diag(r.uniform(0.5, 2.0, d_in)), 0.01)
    res = O.quantize_layer(w, k, None, bits, group=group)
    wq = O.dequantize_layer(res["codes"], res["scale"], res["zero"], group)
    sc = np.asarray(res["scale"], dtype=np.float64).reshape(d_out, -1)
    per_el = sc[:, np.arange(d_in) // group] if group else np.repeat(sc, d_in, axis=1)
    assert np.all(np.abs(wq - w) <= 0.5 * per_el * (1 + 1e-6))


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("shape", [(1, 1), (5, 37), (130, 300), (128, 256)])
def test_pack_roundtrip_size_and_density(bits, shape):
    r = rng(92)
    codes = r.integers(0, 1 << bits, size=shape).astype(np.uint8)
    p = O.pack_codes(codes, bits)
    t, g = -(-shape[0] // 128), -(-shape[1] // 128)
    assert p.dtype == np.uint8 and p.size == O.packed_bytes(*shape, bits) == t * g * 2048 * bits
    np.testing.assert_array_equal(O.unpack_codes(p, *shape, bits), codes)
    # every code bit lands on its own bit, padding stays zero
    pop = lambda a: int(np.unpackbits(a.view(np.uint8)).sum())
    assert pop(p) == pop(codes)


def test_pack_hand_worked_positions():
    # single codes placed by hand; the expected byte follows the format's wording: byte k of
    # row r's string sits at (t G + g) 2048 b + 1024 (k // 8) + 8 r + (k mod 8) of the packed
    # array; word w of the string is its bytes 4w..4w+3
    def one(bits, shape, row, col, code):
        c = np.zeros(shape, dtype=np.uint8)
        c[row, col] = code
        p = O.pack_codes(c, bits)
        return {int(i): int(p[i]) for i in np.flatnonzero(p)}
    # b=2, col 1 (w 0, k 0, j 1): bits 8-9 -> string byte 1, bits 0-1
    assert one(2, (1, 20), 0, 1, 3) == {1: 0x03}
    # b=2, col 6 (w 0, k 1, j 2): bits 18-19 -> byte 2, bits 2-3; code 2 -> bit 3
    assert one(2, (1, 20), 0, 6, 2) == {2: 0x08}
    # b=2, row 1, col 15 (w 0, k 3, j 3): bits 30-31 -> byte 3, bits 6-7; row 1 of piece 0
    # starts at byte 8
    assert one(2, (2, 20), 1, 15, 3) == {11: 0xC0}
    # b=2, row 3, col 40 (w 2, k 2, j 0): bits 4-5 of word 2 -> string byte 8 = piece 1, k 0:
    # 1024 + 24
    assert one(2, (4, 60), 3, 40, 1) == {1048: 0x10}
    # b=4, col 5 (w 0, k 1, j 1): bits 12-15 -> byte 1 high nibble
    assert one(4, (1, 20), 0, 5, 0xA) == {1: 0xA0}
    # b=4, row 2, col 127 (w 15, k 1, j 3): bits 28-31 of word 15 -> string byte 63 = piece 7,
    # k 7: 7168 + 16 + 7
    assert one(4, (3, 128), 2, 127, 0x9) == {7191: 0x90}
    # b=3, col 5 (low bits: w 0, k 1, j 1 -> bits 10-11; top bit: word 2, k 1, j 1 -> bit 9):
    # code 7 -> byte 1 bits 2-3 and byte 9 bit 1 (piece 1, k 1: 1025)
    assert one(3, (1, 40), 0, 5, 7) == {1: 0x0C, 1025: 0x02}
    # b=3, col 30 (low bits: w 1, k 3, j 2 -> bits 22-23 of word 1; top: word 2, k 7, j 2 ->
    # bit 23): code 4 -> top bit only -> string byte 10 (piece 1, k 2: 1026), bit 7
    assert one(3, (1, 40), 0, 30, 4) == {1026: 0x80}
    # b=3, col 33 (chunk 1: w 3, k 0, j 1 -> bits 8-9 of word 3 = string byte 13; top: word 5,
    # bit 8 = byte 21 = piece 2, k 5: 2048 + 5): code 3 -> low bits only
    assert one(3, (1, 40), 0, 33, 3) == {1029: 0x03}
    # second group of tile 0 (G = 2) and first group of tile 1 (row 128)
    assert one(2, (1, 200), 0, 128, 1) == {4096: 0x01}
    assert one(4, (129, 20), 128, 0, 1) == {8192: 0x01}


def test_qlinear_of_codes_is_the_dense_layer_of_their_dequantization():
    r = rng(93)
    d_out, d_in, bits, group = 16, 48, 2, 16
    codes = r.integers(0, 4, size=(d_out, d_in)).astype(np.uint8)
    scale = r.uniform(0.01, 0.1, (d_out, 3)).astype(np.float32)
    zero = r.integers(-1, 4, (d_out, 3)).astype(np.float32)
    s_x = r.uniform(0.5, 2, d_in); s_g = r.uniform(0.5, 2, d_out)
    si = r.choice([-1, 1], d_in); so = r.choice([-1, 1], d_out)
    x = r.standard_normal((3, d_in))
    y = O.qlinear(x, codes, scale, zero, s_x, s_g, si, so, O.BIIP_FULL, group)
    # brute force: element-by-element dequantization, explicit dense transforms
    wq = np.zeros((d_out, d_in))
    for i in range(d_out):
        for j in range(d_in):
            wq[i, j] = float(scale[i, j // group]) * (int(codes[i, j]) - float(zero[i, j // group]))
    u = O.transform_matrix(d_out, so); v = O.transform_matrix(d_in, si)
    want = x @ (np.diag(1 / s_g) @ u.T @ wq @ v @ np.diag(1 / s_x)).T
    np.testing.assert_allclose(y, want, rtol=0, atol=1e-12 * np.abs(want).max())


@pytest.mark.parametrize("group", [0, 128])
def test_pack_grid_places_each_pair(group):
    # every (row, group) pair is found at (t G' + g) 128 + r and nothing else is non-zero
    r = rng(94)
    d_out, d_in = 300, 520
    gp = -(-d_in // 128) if group else 1
    sc = r.uniform(0.1, 1, (d_out, gp)).astype(np.float32)
    zr = r.integers(1, 5, (d_out, gp)).astype(np.float32)
    pk = O.pack_grid(sc if group else sc[:, 0], zr if group else zr[:, 0], d_out, d_in, group)
    assert pk.shape == (3 * gp * 128, 2)
    for row in range(d_out):
        for g in range(gp):
            idx = ((row // 128) * gp + g) * 128 + row % 128
            assert pk[idx, 0] == sc[row, g] and pk[idx, 1] == zr[row, g]
    assert np.count_nonzero(pk[:, 1]) == d_out * gp


# ------------------------------------------------------------------ output-side feedback (comparison variant)

def test_udu_factor_is_the_inverse_factor_rescaled():
    # H = U diag(d) U^T with U unit upper triangular; the same U follows from the damped inverse
    # factor, K^T K = H^-1  =>  H = K^-1 K^-T, so U = K^-1 diag(K_pp) and d = 1 / K_pp^2.
    r = rng(80)
    h = spd(r, 9, cond=40.0)
    u, dg = O.udu_factor(h)
    np.testing.assert_allclose(u @ np.diag(dg) @ u.T, h, rtol=0, atol=1e-12 * np.abs(h).max())
    np.testing.assert_array_equal(np.tril(u, -1), 0)
    np.testing.assert_allclose(np.diag(u), 1.0, rtol=0, atol=1e-15)
    k = O.cholinv(h, 0.0)
    np.testing.assert_allclose(u, np.linalg.inv(k) * np.diag(k)[None, :], rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(dg, 1.0 / np.diag(k) ** 2, rtol=1e-9)


@pytest.mark.parametrize("seed,bits", [(81, 2), (82, 3), (83, 4)])
def test_output_feedback_rounding_reduces_to_the_column_solve(seed, bits):
    # [YAQA notes]: with H_O = I the output-side terms vanish and the fixed point is LDLQ, i.e.
    # the column-wise OBS solve without P (GPTQ); same grid, so the same codes.
    r = rng(seed)
    m, n = 7, 12
    w = r.standard_normal((m, n))
    hi = spd(r, n, cond=50.0)
    res = O.yaqa_round(w, np.eye(m), hi, bits)
    ref = O.quantize_layer(w, O.cholinv(hi, 0.01), None, bits)
    np.testing.assert_array_equal(res["codes"], ref["codes"])
    np.testing.assert_allclose(res["w_hat"], ref["w_hat"], rtol=0, atol=1e-12)


def _yaqa_elementwise(w, ho, hi, bits, damp_rel=0.01):
    """The fixed point evaluated element by element in row-major order (a valid order: element
    (i, j) reads the errors of elements (k, l) with k <= i and l <= j only), scalar loops."""
    m, n = w.shape
    ho = ho + O.damping(ho, damp_rel) * np.eye(m)
    hi = hi + O.damping(hi, damp_rel) * np.eye(n)
    uo = O.udu_factor(ho)[0]
    ui = O.udu_factor(hi)[0]
    scale, zero = O.grid(w, bits)
    maxq = np.float32(2 ** bits - 1)
    delta = np.zeros((m, n))
    codes = np.zeros((m, n), dtype=np.float32)
    for i in range(m):
        for j in range(n):
            t = w[i, j]
            for k in range(i + 1):
                for l in range(j + 1):
                    if (k, l) != (i, j):
                        t += uo[k, i] * delta[k, l] * ui[l, j]
            c = np.clip(np.rint(np.float32(t) / scale[i]) + zero[i], np.float32(0), maxq)
            codes[i, j] = c
            delta[i, j] = w[i, j] - float(np.float32(scale[i] * (c - zero[i])))
    return codes


@pytest.mark.parametrize("seed", [84, 85, 86])
def test_output_feedback_fixed_point_equals_elementwise_order(seed):
    r = rng(seed)
    m, n, bits = 5, 6, 2
    w = r.standard_normal((m, n))
    ho = spd(r, m, cond=20.0); hi = spd(r, n, cond=20.0)
    res = O.yaqa_round(w, ho, hi, bits)
    np.testing.assert_array_equal(res["codes"], _yaqa_elementwise(w, ho, hi, bits))
    # reached within m + n - 1 updates (+1 iteration that finds nothing to change)
    assert res["iterations"] <= m + n
    # a fixed point: one more update changes no code
    again = O.yaqa_round(w, ho, hi, bits, follow_codes=res["codes"], tie_tol=0.0)
    np.testing.assert_array_equal(again["codes"], res["codes"])
