"""KronQ per-layer hot path: plain, slow, fp64 CPU oracle.

TEST INFRASTRUCTURE ONLY. This module is the yardstick the CUDA library is checked against.
Only the test suite, the smoke check and the benchmark's CPU-baseline / reference arm may
import it; the library itself never does, and the two share no code (the oracle uses numpy
and scipy; the library is CUDA C++).

What it computes, step by step, with the passage each step follows. Page names:
  [KronQ-hyper]  "KronQ: LLM Quantization via Kronecker-Factored Hessian", hyper.ai summary
                 (Method section; the only page that prints the equations).
  [KronQ-gist]   the same paper, gist.science technical summary (Methodology, Limitations).

  accumulate      H_X = E[x x^T], H_G = E[g g^T] under the K-FAC split H ~ H_X (x) H_G, and the
                  asymmetric term E[(x - x~) x~^T]            [KronQ-hyper] Method: Fisher eq.,
                                                              K-FAC split, asymmetric objective
  accumulate_diag the diagonal of G^T G alone: S_G and tr(H_G) read only the diagonal, and H_G
                  cancels from the column update           [KronQ-hyper] Method: BiIP equations,
                                                              sensitivity, Proposition 1
  biip            W <- S_G W S_X with S_X = diag(H_X,jj/|W_:,j|^2)^(1/4), S_G likewise on rows;
                  then W <- U W V^T, H_X <- V H_X V^T, H_G <- U H_G U^T, dXX^T <- V dXX^T V^T
                  with U, V random-sign Hadamard          [KronQ-hyper] Method: BiIP equations
  score           s = tr(H_G) * tr(H_X), after BiIP          [KronQ-hyper] Method: sensitivity
  cholinv         K = upper Cholesky factor of (H_X + lambda I)^-1, read as the "[H_X^-1]" rows
                  of the column update                      [KronQ-hyper] Method: OBS update
  p_matrix        P = striu(D K^T) K (GPTAQ's correction matrix; the pages name P but do not
                  define it - this is the documented reading)
  grid            per-output-row asymmetric min-max b-bit grid
  quantize_layer  column-wise OBS update, literally:
                    dW_:,p+1: = -delta_p [H_X^-1]_p,p+1: + W_:,p P_p,p+1:
                                                             [KronQ-hyper] Method: OBS update
  score_allocate  larger s gets more bits, greedy under an average-bit budget
                                                  [KronQ-hyper] Method: mixed precision;
                                                  [KronQ-gist] Experimental results (upgrade the
                                                  higher-scored sublayer first)
  objective       tr[H_G dW H_X dW^T] + 2 tr[H_G W D dW^T]  [KronQ-hyper] Method: objectives
  yaqa_round      comparison variant (prior art, not KronQ): rounding with input- and
                  output-side feedback, the fixed point W^ = Q(W + L_O'^T D L_I' + L_O'^T D +
                  D L_I')                       [YAQA notes] generalized LDLQ
  mu_incoherence  max_ij |Q_ij| over eigenvectors Q of H (mu(H)/sqrt(d))
                                                  [KronQ-hyper] Method: incoherence figure
  qlinear         the quantized layer on activations, y = S_G^-1 U^T W^' V S_X^-1 x with
                  W^' = scale (codes - zero): at inference only the orthogonal transforms are
                  added                                     [KronQ-gist] Limitations
  pack_codes      the library's packed storage of 2/3/4-bit codes (a format of this library,
                  defined in the inference-side section below; the pages fix none)

Precision: all continuous arithmetic is fp64. The two places where floating point decides an
integer (the grid's integer zero point and each quantized code) are evaluated in fp32, the
precision the CUDA kernels decide them in, so that both sides take the same decision.

Readings where the pages are silent or ambiguous (each is also listed in the design notes):
  * statistics are normalised by 1/N; H_X is built from the quantized-path input x~;
  * the asymmetric term is D = E[(x - x~) x~^T] with factor 2 in the objective and "+" in the
    update (exact expansion of E|W x - W^ x~|^2_{H_G});
  * S_X and S_G are both computed from the original W; H_X, D transform as S_X^-1 . S_X^-1,
    H_G as S_G^-1 . S_G^-1 (the only choice that leaves the objective unchanged); a zero norm or
    zero diagonal gives scale 1;
  * U = (1/sqrt(b)) (I (x) H_b) diag(sigma): Sylvester Hadamard blocks of b = largest power of
    two dividing d, caller-supplied signs;
  * damping lambda = damp_rel * mean diag(H_X after BiIP), added before factorisation;
  * grid: lo/hi = row min/max of W' before the solve, scale = (hi-lo)/(2^b-1) (1 if hi == lo),
    zero = rint(-lo/scale), codes clamp(rint(w/scale)+zero, 0, 2^b-1), round half to even;
  * columns in natural order; allocation is the greedy in score_allocate.

Parity pins: every function here is pinned by tests in tests/test_oracle_pins.py against
closed forms, brute force or textbook special cases; none is "parity unpinned".
"""
from __future__ import annotations

import functools
import math

import numpy as np
import scipy.linalg as sla

# flags of the incoherence step (same numeric values as the C header, re-declared here)
SCALE_IN = 1
SCALE_OUT = 2
ROTATE_IN = 4
ROTATE_OUT = 8
BIIP_FULL = SCALE_IN | SCALE_OUT | ROTATE_IN | ROTATE_OUT


class NotPositiveDefinite(Exception):
    pass


# ------------------------------------------------------------------------------------------
# Statistics
# ------------------------------------------------------------------------------------------

def accumulate(xq, xfp=None, g=None):
    """Raw (un-normalised) sums over the N calibration tokens (rows).

    hx_sum = X~^T X~, hg_sum = G^T G, dxx_sum = (X - X~)^T X~.
    [KronQ-hyper] Method: H_X = E[x x^T], H_G = E[g g^T] (K-FAC split of the empirical Fisher
    E[x x^T (x) g g^T]); the asymmetric objective's input-drift term dX X^T.
    """
    xq = np.asarray(xq, dtype=np.float64)
    hx = xq.T @ xq
    hg = None
    if g is not None:
        g = np.asarray(g, dtype=np.float64)
        hg = g.T @ g
    dxx = None
    if xfp is not None:
        xfp = np.asarray(xfp, dtype=np.float64)
        dxx = (xfp - xq).T @ xq
    return hx, hg, dxx


def accumulate_diag(g):
    """Raw diagonal sums diag(G^T G)_j = sum_t G_tj^2 over the N tokens (rows).

    [KronQ-hyper] Method: S_G = diag(H_G,ii / |W_i,:|^2)^(1/4) and the sensitivity tr(H_G) use
    only the diagonal of H_G, and Proposition 1 removes H_G from the column update, so a
    quantization that skips the objective and the incoherence figure needs only these sums.
    """
    g = np.asarray(g, dtype=np.float64)
    return np.einsum("tj,tj->j", g, g)


def fisher_kron(x, g):
    """Empirical Fisher E[vec(dL/dW) vec(dL/dW)^T] with dL/dW = g x^T, column-stacked vec.

    [KronQ-hyper] Method: Fisher equation, vec(g x^T) = x (x) g. Brute force, tiny sizes only.
    """
    x = np.asarray(x, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    n = x.shape[0]
    dim = x.shape[1] * g.shape[1]
    f = np.zeros((dim, dim))
    for t in range(n):
        grad = np.outer(g[t], x[t])           # dL/dW, d_out x d_in
        v = grad.reshape(-1, order="F")       # column-stacked vec
        f += np.outer(v, v)
    return f / n


# ------------------------------------------------------------------------------------------
# Hadamard blocks
# ------------------------------------------------------------------------------------------

def hadamard_block_size(d: int) -> int:
    """Largest power of two dividing d (the Hadamard block size used for dimension d)."""
    if d <= 0:
        raise ValueError("d must be positive")
    return d & (-d)


@functools.lru_cache(maxsize=16)
def _sylvester_cached(b: int) -> np.ndarray:
    i = np.arange(b)
    pc = np.zeros((b, b), dtype=np.int64)
    a = i[:, None] & i[None, :]
    while np.any(a):
        pc += a & 1
        a = a >> 1
    h = np.where(pc % 2 == 0, 1.0, -1.0)
    h.setflags(write=False)
    return h


def sylvester(b: int) -> np.ndarray:
    """Sylvester Hadamard matrix of order b: [H_b]_ij = (-1)^popcount(i & j)."""
    return _sylvester_cached(b)


def transform_matrix(d: int, signs) -> np.ndarray:
    """Dense U (or V) = (1/sqrt(b)) (I_{d/b} (x) H_b) diag(signs). Small d only."""
    b = hadamard_block_size(d)
    blk = np.kron(np.eye(d // b), sylvester(b)) / math.sqrt(b)
    return blk * np.asarray(signs, dtype=np.float64)[None, :]


def apply_transform(m, signs, axis: int):
    """Apply T = (1/sqrt(b)) (I (x) H_b) diag(signs) along one axis of m.

    axis=1 returns m T^T (rows transformed), axis=0 returns T m (columns transformed).
    Implemented with the block structure (reshape into d/b blocks of b and multiply each by the
    Sylvester matrix) so that large d stays tractable.
    """
    m = np.asarray(m, dtype=np.float64)
    d = m.shape[axis]
    b = hadamard_block_size(d)
    h = sylvester(b) / math.sqrt(b)
    s = np.asarray(signs, dtype=np.float64)
    if axis == 1:
        ms = m * s[None, :]
        r = ms.reshape(m.shape[0], d // b, b) @ h.T
        return r.reshape(m.shape[0], d)
    ms = m * s[:, None]
    r = np.matmul(h, ms.reshape(d // b, b, m.shape[1]))     # H_b times each block of rows
    return r.reshape(d, m.shape[1])


# ------------------------------------------------------------------------------------------
# Bidirectional incoherence processing
# ------------------------------------------------------------------------------------------

def biip(w, hx_sum, hg_sum=None, dxx_sum=None, inv_n=1.0, sign_in=None, sign_out=None,
         flags=BIIP_FULL):
    """Normalise the sums, rescale, rotate; return the processed layer and its traces.

    [KronQ-hyper] Method, BiIP equations:
      W <- S_G W S_X,  S_X = diag(H_X,jj / |W_:,j|^2)^(1/4),  S_G = diag(H_G,ii / |W_i,:|^2)^(1/4)
      W <- U W V^T,  H_X <- V H_X V^T,  H_G <- U H_G U^T,  dXX^T <- V dXX^T V^T.
    The Hessians follow the scaling as H_X <- S_X^-1 H_X S_X^-1, H_G <- S_G^-1 H_G S_G^-1,
    D <- S_X^-1 D S_X^-1, which keeps tr[H_G dW H_X dW^T] unchanged.
    Returns dict: w, hx, hg (None if not given), dxx (None if not given), s_x, s_g, tr_hx, tr_hg.
    """
    w0 = np.asarray(w, dtype=np.float64)
    d_out, d_in = w0.shape
    hx = np.asarray(hx_sum, dtype=np.float64) * inv_n
    hg = None if hg_sum is None else np.asarray(hg_sum, dtype=np.float64) * inv_n
    dxx = None if dxx_sum is None else np.asarray(dxx_sum, dtype=np.float64) * inv_n
    if (flags & SCALE_OUT) and hg is None:
        raise ValueError("output-side scaling needs H_G")

    col_sq = (w0 * w0).sum(axis=0)    # |W_:,j|^2 of the original W
    row_sq = (w0 * w0).sum(axis=1)    # |W_i,:|^2 of the original W
    s_x = np.ones(d_in)
    s_g = np.ones(d_out)
    if flags & SCALE_IN:
        dx = np.diag(hx)
        ok = (col_sq > 0) & (dx > 0)
        s_x[ok] = (dx[ok] / col_sq[ok]) ** 0.25
    if flags & SCALE_OUT:
        dg = np.diag(hg)
        ok = (row_sq > 0) & (dg > 0)
        s_g[ok] = (dg[ok] / row_sq[ok]) ** 0.25

    wp = s_g[:, None] * w0 * s_x[None, :]
    hx = hx / np.outer(s_x, s_x)
    if dxx is not None:
        dxx = dxx / np.outer(s_x, s_x)
    if hg is not None:
        hg = hg / np.outer(s_g, s_g)

    if flags & ROTATE_IN:
        wp = apply_transform(wp, sign_in, axis=1)                      # W V^T
        hx = apply_transform(apply_transform(hx, sign_in, axis=0), sign_in, axis=1)  # V H V^T
        if dxx is not None:
            dxx = apply_transform(apply_transform(dxx, sign_in, axis=0), sign_in, axis=1)
    if flags & ROTATE_OUT:
        wp = apply_transform(wp, sign_out, axis=0)                     # U W
        if hg is not None:
            hg = apply_transform(apply_transform(hg, sign_out, axis=0), sign_out, axis=1)

    tr_hx = float(np.trace(hx))
    tr_hg = None if hg is None else float(np.trace(hg))
    return {"w": wp, "hx": hx, "hg": hg, "dxx": dxx, "s_x": s_x, "s_g": s_g,
            "tr_hx": tr_hx, "tr_hg": tr_hg}


def score(tr_hx, tr_hg):
    """s = tr(H_G) * tr(H_X)   [KronQ-hyper] Method: sensitivity score."""
    return float(tr_hg) * float(tr_hx)


# ------------------------------------------------------------------------------------------
# Damped inverse factor
# ------------------------------------------------------------------------------------------

def damping(h, damp_rel: float) -> float:
    return float(damp_rel) * float(np.mean(np.diag(h)))


def cholinv(h, damp_rel: float = 0.01):
    """K upper triangular with K^T K = (H + lambda I)^-1, lambda = damp_rel * mean diag H.

    Plain three-step route: Cholesky of H + lambda I, the explicit inverse, then the upper
    Cholesky factor of that inverse. K's rows are the "[H_X^-1]_p,p+1:" rows of the column
    update ([KronQ-hyper] Method: OBS update).
    """
    h = np.asarray(h, dtype=np.float64)
    d = h.shape[0]
    a = h + damping(h, damp_rel) * np.eye(d)
    try:
        l = np.linalg.cholesky(a)
    except np.linalg.LinAlgError as e:
        raise NotPositiveDefinite(str(e))
    linv = sla.solve_triangular(l, np.eye(d), lower=True)
    ainv = linv.T @ linv
    ainv = 0.5 * (ainv + ainv.T)
    try:
        l2 = np.linalg.cholesky(ainv)
    except np.linalg.LinAlgError as e:
        raise NotPositiveDefinite(str(e))
    return l2.T.copy()


def p_matrix(dxx, k):
    """GPTAQ correction matrix P = striu(D K^T) K (strictly upper triangular)."""
    m = np.asarray(dxx, dtype=np.float64) @ np.asarray(k, dtype=np.float64).T
    return np.triu(m, 1) @ k


# ------------------------------------------------------------------------------------------
# Grid and column-wise solve
# ------------------------------------------------------------------------------------------

def grid(w, bits: int):
    """Per-row asymmetric min-max grid; decisions in fp32. Returns (scale, zero) as float32."""
    w = np.asarray(w)
    maxq = np.float32(2 ** bits - 1)
    lo = w.min(axis=1).astype(np.float32)
    hi = w.max(axis=1).astype(np.float32)
    scale = ((hi - lo) / maxq).astype(np.float32)
    scale = np.where(hi == lo, np.float32(1.0), scale).astype(np.float32)
    zero = np.rint((-lo) / scale).astype(np.float32)
    return scale, zero


def quantize_codes(col, scale, zero, bits):
    """codes = clamp(rint(w/scale) + zero, 0, 2^b - 1), division and rounding in fp32."""
    maxq = np.float32(2 ** bits - 1)
    t = np.rint(col.astype(np.float32) / scale)
    return np.clip(t + zero, np.float32(0), maxq).astype(np.float32)


def dequantize(codes, scale, zero):
    return (scale * (codes - zero)).astype(np.float32)


def quantize_layer(w, k, dxx=None, bits: int = 4, follow_codes=None, tie_tol: float = 1e-3,
                   group: int = 0, follow_grid=None, scale_rtol: float = 1e-5):
    """Column-wise OBS / GPTAQ solve onto the per-row grid, literally, one column at a time.

    [KronQ-hyper] Method, OBS update:
        dW_:,p+1: = -delta_p [H_X^-1]_p,p+1: + W_:,p [P]_p,p+1:
    with delta_p = (w_p - deq(q(w_p))) / K_pp, [H_X^-1]_p,p+1: = K_p,p+1:, W_:,p the weights
    before quantization (after incoherence processing), P = p_matrix(dxx, k).

    follow_codes: optional array of codes from another implementation. Where this oracle's
    value sits within tie_tol grid units of a rounding boundary (a half-integer of w/scale) it
    adopts that code instead of its own, and records a near-tie; where it adopts a code that
    differs from its own decision it also records a disagreement. Every other code is its own.
    group: 0 for one grid per output row (from W before the solve); g > 0 for one grid per row
    and per g consecutive columns ([KronQ-hyper] Experiments, g = 128). A group's grid is taken
    when the solve reaches its first column, from the weights that the solve is about to
    quantize: the current (error-updated) weights plus the P contributions that the group's own
    earlier columns will still add (the solve quantizes W (I + P), updated). With P = 0 this is
    the grouped grid of GPTQ.
    follow_grid: optional (scale, zero) group grids from another implementation (group > 0).
    A group's grid comes from weights that each side has updated in its own arithmetic, so the
    two differ by rounding: this oracle adopts the other scale where it agrees with its own to
    scale_rtol, and the other zero only where its own -lo / scale lies within tie_tol of a
    rounding boundary (grid_tie counts those rows); anywhere else it keeps its own grid.
    Returns dict: codes (uint8), scale, zero (d_out, or d_out x groups), w_hat (fp64), near_tie
    (bool mask), disagree (bool mask), pre (fp64: each column's value just before it was
    quantized), grid_tie (rows x groups that adopted the other zero).
    """
    w0 = np.asarray(w, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    d_out, d_in = w0.shape
    p_mat = None if dxx is None else p_matrix(dxx, k)
    grid_tie = None
    if group:
        n_groups = (d_in + group - 1) // group
        scales = np.zeros((d_out, n_groups), dtype=np.float32)
        zeros = np.zeros((d_out, n_groups), dtype=np.float32)
        grid_tie = np.zeros((d_out, n_groups), dtype=bool)
    else:
        scale, zero = grid(w0, bits)
    cur = w0.copy()
    codes = np.zeros((d_out, d_in), dtype=np.uint8)
    near = np.zeros((d_out, d_in), dtype=bool)
    disagree = np.zeros((d_out, d_in), dtype=bool)
    pre = np.zeros((d_out, d_in))
    for p in range(d_in):
        if group and p % group == 0:
            g1 = min(d_in, p + group)
            target = cur[:, p:g1].copy()
            if p_mat is not None:
                # P terms from the group's own columns, not yet added: column j gets
                # sum over p <= q < j of W_:,q P_q,j
                target += w0[:, p:g1] @ np.triu(p_mat[p:g1, p:g1], 1)
            scale, zero = grid(target, bits)
            if follow_grid is not None:
                gi = p // group
                o_s = np.asarray(follow_grid[0], dtype=np.float32).reshape(d_out, -1)[:, gi]
                o_z = np.asarray(follow_grid[1], dtype=np.float32).reshape(d_out, -1)[:, gi]
                close = np.abs(o_s.astype(np.float64) - scale) <= scale_rtol * np.abs(scale)
                lo = target.min(axis=1).astype(np.float32)
                u = (-lo / scale).astype(np.float64)
                ztie = np.abs(u - (np.floor(u) + 0.5)) <= tie_tol
                take_z = close & ztie & (o_z != zero)
                grid_tie[:, gi] = take_z
                scale = np.where(close, o_s, scale).astype(np.float32)
                zero = np.where(take_z, o_z, zero).astype(np.float32)
            scales[:, p // group] = scale
            zeros[:, p // group] = zero
        col = cur[:, p].copy()
        pre[:, p] = col
        c = quantize_codes(col, scale, zero, bits)
        if follow_codes is not None:
            t = col / scale.astype(np.float64)
            dist = np.abs(t - (np.floor(t) + 0.5))
            tie = dist <= tie_tol
            near[:, p] = tie
            other = np.asarray(follow_codes)[:, p].astype(np.float32)
            disagree[:, p] = tie & (other != c)
            c = np.where(tie, other, c)
        dq = dequantize(c, scale, zero).astype(np.float64)
        delta = (col - dq) / k[p, p]
        if p + 1 < d_in:
            cur[:, p + 1:] -= np.outer(delta, k[p, p + 1:])
            if p_mat is not None:
                cur[:, p + 1:] += np.outer(w0[:, p], p_mat[p, p + 1:])
        cur[:, p] = dq
        codes[:, p] = c.astype(np.uint8)
    if group:
        scale, zero = scales, zeros
    return {"codes": codes, "scale": scale, "zero": zero, "w_hat": cur, "near_tie": near,
            "disagree": disagree, "pre": pre, "grid_tie": grid_tie}


# ------------------------------------------------------------------------------------------
# Inference side: the quantized layer applied to activations
# ------------------------------------------------------------------------------------------
#
# [KronQ-gist] Limitations: at inference the only overhead is the orthogonal transforms (the
# same ones as QuIP#'s). The layer that was quantized is W' = U S_G W S_X V^T; its quantized
# form W^' = scale (codes - zero) stands for W^ = S_G^-1 U^T W^' V S_X^-1 in the original basis,
# so   y = W^ x = S_G^-1 U^T ( W^' ( V S_X^-1 x ) ).
#
# Packed code format (a storage format of this library; the pages do not fix one). Codes of
# b = 2, 3 or 4 bits. Rows are cut into tiles of 128, columns into groups of 128; rows and
# columns past the matrix hold code 0. Tile t, group g is one blob of 128 x 128 x b bits at byte
# offset (t * G + g) * 2048 * b (G = ceil(d_in / 128)). Each row of the blob has a string of
# 16 * b bytes, read as little-endian 32-bit words; the string is stored in 8-byte pieces,
# piece p of row r at byte 1024 * p + 8 * r of the blob (so that 16 consecutive rows' pieces
# are contiguous). Inside the words, code j of each run of 4 columns sits in byte j, so that
# one shift and one mask turn a word into four 8-bit codes of consecutive columns:
#   b = 2: word w holds columns 16 w .. 16 w + 15; column 16 w + 4 k + j (k, j = 0..3) at
#          bits 8 j + 2 k and 8 j + 2 k + 1;
#   b = 4: word w holds columns 8 w .. 8 w + 7; column 8 w + 4 k + j (k = 0, 1) at bits
#          8 j + 4 k .. 8 j + 4 k + 3;
#   b = 3: each 32 columns 32 m .. 32 m + 31 take words 3 m, 3 m + 1, 3 m + 2: the low two bits
#          of columns 32 m .. + 15 and 32 m + 16 .. + 31 in words 3 m and 3 m + 1 as for b = 2,
#          and the top bit of column 32 m + 4 k + j (k = 0..7) at bit 8 j + k of word 3 m + 2.

PACK_ROWS = 128
PACK_COLS = 128
PACK_BITS = (2, 3, 4)


def packed_bytes(d_out: int, d_in: int, bits: int) -> int:
    """Size of the packed form: ceil(d_out/128) * ceil(d_in/128) blobs of 2048 * bits bytes."""
    if bits not in PACK_BITS:
        raise ValueError("packed codes have 2, 3 or 4 bits")
    t = -(-d_out // PACK_ROWS)
    g = -(-d_in // PACK_COLS)
    return t * g * 2048 * bits


def code_bit_positions(bits: int) -> np.ndarray:
    """(128, bits) array: for column c of a group and code bit i, the bit index (32 * word +
    bit in word) of that bit inside the row's string of 16 * bits bytes, following the format
    above."""
    if bits not in PACK_BITS:
        raise ValueError("packed codes have 2, 3 or 4 bits")
    pos = np.zeros((PACK_COLS, bits), dtype=np.int64)
    for c in range(PACK_COLS):
        if bits == 2:
            w, k, j = c // 16, (c % 16) // 4, c % 4
            for i in range(2):
                pos[c, i] = 32 * w + 8 * j + 2 * k + i
        elif bits == 4:
            w, k, j = c // 8, (c % 8) // 4, c % 4
            for i in range(4):
                pos[c, i] = 32 * w + 8 * j + 4 * k + i
        else:
            m, cc = c // 32, c % 32
            w, k, j = 3 * m + cc // 16, (cc % 16) // 4, cc % 4
            for i in range(2):
                pos[c, i] = 32 * w + 8 * j + 2 * k + i
            k8 = cc // 4
            pos[c, 2] = 32 * (3 * m + 2) + 8 * j + k8
    return pos


def _tiled_codes(codes, bits):
    codes = np.asarray(codes)
    d_out, d_in = codes.shape
    if codes.size and int(codes.max()) >= (1 << bits):
        raise ValueError("code out of range for the bit width")
    t = -(-d_out // PACK_ROWS)
    g = -(-d_in // PACK_COLS)
    full = np.zeros((t * PACK_ROWS, g * PACK_COLS), dtype=np.uint8)
    full[:d_out, :d_in] = codes
    # [tile][group][row in tile][column in group]
    return full.reshape(t, PACK_ROWS, g, PACK_COLS).transpose(0, 2, 1, 3)


def pack_codes(codes, bits: int) -> np.ndarray:
    """Packed form (uint8, packed_bytes(d_out, d_in, bits) bytes) of a d_out x d_in code array."""
    tiled = _tiled_codes(codes, bits)
    pos = code_bit_positions(bits)
    t, g = tiled.shape[:2]
    bitarr = np.zeros((t, g, PACK_ROWS, PACK_COLS * bits), dtype=np.uint8)
    for i in range(bits):
        bitarr[..., pos[:, i]] = (tiled >> i) & 1
    # bit j of the row's bit string is bit (j mod 8) of byte j // 8 (little-endian words)
    rowstr = np.packbits(bitarr, axis=-1, bitorder="little")       # t, g, 128 rows, 16 b
    # 8-byte pieces: blob byte 1024 p + 8 r + k holds byte 8 p + k of row r's string
    pieces = rowstr.reshape(t, g, PACK_ROWS, 2 * bits, 8).transpose(0, 1, 3, 2, 4)
    return np.ascontiguousarray(pieces).reshape(-1)


def unpack_codes(packed, d_out: int, d_in: int, bits: int) -> np.ndarray:
    """Inverse of pack_codes: the d_out x d_in uint8 codes."""
    packed = np.asarray(packed, dtype=np.uint8).reshape(-1)
    if packed.size != packed_bytes(d_out, d_in, bits):
        raise ValueError("packed size does not match the shape")
    t = -(-d_out // PACK_ROWS)
    g = -(-d_in // PACK_COLS)
    rowstr = packed.reshape(t, g, 2 * bits, PACK_ROWS, 8).transpose(0, 1, 3, 2, 4)
    bitarr = np.unpackbits(np.ascontiguousarray(rowstr).reshape(t, g, PACK_ROWS, 16 * bits),
                           axis=-1, bitorder="little")
    pos = code_bit_positions(bits)
    tiled = np.zeros((t, g, PACK_ROWS, PACK_COLS), dtype=np.uint8)
    for i in range(bits):
        tiled |= (bitarr[..., pos[:, i]] << i).astype(np.uint8)
    full = tiled.transpose(0, 2, 1, 3).reshape(t * PACK_ROWS, g * PACK_COLS)
    return full[:d_out, :d_in].copy()


def pack_grid(scale, zero, d_out: int, d_in: int, group: int = 0) -> np.ndarray:
    """The grid as (scale, zero) float32 pairs, tile by tile of 128 rows and, within a tile,
    group by group (group 128) or once (group 0): pair (t, g, r) at (t G' + g) 128 + r;
    rows past d_out hold (0, 0). Returns an array of shape (pairs, 2)."""
    t = -(-d_out // PACK_ROWS)
    gp = -(-d_in // PACK_COLS) if group else 1
    sc = np.zeros((t * PACK_ROWS, gp), dtype=np.float32)
    zr = np.zeros((t * PACK_ROWS, gp), dtype=np.float32)
    sc[:d_out] = np.asarray(scale, dtype=np.float32).reshape(d_out, gp)
    zr[:d_out] = np.asarray(zero, dtype=np.float32).reshape(d_out, gp)
    out = np.zeros((t, gp, PACK_ROWS, 2), dtype=np.float32)
    for ti in range(t):
        for gi in range(gp):
            out[ti, gi, :, 0] = sc[ti * PACK_ROWS:(ti + 1) * PACK_ROWS, gi]
            out[ti, gi, :, 1] = zr[ti * PACK_ROWS:(ti + 1) * PACK_ROWS, gi]
    return out.reshape(-1, 2)


def dequantize_layer(codes, scale, zero, group: int = 0) -> np.ndarray:
    """W^' = scale (codes - zero), element by element in fp64. scale/zero: d_out (group 0), or
    d_out x ceil(d_in / group) with column j on grid j // group."""
    c = np.asarray(codes, dtype=np.float64)
    s = np.asarray(scale, dtype=np.float64)
    z = np.asarray(zero, dtype=np.float64)
    if group:
        gi = np.arange(c.shape[1]) // group
        s = s.reshape(c.shape[0], -1)[:, gi]
        z = z.reshape(c.shape[0], -1)[:, gi]
    else:
        s = s.reshape(-1, 1)
        z = z.reshape(-1, 1)
    return s * (c - z)


def fwht_last(m) -> np.ndarray:
    """(I (x) H_b) applied along the last axis (b = largest power of two dividing its length),
    unnormalised, by the Kronecker factorisation H_b = H_2 (x) ... (x) H_2: each factor adds and
    subtracts the two halves of one binary index digit."""
    m = np.array(m, dtype=np.float64)
    d = m.shape[-1]
    b = hadamard_block_size(d)
    lead = m.shape[:-1]
    v = m.reshape(-1, d // b, b)
    h = 1
    while h < b:
        v = v.reshape(v.shape[0], d // b, b // (2 * h), 2, h)
        a0 = v[:, :, :, 0, :].copy()
        a1 = v[:, :, :, 1, :].copy()
        v[:, :, :, 0, :] = a0 + a1
        v[:, :, :, 1, :] = a0 - a1
        h *= 2
    return v.reshape(lead + (d,))


def qlinear_input(x, s_x=None, sign_in=None, flags: int = BIIP_FULL) -> np.ndarray:
    """x' = V S_X^-1 x for each row x of `x` (tokens x d_in), V = (1/sqrt(b)) (I (x) H_b)
    diag(sign_in) as in biip; a flag that is off drops its factor."""
    xt = np.atleast_2d(np.asarray(x, dtype=np.float64)).copy()
    d_in = xt.shape[1]
    if flags & SCALE_IN:
        xt = xt / np.asarray(s_x, dtype=np.float64)[None, :]
    if flags & ROTATE_IN:
        xt = xt * np.asarray(sign_in, dtype=np.float64)[None, :]
        xt = fwht_last(xt) / math.sqrt(hadamard_block_size(d_in))
    return xt


def qlinear_output(yp, s_g=None, sign_out=None, flags: int = BIIP_FULL) -> np.ndarray:
    """y = S_G^-1 U^T y' for each row y' of `yp` (tokens x d_out)."""
    yp = np.atleast_2d(np.asarray(yp, dtype=np.float64)).copy()
    d_out = yp.shape[1]
    if flags & ROTATE_OUT:
        # U^T = diag(sign_out) (I (x) H_b) / sqrt(b): H_b is symmetric
        yp = fwht_last(yp) / math.sqrt(hadamard_block_size(d_out))
        yp = yp * np.asarray(sign_out, dtype=np.float64)[None, :]
    if flags & SCALE_OUT:
        yp = yp / np.asarray(s_g, dtype=np.float64)[None, :]
    return yp


def qlinear_dense(w_hat, x, s_x=None, s_g=None, sign_in=None, sign_out=None,
                  flags: int = BIIP_FULL) -> np.ndarray:
    """y = S_G^-1 U^T W^' V S_X^-1 x for each row x of `x` (tokens x d_in) -> tokens x d_out.

    V = (1/sqrt(b_in)) (I (x) H_b_in) diag(sign_in), U likewise on the output side (the
    transforms of biip); a flag that is off drops its factor.
    """
    w_hat = np.asarray(w_hat, dtype=np.float64)
    xp = qlinear_input(x, s_x, sign_in, flags)
    return qlinear_output(xp @ w_hat.T, s_g, sign_out, flags)


def qlinear(x, codes, scale, zero, s_x=None, s_g=None, sign_in=None, sign_out=None,
            flags: int = BIIP_FULL, group: int = 0) -> np.ndarray:
    """The quantized layer on activations: qlinear_dense of the dequantized codes."""
    return qlinear_dense(dequantize_layer(codes, scale, zero, group), x, s_x, s_g, sign_in,
                         sign_out, flags)


# ------------------------------------------------------------------------------------------
# Comparison variant: rounding with output-side feedback as well (prior art, not KronQ)
# ------------------------------------------------------------------------------------------

def udu_factor(h):
    """Unit upper triangular U and diagonal d with H = U diag(d) U^T.

    The triangular factor of H in the orientation that makes the natural column order causal:
    row p of U - I holds the feedback from column p to the later columns. Computed as the
    Cholesky factor of the index-reversed matrix, reversed back: J H J = L L^T gives
    H = (J L J)(J L J)^T with J L J upper triangular.
    """
    h = np.asarray(h, dtype=np.float64)
    rev = np.arange(h.shape[0])[::-1]
    try:
        l = np.linalg.cholesky(h[np.ix_(rev, rev)])
    except np.linalg.LinAlgError as e:
        raise NotPositiveDefinite(str(e))
    u = l[np.ix_(rev, rev)]
    dg = np.diag(u).copy()
    return u / dg[None, :], dg * dg


def quantize_matrix(t, scale, zero, bits):
    """Per-row grid codes of a whole matrix: clamp(rint(t/scale) + zero, 0, 2^b - 1) in fp32."""
    maxq = np.float32(2 ** bits - 1)
    s = np.asarray(scale, dtype=np.float32)[:, None]
    z = np.asarray(zero, dtype=np.float32)[:, None]
    c = np.rint(np.asarray(t).astype(np.float32) / s)
    return np.clip(c + z, np.float32(0), maxq).astype(np.float32)


def yaqa_round(w, h_out, h_in, bits: int, damp_rel: float = 0.01, follow_codes=None,
               tie_tol: float = 1e-3):
    """Rounding with feedback on both the input and the output side, for comparison with KronQ.

    [YAQA notes], generalized LDLQ: for a Kronecker proxy H_O (x) H_I of the layer Hessian,
    with the triangular factors L_O, L_I of H_O and H_I and L' = L - I, the quantized W^ is the
    fixed point of
        W^ = Q(W + L_O'^T D L_I' + L_O'^T D + D L_I'),    D = W - W^,
    which is reached in at most m + n - 1 iterations. Here H_O = H_G' and H_I = H_X' (after
    incoherence processing), each damped by damp_rel * mean diag, L the unit upper triangular
    factor of udu_factor (so that L_I' is the input-side feedback of the column solve, which
    with H_O = I is KronQ's solve without P), Q the per-row grid of W (grid). The iteration
    starts from W^ = Q(W) and stops when an iteration changes nothing.
    follow_codes / tie_tol: as in quantize_layer, at every iteration.
    Returns dict: codes, scale, zero, w_hat (fp64), iterations, near_tie, disagree.
    """
    w = np.asarray(w, dtype=np.float64)
    m, n = w.shape
    ho = np.asarray(h_out, dtype=np.float64)
    hi = np.asarray(h_in, dtype=np.float64)
    ho = ho + damping(ho, damp_rel) * np.eye(m)
    hi = hi + damping(hi, damp_rel) * np.eye(n)
    lo = udu_factor(ho)[0] - np.eye(m)
    li = udu_factor(hi)[0] - np.eye(n)
    scale, zero = grid(w, bits)
    s64 = scale.astype(np.float64)[:, None]

    def deq(c):   # scale (c - zero) in fp32, as the column solve dequantizes
        return dequantize(c, scale[:, None], zero[:, None]).astype(np.float64)

    codes = quantize_matrix(w, scale, zero, bits)
    near = np.zeros((m, n), dtype=bool)
    disagree = np.zeros((m, n), dtype=bool)
    iterations = 0
    for _ in range(m + n):
        delta = w - deq(codes)
        target = w + lo.T @ delta @ li + lo.T @ delta + delta @ li
        new = quantize_matrix(target, scale, zero, bits)
        if follow_codes is not None:
            u = target / s64
            near = np.abs(u - (np.floor(u) + 0.5)) <= tie_tol
            fc = np.asarray(follow_codes, dtype=np.float32)
            disagree = near & (fc != new)
            new = np.where(near, fc, new).astype(np.float32)
        iterations += 1
        if np.array_equal(new, codes):
            break
        codes = new
    return {"codes": codes.astype(np.uint8), "scale": scale, "zero": zero, "w_hat": deq(codes),
            "iterations": iterations, "near_tie": near, "disagree": disagree}


# ------------------------------------------------------------------------------------------
# Objective and diagnostics
# ------------------------------------------------------------------------------------------

def objective(w, w_hat, hx, hg=None, dxx=None):
    """tr[H_G dW H_X dW^T] + 2 tr[H_G W D dW^T], dW = W - W^ (H_G = I when not given).

    [KronQ-hyper] Method: Kronecker-factored objective and its asymmetric form.
    """
    w = np.asarray(w, dtype=np.float64)
    dw = w - np.asarray(w_hat, dtype=np.float64)
    hx = np.asarray(hx, dtype=np.float64)
    hg_ = np.eye(w.shape[0]) if hg is None else np.asarray(hg, dtype=np.float64)
    val = np.trace(hg_ @ dw @ hx @ dw.T)
    if dxx is not None:
        val += 2.0 * np.trace(hg_ @ w @ np.asarray(dxx, dtype=np.float64) @ dw.T)
    return float(val)


def mu_incoherence(h):
    """mu(H)/sqrt(d) = max_ij |Q_ij| over an orthonormal eigenbasis Q of H."""
    _, q = np.linalg.eigh(np.asarray(h, dtype=np.float64))
    return float(np.abs(q).max())


def cv_norms(w):
    """(CV_in, CV_out): coefficient of variation of column norms and of row norms of W."""
    w = np.asarray(w, dtype=np.float64)
    c = np.sqrt((w * w).sum(axis=0))
    r = np.sqrt((w * w).sum(axis=1))
    return float(c.std() / c.mean()), float(r.std() / r.mean())


# ------------------------------------------------------------------------------------------
# Mixed-precision allocation
# ------------------------------------------------------------------------------------------

def score_allocate(tr_hx, tr_hg, n_params, choices, avg_bits):
    """Scores s_l = tr(H_G) tr(H_X) and a greedy bit allocation under an average-bit budget.

    [KronQ-hyper] Method: sublayers with larger s get higher bit widths;
    [KronQ-gist] Experimental results: the higher-scored sublayer is upgraded first.
    Order: s descending, ties by index ascending. Budget T = floor(avg_bits * sum n) bits.
    Every sublayer starts at min(choices); in that order each takes the largest choice that
    keeps the total within T.
    Returns (scores, bits).
    """
    tr_hx = [float(v) for v in tr_hx]
    tr_hg = [float(v) for v in tr_hg]
    n_params = [int(v) for v in n_params]
    L = len(tr_hx)
    s = [tr_hg[l] * tr_hx[l] for l in range(L)]
    if any(math.isnan(v) for v in s):
        raise ValueError("NaN score")
    total = sum(n_params)
    budget = int(math.floor(float(avg_bits) * float(total)))
    ch = sorted(set(int(c) for c in choices))
    bits = [ch[0]] * L
    used = ch[0] * total
    if used > budget:
        raise ValueError("budget below the smallest bit width")
    order = sorted(range(L), key=lambda l: (-s[l], l))
    for l in order:
        for b in reversed(ch):
            if b <= bits[l]:
                break
            extra = (b - bits[l]) * n_params[l]
            if used + extra <= budget:
                used += extra
                bits[l] = b
                break
    return s, bits
