"""The quantized layer at inference (packed codes, kronq_qlinear) vs the fp64 oracle.

Bars: the GPU packer is bit-exact against the oracle's packer; y is within a relative
Frobenius error of 1e-4 per token of the oracle's y = S_G^-1 U^T W^' V S_X^-1 x, computed from
the unpacked codes (the library splits x' into two bf16 terms, so about 2^-17 relative per
element plus fp32 sums; 1e-4 leaves room and sits well inside the 1e-3 bar of the solve).
"""
import math

import numpy as np
import pytest
import torch

from oracle import kronq_oracle as O
from post_quantization_b200 import synth

pytestmark = pytest.mark.gpu

TOL = 1e-4


@pytest.fixture(scope="module")
def K():
    from post_quantization_b200 import build
    build.build()
    from post_quantization_b200 import kronq
    kronq.load_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    kronq.kronq_device_check()
    return kronq


def rel_rows(a, b):
    a = np.asarray(a, dtype=np.float64); b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b, axis=1)
    return np.linalg.norm(a - b, axis=1) / np.where(nb > 0, nb, 1.0)


def make_layer(d_out, d_in, bits, group, tag, dev="cuda"):
    c = synth.codes(d_out, d_in, bits, synth.seed_for(tag, "codes"), device=dev)
    ng = (d_in + 127) // 128 if group else 0
    scale, zero = synth.grid_params(d_out, ng, bits, synth.seed_for(tag, "grid"), device=dev)
    s_x = synth.positive_scales(d_in, synth.seed_for(tag, "sx"), device=dev)
    s_g = synth.positive_scales(d_out, synth.seed_for(tag, "sg"), device=dev)
    si = synth.rademacher(d_in, synth.seed_for(tag, "si"), device=dev)
    so = synth.rademacher(d_out, synth.seed_for(tag, "so"), device=dev)
    return c, scale, zero, s_x, s_g, si, so


def tokens(n, d_in, tag, dtype=torch.float32, dev="cuda"):
    return synth.activations(n, d_in, synth.seed_for(tag, "x"), dtype=dtype, device=dev)


def np64(t):
    return t.detach().cpu().double().numpy()


def qlin(K, x, packed, grid, s_x, s_g, si, so, d_out, bits, y, group=0, flags=None, **kw):
    K.kronq_qlinear(x, packed, grid, s_x, s_g, si, so, K.BIIP_FULL if flags is None else flags,
                    d_out, bits, y, group=group, **kw)


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("shape", [(1, 1), (5, 37), (130, 300), (256, 1024), (1000, 4096)])
def test_pack_codes_bit_exact(K, bits, shape):
    c = synth.codes(*shape, bits, synth.seed_for("pack", bits, *shape), device="cuda")
    p = K.kronq_pack_codes(c, bits)
    torch.cuda.synchronize()
    want = O.pack_codes(c.cpu().numpy(), bits)
    got = p.cpu().numpy()[:want.size]
    assert got.size == want.size == O.packed_bytes(*shape, bits)
    np.testing.assert_array_equal(got, want)


def _header_bit_positions(bits, d_in, row, col):
    """Byte offset and bit of each code bit of (row, col), read off the packed-format text of
    include/kronq.h (blob, 8-byte pieces of the row string, byte lanes of 32-bit words)."""
    G = (d_in + 127) // 128
    t, r = divmod(row, 128)
    g, c = divmod(col, 128)
    blob = (t * G + g) * 2048 * bits
    j = c % 4
    if bits == 2:
        where = [(c // 16, 8 * j + 2 * ((c % 16) // 4) + i) for i in range(2)]
    elif bits == 4:
        where = [(c // 8, 8 * j + 4 * ((c % 8) // 4) + i) for i in range(4)]
    else:
        m, e = divmod(c, 32)
        where = [(3 * m + e // 16, 8 * j + 2 * ((e % 16) // 4) + i) for i in range(2)]
        where.append((3 * m + 2, 8 * j + e // 4))
    out = []
    for word, bit in where:
        sbyte = 4 * word + bit // 8           # byte of the row string (little-endian words)
        p, k = divmod(sbyte, 8)
        out.append((blob + 1024 * p + 8 * r + k, bit % 8))
    return out


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_pack_codes_follow_the_header_text(K, bits):
    # one code at a time, all others zero: its bits must appear exactly where the format text
    # of the C header puts them, and nowhere else
    d_out, d_in = 300, 520
    placements = [(0, 0), (1, 1), (127, 127), (128, 5), (37, 130), (299, 519), (64, 255),
                  (5, 33), (200, 62)]
    for row, col in placements:
        value = (1 << bits) - 1 if (row + col) % 2 else (1 << (bits - 1)) | 1
        c = torch.zeros(d_out, d_in, dtype=torch.uint8, device="cuda")
        c[row, col] = value
        got = K.kronq_pack_codes(c, bits).cpu().numpy()[:O.packed_bytes(d_out, d_in, bits)]
        want = np.zeros_like(got)
        for i, (byte, bit) in enumerate(_header_bit_positions(bits, d_in, row, col)):
            if (value >> i) & 1:
                want[byte] |= np.uint8(1 << bit)
        np.testing.assert_array_equal(got, want, err_msg=f"bits {bits} at ({row}, {col})")


@pytest.mark.parametrize("group", [0, 128])
@pytest.mark.parametrize("shape", [(1, 1), (300, 520), (1024, 4096)])
def test_pack_grid_bit_exact(K, group, shape):
    d_out, d_in = shape
    ng = (d_in + 127) // 128 if group else 0
    scale, zero = synth.grid_params(d_out, ng, 3, synth.seed_for("pg", group, *shape),
                                    device="cuda")
    got = K.kronq_pack_grid(scale, zero, d_out, d_in, group).cpu().numpy().reshape(-1, 2)
    want = O.pack_grid(scale.cpu().numpy(), zero.cpu().numpy(), d_out, d_in, group)
    np.testing.assert_array_equal(got, want)


CASES = [
    # d_out, d_in, n_tok: several tiles, ragged rows / columns, Hadamard blocks from 4 to 8192
    (256, 256, 1),
    (300, 520, 3),         # ragged tiles and groups; b_out = 4, b_in = 8
    (1024, 4096, 8),
    (4096, 1024, 17),      # 17 tokens: N = 48
    (768, 11008, 5),       # b_in = 256, 86 groups
    (8192, 512, 2),        # b_out = 8192: 64 tiles in one Hadamard block
]


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("group", [0, 128])
@pytest.mark.parametrize("case", CASES)
def test_qlinear_matches_oracle(K, bits, group, case):
    d_out, d_in, n = case
    tag = ("ql", bits, group, *case)
    c, scale, zero, s_x, s_g, si, so = make_layer(d_out, d_in, bits, group, tag)
    x = tokens(n, d_in, tag)
    packed = K.kronq_pack_codes(c, bits)
    y = torch.full((n, d_out), float("nan"), device="cuda")
    grid = K.kronq_pack_grid(scale, zero, d_out, d_in, group)
    qlin(K, x, packed, grid, s_x, s_g, si, so, d_out, bits, y, group)
    torch.cuda.synchronize()
    want = O.qlinear(np64(x), c.cpu().numpy(), np64(scale), np64(zero), np64(s_x), np64(s_g),
                     np64(si), np64(so), O.BIIP_FULL, group)
    err = rel_rows(np64(y), want)
    assert np.all(np.isfinite(np64(y)))
    assert err.max() <= TOL, err


@pytest.mark.parametrize("flags", [0, 1, 2, 4, 8, 5, 10, 15])
def test_qlinear_transform_flags(K, flags):
    d_out, d_in, n, bits = 512, 768, 4, 3
    tag = ("qlf", flags)
    c, scale, zero, s_x, s_g, si, so = make_layer(d_out, d_in, bits, 0, tag)
    x = tokens(n, d_in, tag)
    packed = K.kronq_pack_codes(c, bits)
    y = torch.empty(n, d_out, device="cuda")
    grid = K.kronq_pack_grid(scale, zero, d_out, d_in, 0)
    qlin(K, x, packed, grid, s_x if flags & 1 else None, s_g if flags & 2 else None,
         si if flags & 4 else None, so if flags & 8 else None, d_out, bits, y, flags=flags)
    torch.cuda.synchronize()
    want = O.qlinear(np64(x), c.cpu().numpy(), np64(scale), np64(zero), np64(s_x), np64(s_g),
                     np64(si), np64(so), flags, 0)
    assert rel_rows(np64(y), want).max() <= TOL


def test_qlinear_bf16_input_many_tokens_and_strides(K):
    # 70 tokens: three passes of up to 32; bf16 activations; padded row strides
    d_out, d_in, n, bits = 1024, 2048, 70, 4
    tag = ("qlb",)
    c, scale, zero, s_x, s_g, si, so = make_layer(d_out, d_in, bits, 128, tag)
    xb = torch.zeros(n, d_in + 64, dtype=torch.bfloat16, device="cuda")
    xb[:, :d_in] = tokens(n, d_in, tag, dtype=torch.bfloat16)
    x = xb[:, :d_in]
    packed = K.kronq_pack_codes(c, bits)
    yb = torch.full((n, d_out + 32), -7.0, device="cuda")
    y = yb[:, :d_out]
    grid = K.kronq_pack_grid(scale, zero, d_out, d_in, 128)
    qlin(K, x, packed, grid, s_x, s_g, si, so, d_out, bits, y, 128)
    torch.cuda.synchronize()
    want = O.qlinear(np64(x), c.cpu().numpy(), np64(scale), np64(zero), np64(s_x), np64(s_g),
                     np64(si), np64(so), O.BIIP_FULL, 128)
    assert rel_rows(np64(y), want).max() <= TOL
    assert torch.all(yb[:, d_out:] == -7.0)          # nothing written past the row


def test_qlinear_deterministic_and_graph_replay(K):
    d_out, d_in, n, bits = 2048, 4096, 8, 2
    tag = ("qld",)
    c, scale, zero, s_x, s_g, si, so = make_layer(d_out, d_in, bits, 0, tag)
    x = tokens(n, d_in, tag)
    packed = K.kronq_pack_codes(c, bits)
    ws = torch.empty(K.kronq_qlinear_workspace_size(d_out, d_in, n) + 256, dtype=torch.uint8,
                     device="cuda")
    ws = ws[(-ws.data_ptr()) % 256:][:K.kronq_qlinear_workspace_size(d_out, d_in, n)]
    y1 = torch.empty(n, d_out, device="cuda")
    y2 = torch.empty(n, d_out, device="cuda")
    grid = K.kronq_pack_grid(scale, zero, d_out, d_in, 0)
    qlin(K, x, packed, grid, s_x, s_g, si, so, d_out, bits, y1, workspace=ws)
    qlin(K, x, packed, grid, s_x, s_g, si, so, d_out, bits, y2, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    y3 = torch.empty(n, d_out, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            qlin(K, x, packed, grid, s_x, s_g, si, so, d_out, bits, y3, workspace=ws)
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y1, y3)
    del g


def test_qlinear_under_an_sm_budget(K):
    d_out, d_in, n, bits = 1024, 4096, 3, 3
    tag = ("qls",)
    c, scale, zero, s_x, s_g, si, so = make_layer(d_out, d_in, bits, 128, tag)
    x = tokens(n, d_in, tag)
    packed = K.kronq_pack_codes(c, bits)
    grid = K.kronq_pack_grid(scale, zero, d_out, d_in, 128)
    outs = []
    try:
        for budget in (0, 7, 100):
            K.kronq_set_sm_budget(budget)
            y = torch.empty(n, d_out, device="cuda")
            qlin(K, x, packed, grid, s_x, s_g, si, so, d_out, bits, y, 128)
            torch.cuda.synchronize()
            outs.append(y)
    finally:
        K.kronq_set_sm_budget(0)
    want = O.qlinear(np64(x), c.cpu().numpy(), np64(scale), np64(zero), np64(s_x), np64(s_g),
                     np64(si), np64(so), O.BIIP_FULL, 128)
    for y in outs:
        assert rel_rows(np64(y), want).max() <= TOL
    # partial sums are added in a different grouping when the CTA count changes, so the bits
    # may differ by rounding only
    assert rel_rows(np64(outs[0]), np64(outs[2])).max() <= 1e-6


def test_qlinear_of_a_quantized_layer_approximates_the_layer(K):
    # end to end on the GPU: BiIP -> inverse factor -> solve -> pack -> qlinear; the result is
    # the oracle's map of the GPU's codes, and close to W x (4-bit quantization error)
    from post_quantization_b200 import pipeline as P
    d_out, d_in, n, bits = 512, 1024, 2048, 4
    tag = ("qle",)
    # calibration tokens and 6 held-out tokens of the same distribution
    xall = synth.correlated_x(n + 6, d_in, synth.seed_for(tag, "X"), device="cuda")
    xq = xall[:n]
    g = synth.gradients(n, d_out, synth.seed_for(tag, "G"), device="cuda")
    w = synth.weight(d_out, d_in, synth.seed_for(tag, "W"), dtype=torch.float32, device="cuda")
    si = synth.rademacher(d_in, synth.seed_for(tag, "si"), device="cuda")
    so = synth.rademacher(d_out, synth.seed_for(tag, "so"), device="cuda")
    hx = torch.zeros(d_in, d_in, device="cuda"); hg = torch.zeros(d_out, d_out, device="cuda")
    K.kronq_accumulate(xq, None, g, hx, hg, None)
    r = P.biip(w, hx, hg, None, 1.0 / n, si, so)
    P.cholinv(r)
    P.quantize(r, bits)
    packed = K.kronq_pack_codes(r.codes, bits)
    x = xall[n:].float()
    y = torch.empty(6, d_out, device="cuda")
    grid = K.kronq_pack_grid(r.scale, r.zero, d_out, d_in, 0)
    qlin(K, x, packed, grid, r.s_x, r.s_g, si, so, d_out, bits, y)
    torch.cuda.synchronize()
    want = O.qlinear(np64(x), r.codes.cpu().numpy(), np64(r.scale), np64(r.zero), np64(r.s_x),
                     np64(r.s_g), np64(si), np64(so), O.BIIP_FULL, 0)
    assert rel_rows(np64(y), want).max() <= TOL
    # the same layer through its dequantized weights W^' (the solve's own w_hat)
    dense = O.qlinear_dense(np64(r.w_hat), np64(x), np64(r.s_x), np64(r.s_g), np64(si),
                            np64(so))
    assert rel_rows(np64(y), dense).max() <= TOL
    # and near the unquantized layer in the metric the method minimises, the output error
    # weighted by H_G (channels with tiny gradients may carry large plain errors: S_G^-1
    # scales their share of the quantization noise up), on held-out calibration-like tokens
    full = np64(x) @ np64(w).T
    hgn = np64(hg) / n
    e = np64(y) - full
    num = np.einsum("ti,ij,tj->", e, hgn, e)
    den = np.einsum("ti,ij,tj->", full, hgn, full)
    assert math.sqrt(num / den) <= 0.15


def test_qlinear_llama3_70b_shapes_sampled(K):
    # full-size sublayers of a LLaMA-3-70B block at 2 bits, group 128, decode (1 token) and a
    # batch of 16. The oracle recomputes y' for the rows of one output Hadamard block (all rows
    # when b_out = d_out) in fp64 from the unpacked codes, then that block's output transform.
    for (d_out, d_in) in [(28672, 8192), (8192, 28672), (1024, 8192)]:
        for n in (1, 16):
            bits, group = 2, 128
            tag = ("ql70", d_out, d_in, n)
            c, scale, zero, s_x, s_g, si, so = make_layer(d_out, d_in, bits, group, tag)
            x = tokens(n, d_in, tag)
            packed = K.kronq_pack_codes(c, bits)
            y = torch.empty(n, d_out, device="cuda")
            grid = K.kronq_pack_grid(scale, zero, d_out, d_in, group)
            qlin(K, x, packed, grid, s_x, s_g, si, so, d_out, bits, y, group)
            torch.cuda.synchronize()
            b_out = O.hadamard_block_size(d_out)
            blk = min(1, d_out // b_out - 1)          # second block when there is one
            rows = slice(blk * b_out, (blk + 1) * b_out)
            xp = O.qlinear_input(np64(x), np64(s_x), np64(si))
            cc = c[rows].cpu().numpy()
            yp = np.zeros((n, b_out))
            for r0 in range(0, b_out, 1024):
                wq = O.dequantize_layer(cc[r0:r0 + 1024], np64(scale[rows][r0:r0 + 1024]),
                                        np64(zero[rows][r0:r0 + 1024]), group)
                yp[:, r0:r0 + 1024] = xp @ wq.T
            want = O.qlinear_output(yp, np64(s_g[rows]), np64(so[rows]))
            err = rel_rows(np64(y[:, rows]), want)
            assert err.max() <= TOL, (d_out, d_in, n, err.max())
