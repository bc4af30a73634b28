"""Host-side checks of the C ABI library (no GPU needed).

The library must load, export every entry point include/kronq.h declares, reject bad
arguments before touching a device, and run the (host-only) score/allocation call bit-exactly
like the oracle.
"""
import json
import math
import os
import re

import numpy as np
import pytest

from oracle import kronq_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def K():
    from post_quantization_b200 import build
    build.build()
    from post_quantization_b200 import kronq
    kronq.load_library()
    return kronq


def header_symbols():
    src = open(os.path.join(ROOT, "include", "kronq.h")).read()
    return sorted(set(re.findall(r"\b(kronq_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol(K):
    import ctypes
    lib = ctypes.CDLL(K.LIB_PATH)
    declared = header_symbols()
    assert len(declared) >= 14
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(K.SYMBOLS)


def test_only_kronq_symbols_exported(K):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", K.LIB_PATH], capture_output=True,
                         text=True).stdout
    names = [l.split()[-1] for l in out.splitlines() if " T " in l]
    assert names and all(n.startswith("kronq_") for n in names), names


def test_status_strings(K):
    assert K.kronq_status_string(K.OK) == "ok"
    assert "positive definite" in K.kronq_status_string(K.ERR_NOT_PD)
    assert K.kronq_version() >= 100


def test_workspace_queries(K):
    assert K.kronq_biip_workspace_size(4096, 11008) > 0
    assert K.kronq_cholinv_workspace_size(4096) >= 4096 * 64 * 4
    assert K.kronq_quantize_layer_workspace_size(4096, 4096, 128, False) >= 4096 * 128 * 4
    assert (K.kronq_quantize_layer_workspace_size(64, 64, 128, True)
            > K.kronq_quantize_layer_workspace_size(64, 64, 128, False))
    assert K.kronq_accumulate_workspace_size(1000, 256, 256, False) == 0
    assert K.kronq_accumulate_workspace_size(1000, 256, 256, True) > 0
    assert K.kronq_biip_workspace_size(0, 5) == 0
    # diagonal sums: one fp32 partial per column and block of 2048 tokens
    assert K.kronq_accumulate_diag_workspace_size(4097, 100) == 3 * 100 * 4
    assert K.kronq_accumulate_diag_workspace_size(0, 100) == 0


def test_sm_budget_is_host_state(K):
    assert K.kronq_sm_budget() == 0
    K.kronq_set_sm_budget(16)
    assert K.kronq_sm_budget() == 16
    K.kronq_set_sm_budget(-3)                  # non-positive lifts it
    assert K.kronq_sm_budget() == 0


def test_argument_errors_before_device(K):
    lib = K.load_library()
    # quantize: bad bits / block / missing pointers, no device touched
    assert lib.kronq_quantize_layer(8, 8, None, 16, 16, 9, 128, 0, 8, 8, 8, 16, None, 0, None) \
        == K.ERR_UNSUPPORTED
    assert lib.kronq_quantize_layer(8, 8, None, 16, 16, 4, 64, 0, 8, 8, 8, 16, None, 0, None) \
        == K.ERR_UNSUPPORTED
    assert lib.kronq_quantize_layer(None, 8, None, 16, 16, 4, 128, 0, 8, 8, 8, 16, None, 0, None) \
        == K.ERR_INVALID_ARG
    assert lib.kronq_quantize_layer(8, 8, None, 0, 16, 4, 128, 0, 8, 8, 8, 16, None, 0, None) \
        == K.ERR_SHAPE
    assert lib.kronq_quantize_layer(8, 8, None, 16, 16, 4, 128, 64, 8, 8, 8, 16, None, 0, None) \
        == K.ERR_UNSUPPORTED                                   # group is 0 or the block width
    # biip: SCALE_OUT without hg, rotation without signs, bad dtype, aliasing
    args = [16, 0, 32, 48, None, None, 1.0, None, None, 4, 4]
    tail = [64, 80, 96, 112, None, 0, None]
    assert lib.kronq_biip(*args, K.BIIP_SCALE_OUT, *tail) == K.ERR_INVALID_ARG
    assert lib.kronq_biip(*args, K.BIIP_ROTATE_IN, *tail) == K.ERR_INVALID_ARG
    bad = list(args); bad[1] = 7
    assert lib.kronq_biip(*bad, 0, *tail) == K.ERR_INVALID_ARG
    assert lib.kronq_biip(*args, 1 << 8, *tail) == K.ERR_INVALID_ARG
    # cholinv: negative damping, missing info
    assert lib.kronq_cholinv(16, 4, -1.0, 32, 0, None, 0, None) == K.ERR_INVALID_ARG
    assert lib.kronq_cholinv(16, 4, 0.01, None, 0, None, 0, None) == K.ERR_INVALID_ARG
    assert lib.kronq_cholinv(16, 0, 0.01, 32, 0, None, 0, None) == K.ERR_SHAPE
    # accumulate: misaligned stride (bf16 stride must be a multiple of 8 elements)
    assert lib.kronq_accumulate(256, 12, None, 0, None, 0, 10, 12, 0, 512, None, None, None, 0,
                                None) == K.ERR_INVALID_ARG
    assert lib.kronq_accumulate(256, 16, None, 0, None, 0, 10, 12, 0, None, None, None, None, 0,
                                None) == K.ERR_INVALID_ARG
    assert "no output" in lib.kronq_last_error_detail().decode()
    # accumulate_diag: missing output, bad width, misaligned stride, short workspace
    assert lib.kronq_accumulate_diag(256, 16, 10, 16, None, None, 0, None) == K.ERR_INVALID_ARG
    assert lib.kronq_accumulate_diag(256, 16, 10, 0, 512, None, 0, None) == K.ERR_SHAPE
    assert lib.kronq_accumulate_diag(256, 12, 10, 12, 512, None, 0, None) == K.ERR_INVALID_ARG
    assert lib.kronq_accumulate_diag(256, 16, 10, 16, 512, None, 0, None) == K.ERR_WORKSPACE
    assert lib.kronq_accumulate_diag(256, 16, 0, 16, 512, None, 0, None) == K.OK   # n = 0
    # biip: the diagonal form of H_G needs hg and cannot be written back
    assert lib.kronq_biip(*args, K.BIIP_HG_DIAG, *tail) == K.ERR_INVALID_ARG
    withhg = list(args); withhg[4] = 128
    assert lib.kronq_biip(*withhg, K.BIIP_HG_DIAG | K.BIIP_WRITE_HG, *tail) == K.ERR_INVALID_ARG
    assert "diagonal" in lib.kronq_last_error_detail().decode()


def test_inference_calls_host_checks(K):
    lib = K.load_library()
    # packed sizes follow the format: 128 x 128 blobs of 2048 * bits bytes
    for bits in (2, 3, 4):
        assert K.kronq_packed_codes_bytes(300, 520, bits) == O.packed_bytes(300, 520, bits)
    assert K.kronq_packed_codes_bytes(128, 128, 5) == 0
    assert K.kronq_qlinear_workspace_size(4096, 4096, 1) > 0
    assert K.kronq_qlinear_workspace_size(4096, 4096, 0) == 0
    # pack: unsupported width, short buffer, misaligned destination
    assert lib.kronq_pack_codes(16, 8, 8, 5, 256, 4096, None) == K.ERR_UNSUPPORTED
    assert lib.kronq_pack_codes(16, 8, 8, 2, 256, 16, None) == K.ERR_SHAPE
    assert lib.kronq_pack_codes(16, 8, 8, 2, 257, 4096, None) == K.ERR_INVALID_ARG
    # pack_grid: group, size, alignment
    assert K.kronq_packed_grid_bytes(300, 520, 128) == 3 * 5 * 128 * 8
    assert K.kronq_packed_grid_bytes(300, 520, 0) == 3 * 128 * 8
    assert lib.kronq_pack_grid(16, 32, 8, 8, 64, 256, 4096, None) == K.ERR_UNSUPPORTED
    assert lib.kronq_pack_grid(16, 32, 8, 8, 0, 256, 8, None) == K.ERR_SHAPE
    assert lib.kronq_pack_grid(16, 32, 8, 8, 0, 260, 4096, None) == K.ERR_INVALID_ARG
    # qlinear: x, dtype, ld_x, n_tok, packed, grid, group, s_x, s_g, si, so, flags,
    #          d_out, d_in, bits, y, ld_y, ws, ws_bytes, stream
    ok = [256, K.DTYPE_F32, 64, 2, 512, 768, 0, 1280, 1536, 1792, 2048, K.BIIP_FULL,
          32, 64, 2, 2304, 32, None, 0, None]

    def call(**kw):
        a = list(ok)
        names = ["x", "dtype", "ld_x", "n_tok", "packed", "grid", "group", "s_x", "s_g",
                 "si", "so", "flags", "d_out", "d_in", "bits", "y", "ld_y"]
        for k, v in kw.items():
            a[names.index(k)] = v
        return lib.kronq_qlinear(*a)
    assert call(bits=5) == K.ERR_UNSUPPORTED
    assert call(group=64) == K.ERR_UNSUPPORTED
    assert call(flags=16) == K.ERR_INVALID_ARG
    assert call(dtype=7) == K.ERR_INVALID_ARG
    assert call(n_tok=0) == K.OK                            # nothing to do
    assert call(d_out=0) == K.ERR_SHAPE
    assert call(grid=None) == K.ERR_INVALID_ARG
    assert call(grid=772) == K.ERR_INVALID_ARG              # 16-byte alignment
    assert call(grid=776) == K.ERR_INVALID_ARG
    assert call(s_g=None) == K.ERR_INVALID_ARG              # SCALE_OUT needs s_g
    assert call(s_g=None, flags=K.BIIP_FULL & ~K.BIIP_SCALE_OUT) == K.ERR_WORKSPACE
    assert call(si=None) == K.ERR_INVALID_ARG
    assert call(ld_x=63) == K.ERR_SHAPE
    assert call(packed=520) == K.ERR_INVALID_ARG            # 16-byte alignment
    assert call(x=258) == K.ERR_INVALID_ARG                 # fp32 alignment
    assert call(d_in=3 * 32768, ld_x=3 * 32768) == K.ERR_UNSUPPORTED   # Hadamard block 32768
    assert call() == K.ERR_WORKSPACE                        # everything else valid


def test_allocation_matches_golden_and_oracle(K):
    with open(os.path.join(ROOT, "tests", "golden", "allocation_cases.json")) as f:
        for c in json.load(f)["cases"]:
            s, bits = K.kronq_score_allocate(c["tr_hx"], c["tr_hg"], c["n_params"], c["choices"],
                                             c["avg_bits"])
            assert bits == c["bits"], c["name"]
    r = np.random.default_rng(7)
    for trial in range(200):
        L = int(r.integers(1, 40))
        tr_hx = r.lognormal(0, 2, L)
        tr_hg = r.lognormal(0, 2, L)
        if trial % 5 == 0:                      # ties
            tr_hx[: L // 2] = 1.0; tr_hg[: L // 2] = 2.0
        n = r.integers(1, 10_000_000, L)
        choices = sorted(set(r.choice([1, 2, 3, 4, 5, 6, 8], int(r.integers(1, 4)), replace=False)))
        avg = float(min(choices) + r.uniform(0, max(choices) - min(choices) + 0.5))
        s_o, b_o = O.score_allocate(tr_hx, tr_hg, n, choices, avg)
        s_k, b_k = K.kronq_score_allocate(tr_hx, tr_hg, n, choices, avg)
        assert b_k == b_o
        assert s_k == s_o


def test_allocation_errors(K):
    with pytest.raises(K.KronqError) as e:
        K.kronq_score_allocate([float("nan")], [1.0], [10], [2, 3], 3.0)
    assert e.value.status == K.ERR_INVALID_ARG
    with pytest.raises(K.KronqError):
        K.kronq_score_allocate([1.0], [1.0], [10], [2, 3], 1.0)


def test_llama2_stack_allocation_shape(K):
    # 224 sublayers of LLaMA-2-7B shapes at 2.5 average bits from {2, 3, 4}
    from post_quantization_b200 import synth
    wl = synth.WORKLOADS["llama2_7b_stack"]
    sizes = [s.d_out * s.d_in for s in wl.sublayers] * wl.n_blocks
    r = np.random.default_rng(3)
    tr_hx = r.lognormal(0, 1, len(sizes)); tr_hg = r.lognormal(0, 3, len(sizes))
    s, bits = K.kronq_score_allocate(tr_hx, tr_hg, sizes, [2, 3, 4], 2.5)
    assert sum(b * n for b, n in zip(bits, sizes)) <= math.floor(2.5 * sum(sizes))
    assert bits == O.score_allocate(tr_hx, tr_hg, sizes, [2, 3, 4], 2.5)[1]


def test_twosided_argument_errors_before_device(K):
    lib = K.load_library()
    f = lib.kronq_quantize_layer_twosided
    # (w, k_in, k_out, d_out, d_in, bits, codes, scale, zero, w_hat, iterations, ws, bytes, stream)
    assert f(8, 8, 8, 0, 16, 2, 8, 8, 8, 16, None, None, 0, None) == K.ERR_SHAPE
    assert f(8, 8, 8, 16, 16, 9, 8, 8, 8, 16, None, None, 0, None) == K.ERR_UNSUPPORTED
    assert f(8, None, 8, 16, 16, 2, 8, 8, 8, 16, None, None, 0, None) == K.ERR_INVALID_ARG
    assert f(8, 8, 8, 16, 16, 2, 8, 8, 8, 8, None, None, 0, None) == K.ERR_INVALID_ARG   # w == w_hat
    assert f(8, 8, 8, 70000, 16, 2, 8, 8, 8, 16, None, None, 0, None) == K.ERR_SHAPE
    assert f(8, 8, 8, 16, 16, 2, 8, 8, 8, 16, None, None, 0, None) == K.ERR_WORKSPACE
    need = K.load_library().kronq_quantize_layer_twosided_workspace_size(300, 200)
    # two factors, their splits, four fp32 d_out x d_in buffers and a split of one
    assert need >= 4 * 300 * 200 * 4 + 3 * 300 * 200 * 2 + (300 * 300 + 200 * 200) * 4
