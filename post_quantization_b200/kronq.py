"""Python binding of the KronQ C ABI (libkronq.so): argument marshalling only.

Every function here has the name of the C entry point it calls and does nothing but turn
torch tensors into pointers, sizes and strides, allocate the caller-side workspace with torch,
and raise KronqError on a non-OK status. All arithmetic runs in the CUDA library; there is no
fallback. If the library is missing, importing the functions still works but the first call
raises (build it with `python -m post_quantization_b200.build`).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libkronq.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_SHAPE = 2
ERR_NOT_PD = 3
ERR_CUDA = 4
ERR_WORKSPACE = 5
ERR_UNSUPPORTED = 6
ERR_TIMEOUT = 7

DTYPE_BF16 = 0
DTYPE_F32 = 1

BIIP_SCALE_IN = 1
BIIP_SCALE_OUT = 2
BIIP_ROTATE_IN = 4
BIIP_ROTATE_OUT = 8
BIIP_WRITE_HG = 16
BIIP_HG_DIAG = 32
BIIP_FULL = 15

CHOLINV_SYNC = 1

# every exported symbol of include/kronq.h
SYMBOLS = (
    "kronq_status_string", "kronq_last_error_detail", "kronq_version", "kronq_device_check",
    "kronq_device_error", "kronq_launch_count", "kronq_set_sm_budget", "kronq_sm_budget",
    "kronq_accumulate_workspace_size", "kronq_accumulate",
    "kronq_accumulate_diag_workspace_size", "kronq_accumulate_diag",
    "kronq_biip_workspace_size", "kronq_biip", "kronq_biip_noalloc",
    "kronq_cholinv_workspace_size", "kronq_cholinv",
    "kronq_quantize_layer_workspace_size", "kronq_quantize_layer",
    "kronq_score_allocate",
    "kronq_quantize_layer_twosided_workspace_size", "kronq_quantize_layer_twosided",
    "kronq_packed_codes_bytes", "kronq_pack_codes", "kronq_packed_grid_bytes", "kronq_pack_grid",
    "kronq_qlinear_workspace_size", "kronq_qlinear",
)


class KronqError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: status {status}: {detail}")
        self.status = status
        self.detail = detail


_lib = None

c_void_p = ctypes.c_void_p
c_i32 = ctypes.c_int32
c_i64 = ctypes.c_int64
c_u32 = ctypes.c_uint32
c_sz = ctypes.c_size_t
c_dbl = ctypes.c_double
c_flt = ctypes.c_float


def load_library(path: str = LIB_PATH):
    """Load libkronq.so and declare its signatures (raises if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"KronQ CUDA library not built: {path} is missing "
                           "(python -m post_quantization_b200.build)")
    lib = ctypes.CDLL(path)
    sig = {
        "kronq_status_string": (ctypes.c_char_p, [c_i32]),
        "kronq_last_error_detail": (ctypes.c_char_p, []),
        "kronq_version": (c_i32, []),
        "kronq_device_check": (c_i32, []),
        "kronq_device_error": (c_i32, [c_void_p, c_void_p]),
        "kronq_launch_count": (ctypes.c_uint64, []),
        "kronq_set_sm_budget": (None, [c_i32]),
        "kronq_sm_budget": (c_i32, []),
        "kronq_accumulate_workspace_size": (c_sz, [c_i64, c_i32, c_i32, c_i32]),
        "kronq_accumulate": (c_i32, [c_void_p, c_i64, c_void_p, c_i64, c_void_p, c_i64, c_i64,
                                     c_i32, c_i32, c_void_p, c_void_p, c_void_p, c_void_p, c_sz,
                                     c_void_p]),
        "kronq_accumulate_diag_workspace_size": (c_sz, [c_i64, c_i32]),
        "kronq_accumulate_diag": (c_i32, [c_void_p, c_i64, c_i64, c_i32, c_void_p, c_void_p, c_sz,
                                          c_void_p]),
        "kronq_biip_workspace_size": (c_sz, [c_i32, c_i32]),
        "kronq_biip": (c_i32, [c_void_p, c_i32, c_void_p, c_void_p, c_void_p, c_void_p, c_dbl,
                               c_void_p, c_void_p, c_i32, c_i32, c_u32, c_void_p, c_void_p,
                               c_void_p, c_void_p, c_void_p, c_sz, c_void_p]),
        "kronq_biip_noalloc": (c_i32, [c_void_p, c_i32, c_void_p, c_void_p, c_void_p, c_void_p,
                                       c_dbl, c_void_p, c_void_p, c_i32, c_i32, c_u32, c_void_p,
                                       c_void_p, c_void_p, c_void_p, c_void_p]),
        "kronq_cholinv_workspace_size": (c_sz, [c_i32]),
        "kronq_cholinv": (c_i32, [c_void_p, c_i32, c_flt, c_void_p, c_u32, c_void_p, c_sz,
                                  c_void_p]),
        "kronq_quantize_layer_workspace_size": (c_sz, [c_i32, c_i32, c_i32, c_i32]),
        "kronq_quantize_layer": (c_i32, [c_void_p, c_void_p, c_void_p, c_i32, c_i32, c_i32, c_i32,
                                         c_i32, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                         c_sz, c_void_p]),
        "kronq_score_allocate": (c_i32, [c_void_p, c_void_p, c_void_p, c_i32, c_void_p, c_i32,
                                         c_dbl, c_void_p, c_void_p]),
        "kronq_quantize_layer_twosided_workspace_size": (c_sz, [c_i32, c_i32]),
        "kronq_quantize_layer_twosided": (c_i32, [c_void_p, c_void_p, c_void_p, c_i32, c_i32,
                                                  c_i32, c_void_p, c_void_p, c_void_p, c_void_p,
                                                  c_void_p, c_void_p, c_sz, c_void_p]),
        "kronq_packed_codes_bytes": (c_sz, [c_i32, c_i32, c_i32]),
        "kronq_pack_codes": (c_i32, [c_void_p, c_i32, c_i32, c_i32, c_void_p, c_sz, c_void_p]),
        "kronq_packed_grid_bytes": (c_sz, [c_i32, c_i32, c_i32]),
        "kronq_pack_grid": (c_i32, [c_void_p, c_void_p, c_i32, c_i32, c_i32, c_void_p, c_sz,
                                    c_void_p]),
        "kronq_qlinear_workspace_size": (c_sz, [c_i32, c_i32, c_i32]),
        "kronq_qlinear": (c_i32, [c_void_p, c_i32, c_i64, c_i32, c_void_p, c_void_p,
                                  c_i32, c_void_p, c_void_p, c_void_p, c_void_p, c_u32, c_i32,
                                  c_i32, c_i32, c_void_p, c_i64, c_void_p, c_sz, c_void_p]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int, where: str):
    if status != OK:
        lib = load_library()
        raise KronqError(status, where, lib.kronq_last_error_detail().decode())


def _p(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _workspace(nbytes: int, device, ws):
    if nbytes == 0:
        return None, 0
    if ws is not None:
        return ws, ws.numel() * ws.element_size()
    t = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
    off = (-t.data_ptr()) % 256
    v = t[off:off + nbytes]
    return v, nbytes


def _rowstride(t):
    if t is None:
        return 0
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D tensor with unit column stride")
    return t.stride(0)


# ------------------------------------------------------------------------------ status helpers

def kronq_status_string(status: int) -> str:
    return load_library().kronq_status_string(status).decode()


def kronq_version() -> int:
    return load_library().kronq_version()


def kronq_device_check():
    _check(load_library().kronq_device_check(), "kronq_device_check")


def kronq_launch_count() -> int:
    return int(load_library().kronq_launch_count())


def kronq_set_sm_budget(sms: int) -> None:
    """At most `sms` CTAs (one per SM) for the persistent kernels launched from now on; 0 = all."""
    load_library().kronq_set_sm_budget(int(sms))


def kronq_sm_budget() -> int:
    return int(load_library().kronq_sm_budget())


def kronq_device_error(stream=None) -> int:
    code = ctypes.c_int32(0)
    _check(load_library().kronq_device_error(ctypes.byref(code), _stream(stream)),
           "kronq_device_error")
    return code.value


# ------------------------------------------------------------------------------ 1. accumulate

def kronq_accumulate_workspace_size(n: int, d_in: int, d_out: int, with_dxx: bool) -> int:
    return load_library().kronq_accumulate_workspace_size(n, d_in, d_out, int(bool(with_dxx)))


def kronq_accumulate(xq=None, xfp=None, g=None, hx_sum=None, hg_sum=None, dxx_sum=None,
                     workspace=None, stream=None):
    """hx_sum += xq^T xq, hg_sum += g^T g, dxx_sum += (xfp - xq)^T xq (bf16 in, fp32 sums)."""
    lib = load_library()
    ref = xq if xq is not None else g
    n = ref.shape[0]
    d_in = xq.shape[1] if xq is not None else 0
    d_out = g.shape[1] if g is not None else 0
    ws, wsb = _workspace(lib.kronq_accumulate_workspace_size(n, d_in, d_out,
                                                             int(dxx_sum is not None)),
                         ref.device, workspace)
    st = lib.kronq_accumulate(_p(xq), _rowstride(xq), _p(xfp), _rowstride(xfp), _p(g),
                              _rowstride(g), n, d_in, d_out, _p(hx_sum), _p(hg_sum),
                              _p(dxx_sum), _p(ws), wsb, _stream(stream))
    _check(st, "kronq_accumulate")


def kronq_accumulate_diag_workspace_size(n: int, d: int) -> int:
    return load_library().kronq_accumulate_diag_workspace_size(n, d)


def kronq_accumulate_diag(g, diag_sum, workspace=None, stream=None):
    """diag_sum[j] += sum_t g[t, j]^2 (the diagonal of g^T g; bf16 in, fp32 sums)."""
    lib = load_library()
    n, d = g.shape
    ws, wsb = _workspace(lib.kronq_accumulate_diag_workspace_size(n, d), g.device, workspace)
    st = lib.kronq_accumulate_diag(_p(g), _rowstride(g), n, d, _p(diag_sum), _p(ws), wsb,
                                   _stream(stream))
    _check(st, "kronq_accumulate_diag")


# ------------------------------------------------------------------------------ 2. biip

def kronq_biip_workspace_size(d_out: int, d_in: int) -> int:
    return load_library().kronq_biip_workspace_size(d_out, d_in)


def kronq_biip(w, w_out, hx, hg, dxx, inv_n, sign_in, sign_out, flags, s_x, s_g, tr_hx,
               tr_hg=None, workspace=None, stream=None):
    lib = load_library()
    d_out, d_in = w.shape
    if w.dtype == torch.bfloat16:
        wd = DTYPE_BF16
    elif w.dtype == torch.float32:
        wd = DTYPE_F32
    else:
        raise ValueError("w must be bf16 or fp32")
    ws, wsb = _workspace(lib.kronq_biip_workspace_size(d_out, d_in), w.device, workspace)
    st = lib.kronq_biip(_p(w), wd, _p(w_out), _p(hx), _p(hg), _p(dxx), float(inv_n),
                        _p(sign_in), _p(sign_out), d_out, d_in, int(flags), _p(s_x), _p(s_g),
                        _p(tr_hx), _p(tr_hg), _p(ws), wsb, _stream(stream))
    _check(st, "kronq_biip")


# ------------------------------------------------------------------------------ 3. cholinv

def kronq_cholinv_workspace_size(d: int) -> int:
    return load_library().kronq_cholinv_workspace_size(d)


def kronq_cholinv(h_to_k, damp_rel, info, flags=0, workspace=None, stream=None):
    lib = load_library()
    d = h_to_k.shape[0]
    ws, wsb = _workspace(lib.kronq_cholinv_workspace_size(d), h_to_k.device, workspace)
    st = lib.kronq_cholinv(_p(h_to_k), d, float(damp_rel), _p(info), int(flags), _p(ws), wsb,
                           _stream(stream))
    _check(st, "kronq_cholinv")


# ------------------------------------------------------------------------------ 4. quantize

def kronq_quantize_layer_workspace_size(d_out: int, d_in: int, block: int, with_dxx: bool) -> int:
    return load_library().kronq_quantize_layer_workspace_size(d_out, d_in, block,
                                                              int(bool(with_dxx)))


def kronq_quantize_layer(w, k, dxx, bits, codes, scale, zero, w_hat, block=128, workspace=None,
                         stream=None, group=0):
    lib = load_library()
    d_out, d_in = w.shape
    ws, wsb = _workspace(lib.kronq_quantize_layer_workspace_size(d_out, d_in, block,
                                                                 int(dxx is not None)),
                         w.device, workspace)
    st = lib.kronq_quantize_layer(_p(w), _p(k), _p(dxx), d_out, d_in, int(bits), int(block),
                                  int(group), _p(codes), _p(scale), _p(zero), _p(w_hat), _p(ws),
                                  wsb, _stream(stream))
    _check(st, "kronq_quantize_layer")


# ------------------------------------------------------------------------------ 5. allocation

def kronq_score_allocate(tr_hx, tr_hg, n_params, choices, avg_bits):
    """Host call. Returns (scores, bits) as Python lists."""
    lib = load_library()
    L = len(tr_hx)
    a = (ctypes.c_double * L)(*[float(v) for v in tr_hx])
    b = (ctypes.c_double * L)(*[float(v) for v in tr_hg])
    n = (ctypes.c_int64 * L)(*[int(v) for v in n_params])
    ch = (ctypes.c_int32 * len(choices))(*[int(v) for v in choices])
    s = (ctypes.c_double * L)()
    bits = (ctypes.c_int32 * L)()
    st = lib.kronq_score_allocate(a, b, n, L, ch, len(choices), float(avg_bits), s, bits)
    _check(st, "kronq_score_allocate")
    return list(s), list(bits)


# ------------------------------------------------------------------------------ comparison variant

def kronq_quantize_layer_twosided(w, k_in, k_out, bits, codes=None, scale=None, zero=None,
                                  w_hat=None, workspace=None, stream=None):
    """Rounding with input- and output-side feedback (prior art, for comparison).
    Returns (codes, scale, zero, w_hat, iterations)."""
    lib = load_library()
    d_out, d_in = w.shape
    dev = w.device
    codes = codes if codes is not None else torch.empty(d_out, d_in, dtype=torch.uint8, device=dev)
    scale = scale if scale is not None else torch.empty(d_out, dtype=torch.float32, device=dev)
    zero = zero if zero is not None else torch.empty(d_out, dtype=torch.float32, device=dev)
    w_hat = w_hat if w_hat is not None else torch.empty(d_out, d_in, dtype=torch.float32,
                                                        device=dev)
    ws, wsb = _workspace(lib.kronq_quantize_layer_twosided_workspace_size(d_out, d_in), dev,
                         workspace)
    it = ctypes.c_int32(0)
    st = lib.kronq_quantize_layer_twosided(_p(w), _p(k_in), _p(k_out), d_out, d_in, int(bits),
                                           _p(codes), _p(scale), _p(zero), _p(w_hat),
                                           ctypes.byref(it), _p(ws), wsb, _stream(stream))
    _check(st, "kronq_quantize_layer_twosided")
    return codes, scale, zero, w_hat, it.value


# ------------------------------------------------------------------------------ 6. inference

def kronq_packed_codes_bytes(d_out: int, d_in: int, bits: int) -> int:
    return load_library().kronq_packed_codes_bytes(d_out, d_in, bits)


def kronq_pack_codes(codes, bits, packed=None, stream=None):
    """codes: d_out x d_in uint8 (contiguous). Returns the packed uint8 tensor."""
    lib = load_library()
    d_out, d_in = codes.shape
    if not codes.is_contiguous():
        raise ValueError("codes must be contiguous")
    nbytes = lib.kronq_packed_codes_bytes(d_out, d_in, int(bits))
    if packed is None:
        packed = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=codes.device)
    st = lib.kronq_pack_codes(_p(codes), d_out, d_in, int(bits), _p(packed),
                              packed.numel() * packed.element_size(), _stream(stream))
    _check(st, "kronq_pack_codes")
    return packed


def kronq_packed_grid_bytes(d_out: int, d_in: int, group: int) -> int:
    return load_library().kronq_packed_grid_bytes(d_out, d_in, group)


def kronq_pack_grid(scale, zero, d_out, d_in, group, packed=None, stream=None):
    """scale, zero from kronq_quantize_layer. Returns the packed (scale, zero) pairs (fp32)."""
    lib = load_library()
    nbytes = lib.kronq_packed_grid_bytes(d_out, d_in, int(group))
    if packed is None:
        packed = torch.empty(max(nbytes // 4, 2), dtype=torch.float32, device=scale.device)
    st = lib.kronq_pack_grid(_p(scale), _p(zero), d_out, d_in, int(group), _p(packed),
                             packed.numel() * packed.element_size(), _stream(stream))
    _check(st, "kronq_pack_grid")
    return packed


def kronq_qlinear_workspace_size(d_out: int, d_in: int, n_tok: int) -> int:
    return load_library().kronq_qlinear_workspace_size(d_out, d_in, n_tok)


def kronq_qlinear(x, packed, packed_grid, s_x, s_g, sign_in, sign_out, flags, d_out, bits, y,
                  group=0, workspace=None, stream=None):
    """y (n_tok x d_out fp32) = S_G^-1 U^T W^' V S_X^-1 x for x (n_tok x d_in, bf16 or fp32)."""
    lib = load_library()
    n_tok, d_in = x.shape
    if x.dtype == torch.bfloat16:
        xd = DTYPE_BF16
    elif x.dtype == torch.float32:
        xd = DTYPE_F32
    else:
        raise ValueError("x must be bf16 or fp32")
    ws, wsb = _workspace(lib.kronq_qlinear_workspace_size(d_out, d_in, n_tok), x.device,
                         workspace)
    st = lib.kronq_qlinear(_p(x), xd, _rowstride(x), n_tok, _p(packed), _p(packed_grid),
                           int(group), _p(s_x), _p(s_g), _p(sign_in), _p(sign_out), int(flags),
                           int(d_out), d_in, int(bits), _p(y), _rowstride(y), _p(ws), wsb,
                           _stream(stream))
    _check(st, "kronq_qlinear")
