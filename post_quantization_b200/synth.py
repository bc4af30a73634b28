"""Seeded synthetic inputs for the KronQ layer path.

These generators stand in for the calibration activations, output gradients and weights of
LLaMA-shaped layers (no model weights or calibration corpora are available). They produce
random numbers only: none of the quantizer's arithmetic lives here, so that both the CUDA
path and the fp64 oracle can be fed the very same arrays.

Recipe (per workload):
  * X  = Z A^T / sqrt(d) with Z, A standard normal, so the token covariance is A A^T / d;
         a seeded set of 4 input channels is multiplied by 20 (activation outliers).
  * G  = Z diag(sigma) with log10(sigma_i) uniform on [-3, 1] (output channels whose gradient
         scale spans four orders of magnitude).
  * X~ = X + N(0, s^2): s = 0.01 (small layer), s = 0.05 * rms(X) (drifted input), or X~ = X.
  * W  ~ N(0, 0.02^2).
  * sign vectors: Rademacher +-1 (the random signs of the randomized Hadamard transforms).
Everything is drawn from torch generators seeded from a stable hash of a label, so a tensor
is identical across runs and processes on the same device type.
"""
from __future__ import annotations

import math
import zlib
from dataclasses import dataclass, field

import torch

BASE_SEED = 20260710


def seed_for(*label) -> int:
    """Stable 63-bit seed from a label tuple (config, block, sublayer, tensor, ...)."""
    s = "/".join(str(x) for x in label).encode()
    return (BASE_SEED * 1_000_003 + zlib.crc32(s) * 65_537 + zlib.adler32(s)) & ((1 << 63) - 1)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def rademacher(d: int, seed: int, device="cpu") -> torch.Tensor:
    """d random signs (+1/-1) as int8."""
    g = _gen(seed, device)
    b = torch.randint(0, 2, (d,), generator=g, device=device, dtype=torch.int8)
    return (b * 2 - 1).to(torch.int8)


def weight(d_out: int, d_in: int, seed: int, dtype=torch.bfloat16, device="cpu",
           std: float = 0.02) -> torch.Tensor:
    g = _gen(seed, device)
    w = torch.randn(d_out, d_in, generator=g, device=device, dtype=torch.float32) * std
    return w.to(dtype)


def mixing_matrix(d: int, seed: int, device="cpu") -> torch.Tensor:
    """A with X = Z A^T / sqrt(d); fp32."""
    g = _gen(seed, device)
    return torch.randn(d, d, generator=g, device=device, dtype=torch.float32)


def outlier_channels(d: int, seed: int, count: int = 4) -> list[int]:
    g = _gen(seed, "cpu")
    return sorted(torch.randperm(d, generator=g)[:count].tolist())


def correlated_x(n: int, d: int, seed: int, dtype=torch.bfloat16, device="cpu",
                 n_outliers: int = 4, outlier_scale: float = 20.0,
                 chunk: int = 16384) -> torch.Tensor:
    """n x d activations with covariance A A^T / d and a few x20 outlier channels.

    Generated chunk by chunk (each chunk from its own seed) so large workloads never hold
    Z for all tokens at once.
    """
    a = mixing_matrix(d, seed_for(seed, "A"), device)
    cols = outlier_channels(d, seed_for(seed, "outliers"), n_outliers)
    colscale = torch.ones(d, device=device, dtype=torch.float32)
    colscale[cols] = outlier_scale
    mix = (a.t() / math.sqrt(d)) * colscale[None, :]  # x_row = z_row @ A^T / sqrt(d), outliers scaled
    mm_dtype = torch.float32 if torch.device(device).type == "cpu" else torch.bfloat16
    mix = mix.to(mm_dtype)
    out = torch.empty(n, d, device=device, dtype=dtype)
    for c0 in range(0, n, chunk):
        c1 = min(n, c0 + chunk)
        g = _gen(seed_for(seed, "Z", c0), device)
        z = torch.randn(c1 - c0, d, generator=g, device=device, dtype=torch.float32).to(mm_dtype)
        out[c0:c1] = (z @ mix).to(dtype)
        del z
    return out


def gradient_scales(d_out: int, seed: int, log10_lo: float = -3.0, log10_hi: float = 1.0,
                    device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    u = torch.rand(d_out, generator=g, device=device, dtype=torch.float32)
    return torch.pow(10.0, log10_lo + (log10_hi - log10_lo) * u)


def gradients(n: int, d_out: int, seed: int, dtype=torch.bfloat16, device="cpu",
              log10_lo: float = -3.0, log10_hi: float = 1.0, multiplier: float = 1.0,
              chunk: int = 16384) -> torch.Tensor:
    """n x d_out output gradients g_n = sigma * z_n, log-uniform per-channel sigma."""
    sig = gradient_scales(d_out, seed_for(seed, "sigma"), log10_lo, log10_hi, device) * multiplier
    out = torch.empty(n, d_out, device=device, dtype=dtype)
    for c0 in range(0, n, chunk):
        c1 = min(n, c0 + chunk)
        g = _gen(seed_for(seed, "Zg", c0), device)
        z = torch.randn(c1 - c0, d_out, generator=g, device=device, dtype=torch.float32)
        out[c0:c1] = (z * sig[None, :]).to(dtype)
        del z
    return out


def perturbed(x: torch.Tensor, seed: int, abs_std: float | None = None,
              rel_std: float | None = None, chunk: int = 16384) -> torch.Tensor:
    """X~ = X + Gaussian noise; abs_std, or rel_std * rms(X) over the whole tensor."""
    if rel_std is not None:
        ss = 0.0
        for c0 in range(0, x.shape[0], chunk):
            ss += float(x[c0:c0 + chunk].float().pow(2).sum())
        std = rel_std * math.sqrt(ss / x.numel())
    else:
        std = float(abs_std)
    out = torch.empty_like(x)
    for c0 in range(0, x.shape[0], chunk):
        c1 = min(x.shape[0], c0 + chunk)
        g = _gen(seed_for(seed, "noise", c0), x.device)
        nz = torch.randn(c1 - c0, x.shape[1], generator=g, device=x.device, dtype=torch.float32)
        out[c0:c1] = (x[c0:c1].float() + std * nz).to(x.dtype)
        del nz
    return out


# ----------------------------------------------------------------------------------------------
# Workload shapes (LLaMA-family linear layers: d_out x d_in)
# ----------------------------------------------------------------------------------------------

@dataclass(frozen=True)
class Sublayer:
    name: str
    d_out: int
    d_in: int
    x_stream: str  # sublayers with the same stream share their input activations


@dataclass
class Workload:
    name: str
    sublayers: list[Sublayer]
    n_tokens: int
    bits: int
    drift: str          # "abs0.01", "rel0.05" or "none" (X~ = X, asymmetric term off)
    w_dtype: torch.dtype = torch.bfloat16
    n_blocks: int = 1
    extra: dict = field(default_factory=dict)

    @property
    def params_per_block(self) -> int:
        return sum(s.d_out * s.d_in for s in self.sublayers)

    def streams(self) -> dict[str, int]:
        out = {}
        for s in self.sublayers:
            out.setdefault(s.x_stream, s.d_in)
        return out


def _block(h, kv, ff, own_x=False):
    def st(name, shared):
        return name if own_x else shared
    return [
        Sublayer("q_proj", h, h, st("q_proj", "attn_in")),
        Sublayer("k_proj", kv, h, st("k_proj", "attn_in")),
        Sublayer("v_proj", kv, h, st("v_proj", "attn_in")),
        Sublayer("o_proj", h, h, st("o_proj", "o_in")),
        Sublayer("gate_proj", ff, h, st("gate_proj", "mlp_in")),
        Sublayer("up_proj", ff, h, st("up_proj", "mlp_in")),
        Sublayer("down_proj", h, ff, st("down_proj", "down_in")),
    ]


WORKLOADS = {
    # single 256x256 layer, 2048 tokens, fp32 weights, drifted input (asymmetric term on)
    "layer256": Workload("layer256", [Sublayer("layer", 256, 256, "x")], 2048, 2, "abs0.01",
                         w_dtype=torch.float32),
    # LLaMA-2-7B-shaped block, 262144 tokens, 4-bit, X~ = X
    "llama2_7b_block": Workload("llama2_7b_block", _block(4096, 4096, 11008), 262144, 4, "none"),
    # LLaMA-3-8B-shaped block (GQA), 262144 tokens, 3-bit, drifted input
    "llama3_8b_block": Workload("llama3_8b_block", _block(4096, 1024, 14336), 262144, 3, "rel0.05"),
    # LLaMA-3-70B-shaped block, 262144 tokens, 2-bit, drifted input
    "llama3_70b_block": Workload("llama3_70b_block", _block(8192, 1024, 28672), 262144, 2,
                                 "rel0.05"),
    # 32 LLaMA-2-7B-shaped blocks, every sublayer its own X and G, 65536 tokens, mixed precision
    "llama2_7b_stack": Workload("llama2_7b_stack", _block(4096, 4096, 11008, own_x=True), 65536,
                                0, "none", n_blocks=32,
                                extra={"choices": (2, 3, 4), "avg_bits": 2.5,
                                       "g_block_multiplier_log10": (-2.0, 1.0)}),
}


def block_g_multiplier(block: int, log10_lo: float, log10_hi: float, seed: int) -> float:
    """Per-block output-gradient scale of a stack, log-uniform on [10^lo, 10^hi]."""
    g = _gen(seed_for(seed, "block", block), "cpu")
    u = float(torch.rand(1, generator=g, dtype=torch.float64))
    return 10.0 ** (log10_lo + (log10_hi - log10_lo) * u)


# ------------------------------------------------------------------ a quantized layer's storage
# Stand-ins for what the solve returns (codes, grid) and for the incoherence scales, so that
# the inference path can be exercised at any size without running the solve first.

def codes(d_out: int, d_in: int, bits: int, seed: int, device="cpu") -> torch.Tensor:
    """Uniform random b-bit codes (uint8)."""
    g = _gen(seed, device)
    return torch.randint(0, 1 << bits, (d_out, d_in), generator=g, device=device,
                         dtype=torch.int32).to(torch.uint8)


def grid_params(d_out: int, n_groups: int, bits: int, seed: int, device="cpu"):
    """(scale, zero) fp32 of shape d_out (n_groups 0) or d_out x n_groups: scale log-uniform on
    [1e-3, 1e-1], zero an integer in [-1, 2^bits]."""
    g = _gen(seed, device)
    shape = (d_out,) if n_groups == 0 else (d_out, n_groups)
    scale = torch.exp(torch.empty(shape, device=device).uniform_(math.log(1e-3), math.log(1e-1),
                                                                generator=g))
    zero = torch.randint(-1, (1 << bits) + 1, shape, generator=g, device=device).float()
    return scale.float(), zero


def positive_scales(d: int, seed: int, device="cpu", lo: float = 0.25, hi: float = 4.0):
    """d fp32 values log-uniform on [lo, hi] (stand-ins for the diagonal BiIP scales)."""
    g = _gen(seed, device)
    return torch.exp(torch.empty(d, device=device).uniform_(math.log(lo), math.log(hi),
                                                            generator=g)).float()


def activations(n: int, d: int, seed: int, dtype=torch.float32, device="cpu",
                n_outliers: int = 4, outlier_scale: float = 20.0) -> torch.Tensor:
    """n x d independent N(0, 1) activations with a few x20 outlier channels (decode-time
    inputs of a layer; no mixing matrix, so any d is cheap)."""
    g = _gen(seed, device)
    x = torch.randn(n, d, generator=g, device=device, dtype=torch.float32)
    cols = outlier_channels(d, seed_for(seed, "outliers"), n_outliers)
    x[:, cols] *= outlier_scale
    return x.to(dtype)


# ------------------------------------------------------------ a synthetic block's own backward
# The KronQ pages obtain G from one backward pass of the model over the calibration set. This
# stands in for that with a random-weight LLaMA-style block (no trained weights, no dataset):
# its forward over correlated synthetic inputs gives each linear's input X, and its backward
# from a synthetic gradient of the block output gives each linear's output gradient G. It is
# input generation, like the generators above: plain torch ops in fp32, stored as bf16.

def _rms_norm(x: torch.Tensor, eps: float = 1e-5) -> torch.Tensor:
    return x * torch.rsqrt(x.pow(2).mean(dim=-1, keepdim=True) + eps)


def block_calibration(wl: Workload, n: int, seed: int, device="cpu", seq_len: int = 2048,
                      head_dim: int = 128, seqs_per_chunk: int = 4, dtype=torch.bfloat16,
                      weights: dict | None = None):
    """X (per input stream) and G (per sublayer) of one forward + backward of a random-weight block.

    Block: u = x + o_proj(attn(q_proj(n1), k_proj(n1), v_proj(n1))) with n1 = rmsnorm(x), causal
    attention per sequence of seq_len tokens (k/v heads shared by groups of query heads when
    k_proj is narrower than q_proj); y = u + down_proj(silu(gate_proj(n2)) * up_proj(n2)) with
    n2 = rmsnorm(u). x is the correlated synthetic activation of the block input; the gradient
    of the block output dL/dy is the log-uniform per-channel synthetic gradient. Weights are
    N(0, 0.02^2) in wl's shapes, or `weights` ({sublayer: W}) when given, so that the statistics
    belong to the layers being quantized. Returns ({stream: X}, {sublayer: G}) with the streams
    of wl: the inputs of q/k/v, o, gate/up and down.
    """
    subs = {s.name: s for s in wl.sublayers}
    h = subs["q_proj"].d_in
    heads = subs["q_proj"].d_out // head_dim
    kv_heads = subs["k_proj"].d_out // head_dim
    f32 = torch.float32
    w = weights if weights is not None else {
        name: weight(s.d_out, s.d_in, seed_for(seed, name, "W"), dtype=dtype, device=device)
        for name, s in subs.items()}
    x_all = correlated_x(n, h, seed_for(seed, "x"), dtype=dtype, device=device)
    gy_all = gradients(n, h, seed_for(seed, "gy"), dtype=dtype, device=device)
    stream_of = {s.name: s.x_stream for s in wl.sublayers}
    xs = {st: torch.empty(n, subs[name].d_in, dtype=dtype, device=device)
          for name, st in stream_of.items()}
    gs = {name: torch.empty(n, s.d_out, dtype=dtype, device=device) for name, s in subs.items()}
    chunk = seq_len * seqs_per_chunk
    for c0 in range(0, n, chunk):
        c1 = min(n, c0 + chunk)
        nb = (c1 - c0) // seq_len
        x = x_all[c0:c1].to(f32).requires_grad_(True)    # so that every output carries a grad
        outs = {}

        def lin(name, inp):
            out = inp @ w[name].to(f32).t()
            out.retain_grad()
            outs[name] = (inp, out)
            return out

        with torch.enable_grad():
            n1 = _rms_norm(x)
            q = lin("q_proj", n1)
            k = lin("k_proj", n1)
            v = lin("v_proj", n1)
            qh = q.view(nb, seq_len, heads, head_dim).transpose(1, 2)
            kh = k.view(nb, seq_len, kv_heads, head_dim).transpose(1, 2)
            vh = v.view(nb, seq_len, kv_heads, head_dim).transpose(1, 2)
            if kv_heads != heads:
                kh = kh.repeat_interleave(heads // kv_heads, dim=1)
                vh = vh.repeat_interleave(heads // kv_heads, dim=1)
            att = torch.nn.functional.scaled_dot_product_attention(qh, kh, vh, is_causal=True)
            att = att.transpose(1, 2).reshape(c1 - c0, heads * head_dim)
            u = x + lin("o_proj", att)
            n2 = _rms_norm(u)
            a = lin("gate_proj", n2)
            b = lin("up_proj", n2)
            y = u + lin("down_proj", torch.nn.functional.silu(a) * b)
            y.backward(gy_all[c0:c1].to(f32))
        for name, (inp, out) in outs.items():
            xs[stream_of[name]][c0:c1] = inp.detach().to(dtype)
            gs[name][c0:c1] = out.grad.to(dtype)
        del outs, x
    return xs, gs
