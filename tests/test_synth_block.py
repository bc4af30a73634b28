"""The synthetic block's forward and backward (the calibration inputs with a real G).

The generator uses autograd; these checks restate the MLP half of the backward by hand: the
gradient of down_proj's output is the block-output gradient itself (residual connection), and
the gradients of gate_proj's and up_proj's outputs follow from the SwiGLU product rule,
dL/da = (dL/dh) b silu'(a) and dL/db = (dL/dh) silu(a) with dL/dh = (dL/dy) W_down. down_proj's
input must be silu(a) b recomputed from gate/up's input.
"""
import torch

from post_quantization_b200 import synth


def test_block_backward_matches_hand_written_mlp_backward():
    wl = synth.Workload("tiny", synth._block(256, 128, 512), 2048, 2, "none")
    n, seed = 2048, 11
    xs, gs = synth.block_calibration(wl, n, seed, seq_len=512, head_dim=64, seqs_per_chunk=2,
                                     dtype=torch.float32)
    w = {s.name: synth.weight(s.d_out, s.d_in, synth.seed_for(seed, s.name, "W"),
                              dtype=torch.float32) for s in wl.sublayers}
    gy = synth.gradients(n, 256, synth.seed_for(seed, "gy"), dtype=torch.float32)
    torch.testing.assert_close(gs["down_proj"], gy, rtol=0, atol=0)
    n2 = xs["mlp_in"].double()
    a = n2 @ w["gate_proj"].double().t()
    b = n2 @ w["up_proj"].double().t()
    sig = torch.sigmoid(a)
    silu = a * sig
    dsilu = sig * (1 + a * (1 - sig))
    gh = gy.double() @ w["down_proj"].double()
    torch.testing.assert_close(xs["down_in"].double(), silu * b, rtol=1e-4, atol=1e-5)
    torch.testing.assert_close(gs["up_proj"].double(), gh * silu, rtol=1e-4, atol=1e-6)
    torch.testing.assert_close(gs["gate_proj"].double(), gh * b * dsilu, rtol=1e-4, atol=1e-6)
    # attention-side gradients exist and are finite; k/v narrower than q (grouped heads)
    for name in ("q_proj", "k_proj", "v_proj", "o_proj"):
        assert torch.isfinite(gs[name]).all() and gs[name].abs().sum() > 0
    assert gs["k_proj"].shape == (n, 128)
