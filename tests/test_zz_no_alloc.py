"""kronq_biip_noalloc: the incoherence step for callers that cannot allocate device memory.

Such callers (code under CUDA graph capture, plug-ins that only see buffers their host
framework hands them, services that reserve all device memory up front) cannot pass a
workspace. The variant uses a fixed scratch array in device memory instead. This test calls
it through the C ABI, twice in a row, and checks each result against kronq_biip with a caller
workspace on the same inputs. It lives in its own file, collected last, and passes on its own
in a fresh process as well as after the other GPU tests.
"""
import numpy as np
import pytest
import torch

from post_quantization_b200 import synth

pytestmark = pytest.mark.gpu

TOL = 1e-3


def rel(a, b):
    a = a.double().cpu().numpy(); b = b.double().cpu().numpy()
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def test_biip_noalloc_matches_workspace_variant():
    from post_quantization_b200 import build
    build.build()
    from post_quantization_b200 import kronq as K
    lib = K.load_library()
    assert torch.cuda.is_available()
    K.kronq_device_check()
    dev = "cuda"
    stream = torch.cuda.current_stream().cuda_stream
    for call, (d_out, d_in) in enumerate([(512, 768), (1024, 256)]):
        n = 1024
        tag = ("noalloc", call)
        x = synth.correlated_x(n, d_in, synth.seed_for(tag, "x"), device=dev)
        xq = synth.perturbed(x, synth.seed_for(tag, "xq"), abs_std=0.01)
        g = synth.gradients(n, d_out, synth.seed_for(tag, "g"), device=dev)
        w = synth.weight(d_out, d_in, synth.seed_for(tag, "w"), device=dev)
        si = synth.rademacher(d_in, synth.seed_for(tag, "si"), device=dev)
        so = synth.rademacher(d_out, synth.seed_for(tag, "so"), device=dev)
        hx = torch.zeros(d_in, d_in, device=dev); hg = torch.zeros(d_out, d_out, device=dev)
        dxx = torch.zeros(d_in, d_in, device=dev)
        K.kronq_accumulate(xq, x, g, hx, hg, dxx)
        outs = {}
        for variant in ("workspace", "noalloc"):
            o = {"w": torch.empty(d_out, d_in, device=dev), "hx": hx.clone(), "hg": hg.clone(),
                 "dxx": dxx.clone(), "sx": torch.empty(d_in, device=dev),
                 "sg": torch.empty(d_out, device=dev),
                 "tr": torch.zeros(2, dtype=torch.float64, device=dev)}
            flags = K.BIIP_FULL | K.BIIP_WRITE_HG
            args = (w.data_ptr(), K.DTYPE_BF16, o["w"].data_ptr(), o["hx"].data_ptr(),
                    o["hg"].data_ptr(), o["dxx"].data_ptr(), 1.0 / n, si.data_ptr(),
                    so.data_ptr(), d_out, d_in, flags, o["sx"].data_ptr(), o["sg"].data_ptr(),
                    o["tr"].data_ptr(), o["tr"].data_ptr() + 8)
            if variant == "workspace":
                nb = lib.kronq_biip_workspace_size(d_out, d_in)
                ws = torch.empty(nb + 256, dtype=torch.uint8, device=dev)
                wp = ws.data_ptr() + (-ws.data_ptr()) % 256
                st = lib.kronq_biip(*args, wp, nb, stream)
            else:
                st = lib.kronq_biip_noalloc(*args, stream)
            assert st == K.OK, lib.kronq_last_error_detail().decode()
            torch.cuda.synchronize()
            outs[variant] = o
        a, b = outs["noalloc"], outs["workspace"]
        for key in ("w", "hx", "hg", "dxx", "sx", "sg", "tr"):
            assert rel(a[key], b[key]) <= TOL, (call, key)
    # a layer too large for the fixed scratch is refused with a clear status
    st = lib.kronq_biip_noalloc(8, 0, 16, 32, None, None, 1.0, None, None, 40000, 40000, 0,
                                48, 64, 80, None, stream)
    assert st == K.ERR_UNSUPPORTED
    assert "static scratch" in lib.kronq_last_error_detail().decode()


def test_biip_noalloc_near_the_scratch_limit():
    """A layer whose scratch fills the fixed array almost to its end.

    d_out = 57088, d_in = 8192 needs 1046528 of the 1048576 bytes; the last region of the
    scratch holds the partial sums of the output-side trace, so tr(H_G) checks that it is
    written and read back correctly. H_G is passed as its diagonal (KRONQ_BIIP_HG_DIAG), which
    keeps the test's own device memory small. Two calls in a row, each against kronq_biip.
    """
    from post_quantization_b200 import build
    build.build()
    from post_quantization_b200 import kronq as K
    lib = K.load_library()
    K.kronq_device_check()
    dev = "cuda"
    stream = torch.cuda.current_stream().cuda_stream
    d_out, d_in, n = 57088, 8192, 512
    nb = lib.kronq_biip_workspace_size(d_out, d_in)
    assert (1 << 20) - 4096 <= nb <= (1 << 20)
    assert lib.kronq_biip_workspace_size(d_out + 256, d_in) > (1 << 20)
    tag = ("noalloc-limit",)
    x = synth.correlated_x(n, d_in, synth.seed_for(tag, "x"), device=dev)
    g = synth.gradients(n, d_out, synth.seed_for(tag, "g"), device=dev)
    w = synth.weight(d_out, d_in, synth.seed_for(tag, "w"), device=dev)
    si = synth.rademacher(d_in, synth.seed_for(tag, "si"), device=dev)
    so = synth.rademacher(d_out, synth.seed_for(tag, "so"), device=dev)
    hx = torch.zeros(d_in, d_in, device=dev)
    hgd = torch.zeros(d_out, device=dev)
    K.kronq_accumulate(xq=x, hx_sum=hx)
    K.kronq_accumulate_diag(g, hgd)
    flags = K.BIIP_FULL | K.BIIP_HG_DIAG
    ws = torch.empty(nb + 256, dtype=torch.uint8, device=dev)
    wp = ws.data_ptr() + (-ws.data_ptr()) % 256

    def run(variant):
        o = {"w": torch.empty(d_out, d_in, device=dev), "hx": hx.clone(),
             "sx": torch.empty(d_in, device=dev), "sg": torch.empty(d_out, device=dev),
             "tr": torch.zeros(2, dtype=torch.float64, device=dev)}
        args = (w.data_ptr(), K.DTYPE_BF16, o["w"].data_ptr(), o["hx"].data_ptr(),
                hgd.data_ptr(), None, 1.0 / n, si.data_ptr(), so.data_ptr(), d_out, d_in, flags,
                o["sx"].data_ptr(), o["sg"].data_ptr(), o["tr"].data_ptr(),
                o["tr"].data_ptr() + 8)
        if variant == "workspace":
            st = lib.kronq_biip(*args, wp, nb, stream)
        else:
            st = lib.kronq_biip_noalloc(*args, stream)
        assert st == K.OK, lib.kronq_last_error_detail().decode()
        torch.cuda.synchronize()
        return o

    ref = run("workspace")
    assert float(ref["tr"][1]) > 0.0
    for _ in range(2):
        got = run("noalloc")
        for key in ("w", "hx", "sx", "sg", "tr"):
            assert rel(got[key], ref[key]) <= TOL, key
        del got
