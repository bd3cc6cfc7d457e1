"""GPU parity of the optional per-head RMS normalisation of the GLA output
(the per-branch normalisation that Sec. 3.2 of the MS-GLA reading notes lists
without defining it, read as o_h / sqrt(mean(o_h^2) + eps) * norm_w) against
the fp64 oracle, through the C ABI. Same bar as the other parity tests."""
import numpy as np
import pytest

from helpers import MAX_REL, MEAN_REL, gpu_inputs, oracle_forward, rel_errors
from scale_gated_linear_b200 import workloads as wl

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

needs_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")

SMALL = wl.WORKLOADS["tiny"].replace(name="small_norm", B=2, L=203, d=128, d_k=64, d_v=128, chunk=64,
                                     head_norm=True)


def run(w, inp, mask=None):
    from scale_gated_linear_b200 import MSGLA
    layer = MSGLA.from_workload(w, inp, device=0)
    X = inp["X"].cuda()
    B, L, _ = X.shape
    ws = layer.alloc_workspace(B, L)
    O = layer.forward(X, workspace=ws, mask=None if mask is None else mask.cuda())
    torch.cuda.synchronize()
    layer.check_status()
    names = layer.launch_names(B, L)
    out = O.float().cpu().numpy()
    layer.close()
    return out, names


def assert_parity(got, ref):
    mx, mn = rel_errors(got, ref)
    assert np.isfinite(got).all()
    assert mx <= MAX_REL and mn <= MEAN_REL, f"max_rel={mx:.3e} mean_rel={mn:.3e}"


@needs_gpu
@pytest.mark.parametrize("dv,scales,heads", [(128, (1, 2, 4), (2, 1, 1)), (200, (1, 2, 4), (2, 1, 1)),
                                              (48, (2, 4), (2, 2)), (384, (1,), (2,))])
def test_head_norm_matches_oracle(dv, scales, heads):
    """One to three value tiles per head, padded head widths (200 -> 256, 48 ->
    128: the mean is over the true d_v), with and without the scale-1 branch."""
    w = SMALL.replace(d_v=dv, scales=scales, heads=heads)
    inp = gpu_inputs(w)
    got, names = run(w, inp)
    assert names[names.index("gla") + 1] == "head_norm"
    assert_parity(got, oracle_forward(w, inp))


@needs_gpu
def test_head_norm_default_weight_is_one():
    w = SMALL
    inp = gpu_inputs(w)
    for br in inp["branches"]:
        del br["norm_w"]
    got, _ = run(w, inp)
    assert_parity(got, oracle_forward(w, inp))


@needs_gpu
def test_head_norm_with_padding_mask():
    """All-padding rows give o = 0, which eps > 0 keeps at zero."""
    w = SMALL
    inp = gpu_inputs(w)
    M = wl.make_mask(w.B, w.L, "left", seed=9)
    got, _ = run(w, inp, M)
    assert_parity(got, oracle_forward(w, inp, mask=M.numpy()))


@needs_gpu
def test_head_norm_340m_shape():
    """d_v = 512 (four value tiles per head), the tcgen05 GEMM/GLA path."""
    w = wl.WORKLOADS["msgla_340m"].replace(name="msgla_340m_norm", head_norm=True)
    inp = gpu_inputs(w, B=2, L=300)
    got, _ = run(w, inp)
    assert_parity(got, oracle_forward(w, inp))
