"""GPU parity of the masked forward (valid-token mask in the pooling of Eq. (8),
MS-GLA reading notes Sec. 3.1) against the fp64 oracle, through the C ABI.

The cases reach every pooling kernel the library picks: the pool-only kernel
for scale sets with a scale-1 branch (blocks of 4, 6 and 8 rows; powers of two
through the pairwise tree, s = 3 through the general loop), the pooling +
fusion-weight kernel of the no-fine-branch layer (blocks of 4 and 6 rows), the
generic kernel (least common multiple 5 or 10) and the lone scale-1 branch (no
pooling launch: the projection epilogue zeroes the padded rows). Same bar as
the unmasked parity tests.
"""
import numpy as np
import pytest

from helpers import MAX_REL, MEAN_REL, gpu_inputs, oracle_forward, rel_errors
from scale_gated_linear_b200 import workloads as wl

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

needs_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")

SMALL = wl.WORKLOADS["tiny"].replace(name="small", B=3, L=203, d=128, d_k=64, d_v=128, chunk=64)
CASES = {
    "fine_124": SMALL,
    "fine_13": SMALL.replace(name="fine_13", scales=(1, 3), heads=(2, 1)),
    "fine_1248": SMALL.replace(name="fine_1248", scales=(1, 2, 4, 8), heads=(2, 1, 1, 1)),
    "nofine_24": SMALL.replace(name="nofine_24", scales=(2, 4), heads=(2, 2)),
    "nofine_23": SMALL.replace(name="nofine_23", scales=(2, 3), heads=(1, 1)),
    "nofine_25": SMALL.replace(name="nofine_25", scales=(2, 5), heads=(1, 1)),
    "fine_15": SMALL.replace(name="fine_15", scales=(1, 5), heads=(1, 1)),
    "single_1": SMALL.replace(name="single_1", scales=(1,), heads=(4,)),
}


def run_masked(w, inp, mask):
    from scale_gated_linear_b200 import MSGLA
    layer = MSGLA.from_workload(w, inp, device=0)
    X = inp["X"].cuda()
    B, L, _ = X.shape
    ws = layer.alloc_workspace(B, L)
    O = layer.forward(X, workspace=ws, mask=None if mask is None else mask.cuda())
    torch.cuda.synchronize()
    layer.check_status()
    out = O.float().cpu().numpy()
    layer.close()
    return out


def assert_parity(got, ref):
    mx, mn = rel_errors(got, ref)
    assert np.isfinite(got).all()
    assert mx <= MAX_REL and mn <= MEAN_REL, f"max_rel={mx:.3e} mean_rel={mn:.3e}"


@needs_gpu
@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("kind", ["left", "right", "random"])
def test_masked_matches_oracle(case, kind):
    w = CASES[case]
    inp = gpu_inputs(w)
    M = wl.make_mask(w.B, w.L, kind, seed=7)
    assert_parity(run_masked(w, inp, M), oracle_forward(w, inp, mask=M.numpy()))


@needs_gpu
@pytest.mark.parametrize("case", ["fine_124", "nofine_24"])
def test_all_padding_mask(case):
    """Every pooled row is zero (denominator clamped to 1); only the fusion
    weights still read x_t."""
    w = CASES[case]
    inp = gpu_inputs(w)
    M = wl.make_mask(w.B, w.L, "all_padding")
    got = run_masked(w, inp, M)
    ref = oracle_forward(w, inp, mask=M.numpy())
    # q = k = v = 0 everywhere: the layer output is exactly zero
    assert np.abs(ref).max() == 0.0
    assert np.abs(got).max() == 0.0


@needs_gpu
@pytest.mark.parametrize("case", sorted(CASES))
def test_all_valid_mask_is_bitwise_the_unmasked_forward(case):
    w = CASES[case]
    inp = gpu_inputs(w)
    a = run_masked(w, inp, wl.make_mask(w.B, w.L, "none"))
    b = run_masked(w, inp, None)
    np.testing.assert_array_equal(a, b)


@needs_gpu
def test_bool_mask_and_340m_shape():
    """The 340M-shaped layer (tcgen05 CTA-pair projection GEMM) with a bool
    left-padding mask over several GEMM tiles and GLA chunks."""
    w = wl.WORKLOADS["msgla_340m"]
    inp = gpu_inputs(w, B=2, L=600)
    M = wl.make_mask(2, 600, "left", seed=3)
    got = run_masked(w, inp, M.bool())
    assert_parity(got, oracle_forward(w, inp, mask=M.numpy()))


@needs_gpu
def test_masked_rows_do_not_reach_pooled_rows():
    """Eq. (8) weights padded rows by zero, so in a layer without a scale-1
    branch X at padded positions reaches the output only through the fusion
    weights of those same positions: changing it leaves every valid position's
    output unchanged, bit for bit."""
    w = CASES["nofine_24"]
    inp = gpu_inputs(w)
    M = wl.make_mask(w.B, w.L, "random", seed=5)
    inp2 = dict(inp)
    X2 = inp["X"].clone()
    X2[M == 0] = (X2[M == 0].float() + 3.0).to(X2.dtype)
    inp2["X"] = X2
    a = run_masked(w, inp, M)
    b = run_masked(w, inp2, M)
    keep = M.numpy().astype(bool)
    np.testing.assert_array_equal(a[keep], b[keep])
