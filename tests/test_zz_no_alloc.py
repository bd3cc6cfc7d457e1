"""msgla_forward_noalloc: the forward for callers that cannot allocate device
memory when they run the layer (a fixed memory arena, a runtime that forbids
allocation after start-up). Its intermediates live in a fixed scratch array
inside the library instead of a caller workspace.

Checked through the C ABI against msgla_forward (the workspace entry point) on
two calls in a row, so that the second call runs on the scratch contents the
first one left behind. Collected last on purpose: it needs nothing from the
other tests and passes alone in a fresh process as well.
"""
import ctypes

import numpy as np
import pytest

from helpers import MAX_REL, MEAN_REL, gpu_inputs, rel_errors
from scale_gated_linear_b200 import _lib
from scale_gated_linear_b200 import workloads as wl

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
needs_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


@needs_gpu
def test_noalloc_forward_matches_workspace_forward_twice():
    from scale_gated_linear_b200 import MSGLA
    w = wl.WORKLOADS["msgla_340m"]
    B, L = 1, 1000
    inp = gpu_inputs(w, B=B, L=L)
    layer = MSGLA.from_workload(w, inp, device=0)
    assert layer.workspace_size(B, L) <= 32 << 20
    X = inp["X"].cuda()
    ref = layer(X).float().cpu().numpy()
    lib = _lib.load()
    stream = torch.cuda.current_stream()
    for call in range(2):
        O = torch.full_like(X, float("nan"))
        _lib.check(lib.msgla_forward_noalloc(layer._h, X.data_ptr(), B, L, O.data_ptr(),
                                             ctypes.c_void_p(stream.cuda_stream)))
        torch.cuda.synchronize()
        layer.check_status()
        got = O.float().cpu().numpy()
        assert np.isfinite(got).all(), f"call {call}"
        mx, mn = rel_errors(got, ref.astype(np.float64))
        assert mx <= MAX_REL and mn <= MEAN_REL, f"call {call}: max_rel={mx:.3e} mean_rel={mn:.3e}"
    layer.close()


@needs_gpu
def test_noalloc_forward_rejects_sizes_beyond_its_scratch():
    from scale_gated_linear_b200 import MSGLA
    w = wl.WORKLOADS["msgla_340m"]
    inp = gpu_inputs(w, B=1, L=64)
    layer = MSGLA.from_workload(w, inp, device=0)
    B, L = 8, 2048
    assert layer.workspace_size(B, L) > 32 << 20
    X = torch.zeros(B, L, w.d, dtype=torch.bfloat16, device="cuda")
    O = torch.empty_like(X)
    lib = _lib.load()
    st = lib.msgla_forward_noalloc(layer._h, X.data_ptr(), B, L, O.data_ptr(), None)
    assert st == -6, lib.msgla_last_error()
    assert b"fixed scratch" in lib.msgla_last_error()
    layer.close()
