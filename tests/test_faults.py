"""Failure detection on the GPU without faulting it: a withheld barrier arrival
makes a bounded wait inside the GLA kernel run out; the kernel exits through its
normal path, the host reads MSGLA_ERR_DEVICE_TIMEOUT, and the next forward on the
same handle is correct."""
import pytest

from helpers import gpu_inputs
from scale_gated_linear_b200 import _lib
from scale_gated_linear_b200 import workloads as wl

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
needs_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


@needs_gpu
def test_bounded_wait_times_out_and_handle_recovers():
    from scale_gated_linear_b200 import MSGLA
    w = wl.WORKLOADS["tiny"].replace(name="fault", B=2, L=300, d=128, d_k=64, d_v=128)
    inp = gpu_inputs(w)
    layer = MSGLA.from_workload(w, inp, device=0)
    X = inp["X"].cuda()
    ref = layer(X).clone()
    layer.check_status()
    lib = _lib.load()
    _lib.check(lib.msgla_test_skip_arrival(layer._h, 1))
    layer(X)
    assert layer.sync_status() == -4          # MSGLA_ERR_DEVICE_TIMEOUT, read on the host
    assert layer.sync_status() == 0           # latched once, then cleared
    again = layer(X)                          # the switch reset itself
    layer.check_status()
    assert torch.equal(again, ref)
    layer.close()
