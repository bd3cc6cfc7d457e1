"""GPU parity of the token-by-token decode (msgla_step with the per-branch cache)
against the fp64 oracle, through the C ABI: feeding a sequence one token at a
time must give the layer output at every position (the oracle's whole-sequence
layer, which its own pins tie to the decode recurrence). Same bar as the other
parity tests, over all positions."""
import numpy as np
import pytest

from helpers import MAX_REL, MEAN_REL, gpu_inputs, oracle_forward, rel_errors
from scale_gated_linear_b200 import workloads as wl

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

needs_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")

SMALL = wl.WORKLOADS["tiny"].replace(name="dec_small", B=3, L=37, d=128, d_k=64, d_v=128, chunk=64)


def decode_all(layer, X):
    B, L, _ = X.shape
    cache = layer.new_cache(B)
    outs = []
    for t in range(L):
        outs.append(layer.step(X[:, t].contiguous(), t, cache).clone())
    torch.cuda.synchronize()
    layer.check_status()
    return torch.stack(outs, dim=1).float().cpu().numpy(), cache


def assert_parity(got, ref):
    mx, mn = rel_errors(got, ref)
    assert np.isfinite(got).all()
    assert mx <= MAX_REL and mn <= MEAN_REL, f"max_rel={mx:.3e} mean_rel={mn:.3e}"


@needs_gpu
@pytest.mark.parametrize("scales,heads", [((1, 2, 4), (2, 1, 1)), ((2, 4), (2, 2)), ((1, 3), (2, 1)),
                                          ((1,), (4,)), ((1, 2, 4, 8), (2, 1, 1, 1))])
def test_decode_matches_oracle(scales, heads):
    from scale_gated_linear_b200 import MSGLA
    w = SMALL.replace(scales=scales, heads=heads)
    inp = gpu_inputs(w)
    layer = MSGLA.from_workload(w, inp, device=0)
    got, _ = decode_all(layer, inp["X"].cuda())
    layer.close()
    assert_parity(got, oracle_forward(w, inp))


@needs_gpu
def test_decode_padded_widths_and_head_norm():
    from scale_gated_linear_b200 import MSGLA
    w = SMALL.replace(d_k=100, d_v=200, head_norm=True)
    inp = gpu_inputs(w)
    layer = MSGLA.from_workload(w, inp, device=0)
    got, _ = decode_all(layer, inp["X"].cuda())
    layer.close()
    assert_parity(got, oracle_forward(w, inp))


@needs_gpu
def test_decode_equals_forward_and_reset_restarts():
    """Decode and the whole-sequence forward agree, and emptying the cache makes
    a second pass over the same tokens repeat the first bit for bit."""
    from scale_gated_linear_b200 import MSGLA
    w = SMALL
    inp = gpu_inputs(w)
    layer = MSGLA.from_workload(w, inp, device=0)
    X = inp["X"].cuda()
    first, cache = decode_all(layer, X)
    B, L, _ = X.shape
    layer.reset_cache(cache, B)
    again = []
    for t in range(L):
        again.append(layer.step(X[:, t].contiguous(), t, cache).clone())
    again = torch.stack(again, dim=1).float().cpu().numpy()
    np.testing.assert_array_equal(first, again)
    full = layer.forward(X).float().cpu().numpy()
    layer.close()
    assert_parity(first, full.astype(np.float64))


@needs_gpu
def test_decode_340m_shape():
    """The 340M-shaped layer (d_k = 256, d_v = 512, CTA-pair GEMMs with the
    sequences as rows) over 20 tokens of 5 sequences."""
    from scale_gated_linear_b200 import MSGLA
    w = wl.WORKLOADS["msgla_340m"]
    inp = gpu_inputs(w, B=5, L=20)
    layer = MSGLA.from_workload(w, inp, device=0)
    got, _ = decode_all(layer, inp["X"].cuda())
    layer.close()
    assert_parity(got, oracle_forward(w, inp))


@needs_gpu
def test_decode_long_memory_gates():
    """Gates near 1 (b_g = +3): the state carries information over all 300
    positions, so an error in the per-step decay would accumulate."""
    from scale_gated_linear_b200 import MSGLA
    w = SMALL.replace(gate_bias=3.0, gate_fan_in_init=True, B=2, L=300)
    inp = gpu_inputs(w)
    layer = MSGLA.from_workload(w, inp, device=0)
    got, _ = decode_all(layer, inp["X"].cuda())
    layer.close()
    assert_parity(got, oracle_forward(w, inp))


@needs_gpu
def test_decode_cycle_replays_as_cuda_graph():
    """Which branches step depends only on t modulo lcm(scales), so one captured
    cycle of msgla_step calls replays every later cycle: graph replay and eager
    calls give bit-identical outputs and caches."""
    from scale_gated_linear_b200 import MSGLA
    w = SMALL.replace(L=12)
    inp = gpu_inputs(w)
    X = inp["X"].cuda()
    B = w.B
    period = 4
    outs_eager = []
    layer = MSGLA.from_workload(w, inp, device=0)
    cache = layer.new_cache(B)
    for t in range(w.L):
        outs_eager.append(layer.step(X[:, t].contiguous(), t, cache).clone())
    torch.cuda.synchronize()
    eager_cache = cache.clone()

    layer.reset_cache(cache, B)
    xs = [torch.empty(B, w.d, dtype=torch.bfloat16, device="cuda") for _ in range(period)]
    outs = [torch.empty(B, w.d, dtype=torch.bfloat16, device="cuda") for _ in range(period)]
    ws = torch.empty(layer.step_workspace_size(B), dtype=torch.uint8, device="cuda")
    for i in range(period):  # the first cycle runs eagerly (also warms the launch paths)
        xs[i].copy_(X[:, i])
        layer.step(xs[i], i, cache, out=outs[i], workspace=ws)
    got = [o.clone() for o in outs]
    graph = torch.cuda.CUDAGraph()
    snapshot = cache.clone()
    with torch.cuda.graph(graph):
        for i in range(period):
            layer.step(xs[i], period + i, cache, out=outs[i], workspace=ws, stream=torch.cuda.current_stream())
    cache.copy_(snapshot)  # capture does not run the kernels; start the replays from cycle 1
    for c in range(1, w.L // period):
        for i in range(period):
            xs[i].copy_(X[:, c * period + i])
        graph.replay()
        got += [o.clone() for o in outs]
    torch.cuda.synchronize()
    layer.check_status()
    del graph
    layer.close()
    np.testing.assert_array_equal(torch.stack(got, 1).float().cpu().numpy(),
                                  torch.stack(outs_eager, 1).float().cpu().numpy())
    assert torch.equal(cache, eager_cache)
