"""GPU parity of the CUDA path (through the C ABI) against the fp64 oracle.

Bar (bf16 inputs/outputs, fp32 accumulation): max|gpu - oracle| / max|oracle|
<= 1e-2 and mean|gpu - oracle| / mean|oracle| <= 2e-3 on the layer output.
Intermediate stages are checked against the oracle's own intermediates with a
bar of 2e-3 (max) for the fp16 projections and 4e-3 for the GLA output.
"""
import numpy as np
import pytest

from helpers import MAX_REL, MEAN_REL, gpu_inputs, oracle_forward, rel_errors
from scale_gated_linear_b200 import workloads as wl

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

needs_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def _layer(w, inp, **kw):
    from scale_gated_linear_b200 import MSGLA
    return MSGLA.from_workload(w, inp, device=0, **kw)


def run_gpu(w, inp, **kw):
    layer = _layer(w, inp, **kw)
    X = inp["X"].cuda()
    B, L, _ = X.shape
    ws = layer.alloc_workspace(B, L)
    O = layer.forward(X, workspace=ws)
    torch.cuda.synchronize()
    layer.check_status()
    return O.float().cpu().numpy(), layer, ws


def assert_parity(got, ref, max_rel=MAX_REL, mean_rel=MEAN_REL):
    mx, mn = rel_errors(got, ref)
    assert np.isfinite(got).all()
    assert mx <= max_rel and mn <= mean_rel, f"max_rel={mx:.3e} mean_rel={mn:.3e}"


SMALL = wl.WORKLOADS["tiny"].replace(name="small", B=2, L=200, d=128, d_k=64, d_v=128, chunk=64)


@needs_gpu
def test_tiny_workload():
    w = wl.WORKLOADS["tiny"]
    inp = gpu_inputs(w)
    got, layer, _ = run_gpu(w, inp)
    assert_parity(got, oracle_forward(w, inp))
    layer.close()


def chunk_scaled(q, k, log_alpha, chunk=128):
    """Decay-scaled queries and keys of the chunkwise GLA form: within each
    chunk of `chunk` rows, b = cumulative sum of log alpha from the chunk's first
    row, m = b at the chunk's row 63 (its last row if shorter); Qs = q e^{b-m},
    Ks = k e^{m-b}, gamma = e^{b_last - m}, mid = e^{m} per chunk and channel."""
    n = q.shape[0]
    Qs, Ks = np.zeros_like(q), np.zeros_like(k)
    gamma, mid = [], []
    for c0 in range(0, n, chunk):
        b = np.cumsum(log_alpha[c0:c0 + chunk], axis=0)
        m = b[min(63, b.shape[0] - 1)]
        Qs[c0:c0 + chunk] = q[c0:c0 + chunk] * np.exp(b - m)
        Ks[c0:c0 + chunk] = k[c0:c0 + chunk] * np.exp(m - b)
        gamma.append(np.exp(b[-1] - m))
        mid.append(np.exp(m))
    return Qs, Ks, np.array(gamma), np.array(mid)


@needs_gpu
def test_intermediate_stages():
    """Pooled rows, the gate inputs and fusion logits, the decay-scaled queries and
    keys with their chunk decays, v, the GLA output and the fusion weights each
    match the oracle's intermediates (several chunks, ragged tail)."""
    from scale_gated_linear_b200 import WS_FUSION, WS_GAMMA, WS_KS, WS_MID, WS_O, WS_POOLED, WS_QS, WS_U, WS_V
    w = wl.WORKLOADS["msgla_340m"].replace(name="mid")
    B, L = 2, 300
    inp = gpu_inputs(w, B=B, L=L)
    got, layer, ws = run_gpu(w, inp)
    ref, inter = oracle_forward(w, inp, intermediates=True)
    assert_parity(got, ref)
    f = wl.to_float64(inp)

    def close(name, a, b, tol):
        d = np.abs(a - b).max() / np.abs(b).max()
        assert d <= tol, f"{name}: {d:.3e}"

    def heads_only(t, h, width):
        pad = t.shape[-1] // h
        return np.concatenate([t[..., x * pad:x * pad + width] for x in range(h)], axis=-1)

    close("w", layer.workspace_tensor(ws, B, L, 0, WS_FUSION).cpu().numpy(), inter["w"], 1e-5)
    U = layer.workspace_tensor(ws, B, L, 0, WS_U).cpu().numpy()
    ns = len(w.scales)
    close("fusion logits", U[:, :, :ns], f["X"] @ f["Wfuse"].T, 2e-3)
    rp = -(-w.gate_rank // 16) * 16
    for j, (s, h) in enumerate(zip(w.scales, w.heads)):
        bi = inter["branches"][j]
        if s > 1:
            close(f"pooled s={s}", layer.workspace_tensor(ws, B, L, j, WS_POOLED).float().cpu().numpy(), bi["Xp"],
                  1e-3)
        # the branch's gate input: block means of the unpooled rows' columns
        gu = U[:, :, 16 + j * rp:16 + j * rp + w.gate_rank]
        n = bi["Xp"].shape[1]
        gp = np.stack([gu[:, i * s:min(L, i * s + s)].mean(axis=1) for i in range(n)], axis=1)
        close(f"g s={s}", gp, bi["Xp"] @ f["branches"][j]["Wg1"].T, 2e-3)
        qs = heads_only(layer.workspace_tensor(ws, B, L, j, WS_QS).float().cpu().numpy(), h, w.d_k)
        ks = heads_only(layer.workspace_tensor(ws, B, L, j, WS_KS).float().cpu().numpy(), h, w.d_k)
        gam = heads_only(layer.workspace_tensor(ws, B, L, j, WS_GAMMA).cpu().numpy(), h, w.d_k)
        mid = heads_only(layer.workspace_tensor(ws, B, L, j, WS_MID).cpu().numpy(), h, w.d_k)
        for b in range(B):
            Qr, Kr, Gr, Mr = chunk_scaled(bi["q"][b], bi["k"][b], bi["log_alpha"][b])
            close(f"Qs s={s} b={b}", qs[b], Qr, 2e-3)
            close(f"Ks s={s} b={b}", ks[b], Kr, 2e-3)
            close(f"gamma s={s} b={b}", gam[b], Gr, 1e-4)
            close(f"mid s={s} b={b}", mid[b], Mr, 1e-4)
        for name, which, width, ref_t, tol in (("v", WS_V, w.d_v, bi["v"], 2e-3), ("o", WS_O, w.d_v, bi["o"], 4e-3)):
            t = heads_only(layer.workspace_tensor(ws, B, L, j, which).float().cpu().numpy(), h, width)
            close(f"{name} s={s}", t, ref_t, tol)
    layer.close()


@needs_gpu
@pytest.mark.parametrize("L", [1, 2, 3, 4, 5, 63, 64, 65, 127, 128, 129, 200, 255, 257, 520])
def test_ragged_lengths(L):
    """L below a pooling factor, at and around the gate block (64), GLA chunk and
    GEMM tile (128) edges, for every branch's pooled length."""
    inp = gpu_inputs(SMALL, L=L)
    got, layer, _ = run_gpu(SMALL, inp)
    assert_parity(got, oracle_forward(SMALL, inp))
    layer.close()


@needs_gpu
def test_single_scale_plain_gla():
    w = wl.WORKLOADS["gla_340m"].replace(name="gla_small", B=2, d=256)
    inp = gpu_inputs(w, L=333)
    got, layer, _ = run_gpu(w, inp)
    assert_parity(got, oracle_forward(w, inp))
    layer.close()


@needs_gpu
def test_no_fine_branch():
    """{2,4} without the scale-1 branch takes the materialised hold + fusion path."""
    w = wl.WORKLOADS["wide_8k_no_fine"].replace(name="nofine_small", d=256)
    inp = gpu_inputs(w, B=2, L=150)
    got, layer, _ = run_gpu(w, inp)
    assert_parity(got, oracle_forward(w, inp))
    layer.close()


@needs_gpu
def test_wide_scale_set_small():
    w = wl.WORKLOADS["wide_8k"].replace(name="wide_small", d=256)
    inp = gpu_inputs(w, B=2, L=260)
    got, layer, _ = run_gpu(w, inp)
    assert_parity(got, oracle_forward(w, inp))
    layer.close()


@needs_gpu
@pytest.mark.parametrize("L", [200, 201])
def test_two_row_pooling(L):
    """Scales {1, 2}: with an even length and no mask the pooling runs the flat
    2-row kernel, with an odd one the per-block kernel; pooled rows and output
    match the oracle either way."""
    from scale_gated_linear_b200 import WS_POOLED
    w = SMALL.replace(name="s12", scales=(1, 2), heads=(2, 1))
    inp = gpu_inputs(w, L=L)
    got, layer, ws = run_gpu(w, inp)
    ref, inter = oracle_forward(w, inp, intermediates=True)
    assert_parity(got, ref)
    pooled = layer.workspace_tensor(ws, w.B, L, 1, WS_POOLED).float().cpu().numpy()
    want = inter["branches"][1]["Xp"]
    assert np.abs(pooled - want).max() <= 1e-3 * np.abs(want).max()
    layer.close()


@needs_gpu
@pytest.mark.parametrize("scales,heads", [((1, 3), (2, 1)), ((2, 3), (1, 1)), ((1, 2, 6), (1, 1, 1)),
                                          ((1, 5), (1, 1)), ((2, 5), (1, 1)), ((3,), (2,))])
def test_scale_sets_beyond_powers_of_two(scales, heads):
    """Scales that do not divide 4 or 8: the pooling picks 6-row blocks or its
    generic kernel; the hold index floor((t+1)/s) - 1 at odd s."""
    w = SMALL.replace(name="odd", scales=scales, heads=heads)
    inp = gpu_inputs(w, B=2, L=211)
    got, layer, _ = run_gpu(w, inp)
    assert_parity(got, oracle_forward(w, inp))
    layer.close()


@needs_gpu
@pytest.mark.parametrize("dk,dv", [(16, 16), (100, 200), (128, 384)])
def test_padded_head_widths(dk, dv):
    w = SMALL.replace(name=f"pad{dk}x{dv}", d_k=dk, d_v=dv)
    inp = gpu_inputs(w, B=1, L=150)
    got, layer, _ = run_gpu(w, inp)
    assert_parity(got, oracle_forward(w, inp))
    layer.close()


@needs_gpu
def test_qk_scale_and_long_memory_gates():
    w = SMALL.replace(name="qk", gate_bias=3.0, gate_fan_in_init=True)
    inp = gpu_inputs(w, B=1, L=300)
    from scale_gated_linear_b200 import MSGLA
    import oracle
    layer = MSGLA.from_workload(w, inp, device=0, qk_scale=0.125)
    O = layer(inp["X"].cuda())
    torch.cuda.synchronize()
    layer.check_status()
    f = wl.to_float64(inp)
    ref = oracle.layer_forward(f["X"], f, w.scales, w.heads, w.d_k, w.d_v, qk_scale=0.125)
    assert_parity(O.float().cpu().numpy(), ref)
    layer.close()


@needs_gpu
def test_empty_inputs_launch_nothing():
    inp = gpu_inputs(SMALL, L=8)
    layer = _layer(SMALL, inp)
    assert layer.workspace_size(0, 100) == 0 and layer.workspace_size(3, 0) == 0
    for B, L in ((0, 100), (3, 0)):
        X = torch.zeros(B, L, SMALL.d, dtype=torch.bfloat16, device="cuda")
        O = layer.forward(X, workspace=torch.empty(1, dtype=torch.uint8, device="cuda"))
        assert O.shape == (B, L, SMALL.d)
    assert layer.sync_status() == 0
    layer.close()


@needs_gpu
def test_deterministic_and_batch_independent():
    inp = gpu_inputs(SMALL, B=3, L=190)
    layer = _layer(SMALL, inp)
    X = inp["X"].cuda()
    O1 = layer(X).clone()
    O2 = layer(X).clone()
    assert torch.equal(O1, O2)
    for b in range(3):
        Ob = layer(X[b:b + 1].contiguous())
        assert torch.equal(Ob[0], O1[b])
    layer.check_status()
    layer.close()


@needs_gpu
def test_chunk_argument():
    inp = gpu_inputs(SMALL, L=130)
    a = _layer(SMALL, inp, chunk=0)
    b = _layer(SMALL, inp, chunk=128)
    X = inp["X"].cuda()
    assert torch.equal(a(X), b(X))
    a.close(), b.close()


@needs_gpu
@pytest.mark.parametrize("B", [2, 11])
def test_host_buffer_forward_matches_device_forward(B):
    """The host-buffer forward pipelines its copies over chunks of whole
    sequences (one first and last, max(2, ceil((B - 2) / 4)) in each chunk
    between): bit-identical to device forwards of the same chunks, and within
    the parity tolerance of one batched forward (the GLA's segment plan, and so
    its summation order, depends on the batch size)."""
    inp = gpu_inputs(SMALL, B=B, L=150)
    layer = _layer(SMALL, inp)
    X = inp["X"].cuda()
    Od = layer(X)
    mid = 1 if B <= 2 else max(2, -(-(B - 2) // 4))
    sizes, b0 = [], 0
    while b0 < B:
        sizes.append(1 if b0 == 0 or B - b0 <= 1 else min(mid, B - b0 - 1))
        b0 += sizes[-1]
    Oc = torch.cat([layer(x.contiguous()) for x in torch.split(X, sizes)])
    Xh = inp["X"].pin_memory()
    Oh = torch.empty_like(Xh).pin_memory()
    ws = layer.alloc_workspace(B, 150, host_staging=True)
    layer.forward_host(Xh, Oh, ws)
    assert torch.equal(Oh, Oc.cpu())
    assert_parity(Oh.float().numpy(), Od.double().cpu().numpy())
    layer.close()


@needs_gpu
def test_fp16_range_overflow_is_reported():
    """Rows far outside the fp16 range make the pooled fp16 operand overflow: the
    kernel latches MSGLA_ERR_RANGE (no fault) and the handle stays usable."""
    from scale_gated_linear_b200 import MSGLAError
    inp = gpu_inputs(SMALL, L=16)
    layer = _layer(SMALL, inp)
    X = (inp["X"].float() * 1e6).to(torch.bfloat16).cuda()
    layer(X)
    assert layer.sync_status() == -5
    assert layer.sync_status() == 0  # cleared
    O = layer(inp["X"].cuda())
    layer.check_status()
    assert torch.isfinite(O.float()).all()
    layer.close()


@needs_gpu
def test_gate_range_overflow_is_reported():
    """A gate bias far below zero (log alpha near -200/16 per pooled step) makes
    the decay-scaled queries and keys formed in the projection's epilogue leave
    the fp16 range on both halves of a chunk: the kernel latches MSGLA_ERR_RANGE
    and the handle stays usable."""
    inp = gpu_inputs(SMALL, L=200)
    strong = {k: v for k, v in inp.items()}
    strong["branches"] = [dict(br) for br in inp["branches"]]
    for br in strong["branches"]:
        br["bg"] = torch.full_like(br["bg"], -200.0)
    layer = _layer(SMALL, strong)
    layer(inp["X"].cuda())
    assert layer.sync_status() == -5
    assert layer.sync_status() == 0
    layer.close()


@needs_gpu
def test_forward_profiled_records_every_launch():
    inp = gpu_inputs(SMALL, L=100)
    layer = _layer(SMALL, inp)
    X = inp["X"].cuda()
    ws = layer.alloc_workspace(*X.shape[:2])
    names = layer.launch_names(*X.shape[:2])
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
    n = layer.forward_profiled(X, torch.empty_like(X), ws, ev)
    torch.cuda.synchronize()
    # the coarse output projection runs on the handle's second stream alongside
    # the GLA, after a one-warp wait for the GLA CTAs to start (no plan entries,
    # counted as launches)
    assert n == len(names) + 2
    assert names == ["pool_u", "gate", "proj_gemm", "gla", "out_gemm_fused"]
    assert all(ev[i].elapsed_time(ev[i + 1]) >= 0 for i in range(len(names)))
    layer.close()


@needs_gpu
def test_forward_replays_as_cuda_graph():
    """A captured forward (the coarse output projection on the handle's second
    stream beside the GLA, waiting on the GLA's start and completion counters)
    replays three times with outputs bit-identical to an eager forward, and an
    eager forward after the replays still matches: every launch starts its
    counters from zero and waits for per-launch targets."""
    w = wl.WORKLOADS["msgla_340m"].replace(name="graph", L=300)
    inp = gpu_inputs(w)
    layer = _layer(w, inp)
    X = inp["X"].cuda()
    B, L = X.shape[:2]
    assert "out_gemm_coarse" not in layer.launch_names(B, L)  # overlapped with the GLA
    ws = layer.alloc_workspace(B, L)
    ref = torch.empty_like(X)
    layer.forward(X, out=ref, workspace=ws)
    torch.cuda.synchronize()
    layer.check_status()
    O = torch.empty_like(X)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        layer.forward(X, out=O, workspace=ws, stream=torch.cuda.current_stream())
    for _ in range(3):
        O.zero_()
        graph.replay()
        torch.cuda.synchronize()
        layer.check_status()
        assert torch.equal(O, ref)
    again = layer.forward(X, workspace=ws)
    torch.cuda.synchronize()
    layer.check_status()
    assert torch.equal(again, ref)
    del graph
    layer.close()


_SERIAL_CHILD = """
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
sys.path.insert(0, sys.argv[1] + "/tests")
from helpers import gpu_inputs
from scale_gated_linear_b200 import MSGLA
from scale_gated_linear_b200 import workloads as wl
w = wl.WORKLOADS["tiny"].replace(name="small", B=2, L=200, d=128, d_k=64, d_v=128, chunk=64)
inp = gpu_inputs(w, L=100)
layer = MSGLA.from_workload(w, inp, device=0)
X = inp["X"].cuda()
O = layer.forward(X, workspace=layer.alloc_workspace(*X.shape[:2]))
torch.cuda.synchronize()
layer.check_status()
np.save(sys.argv[2], O.float().cpu().numpy())
print(",".join(layer.launch_names(*X.shape[:2])))
layer.close()
"""


@needs_gpu
def test_serial_switch_runs_one_stream_with_identical_output(tmp_path):
    """MSGLA_SERIAL=1 (read once per process, so in a child process) puts the
    coarse output projection back on the caller's stream; the output is
    bit-identical to the two-stream forward."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = tmp_path / "serial.npy"
    env = dict(os.environ, MSGLA_SERIAL="1")
    r = subprocess.run([sys.executable, "-c", _SERIAL_CHILD, root, str(out)], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    names = r.stdout.strip().splitlines()[-1].split(",")
    assert names == ["pool_u", "gate", "proj_gemm", "gla", "out_gemm_coarse", "out_gemm_fused"]
    inp = gpu_inputs(SMALL, L=100)
    got, layer, _ = run_gpu(SMALL, inp)
    assert layer.launch_names(2, 100) == ["pool_u", "gate", "proj_gemm", "gla", "out_gemm_fused"]
    layer.close()
    np.testing.assert_array_equal(np.load(out), got)


@needs_gpu
def test_forward_profiled_rejects_aliased_output():
    """The profiled forward checks its buffers like msgla_forward_masked: an
    output that overlaps the input or the mask is an invalid argument (no kernel
    is launched), and the handle stays usable."""
    from scale_gated_linear_b200 import MSGLAError
    inp = gpu_inputs(SMALL, L=100)
    layer = _layer(SMALL, inp)
    X = inp["X"].cuda()
    B, L, d = X.shape
    ws = layer.alloc_workspace(B, L)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(layer.launch_names(B, L)) + 1)]
    with pytest.raises(MSGLAError) as e:
        layer.forward_profiled(X, X, ws, ev)  # O is X
    assert e.value.status == -1
    # a mask placed inside the output buffer
    O = torch.empty_like(X)
    M = O.view(torch.uint8).view(-1)[: B * L].view(B, L)
    with pytest.raises(MSGLAError) as e:
        layer.forward_profiled(X, O, ws, ev, mask=M)
    assert e.value.status == -1
    n = layer.forward_profiled(X, O, ws, ev)
    torch.cuda.synchronize()
    layer.check_status()
    assert n >= len(ev) - 1
    layer.close()


# ----------------------------------------------------------------- full sizes
@needs_gpu
def test_340m_layer_full_size_sampled_rows():
    """The measured configuration (B=8, L=2048, d=1024) in the launch the bench
    times; batch rows 0 and 7 are compared with the oracle in full."""
    w = wl.WORKLOADS["msgla_340m"]
    inp = gpu_inputs(w)
    got, layer, _ = run_gpu(w, inp)
    for b in (0, 7):
        assert_parity(got[b:b + 1], oracle_forward(w, inp, batch=slice(b, b + 1)))
    layer.close()


@needs_gpu
def test_gla_340m_full_size_sampled_row():
    w = wl.WORKLOADS["gla_340m"]
    inp = gpu_inputs(w)
    got, layer, _ = run_gpu(w, inp)
    assert_parity(got[3:4], oracle_forward(w, inp, batch=slice(3, 4)))
    layer.close()


@needs_gpu
def test_long_32k_full_sequence():
    """L = 32768 (B = 1) in the launch the bench times (sequence segments, state
    pass and scan): every one of the 32768 positions against the oracle, and the
    last 4096 on their own (they depend on the whole carried state)."""
    w = wl.WORKLOADS["long_32k"]
    inp = gpu_inputs(w)
    got, layer, _ = run_gpu(w, inp)
    assert "gla_state" in layer.launch_names(w.B, w.L)
    ref = oracle_forward(w, inp)
    assert_parity(got, ref)
    assert_parity(got[:, -4096:], ref[:, -4096:])
    layer.close()


@needs_gpu
@pytest.mark.parametrize("name", ["wide_8k", "wide_8k_no_fine"])
def test_wide_8k_full_row(name):
    """The wide scale set (d = 2048, B = 4, L = 8192) and its no-fine-branch
    ablation in the launch the bench times: batch row 0 against the oracle at
    all 8192 positions, and the other rows finite."""
    w = wl.WORKLOADS[name]
    inp = gpu_inputs(w)
    got, layer, _ = run_gpu(w, inp)
    ref = oracle_forward(w, inp, batch=slice(0, 1))
    assert_parity(got[0:1], ref)
    assert_parity(got[0:1, -1024:], ref[:, -1024:])
    assert np.isfinite(got).all()
    layer.close()


@needs_gpu
def test_overlap_plan_falls_back_to_serial_when_gla_fills_the_gpu():
    """The coarse output projection runs beside the GLA kernel only when the GLA
    CTAs (one per SM) leave SMs free; at B = 10 (160 CTAs of the 340M-shaped
    layer) they do not, and the plan runs it on the caller's stream."""
    w = wl.WORKLOADS["msgla_340m"]
    inp = gpu_inputs(w, B=1, L=64)
    layer = _layer(w, inp)
    assert "out_gemm_coarse" not in layer.launch_names(8, 2048)  # 128 GLA CTAs
    assert "out_gemm_coarse" in layer.launch_names(10, 2048)     # 160 GLA CTAs
    layer.close()


# ----------------------------------------------------------------- long sequences
@needs_gpu
def test_segment_plan():
    w = wl.WORKLOADS["msgla_340m"]
    inp = gpu_inputs(w, B=1, L=64)
    layer = _layer(w, inp)
    assert "gla_state" not in layer.launch_names(8, 2048)   # 128 CTAs: one pass
    plan = layer.launch_names(1, 4096)                       # 16 CTAs: segmented
    assert plan[plan.index("gla_state"):plan.index("gla") + 1] == ["gla_state", "gla_scan", "gla"]
    layer.close()


@needs_gpu
def test_segmented_long_sequence_matches_oracle():
    """One 4096-token sequence of the 340M-shaped layer: the GLA kernel cuts each
    branch into segments (state pass, scan, full pass from carried states)."""
    w = wl.WORKLOADS["msgla_340m"]
    inp = gpu_inputs(w, B=1, L=4096)
    got, layer, _ = run_gpu(w, inp)
    assert "gla_state" in layer.launch_names(1, 4096)
    assert_parity(got, oracle_forward(w, inp))
    layer.close()
