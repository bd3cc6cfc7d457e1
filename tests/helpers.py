"""Shared helpers of the test-suite: running the CUDA path and the oracle on the
same seeded inputs, and the error metrics of the parity bar."""
from __future__ import annotations

import numpy as np

from scale_gated_linear_b200 import workloads as wl

# parity bar for the layer output (bf16 in/out, fp32 accumulation)
MAX_REL = 1e-2    # max|gpu - oracle| / max|oracle|
MEAN_REL = 2e-3   # mean|gpu - oracle| / mean|oracle|


def rel_errors(got: np.ndarray, ref: np.ndarray):
    d = np.abs(got.astype(np.float64) - ref)
    return float(d.max() / np.abs(ref).max()), float(d.mean() / np.abs(ref).mean())


def gpu_inputs(w: wl.Workload, B=None, L=None, seed=None):
    """Inputs as the CUDA path stores them (bf16 X and weights)."""
    inp = wl.make_inputs(w, B=B, L=L, seed=seed)
    if w.dtype != "bf16":
        inp = wl.round_inputs_to_bf16(inp)
    return inp


def oracle_forward(w: wl.Workload, inp: dict, rows=None, intermediates=False, batch=None, mask=None):
    import oracle
    f = wl.to_float64(inp)
    X = f["X"] if batch is None else f["X"][batch]
    if rows is not None:
        X = X[:, :rows]
    if mask is not None:
        mask = np.asarray(mask, dtype=np.float64)
    return oracle.layer_forward(X, f, w.scales, w.heads, w.d_k, w.d_v,
                                gate_normalizer=w.gate_normalizer, intermediates=intermediates, mask=mask,
                                head_norm_eps=w.norm_eps if w.head_norm else None)
