"""MS-GLA (multi-scale gated linear attention) layer forward pass for B200.

The computation runs in libmsgla.so (hand-written sm_100a CUDA behind the C ABI
of include/msgla.h). This package only marshals torch tensors into that ABI;
PyTorch provides device memory and streams.

    from scale_gated_linear_b200 import MSGLA
    layer = MSGLA(d=1024, scales=(1, 2, 4), heads=(2, 1, 1), d_k=256, d_v=512,
                  weights=weights_dict, device=0)
    O = layer(X)          # X: cuda bf16 [B, L, d] -> O: cuda bf16 [B, L, d]
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence

from . import _lib
from ._lib import (MSGLAError, WS_FUSION, WS_GAMMA, WS_KS, WS_MID, WS_O, WS_POOLED, WS_QS, WS_U, WS_V,
                   WS_Y)

__all__ = ["MSGLA", "MSGLAError", "load_library"]


def load_library():
    return _lib.load()


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


class MSGLA:
    """One MS-GLA layer on one CUDA device (owns a C handle)."""

    def __init__(self, d: int, scales: Sequence[int], heads: Sequence[int], d_k: int, d_v: int,
                 weights: dict, gate_rank: int = 16, gate_normalizer: float = 16.0,
                 qk_scale: float = 1.0, chunk: int = 0, device: int = 0,
                 head_norm_eps: Optional[float] = None):
        import torch

        lib = _lib.load()
        self.d, self.scales, self.heads = d, tuple(scales), tuple(heads)
        self.d_k, self.d_v, self.device = d_k, d_v, device
        cfg = _lib.Config()
        cfg.d, cfg.n_scales = d, len(self.scales)
        for j, (s, h) in enumerate(zip(self.scales, self.heads)):
            cfg.scales[j], cfg.heads[j] = s, h
        cfg.d_k, cfg.d_v, cfg.gate_rank, cfg.chunk = d_k, d_v, gate_rank, chunk
        cfg.gate_normalizer, cfg.qk_scale = gate_normalizer, qk_scale
        if head_norm_eps is not None:  # per-head RMS norm of the GLA output (off by default)
            cfg.head_norm, cfg.head_norm_eps = 1, head_norm_eps
        dev = torch.device("cuda", device)

        def on_dev(t, dtype):
            return None if t is None else t.to(device=dev, dtype=dtype).contiguous()

        keep = []
        w = _lib.Weights()
        for j, br in enumerate(weights["branches"]):
            ts = {k: on_dev(br[k], torch.bfloat16) for k in ("Wq", "Wk", "Wv", "Wg1", "Wo")}
            ts["Wg2"] = on_dev(br["Wg2"], torch.float32)
            ts["bg"] = on_dev(br.get("bg"), torch.float32)
            ts["norm_w"] = on_dev(br.get("norm_w"), torch.float32)
            keep.append(ts)
            for k, t in ts.items():
                getattr(w, k)[j] = _ptr(t)
        wf = on_dev(weights["Wfuse"], torch.bfloat16)
        bf = on_dev(weights.get("bfuse"), torch.float32)
        keep += [wf, bf]
        w.Wfuse, w.bfuse = _ptr(wf), _ptr(bf)
        handle = ctypes.c_void_p()
        _lib.check(lib.msgla_create(ctypes.byref(handle), ctypes.byref(cfg), ctypes.byref(w), device))
        self._h = handle
        self._lib = lib
        self._ws = None

    # ------------------------------------------------------------- sizes
    def workspace_size(self, B: int, L: int) -> int:
        n = ctypes.c_size_t()
        _lib.check(self._lib.msgla_workspace_size(self._h, B, L, ctypes.byref(n)))
        return n.value

    def workspace_size_host(self, B: int, L: int) -> int:
        n = ctypes.c_size_t()
        _lib.check(self._lib.msgla_workspace_size_host(self._h, B, L, ctypes.byref(n)))
        return n.value

    def alloc_workspace(self, B: int, L: int, host_staging: bool = False):
        import torch
        n = self.workspace_size_host(B, L) if host_staging else self.workspace_size(B, L)
        return torch.empty(max(n, 1), dtype=torch.uint8, device=torch.device("cuda", self.device))

    # ------------------------------------------------------------- forward
    def forward(self, X, out=None, workspace=None, stream=None, mask=None):
        """O = MS-GLA(X) for cuda bf16 X [B, L, d]; asynchronous on `stream`
        (default: torch's current stream). ``mask``: optional cuda [B, L] tensor
        of valid tokens (bool or uint8, nonzero = valid) for the pooling of
        Eq. (8)."""
        import torch
        B, L, d = X.shape
        assert d == self.d and X.dtype == torch.bfloat16 and X.is_cuda and X.is_contiguous()
        if mask is not None:
            assert mask.shape == (B, L) and mask.is_cuda and mask.is_contiguous()
            assert mask.dtype in (torch.bool, torch.uint8)
        if out is None:
            out = torch.empty_like(X)
        if workspace is None:
            need = self.workspace_size(B, L)
            if self._ws is None or self._ws.numel() < need:
                self._ws = self.alloc_workspace(B, L)
            workspace = self._ws
        if stream is None:
            stream = torch.cuda.current_stream(X.device)
        if mask is None:
            _lib.check(self._lib.msgla_forward(self._h, X.data_ptr(), B, L, out.data_ptr(), workspace.data_ptr(),
                                               workspace.numel(), ctypes.c_void_p(stream.cuda_stream)))
        else:
            _lib.check(self._lib.msgla_forward_masked(self._h, X.data_ptr(), mask.data_ptr(), B, L, out.data_ptr(),
                                                      workspace.data_ptr(), workspace.numel(),
                                                      ctypes.c_void_p(stream.cuda_stream)))
        return out

    __call__ = forward

    # ------------------------------------------------------------- decode
    def cache_size(self, B: int) -> int:
        n = ctypes.c_size_t()
        _lib.check(self._lib.msgla_cache_size(self._h, B, ctypes.byref(n)))
        return n.value

    def new_cache(self, B: int, stream=None):
        """Device buffer holding the per-branch decode cache of B sequences,
        emptied (the state before the first token)."""
        import torch
        cache = torch.empty(max(self.cache_size(B), 1), dtype=torch.uint8, device=torch.device("cuda", self.device))
        self.reset_cache(cache, B, stream)
        return cache

    def reset_cache(self, cache, B: int, stream=None):
        import torch
        if stream is None:
            stream = torch.cuda.current_stream(cache.device)
        _lib.check(self._lib.msgla_cache_reset(self._h, cache.data_ptr(), B, ctypes.c_void_p(stream.cuda_stream)))

    def step_workspace_size(self, B: int) -> int:
        n = ctypes.c_size_t()
        _lib.check(self._lib.msgla_step_workspace_size(self._h, B, ctypes.byref(n)))
        return n.value

    def step(self, x, t: int, cache, out=None, workspace=None, stream=None):
        """Layer output at position t for token x (cuda bf16 [B, d]) of every
        sequence, updating ``cache`` (from new_cache); tokens must come in order
        t = 0, 1, 2, ... after the cache was emptied."""
        import torch
        B, d = x.shape
        assert d == self.d and x.dtype == torch.bfloat16 and x.is_cuda and x.is_contiguous()
        if out is None:
            out = torch.empty_like(x)
        if workspace is None:
            need = self.step_workspace_size(B)
            if getattr(self, "_step_ws", None) is None or self._step_ws.numel() < need:
                self._step_ws = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
            workspace = self._step_ws
        if stream is None:
            stream = torch.cuda.current_stream(x.device)
        _lib.check(self._lib.msgla_step(self._h, cache.data_ptr(), x.data_ptr(), B, t, out.data_ptr(),
                                        workspace.data_ptr(), workspace.numel(), ctypes.c_void_p(stream.cuda_stream)))
        return out

    def launch_names(self, B: int, L: int):
        """Kernel names of one forward of a [B, L, d] input, in launch order."""
        buf = ctypes.create_string_buffer(512)
        _lib.check(self._lib.msgla_launch_plan(self._h, B, L, buf, len(buf)))
        return buf.value.decode().split(",") if buf.value else []

    def forward_profiled(self, X, out, workspace, events, stream=None, mask=None):
        """forward() recording events[0] before the first kernel and events[i+1]
        after kernel i (torch.cuda.Event objects with timing enabled; None skips a
        record -- an event between two kernels keeps the second from starting
        early). Returns the number of kernels launched. ``mask`` as for forward()."""
        import torch
        B, L, d = X.shape
        if stream is None:
            stream = torch.cuda.current_stream(X.device)
        for e in events:  # torch creates the underlying cudaEvent_t on first record
            if e is not None and not e.cuda_event:
                e.record(stream)
        arr = (ctypes.c_void_p * len(events))(*[None if e is None else e.cuda_event for e in events])
        n = ctypes.c_int()
        if mask is not None:
            assert mask.shape == (B, L) and mask.is_cuda and mask.is_contiguous()
            assert mask.dtype in (torch.bool, torch.uint8)
        _lib.check(self._lib.msgla_forward_profiled(self._h, X.data_ptr(), None if mask is None else mask.data_ptr(),
                                                    B, L, out.data_ptr(),
                                                    workspace.data_ptr(), workspace.numel(),
                                                    ctypes.c_void_p(stream.cuda_stream), arr, len(events),
                                                    ctypes.byref(n)))
        return n.value

    def forward_host(self, X_host, O_host, workspace, stream=None):
        """Host-buffer forward: X_host, O_host are CPU bf16 [B, L, d] (pinned for
        speed); copies in, runs, copies out and synchronises."""
        import torch
        B, L, d = X_host.shape
        s = stream if stream is not None else torch.cuda.current_stream(torch.device("cuda", self.device))
        _lib.check(self._lib.msgla_forward_host(self._h, X_host.data_ptr(), B, L, O_host.data_ptr(),
                                                workspace.data_ptr(), workspace.numel(),
                                                ctypes.c_void_p(s.cuda_stream)))
        return O_host

    def sync_status(self) -> int:
        """Synchronise and return the latched device-side status (0 = ok)."""
        return self._lib.msgla_sync_status(self._h)

    def check_status(self) -> None:
        _lib.check(self.sync_status())

    def workspace_tensor(self, workspace, B: int, L: int, scale_index: int, which: int):
        """View of an intermediate tensor inside `workspace` (after a forward)."""
        import torch
        off = ctypes.c_size_t()
        dims = (ctypes.c_int * 3)()
        _lib.check(self._lib.msgla_workspace_tensor(self._h, B, L, scale_index, which, ctypes.byref(off), dims))
        dtype = torch.float32 if which in (WS_FUSION, WS_U, WS_GAMMA, WS_MID) else torch.float16
        esz = 4 if dtype == torch.float32 else 2
        n = dims[0] * dims[1] * dims[2]
        raw = workspace[off.value: off.value + n * esz]
        return raw.view(dtype).view(dims[0], dims[1], dims[2])

    def close(self) -> None:
        if getattr(self, "_h", None):
            self._lib.msgla_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @classmethod
    def from_workload(cls, w, weights: dict, device: int = 0, **kw) -> "MSGLA":
        if getattr(w, "head_norm", False):
            kw.setdefault("head_norm_eps", w.norm_eps)
        return cls(d=w.d, scales=w.scales, heads=w.heads, d_k=w.d_k, d_v=w.d_v, weights=weights,
                   gate_rank=w.gate_rank, gate_normalizer=w.gate_normalizer, device=device, **kw)
