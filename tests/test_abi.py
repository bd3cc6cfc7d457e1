"""C ABI checks that need no GPU: the library loads, exports every function the
header declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

from scale_gated_linear_b200 import MSGLA, _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "msgla.h")


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:int|void|const char\*)\s+(msgla_\w+)\s*\(", text, re.M)))


def test_header_declares_the_abi():
    names = declared_functions()
    for must in ("msgla_create", "msgla_forward", "msgla_destroy", "msgla_workspace_size"):
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_covers_every_declared_symbol():
    assert set(declared_functions()) == set(_lib._SIGNATURES)


def test_status_strings():
    lib = _lib.load()
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert lib.msgla_status_string(code).decode() != "unknown status"
    assert lib.msgla_status_string(42).decode() == "unknown status"


def _cfg(**kw):
    c = _lib.Config()
    c.d, c.n_scales = 64, 3
    for j, (s, h) in enumerate(zip((1, 2, 4), (2, 1, 1))):
        c.scales[j], c.heads[j] = s, h
    c.d_k, c.d_v, c.gate_rank, c.chunk, c.gate_normalizer, c.qk_scale = 16, 16, 16, 0, 16.0, 1.0
    for k, v in kw.items():
        if k in ("scales", "heads"):
            for j, x in enumerate(v):
                getattr(c, k)[j] = x
        else:
            setattr(c, k, v)
    return c


@pytest.mark.parametrize("kw,code", [
    (dict(d=100), -2), (dict(d=0), -2), (dict(n_scales=0), -1), (dict(n_scales=9), -1),
    (dict(scales=(1, 4, 2)), -1), (dict(scales=(0, 2, 4)), -1), (dict(heads=(2, 0, 1)), -1),
    (dict(d_k=300), -2), (dict(d_v=0), -2), (dict(gate_rank=33), -2), (dict(chunk=16), -2), (dict(chunk=64), -2),
    (dict(gate_normalizer=0.0), -1), (dict(gate_normalizer=float("nan")), -1),
    (dict(qk_scale=float("inf")), -1), (dict(scales=(1, 7, 11)), -2),
    (dict(head_norm=2, head_norm_eps=1e-5), -1), (dict(head_norm=1, head_norm_eps=0.0), -1),
    (dict(head_norm=1, head_norm_eps=float("nan")), -1),
])
def test_create_rejects_bad_config(kw, code):
    lib = _lib.load()
    h = ctypes.c_void_p(123)
    w = _lib.Weights()
    st = lib.msgla_create(ctypes.byref(h), ctypes.byref(_cfg(**kw)), ctypes.byref(w), 0)
    assert st == code, lib.msgla_last_error()
    assert h.value is None
    assert lib.msgla_last_error().decode()


def test_null_arguments():
    lib = _lib.load()
    n = ctypes.c_size_t()
    assert lib.msgla_create(None, ctypes.byref(_cfg()), None, 0) == -1
    assert lib.msgla_workspace_size(None, 1, 1, ctypes.byref(n)) == -1
    assert lib.msgla_forward(None, None, 1, 1, None, None, 0, None) == -1
    assert lib.msgla_forward_masked(None, None, None, 1, 1, None, None, 0, None) == -1
    assert lib.msgla_cache_size(None, 1, ctypes.byref(n)) == -1
    assert lib.msgla_cache_reset(None, None, 1, None) == -1
    assert lib.msgla_step_workspace_size(None, 1, ctypes.byref(n)) == -1
    assert lib.msgla_step(None, None, None, 1, 0, None, None, 0, None) == -1
    assert lib.msgla_forward_host(None, None, 1, 1, None, None, 0, None) == -1
    assert lib.msgla_sync_status(None) == -1
    lib.msgla_destroy(None)


def test_product_does_not_use_the_oracle():
    pkg = os.path.join(ROOT, "scale_gated_linear_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle", text, re.M), f
                assert "msgla_oracle" not in text, f
