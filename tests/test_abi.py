"""The C-ABI library loads and exports every entry point include/q2.h declares
(CPU only: no compute calls), and host-side argument checks reject bad
arguments before any device work."""

import ctypes
import os
import re

import pytest

import qwen2_decode_step_b200 as q2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_entry_points():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"^\s*(?:q2_status|const char\*)\s+(q2_\w+)\s*\(", src, re.M))
    return sorted(names)


def test_header_declares_the_operator_and_model_entry_points():
    names = declared_entry_points()
    for op in ("add", "argmax", "embedding", "linear", "rms_norm", "rope", "self_attention",
               "swiglu", "rearrange"):
        assert f"q2_{op}" in names
    for fn in ("create", "destroy", "load_weight", "prefill", "decode_step", "reset_kv"):
        assert f"q2_model_{fn}" in names


def test_library_exports_every_declared_symbol():
    L = q2.lib()
    missing = [n for n in declared_entry_points() if not hasattr(L, n)]
    assert not missing, missing


def test_binding_covers_every_declared_symbol():
    from qwen2_decode_step_b200 import _SIGS
    bound = set(_SIGS) | {"q2_last_error", "q2_version"}
    assert set(declared_entry_points()) <= bound


def test_version_string():
    assert q2.q2_version().startswith("q2 ")


def _raw(name, *args):
    return getattr(q2.lib(), name)(*args)


def test_host_side_argument_checks_need_no_device():
    # Each of these is rejected before any CUDA call.
    assert _raw("q2_add", None, None, None, 10, 7, None) == 2          # bad dtype
    assert _raw("q2_add", None, None, None, 10, 0, None) == 1          # NULL pointers
    assert _raw("q2_linear", 1, 1, 1, None, 4, 4, 0, 1, None) == 3     # K == 0
    assert _raw("q2_rope", 1, 1, 1, 2, 2, 7, ctypes.c_float(1e4), 1, None) == 3  # odd head dim
    assert _raw("q2_self_attention", 1, 1, 1, 1, 5, 4, 12, 2, 128, ctypes.c_float(1.0), 1, None) == 3
    assert _raw("q2_self_attention", 1, 1, 1, 1, 1, 4, 12, 5, 128, ctypes.c_float(1.0), 1, None) == 3
    assert _raw("q2_self_attention", 1, 1, 1, 1, 1, 4, 12, 2, 96, ctypes.c_float(1.0), 1, None) == 3
    assert _raw("q2_rearrange", 1, 1, 9, None, None, None, 2, None) == 3  # ndim > 8
    assert _raw("q2_argmax", 1, None, 1, 3, 0, 0, None) == 3           # empty rows
    assert b"dtype" in q2.lib().q2_last_error() or q2.lib().q2_last_error() != b""


def test_model_create_rejects_bad_meta_before_touching_a_device():
    meta = q2._Meta(1, 2, 128, 4, 3, 32, 384, 1024, 1e-6, 1e4, 64, 1, 0)  # 4 % 3 != 0
    h = ctypes.c_void_p()
    assert q2.lib().q2_model_create(ctypes.byref(meta), 0, ctypes.byref(h)) == 3
    meta = q2._Meta(1, 2, 128, 4, 2, 48, 384, 1024, 1e-6, 1e4, 64, 1, 0)  # head_dim 48
    assert q2.lib().q2_model_create(ctypes.byref(meta), 0, ctypes.byref(h)) == 3
    meta = q2._Meta(5, 2, 128, 4, 2, 32, 384, 1024, 1e-6, 1e4, 64, 1, 0)  # dtype
    assert q2.lib().q2_model_create(ctypes.byref(meta), 0, ctypes.byref(h)) == 2


def test_model_calls_reject_null_model():
    assert q2.lib().q2_model_reset_kv(None, -1) == 1
    assert q2.lib().q2_model_decode_step(None, None, 1, None, None, None) == 1
    assert q2.lib().q2_model_destroy(None) == 0
