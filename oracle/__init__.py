"""Python face of the CPU oracle (oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg use this module; the library under
``qwen2_decode_step_b200/`` never imports it.  The oracle shares no code with
the CUDA path.

Tensors are torch CPU tensors used as plain containers (float32 or bfloat16);
every computation happens in oracle.c.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Tuple

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_HDR = os.path.join(_HERE, "oracle.h")
_BUILD = os.path.join(_HERE, "_build")
# ORACLE_FP32_ACCUMULATION=1 in the environment selects the fp32-accumulating
# copy (a tolerance-derivation tool, see oracle/drift.py), never the default.
_F32ACC = os.environ.get("ORACLE_FP32_ACCUMULATION") == "1"
_LIB_PATH = os.path.join(_BUILD, "liboracle_f32acc.so" if _F32ACC else "liboracle.so")

F32, BF16 = 0, 1
_CODE = {torch.float32: F32, torch.bfloat16: BF16}
_TORCH = {F32: torch.float32, BF16: torch.bfloat16}
DTYPE_CODE = {"f32": F32, "bf16": BF16}

W_KINDS = ["embed", "lm_head", "final_norm", "in_norm", "q_w", "q_b", "k_w", "k_b", "v_w", "v_b",
           "o_w", "post_norm", "gate_w", "up_w", "down_w"]

_lock = threading.Lock()
_lib = None


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile oracle.c into a shared library with gcc (plain C, no SIMD intrinsics)."""
    os.makedirs(_BUILD, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < max(os.path.getmtime(_SRC), os.path.getmtime(_HDR)))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
               *(["-DORACLE_FP32_ACCUMULATION"] if _F32ACC else []), "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Meta(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("n_layers", ctypes.c_int), ("hidden", ctypes.c_int),
                ("n_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("intermediate", ctypes.c_int), ("vocab", ctypes.c_int), ("eps", ctypes.c_double),
                ("theta", ctypes.c_double), ("max_seq", ctypes.c_int), ("max_batch", ctypes.c_int)]


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            vp, sz, i64p = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p
            sig = {
                "oracle_round": [vp, vp, sz, ctypes.c_int],
                "oracle_add": [vp, vp, vp, sz, ctypes.c_int],
                "oracle_argmax": [i64p, vp, vp, sz, sz, ctypes.c_int],
                "oracle_embedding": [vp, i64p, vp, sz, sz, sz, ctypes.c_int],
                "oracle_linear": [vp, vp, vp, vp, sz, sz, sz, ctypes.c_int, ctypes.c_int],
                "oracle_rms_norm": [vp, vp, vp, sz, sz, ctypes.c_double, ctypes.c_int],
                "oracle_rope": [vp, vp, i64p, sz, sz, sz, ctypes.c_double, ctypes.c_int],
                "oracle_self_attention": [vp, vp, vp, vp, sz, sz, sz, sz, sz, ctypes.c_double,
                                          ctypes.c_int],
                "oracle_swiglu": [vp, vp, vp, sz, ctypes.c_int],
                "oracle_rearrange": [vp, vp, ctypes.c_int, i64p, i64p, i64p, sz],
                "oracle_model_set_weight": [vp, ctypes.c_int, ctypes.c_int, vp, sz],
                "oracle_model_kv": [vp, ctypes.c_int, ctypes.c_int, ctypes.POINTER(vp),
                                    ctypes.POINTER(vp)],
                "oracle_model_set_len": [vp, ctypes.c_int, ctypes.c_int],
                "oracle_model_get_len": [vp, ctypes.c_int],
                "oracle_model_forward": [vp, ctypes.c_int, i64p, ctypes.c_int, vp, vp, i64p],
                "oracle_model_forward_hidden": [vp, ctypes.c_int, vp, ctypes.c_int, vp],
            }
            for name, args in sig.items():
                f = getattr(L, name)
                f.argtypes = args
                f.restype = ctypes.c_int
            L.oracle_bf16_from_double.argtypes = [ctypes.c_double]
            L.oracle_bf16_from_double.restype = ctypes.c_uint16
            L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
            L.oracle_bf16_to_double.restype = ctypes.c_double
            L.oracle_model_create.argtypes = [ctypes.POINTER(_Meta)]
            L.oracle_model_create.restype = vp
            L.oracle_model_destroy.argtypes = [vp]
            L.oracle_model_destroy.restype = None
            _lib = L
    return _lib


def _check(rc: int, what: str, allow=()):
    if rc != 0 and rc not in allow:
        raise OracleError(f"{what} failed with code {rc}")
    return rc


def _c(t: torch.Tensor) -> torch.Tensor:
    assert t.device.type == "cpu"
    return t.contiguous()


def _code(t: torch.Tensor) -> int:
    if t.dtype not in _CODE:
        raise TypeError(f"oracle takes float32 or bfloat16 tensors, got {t.dtype}")
    return _CODE[t.dtype]


# ---------------------------------------------------------------- operators

def round_to(values: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    """Round float64 values to the storage dtype (nearest, ties to even)."""
    v = np.ascontiguousarray(values, dtype=np.float64)
    out = torch.empty(v.shape, dtype=dtype)
    _check(lib().oracle_round(out.data_ptr(), v.ctypes.data, v.size, _CODE[dtype]), "round")
    return out


def add(a: torch.Tensor, b: torch.Tensor) -> torch.Tensor:
    a, b = _c(a), _c(b)
    assert a.shape == b.shape and a.dtype == b.dtype
    c = torch.empty_like(a)
    _check(lib().oracle_add(c.data_ptr(), a.data_ptr(), b.data_ptr(), a.numel(), _code(a)), "add")
    return c


def argmax(x: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor]:
    """Row-wise argmax of a 2-D (or 1-D) tensor: (int64 indices, values)."""
    x = _c(x)
    x2 = x.reshape(1, -1) if x.dim() == 1 else x
    rows, n = x2.shape
    idx = torch.empty(rows, dtype=torch.int64)
    val = torch.empty(rows, dtype=x.dtype)
    _check(lib().oracle_argmax(idx.data_ptr(), val.data_ptr(), x2.data_ptr(), rows, n, _code(x)),
           "argmax")
    return idx, val


def embedding(ids: torch.Tensor, table: torch.Tensor, allow_range_error: bool = False):
    ids, table = _c(ids.to(torch.int64)), _c(table)
    V, d = table.shape
    out = torch.empty((ids.numel(), d), dtype=table.dtype)
    rc = lib().oracle_embedding(out.data_ptr(), ids.data_ptr(), table.data_ptr(), ids.numel(), V, d,
                                _code(table))
    _check(rc, "embedding", allow=(-2,) if allow_range_error else ())
    return (out, rc) if allow_range_error else out


def linear(x: torch.Tensor, w: torch.Tensor, b: Optional[torch.Tensor] = None,
           out_dtype: Optional[torch.dtype] = None) -> torch.Tensor:
    x, w = _c(x), _c(w)
    N, K = w.shape
    x2 = x.reshape(-1, K)
    M = x2.shape[0]
    od = out_dtype or x.dtype
    y = torch.empty((M, N), dtype=od)
    bp = _c(b).data_ptr() if b is not None else None
    _check(lib().oracle_linear(y.data_ptr(), x2.data_ptr(), w.data_ptr(), bp, M, N, K, _code(x),
                               _CODE[od]), "linear")
    return y.reshape(*x.shape[:-1], N)


def rms_norm(x: torch.Tensor, w: torch.Tensor, eps: float) -> torch.Tensor:
    x, w = _c(x), _c(w)
    d = x.shape[-1]
    y = torch.empty_like(x)
    _check(lib().oracle_rms_norm(y.data_ptr(), x.data_ptr(), w.data_ptr(), x.numel() // d, d, eps,
                                 _code(x)), "rms_norm")
    return y


def rope(x: torch.Tensor, pos: torch.Tensor, theta: float) -> torch.Tensor:
    """x [ntok, nhead, hd], pos [ntok] int64."""
    x, pos = _c(x), _c(pos.to(torch.int64))
    ntok, nhead, hd = x.shape
    y = torch.empty_like(x)
    _check(lib().oracle_rope(y.data_ptr(), x.data_ptr(), pos.data_ptr(), ntok, nhead, hd, theta,
                             _code(x)), "rope")
    return y


def self_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                   scale: Optional[float] = None) -> torch.Tensor:
    """q [seqlen, nh, hd]; k, v [total_len, nkv, hd]."""
    q, k, v = _c(q), _c(k), _c(v)
    seqlen, nh, hd = q.shape
    total, nkv, _ = k.shape
    if scale is None:
        scale = 1.0 / float(np.sqrt(hd))
    out = torch.empty_like(q)
    _check(lib().oracle_self_attention(out.data_ptr(), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                       seqlen, total, nh, nkv, hd, scale, _code(q)),
           "self_attention")
    return out


def swiglu(gate: torch.Tensor, up: torch.Tensor) -> torch.Tensor:
    gate, up = _c(gate), _c(up)
    out = torch.empty_like(gate)
    _check(lib().oracle_swiglu(out.data_ptr(), gate.data_ptr(), up.data_ptr(), gate.numel(),
                               _code(gate)), "swiglu")
    return out


def rearrange(out: torch.Tensor, inp: torch.Tensor, shape, out_strides, in_strides) -> torch.Tensor:
    """Strided copy into `out` (modified in place); strides in elements, relative to
    the start of each tensor's storage."""
    nd = len(shape)
    arr = (ctypes.c_int64 * max(nd, 1))
    s, os_, is_ = arr(*shape), arr(*out_strides), arr(*in_strides)
    _check(lib().oracle_rearrange(out.data_ptr(), inp.data_ptr(), nd, s, os_, is_,
                                  out.element_size()), "rearrange")
    return out


# ------------------------------------------------------------------- model

class OracleModel:
    """The whole decoder on the CPU.  Weight tensors are borrowed (kept alive here)."""

    def __init__(self, shape, max_seq: int, max_batch: int = 1):
        self.shape = shape
        self.max_seq, self.max_batch = max_seq, max_batch
        self.dtype = torch.float32 if shape.dtype == "f32" else torch.bfloat16
        meta = _Meta(DTYPE_CODE[shape.dtype], shape.n_layers, shape.hidden, shape.n_heads,
                     shape.n_kv_heads, shape.head_dim, shape.intermediate, shape.vocab, shape.eps,
                     shape.theta, max_seq, max_batch)
        self._h = lib().oracle_model_create(ctypes.byref(meta))
        if not self._h:
            raise OracleError("oracle_model_create failed")
        self._keep = {}

    def __del__(self):
        h = getattr(self, "_h", None)
        if h:
            lib().oracle_model_destroy(h)
            self._h = None

    def set_weight(self, name: str, layer: int, t: torch.Tensor):
        t = _c(t)
        assert t.dtype == self.dtype, (name, t.dtype)
        self._keep[(name, layer)] = t
        _check(lib().oracle_model_set_weight(self._h, W_KINDS.index(name), layer, t.data_ptr(),
                                             t.numel() * t.element_size()), f"set_weight {name}")

    def load(self, weights):
        for (name, layer), t in weights.items():
            if layer >= self.shape.n_layers:
                continue
            self.set_weight(name, layer, t)

    def kv(self, layer: int, seq: int) -> Tuple[torch.Tensor, torch.Tensor]:
        """Views of the cache of (layer, seq): K, V as [max_seq, nkv, hd]."""
        kp, vp = ctypes.c_void_p(), ctypes.c_void_p()
        _check(lib().oracle_model_kv(self._h, layer, seq, ctypes.byref(kp), ctypes.byref(vp)), "kv")
        shp = (self.max_seq, self.shape.n_kv_heads, self.shape.head_dim)
        n = int(np.prod(shp))
        out = []
        for p in (kp, vp):
            if self.dtype == torch.float32:
                a = np.ctypeslib.as_array(ctypes.cast(p, ctypes.POINTER(ctypes.c_float)), (n,))
                out.append(torch.from_numpy(a).view(shp))
            else:
                a = np.ctypeslib.as_array(ctypes.cast(p, ctypes.POINTER(ctypes.c_int16)), (n,))
                out.append(torch.from_numpy(a).view(torch.bfloat16).view(shp))
        return out[0], out[1]

    def set_len(self, seq: int, n: int):
        _check(lib().oracle_model_set_len(self._h, seq, n), "set_len")

    def get_len(self, seq: int) -> int:
        return lib().oracle_model_get_len(self._h, seq)

    def forward(self, seq: int, ids: torch.Tensor, all_logits: bool = False):
        """Run ids (1-D) of sequence seq; returns (next_id, logits_last[V] fp32[, logits_all])."""
        ids = _c(ids.to(torch.int64).reshape(-1))
        T = ids.numel()
        V = self.shape.vocab
        last = torch.empty(V, dtype=torch.float32)
        allg = torch.empty((T, V), dtype=torch.float32) if all_logits else None
        nxt = torch.empty(1, dtype=torch.int64)
        _check(lib().oracle_model_forward(self._h, seq, ids.data_ptr(), T, last.data_ptr(),
                                          allg.data_ptr() if allg is not None else None,
                                          nxt.data_ptr()), "model_forward")
        if all_logits:
            return int(nxt[0]), last, allg
        return int(nxt[0]), last

    def forward_hidden(self, seq: int, x: torch.Tensor) -> torch.Tensor:
        x = _c(x)
        assert x.dtype == self.dtype
        T = x.shape[0]
        out = torch.empty_like(x)
        _check(lib().oracle_model_forward_hidden(self._h, seq, x.data_ptr(), T, out.data_ptr()),
               "forward_hidden")
        return out

    def generate(self, seq: int, prompt: torch.Tensor, n_decode: int, teacher=None):
        """Prefill `prompt`, then n_decode greedy steps.  With `teacher` (a list of
        ids), step i is fed teacher[i] instead of the oracle's own choice.
        Returns (tokens fed/chosen, list of fp32 logits per step: prefill last + each decode)."""
        nxt, lg = self.forward(seq, prompt)
        logits = [lg]
        chosen = [nxt]
        for i in range(n_decode):
            feed = chosen[-1] if teacher is None else int(teacher[i])
            nxt, lg = self.forward(seq, torch.tensor([feed], dtype=torch.int64))
            logits.append(lg)
            chosen.append(nxt)
        return chosen, logits
