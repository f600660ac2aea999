"""B200 (sm_100a) Qwen2-style decoder: Python binding of libq2.so.

Argument marshalling only: every function below hands device pointers of
torch tensors (torch supplies device memory and streams) to the C ABI
declared in include/q2.h, whose names it keeps.  All computation happens in
the library's CUDA kernels; there is no fallback of any kind -- importing
this module fails loudly when libq2.so is missing.

Streams: every call is enqueued on torch's current CUDA stream.
"""

from __future__ import annotations

import ctypes
import os
from typing import Dict, Iterable, Optional, Sequence, Tuple

import torch

__all__ = [
    "Q2Error", "lib", "q2_version", "q2_check_device_error", "q2_add", "q2_argmax",
    "q2_argmax_noalloc", "q2_embedding", "q2_test_raise_device_error", "q2_test_attn_plan",
    "q2_test_gemm_tile",
    "q2_linear", "q2_test_tc_gemm", "q2_rms_norm", "q2_add_rms_norm", "q2_rope", "q2_self_attention", "q2_swiglu",
    "q2_rearrange", "Model", "W_KIND", "STATUS", "KCLASS",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libq2.so")

STATUS = {0: "Q2_OK", 1: "Q2_ERR_INVALID_ARG", 2: "Q2_ERR_DTYPE", 3: "Q2_ERR_SHAPE",
          4: "Q2_ERR_CAPACITY", 5: "Q2_ERR_INDEX", 6: "Q2_ERR_CUDA", 7: "Q2_ERR_OOM",
          8: "Q2_ERR_STATE", 9: "Q2_ERR_TIMEOUT"}
F32, BF16 = 0, 1
_DT = {torch.float32: F32, torch.bfloat16: BF16}
W_KIND = {"embed": 0, "lm_head": 1, "final_norm": 2, "in_norm": 3, "q_w": 4, "q_b": 5, "k_w": 6,
          "k_b": 7, "v_w": 8, "v_b": 9, "o_w": 10, "post_norm": 11, "gate_w": 12, "up_w": 13,
          "down_w": 14}


class Q2Error(RuntimeError):
    def __init__(self, code: int, fn: str, msg: str):
        self.code = code
        self.status = STATUS.get(code, str(code))
        super().__init__(f"{fn}: {self.status}: {msg}")


class _Meta(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("n_layers", ctypes.c_int), ("hidden", ctypes.c_int),
                ("n_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("intermediate", ctypes.c_int), ("vocab", ctypes.c_int), ("eps", ctypes.c_float),
                ("theta", ctypes.c_float), ("max_seq", ctypes.c_int), ("max_batch", ctypes.c_int),
                ("max_prefill_tokens", ctypes.c_int)]


_VP, _SZ, _I, _F = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
_SIGS = {
    "q2_check_device_error": [_VP],
    "q2_add": [_VP, _VP, _VP, _SZ, _I, _VP],
    "q2_argmax": [_VP, _VP, _VP, _SZ, _SZ, _I, _VP],
    "q2_argmax_noalloc": [_VP, _VP, _VP, _SZ, _SZ, _I, _VP],
    "q2_embedding": [_VP, _VP, _VP, _SZ, _SZ, _SZ, _I, _VP],
    "q2_linear": [_VP, _VP, _VP, _VP, _SZ, _SZ, _SZ, _I, _VP],
    "q2_test_tc_gemm": [_VP, _SZ, _I, _I, _VP, _VP, _VP, _SZ, _SZ, _SZ, _I, _VP],
    "q2_rms_norm": [_VP, _VP, _VP, _SZ, _SZ, _F, _I, _VP],
    "q2_add_rms_norm": [_VP, _VP, _VP, _VP, _SZ, _SZ, _F, _I, _VP],
    "q2_rope": [_VP, _VP, _VP, _SZ, _SZ, _SZ, _F, _I, _VP],
    "q2_self_attention": [_VP, _VP, _VP, _VP, _SZ, _SZ, _SZ, _SZ, _SZ, _F, _I, _VP],
    "q2_swiglu": [_VP, _VP, _VP, _SZ, _I, _VP],
    "q2_rearrange": [_VP, _VP, _I, _VP, _VP, _VP, _SZ, _VP],
    "q2_model_create": [ctypes.POINTER(_Meta), _I, ctypes.POINTER(_VP)],
    "q2_model_destroy": [_VP],
    "q2_model_load_weight": [_VP, _I, _I, _VP, _SZ, _VP],
    "q2_model_prefill": [_VP, _VP, _I, _VP, _VP, _VP, _VP],
    "q2_model_decode_step": [_VP, _VP, _I, _VP, _VP, _VP],
    "q2_model_decode_step_host": [_VP, _VP, _I, _VP, _VP],
    "q2_model_forward_hidden": [_VP, _VP, _I, _VP, _VP],
    "q2_model_reset_kv": [_VP, _I],
    "q2_model_set_seq_len": [_VP, _I, _I],
    "q2_model_get_seq_len": [_VP, _I, ctypes.POINTER(_I)],
    "q2_model_kv_cache": [_VP, _I, _I, ctypes.POINTER(_VP), ctypes.POINTER(_VP)],
    "q2_model_check_error": [_VP, _VP],
    "q2_model_set_graphs": [_VP, _I],
    "q2_model_time_kernels": [_VP, _VP, _I, _I, _VP, _VP, ctypes.POINTER(_I), _VP],
    "q2_model_prefill_hidden": [_VP, _I, _VP, _I, _VP, _VP],
    "q2_model_head": [_VP, _VP, _I, _VP, _VP, _VP],
    "q2_model_set_decode_path": [_VP, _I],
    "q2_test_raise_device_error": [_I, _VP],
    "q2_test_attn_plan": [_SZ, _SZ, _SZ, _I, _VP],
    "q2_test_gemm_tile": [_SZ, _SZ, _I, _VP],
    "q2_test_model_raise_error": [_VP, _I, _VP],
    "q2_test_set_wait_fault": [_VP, _I, ctypes.c_ulonglong],
    "q2_test_trace_stream_step": [_VP, _VP, _VP, _SZ, ctypes.POINTER(_I), _VP],
}

KCLASS = ["embed", "norm", "qkv", "rope_kv", "attn", "o", "gate_up", "swiglu", "down", "lm_head",
          "argmax", "other", "step"]
PATH = {"auto": 0, "persistent": 1, "kernels": 2, "generic": 3, "stream": 4}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libq2.so.  Raises if it has not been built: there is no fallback."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libq2.so not found at {LIB_PATH}; build it with "
                              "`python -m qwen2_decode_step_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        L.q2_last_error.argtypes = []
        L.q2_last_error.restype = ctypes.c_char_p
        L.q2_version.argtypes = []
        L.q2_version.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _call(name: str, *args) -> int:
    rc = getattr(lib(), name)(*args)
    if rc != 0:
        raise Q2Error(rc, name, lib().q2_last_error().decode())
    return rc


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    return t.data_ptr()


def _dense(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("expected contiguous tensors")


def _dtype(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise TypeError(f"dtype must be float32 or bfloat16, got {t.dtype}")
    return _DT[t.dtype]


# ------------------------------------------------------------------ operators

def q2_version() -> str:
    return lib().q2_version().decode()


def q2_check_device_error() -> None:
    _call("q2_check_device_error", _stream())


def q2_test_raise_device_error(bits: int) -> None:
    """Test hook: OR `bits` into the operators' device error word."""
    _call("q2_test_raise_device_error", bits, _stream())


def q2_test_attn_plan(rows: int, pos0: int, nh: int, sms: int) -> dict:
    """Test hook: the tcgen05 prefill attention's work plan on a machine of
    `sms` SMs (host only, no device)."""
    out = (ctypes.c_int * 6)()
    _call("q2_test_attn_plan", rows, pos0, nh, sms, ctypes.cast(out, _VP))
    keys = ("n_whole", "ts", "ctas", "items", "slot_capacity", "counter_capacity")
    return dict(zip(keys, list(out)))


def q2_test_gemm_tile(M: int, N: int, sms: int) -> int:
    """Test hook: the token tile width the tcgen05 GEMM takes for M x N (host only)."""
    bn = ctypes.c_int(0)
    _call("q2_test_gemm_tile", M, N, sms, ctypes.cast(ctypes.pointer(bn), _VP))
    return bn.value


def q2_add(c, a, b):
    _dense(c, a, b)
    _call("q2_add", _p(c), _p(a), _p(b), a.numel(), _dtype(a), _stream())
    return c


def q2_argmax(max_idx, max_val, vals):
    """vals [rows, n] (or [n]); max_idx int64 [rows]; max_val [rows] or None."""
    _dense(vals, max_idx, max_val)
    rows = 1 if vals.dim() == 1 else vals.shape[0]
    n = vals.shape[-1]
    _call("q2_argmax", _p(max_idx), _p(max_val), _p(vals), rows, n, _dtype(vals), _stream())
    return max_idx, max_val


def q2_argmax_noalloc(max_idx, max_val, vals):
    """q2_argmax with no device allocation (fixed library-owned partials array;
    rows <= 16384).  Same arguments as q2_argmax."""
    _dense(vals, max_idx, max_val)
    rows = 1 if vals.dim() == 1 else vals.shape[0]
    n = vals.shape[-1]
    _call("q2_argmax_noalloc", _p(max_idx), _p(max_val), _p(vals), rows, n, _dtype(vals), _stream())
    return max_idx, max_val


def q2_embedding(out, ids, weight):
    _dense(out, ids, weight)
    V, d = weight.shape
    _call("q2_embedding", _p(out), _p(ids), _p(weight), ids.numel(), V, d, _dtype(weight), _stream())
    return out


def q2_linear(out, inp, weight, bias=None):
    _dense(out, inp, weight, bias)
    N, K = weight.shape
    M = inp.numel() // K
    _call("q2_linear", _p(out), _p(inp), _p(weight), _p(bias), M, N, K, _dtype(inp), _stream())
    return out


TC_EPI = {"plain": 0, "swiglu": 1, "resid": 2}


def q2_test_tc_gemm(out, x, weight, bias=None, epilogue="plain", split=False):
    """Test hook: the tcgen05 GEMM with one of its epilogues (see q2.h)."""
    _dense(out, x, weight, bias)
    N, K = weight.shape
    M = x.numel() // K
    _call("q2_test_tc_gemm", _p(out), out.shape[-1], _dtype(out), TC_EPI[epilogue], _p(x),
          _p(weight), _p(bias), M, N, K, 1 if split else 0, _stream())
    return out


def q2_rms_norm(out, inp, weight, eps):
    _dense(out, inp, weight)
    d = inp.shape[-1]
    _call("q2_rms_norm", _p(out), _p(inp), _p(weight), inp.numel() // d, d, eps, _dtype(inp),
          _stream())
    return out


def q2_add_rms_norm(residual, y, h, weight, eps):
    _dense(residual, y, h, weight)
    d = residual.shape[-1]
    _call("q2_add_rms_norm", _p(residual), _p(y), _p(h), _p(weight), residual.numel() // d, d, eps,
          _dtype(residual), _stream())
    return residual, h


def q2_rope(out, inp, pos, theta):
    """inp [ntok, nhead, hd]; pos int64 [ntok]."""
    _dense(out, inp, pos)
    ntok, nhead, hd = inp.shape
    _call("q2_rope", _p(out), _p(inp), _p(pos), ntok, nhead, hd, theta, _dtype(inp), _stream())
    return out


def q2_self_attention(out, q, k, v, scale):
    """q [seqlen, nh, hd]; k, v [total_len, nkv, hd]."""
    _dense(out, q, k, v)
    seqlen, nh, hd = q.shape
    total, nkv, _ = k.shape
    _call("q2_self_attention", _p(out), _p(q), _p(k), _p(v), seqlen, total, nh, nkv, hd, scale,
          _dtype(q), _stream())
    return out


def q2_swiglu(out, gate, up):
    _dense(out, gate, up)
    _call("q2_swiglu", _p(out), _p(gate), _p(up), gate.numel(), _dtype(gate), _stream())
    return out


def q2_rearrange(out, inp, shape: Sequence[int], out_strides: Sequence[int],
                 in_strides: Sequence[int]):
    """Strided copy between the storages starting at out.data_ptr() / inp.data_ptr()."""
    nd = len(shape)
    arr = ctypes.c_int64 * max(nd, 1)
    _call("q2_rearrange", _p(out), _p(inp), nd, arr(*shape), arr(*out_strides), arr(*in_strides),
          out.element_size(), _stream())
    return out


# ---------------------------------------------------------------------- model

class _DevArray:
    """A raw device buffer exposed through __cuda_array_interface__."""

    def __init__(self, ptr: int, shape: Tuple[int, ...], typestr: str):
        self.__cuda_array_interface__ = {"shape": shape, "typestr": typestr, "data": (ptr, False),
                                         "version": 3, "strides": None}


class Model:
    """A Qwen2-style decoder on one GPU (q2_model_*)."""

    def __init__(self, shape, max_seq: int, max_batch: int = 1, max_prefill_tokens: int = 0,
                 device: Optional[int] = None):
        self.shape = shape
        self.max_seq, self.max_batch = max_seq, max_batch
        self.device = torch.cuda.current_device() if device is None else device
        self.dtype = torch.float32 if shape.dtype == "f32" else torch.bfloat16
        meta = _Meta(F32 if shape.dtype == "f32" else BF16, shape.n_layers, shape.hidden,
                     shape.n_heads, shape.n_kv_heads, shape.head_dim, shape.intermediate,
                     shape.vocab, shape.eps, shape.theta, max_seq, max_batch, max_prefill_tokens)
        h = ctypes.c_void_p()
        _call("q2_model_create", ctypes.byref(meta), self.device, ctypes.byref(h))
        self._h = h

    def close(self):
        if getattr(self, "_h", None):
            torch.cuda.synchronize(self.device)
            _call("q2_model_destroy", self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def load_weight(self, name: str, layer: int, t: torch.Tensor):
        _dense(t)
        _call("q2_model_load_weight", self._h, W_KIND[name], layer, _p(t),
              t.numel() * t.element_size(), _stream())

    def load(self, weights: Dict[Tuple[str, int], torch.Tensor]):
        """Copies every (name, layer) tensor (moved to this GPU first if needed)."""
        for (name, layer), t in weights.items():
            if layer >= self.shape.n_layers:
                continue
            if not t.is_cuda:
                t = t.to(f"cuda:{self.device}")
            self.load_weight(name, layer, t)
        torch.cuda.current_stream().synchronize()

    def prefill(self, ids: torch.Tensor, lens: Iterable[int], want_logits: bool = False):
        lens = [int(x) for x in lens]
        B = len(lens)
        arr = (ctypes.c_int32 * B)(*lens)
        nxt = torch.empty(B, dtype=torch.int64, device=ids.device)
        lg = torch.empty((B, self.shape.vocab), dtype=torch.float32, device=ids.device) \
            if want_logits else None
        _dense(ids)
        _call("q2_model_prefill", self._h, _p(ids), B, arr, _p(nxt), _p(lg), _stream())
        return (nxt, lg) if want_logits else nxt

    def decode_step(self, ids: torch.Tensor, want_logits: bool = False, out: Optional[torch.Tensor] = None):
        _dense(ids)
        B = ids.numel()
        nxt = out if out is not None else torch.empty(B, dtype=torch.int64, device=ids.device)
        lg = torch.empty((B, self.shape.vocab), dtype=torch.float32, device=ids.device) \
            if want_logits else None
        _call("q2_model_decode_step", self._h, _p(ids), B, _p(nxt), _p(lg), _stream())
        return (nxt, lg) if want_logits else nxt

    def decode_step_host(self, ids_host: torch.Tensor, next_host: torch.Tensor):
        """Host (ideally pinned) int64 ids -> host int64 next ids; synchronises."""
        assert ids_host.device.type == "cpu" and next_host.device.type == "cpu"
        _call("q2_model_decode_step_host", self._h, ids_host.data_ptr(), ids_host.numel(),
              next_host.data_ptr(), _stream())
        return next_host

    def forward_hidden(self, x: torch.Tensor) -> torch.Tensor:
        _dense(x)
        out = torch.empty_like(x)
        _call("q2_model_forward_hidden", self._h, _p(x), x.shape[0], _p(out), _stream())
        return out

    def prefill_hidden(self, seq: int, x: torch.Tensor) -> torch.Tensor:
        """Decoder layers over x [T, H] at the next T positions of `seq`."""
        _dense(x)
        out = torch.empty_like(x)
        _call("q2_model_prefill_hidden", self._h, seq, _p(x), x.shape[0], _p(out), _stream())
        return out

    def head(self, x: torch.Tensor):
        """Final RMSNorm + lm_head + argmax on hidden states x [rows, H]: (next, fp32 logits)."""
        _dense(x)
        rows = x.shape[0]
        nxt = torch.empty(rows, dtype=torch.int64, device=x.device)
        lg = torch.empty((rows, self.shape.vocab), dtype=torch.float32, device=x.device)
        _call("q2_model_head", self._h, _p(x), rows, _p(nxt), _p(lg), _stream())
        return nxt, lg

    def reset_kv(self, seq: int = -1):
        _call("q2_model_reset_kv", self._h, seq)

    def set_seq_len(self, seq: int, n: int):
        _call("q2_model_set_seq_len", self._h, seq, n)

    def get_seq_len(self, seq: int) -> int:
        v = ctypes.c_int()
        _call("q2_model_get_seq_len", self._h, seq, ctypes.byref(v))
        return v.value

    def kv_cache(self, layer: int, seq: int) -> Tuple[torch.Tensor, torch.Tensor]:
        """Views (not copies) of the cache of (layer, seq): K, V as [nkv, max_seq, hd]."""
        kp, vp = ctypes.c_void_p(), ctypes.c_void_p()
        _call("q2_model_kv_cache", self._h, layer, seq, ctypes.byref(kp), ctypes.byref(vp))
        shp = (self.shape.n_kv_heads, self.max_seq, self.shape.head_dim)
        out = []
        for p in (kp, vp):
            if self.dtype == torch.float32:
                t = torch.as_tensor(_DevArray(p.value, shp, "<f4"), device=f"cuda:{self.device}")
            else:
                t = torch.as_tensor(_DevArray(p.value, shp, "<i2"), device=f"cuda:{self.device}")
                t = t.view(torch.bfloat16)
            out.append(t)
        return out[0], out[1]

    def check_error(self):
        _call("q2_model_check_error", self._h, _stream())

    def test_raise_error(self, bits: int):
        """Test hook: OR `bits` into the model's device error word (q2_test_model_raise_error)."""
        _call("q2_test_model_raise_error", self._h, bits, _stream())

    def test_set_wait_fault(self, phase: int, deadline_ns: int = 200_000_000):
        """Test hook: make one phase's grid counter of the streaming step
        unreachable, with every wait bounded by deadline_ns (q2_test_set_wait_fault)."""
        _call("q2_test_set_wait_fault", self._h, phase, deadline_ns)

    def trace_stream_step(self, ids: torch.Tensor):
        """Profiling hook: per-CTA timestamps of one streaming step,
        [phases, grid, 4] int64 ns (q2_test_trace_stream_step)."""
        import numpy as np
        n = (5 * self.shape.n_layers + 1) * 160 * 4
        buf = np.zeros(n, dtype=np.uint64)
        g = ctypes.c_int()
        _dense(ids)
        _call("q2_test_trace_stream_step", self._h, _p(ids), buf.ctypes.data, n, ctypes.byref(g), _stream())
        G = g.value
        return torch.from_numpy(buf[: (5 * self.shape.n_layers + 1) * G * 4].astype(np.int64)).view(-1, G, 4)

    def set_graphs(self, enable: bool):
        _call("q2_model_set_graphs", self._h, 1 if enable else 0)

    def set_decode_path(self, path: str):
        """'auto' | 'persistent' | 'kernels' | 'generic' | 'stream' (q2_model_set_decode_path)."""
        _call("q2_model_set_decode_path", self._h, PATH[path])

    def time_kernels(self, ids: torch.Tensor, steps: int):
        """Per kernel class: (mean ms per instance, instances per step), plus the
        kernel launches of one step (q2_model_time_kernels)."""
        n = len(KCLASS)
        ms = (ctypes.c_float * n)()
        per = (ctypes.c_int * n)()
        kern = ctypes.c_int()
        _dense(ids)
        _call("q2_model_time_kernels", self._h, _p(ids), ids.numel(), steps, ms, per,
              ctypes.byref(kern), _stream())
        return {KCLASS[i]: (ms[i], per[i]) for i in range(n)}, kern.value
