"""Seeded synthetic inputs for the Qwen2-style decoder.

This module only draws numbers and stores them in the requested storage
type; it holds none of the model's arithmetic.  The oracle tests, the CUDA
parity tests and the benchmark all take their inputs from here, so both sides
of every comparison see identical bits.

Recipe (what the workloads are made of):

* weight matrices ~ N(0, 0.02), q/k/v biases ~ N(0, 0.01), RMSNorm weights
  ~ 1 + N(0, 0.05), embedding and (untied) lm_head ~ N(0, 0.02);
* prompt ids uniform in [0, vocab);
* pre-filled KV-cache entries and hidden-state inputs ~ N(0, 1).

Every tensor is drawn in float32 from its own torch generator, seeded from
(workload seed, tensor name, layer), then rounded to the storage type with
torch's round-to-nearest-even cast.  Drawing on a CUDA device (for the
multi-GB full-size weights) gives different values than drawing on the CPU
with the same seed; within one run both sides always get the same tensor.
"""

from __future__ import annotations

import dataclasses
import zlib
from typing import Dict, Iterable, Tuple

import torch

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class ModelShape:
    """Shape of a Qwen2-style decoder (the names follow the HF Qwen2 config)."""

    n_layers: int
    hidden: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    intermediate: int
    vocab: int
    eps: float = 1e-6
    theta: float = 10000.0
    dtype: str = "bf16"  # storage dtype of weights / activations / KV: "f32" | "bf16"

    @property
    def q_dim(self) -> int:
        return self.n_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    def weight_shapes(self) -> Dict[Tuple[str, int], Tuple[int, ...]]:
        """(name, layer) -> shape.  Global tensors use layer -1."""
        H, I, V = self.hidden, self.intermediate, self.vocab
        out: Dict[Tuple[str, int], Tuple[int, ...]] = {
            ("embed", -1): (V, H),
            ("lm_head", -1): (V, H),
            ("final_norm", -1): (H,),
        }
        for l in range(self.n_layers):
            out[("in_norm", l)] = (H,)
            out[("q_w", l)] = (self.q_dim, H)
            out[("q_b", l)] = (self.q_dim,)
            out[("k_w", l)] = (self.kv_dim, H)
            out[("k_b", l)] = (self.kv_dim,)
            out[("v_w", l)] = (self.kv_dim, H)
            out[("v_b", l)] = (self.kv_dim,)
            out[("o_w", l)] = (H, self.q_dim)
            out[("post_norm", l)] = (H,)
            out[("gate_w", l)] = (I, H)
            out[("up_w", l)] = (I, H)
            out[("down_w", l)] = (H, I)
        return out

    def param_count(self) -> int:
        n = 0
        for shp in self.weight_shapes().values():
            c = 1
            for s in shp:
                c *= s
            n += c
        return n


# The five workloads: a tiny fp32 model, one Qwen2-1.5B-shaped layer, and
# the full 28-layer Qwen2-1.5B shape (DeepSeek-R1-Distill-Qwen-1.5B is such a
# model) with random-init weights.
TINY_F32 = ModelShape(n_layers=2, hidden=128, n_heads=4, n_kv_heads=2, head_dim=32,
                      intermediate=384, vocab=1024, dtype="f32")
QWEN2_1P5B = ModelShape(n_layers=28, hidden=1536, n_heads=12, n_kv_heads=2, head_dim=128,
                        intermediate=8960, vocab=151936, dtype="bf16")
QWEN2_1P5B_ONE_LAYER = dataclasses.replace(QWEN2_1P5B, n_layers=1)

WORKLOADS = {
    "tiny-2l-f32-prompt16-decode16": dict(shape=TINY_F32, batch=1, prompt=16, decode=16, seed=1001),
    "qwen2-1.5b-layer-decode-ctx4096": dict(shape=QWEN2_1P5B_ONE_LAYER, batch=1, past=4095, decode=1, seed=1002),
    "qwen2-1.5b-b1-prompt512-decode128": dict(shape=QWEN2_1P5B, batch=1, prompt=512, decode=128, seed=1003),
    "qwen2-1.5b-b64-ctx4096-decode32": dict(shape=QWEN2_1P5B, batch=64, past=4096, decode=32, seed=1004),
    "qwen2-1.5b-b1-prompt32768-decode64": dict(shape=QWEN2_1P5B, batch=1, prompt=32768, decode=64, seed=1005),
}


def tensor_seed(seed: int, name: str, index: int = 0) -> int:
    """Stable per-tensor seed (independent of Python's hash randomisation)."""
    return (seed * 1_000_003 + zlib.crc32(f"{name}:{index}".encode())) % (2**62)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal(shape: Iterable[int], std: float, seed: int, dtype: str = "f32",
           device="cpu", mean: float = 0.0) -> torch.Tensor:
    """N(mean, std^2) draws in float32, rounded to the storage dtype."""
    t = torch.randn(tuple(shape), generator=_gen(device, seed), device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    if mean != 0.0:
        t.add_(mean)
    return t.to(TORCH_DTYPE[dtype])


def uniform_ids(n: int, vocab: int, seed: int, device="cpu") -> torch.Tensor:
    """n token ids, uniform in [0, vocab), int64."""
    return torch.randint(0, vocab, (n,), generator=_gen(device, seed), device=device, dtype=torch.int64)


def init_std(name: str) -> Tuple[float, float]:
    """(mean, std) of the random init of a weight tensor by kind."""
    if name.endswith("norm"):
        return 1.0, 0.05
    if name.endswith("_b"):
        return 0.0, 0.01
    return 0.0, 0.02


def weight(shape: ModelShape, name: str, layer: int, seed: int, device="cpu") -> torch.Tensor:
    shp = shape.weight_shapes()[(name, layer)]
    mean, std = init_std(name)
    return normal(shp, std, tensor_seed(seed, name, layer), shape.dtype, device, mean)


def model_weights(shape: ModelShape, seed: int, device="cpu") -> Dict[Tuple[str, int], torch.Tensor]:
    """All weights of a random-init model, keyed by (name, layer)."""
    return {key: weight(shape, key[0], key[1], seed, device) for key in shape.weight_shapes()}


def prompt_ids(shape: ModelShape, n: int, seed: int, seq: int = 0, device="cpu") -> torch.Tensor:
    return uniform_ids(n, shape.vocab, tensor_seed(seed, "ids", seq), device)


def kv_fill(shape: ModelShape, n_pos: int, seed: int, layer: int, seq: int, device="cpu"):
    """N(0,1) K and V entries for n_pos cached positions, each [n_pos, n_kv_heads, head_dim]."""
    shp = (n_pos, shape.n_kv_heads, shape.head_dim)
    k = normal(shp, 1.0, tensor_seed(seed, f"kcache:{seq}", layer), shape.dtype, device)
    v = normal(shp, 1.0, tensor_seed(seed, f"vcache:{seq}", layer), shape.dtype, device)
    return k, v


def hidden_input(shape: ModelShape, n_tok: int, seed: int, device="cpu") -> torch.Tensor:
    """N(0,1) hidden-state input [n_tok, hidden]."""
    return normal((n_tok, shape.hidden), 1.0, tensor_seed(seed, "hidden", 0), shape.dtype, device)
