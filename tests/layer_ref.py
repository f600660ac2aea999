"""The oracle's decoder layer and head, composed in the test from the oracle's
own operators and run row-parallel on the host's cores: what the prefill
parity tests need at the workloads' sizes (hundreds to thousands of rows),
where the oracle model's one-thread layer would take minutes.

Same operators, same order, same roundings as ``oracle.OracleModel``'s layer
(RMSNorm, q/k/v linears with bias, RoPE, KV write-back, causal GQA attention,
o linear, residual add, RMSNorm, gate/up linears, SwiGLU, down linear,
residual add -- the Qwen2 layer of the LLAISYS report, section 3.2);
``tests/test_layer_ref.py`` checks bit for bit that the two agree.  Threads
only split rows that do not depend on each other: a linear's rows, and the
query rows of attention (row i of a chunk at position pos0 sees keys
0 .. pos0 + i, which is one single-row attention call over the first
pos0 + i + 1 cache rows).  ctypes releases the GIL inside every oracle call.

Test infrastructure only: nothing here touches the GPU or the CUDA library.
"""

from __future__ import annotations

import concurrent.futures as cf
import os
from typing import Dict, Iterable, List, Optional, Tuple

import torch

import oracle


def make_pool(workers: Optional[int] = None) -> cf.ThreadPoolExecutor:
    return cf.ThreadPoolExecutor(max_workers=workers or max(1, os.cpu_count() or 1))


def _chunks(n: int, parts: int) -> List[Tuple[int, int]]:
    parts = max(1, min(parts, n))
    return [(n * i // parts, n * (i + 1) // parts) for i in range(parts)]


def linear(pool, x: torch.Tensor, w: torch.Tensor, b: Optional[torch.Tensor] = None,
           out_dtype: Optional[torch.dtype] = None) -> torch.Tensor:
    """oracle.linear with the rows of x (or, for one row, the rows of w) split over the pool."""
    workers = pool._max_workers
    if x.shape[0] > 1:
        parts = _chunks(x.shape[0], 4 * workers)
        outs = list(pool.map(lambda c: oracle.linear(x[c[0]:c[1]], w, b, out_dtype=out_dtype), parts))
        return torch.cat(outs, 0)
    parts = _chunks(w.shape[0], 4 * workers)
    outs = list(pool.map(lambda c: oracle.linear(x, w[c[0]:c[1]], None if b is None else b[c[0]:c[1]],
                                                 out_dtype=out_dtype), parts))
    return torch.cat(outs, -1)


def layer_weights(weights: Dict, layer: int) -> Dict[str, torch.Tensor]:
    return {name: t for (name, l), t in weights.items() if l == layer}


def layer_prefill(pool, shape, lw: Dict[str, torch.Tensor], x: torch.Tensor, pos0: int,
                  k_cache: torch.Tensor, v_cache: torch.Tensor,
                  rows: Optional[Iterable[int]] = None) -> torch.Tensor:
    """One decoder layer for the chunk x [T, H] at positions pos0 .. pos0 + T - 1.

    k_cache, v_cache: [>= pos0 + T, nkv, hd], rows < pos0 already filled; the
    chunk's K/V rows (k after RoPE) are written at pos0 .. pos0 + T - 1.
    Returns the layer output of the chunk rows `rows` (all rows if None),
    [len(rows), H]."""
    T, H = x.shape
    nh, nkv, hd = shape.n_heads, shape.n_kv_heads, shape.head_dim
    rows = list(range(T)) if rows is None else list(rows)
    h = oracle.rms_norm(x, lw["in_norm"], shape.eps)
    q = linear(pool, h, lw["q_w"], lw["q_b"])
    k = linear(pool, h, lw["k_w"], lw["k_b"])
    v = linear(pool, h, lw["v_w"], lw["v_b"])
    pos = torch.arange(pos0, pos0 + T, dtype=torch.int64)
    q = oracle.rope(q.reshape(T, nh, hd), pos, shape.theta)
    k = oracle.rope(k.reshape(T, nkv, hd), pos, shape.theta)
    k_cache[pos0:pos0 + T] = k
    v_cache[pos0:pos0 + T] = v.reshape(T, nkv, hd)

    def attend(i):
        n = pos0 + i + 1
        return oracle.self_attention(q[i:i + 1], k_cache[:n], v_cache[:n]).reshape(1, nh * hd)

    a = torch.cat(list(pool.map(attend, rows)), 0)
    xs = x[rows]
    o = linear(pool, a, lw["o_w"])
    xs = oracle.add(xs, o)
    h2 = oracle.rms_norm(xs, lw["post_norm"], shape.eps)
    g = linear(pool, h2, lw["gate_w"])
    u = linear(pool, h2, lw["up_w"])
    s = oracle.swiglu(g, u)
    d = linear(pool, s, lw["down_w"])
    return oracle.add(xs, d)


def head(pool, shape, final_norm: torch.Tensor, lm_head: torch.Tensor,
         x_last: torch.Tensor) -> Tuple[int, torch.Tensor]:
    """Final RMSNorm, lm_head (fp32 logits) and greedy argmax of one row x_last [1, H]."""
    h = oracle.rms_norm(x_last.reshape(1, -1), final_norm, shape.eps)
    logits = linear(pool, h, lm_head, None, out_dtype=torch.float32)[0]
    idx, _ = oracle.argmax(logits)
    return int(idx[0]), logits


def prefill(pool, shape, weights: Dict, ids: torch.Tensor, max_seq: int, keep_layer_inputs=False):
    """The whole prompt through every layer (all rows), then the head on the
    last position.  Returns (next id, last-position logits, list of the layer
    inputs if asked, the K/V caches per layer)."""
    T = ids.numel()
    x = oracle.embedding(ids, weights[("embed", -1)])
    dt = x.dtype
    caches = []
    inputs = []
    for l in range(shape.n_layers):
        kc = torch.zeros((max_seq, shape.n_kv_heads, shape.head_dim), dtype=dt)
        vc = torch.zeros_like(kc)
        if keep_layer_inputs:
            inputs.append(x)
        x = layer_prefill(pool, shape, layer_weights(weights, l), x, 0, kc, vc)
        caches.append((kc, vc))
    nxt, logits = head(pool, shape, weights[("final_norm", -1)], weights[("lm_head", -1)], x[T - 1:T])
    return nxt, logits, inputs, caches, x


def decode_step(pool, shape, weights: Dict, caches, token: int, pos: int):
    """One greedy decode step of token `token` at position `pos` over the
    per-layer caches (rows < pos filled; row pos written): (next id, logits)."""
    x = oracle.embedding(torch.tensor([token], dtype=torch.int64), weights[("embed", -1)])
    for l in range(shape.n_layers):
        kc, vc = caches[l]
        x = layer_prefill(pool, shape, layer_weights(weights, l), x, pos, kc, vc)
    return head(pool, shape, weights[("final_norm", -1)], weights[("lm_head", -1)], x)
