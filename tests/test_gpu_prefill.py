"""The model's tensor-core prefill against the oracle, layer by layer, at the
workloads' sizes.

Every prompt of 64 tokens or more takes this path: per 4096-token chunk, the
tcgen05 GEMM for the q/k/v linear (bias fused), RoPE and the K/V write-back at
positions pos0 + t, flash attention over the cache, and the tcgen05 GEMM with
fused epilogues for o (+ residual), gate/up (+ SwiGLU) and down (+ residual).
The oracle side is the oracle's own layer, composed from its operators and
run row-parallel (tests/layer_ref.py, bit-identical to the oracle model).

* every one of the 28 full-size layers at the 512-token prompt length, each
  on its own seeded N(0,1) input: the K/V rows of all 512 positions and the
  layer output on rows on both sides of the 64-row, 128- and 256-token tile
  edges (the per-layer bisection of the Day-0 tutorial, step 6);
* the whole 28-layer model on a 128-token prompt prefilled in two 64-token
  chunks: each layer fed the oracle's own input for that layer (all rows, K/V
  at pos0 = 0 and 64), the head on the oracle's final state, and the model's
  own prefill from ids (first greedy token, last-position logits);
* the last 4096-token chunk of the 32768-token prompt (positions 28672 ..
  32767) over a cache holding the earlier positions, for the first and the
  last layer.
Bounds: V rows per operator (1e-2 of max(|ref|, rms(ref))), K rows (a linear
with RoPE in its epilogue: two roundings) twice that; layer outputs
the layer bound (3.5e-2 elementwise, 1e-2 in norm); logits on the oracle's
final state 5e-2 / 0.9995; free-running logits 0.15 / 0.9995 (tests/tol.py).
"""
import dataclasses

import pytest
import torch

import layer_ref
import oracle
import qwen2_decode_step_b200 as q2
import synth
from tol import (assert_bf16_logits, assert_bf16_logits_free_running, assert_fused_close,
                 assert_layer_close, assert_op_close)

pytestmark = pytest.mark.gpu

SHAPE = synth.QWEN2_1P5B
ONE = dataclasses.replace(SHAPE, n_layers=1)
SEED = synth.WORKLOADS["qwen2-1.5b-b1-prompt512-decode128"]["seed"]


@pytest.fixture(autouse=True)
def _gpu(cuda_ok):
    yield
    torch.cuda.synchronize()


@pytest.fixture(scope="module")
def full_w():
    w = synth.model_weights(SHAPE, SEED, device="cuda")  # drawn on the GPU (fast) ...
    return {k: t.cpu() for k, t in w.items()}           # ... same bits on both sides


@pytest.fixture(scope="module")
def pool():
    p = layer_ref.make_pool()
    yield p
    p.shutdown()


def one_layer(full_w, l):
    """Layer l's weights as a one-layer model's (layer 0)."""
    return {(n, 0): t for (n, ll), t in full_w.items() if ll == l}


def globals_of(full_w):
    return {k: t for k, t in full_w.items() if k[1] == -1}


def gpu_kv(gm, n0, n1):
    k, v = gm.kv_cache(0, 0)  # [nkv, max_seq, hd]
    return k[:, n0:n1].permute(1, 0, 2).cpu(), v[:, n0:n1].permute(1, 0, 2).cpu()


def empty_cache(n):
    kc = torch.zeros((n, SHAPE.n_kv_heads, SHAPE.head_dim), dtype=torch.bfloat16)
    return kc, torch.zeros_like(kc)


# rows on both sides of the 64-row (attention block), 128- and 256-token (GEMM
# tile) edges, the first and the last row
ROWS_512 = [0, 1, 2, 63, 64, 65, 127, 128, 191, 192, 255, 256, 257, 319, 320, 383, 384, 447, 448, 449,
            500, 509, 510, 511]


def test_prefill_512_every_layer(full_w, pool):
    gm = q2.Model(ONE, max_seq=512)
    errs = []
    for l in range(SHAPE.n_layers):
        w = one_layer(full_w, l)
        x = synth.normal((512, SHAPE.hidden), 1.0, synth.tensor_seed(SEED, "prefill-input", l), "bf16")
        kc, vc = empty_cache(512)
        ref = layer_ref.layer_prefill(pool, ONE, layer_ref.layer_weights(w, 0), x, 0, kc, vc, rows=ROWS_512)
        gm.reset_kv()
        gm.load(w)
        y = gm.prefill_hidden(0, x.cuda()).cpu()
        gk, gv = gpu_kv(gm, 0, 512)
        assert_fused_close(gk, kc[:512], f"layer {l}: K rows 0..511")
        assert_op_close(gv, vc[:512], f"layer {l}: V rows 0..511")
        errs.append(assert_layer_close(y[ROWS_512], ref, f"layer {l}: output rows"))
    gm.check_error()
    gm.close()
    assert max(errs) <= 1e-2, errs


def test_prefill_two_chunks_full_model_against_the_oracle_chain(full_w, pool):
    T, chunk = 128, 64
    prompt = synth.prompt_ids(SHAPE, T, SEED + 500)
    nxt_ref, lg_ref, inputs, caches, x_final = layer_ref.prefill(pool, SHAPE, full_w, prompt, T,
                                                                 keep_layer_inputs=True)
    # (a) layer by layer, each fed the oracle's input for that layer, in two chunks
    gm = q2.Model(ONE, max_seq=T, max_prefill_tokens=chunk)
    gm.load(globals_of(full_w))
    errs = []
    for l in range(SHAPE.n_layers):
        gm.reset_kv()
        gm.load(one_layer(full_w, l))
        y = gm.prefill_hidden(0, inputs[l].cuda()).cpu()
        ref = inputs[l + 1] if l + 1 < SHAPE.n_layers else x_final
        gk, gv = gpu_kv(gm, 0, T)
        assert_fused_close(gk, caches[l][0][:T], f"layer {l}: K rows")
        assert_op_close(gv, caches[l][1][:T], f"layer {l}: V rows")
        errs.append(assert_layer_close(y, ref, f"layer {l}: output"))
    # the head on the oracle's final state of the last position
    nxt, lg = gm.head(x_final[T - 1:T].cuda())
    assert_bf16_logits(lg[0].cpu(), lg_ref, "head on the oracle's final state")
    top2 = torch.topk(lg_ref, 2).values
    if float(top2[0] - top2[1]) > 1e-2:
        assert int(nxt[0]) == nxt_ref
    gm.check_error()
    gm.close()
    assert max(errs) <= 1e-2 and max(errs[-7:]) <= 2 * max(errs[:7]) + 1e-3, errs
    # (b) the model's own prefill from ids: first greedy token and logits
    gm = q2.Model(SHAPE, max_seq=T + 8, max_prefill_tokens=chunk)
    gm.load(full_w)
    nxt, lg = gm.prefill(prompt.cuda(), [T], want_logits=True)
    assert_bf16_logits_free_running(lg[0].cpu(), lg_ref, "prefill logits (free-running)")
    if float(top2[0] - top2[1]) > 5e-2:
        assert int(nxt[0]) == nxt_ref
    gm.check_error()
    gm.close()


ROWS_4096 = [0, 1, 63, 64, 127, 128, 255, 256, 1023, 1024, 2047, 2048, 2049, 3071, 3072, 4031, 4032, 4093,
             4094, 4095]


@pytest.mark.parametrize("layer", [0, SHAPE.n_layers - 1])
def test_prefill_last_4096_chunk_of_32768(full_w, pool, layer):
    past, T = 28672, 4096
    seed = synth.WORKLOADS["qwen2-1.5b-b1-prompt32768-decode64"]["seed"]
    w = one_layer(full_w, layer)
    k, v = synth.kv_fill(ONE, past, seed, layer, 0)  # [past, nkv, hd] N(0,1)
    x = synth.normal((T, SHAPE.hidden), 1.0, synth.tensor_seed(seed, "chunk-input", layer), "bf16")
    kc, vc = empty_cache(past + T)
    kc[:past], vc[:past] = k, v
    ref = layer_ref.layer_prefill(pool, ONE, layer_ref.layer_weights(w, 0), x, past, kc, vc, rows=ROWS_4096)
    gm = q2.Model(ONE, max_seq=past + T)
    gm.load(w)
    gk, gv = gm.kv_cache(0, 0)
    gk[:, :past] = k.permute(1, 0, 2).cuda()
    gv[:, :past] = v.permute(1, 0, 2).cuda()
    gm.set_seq_len(0, past)
    y = gm.prefill_hidden(0, x.cuda()).cpu()
    nk, nv = gpu_kv(gm, past, past + T)
    assert_fused_close(nk, kc[past:past + T], f"layer {layer}: K rows {past}..{past + T - 1}")
    assert_op_close(nv, vc[past:past + T], f"layer {layer}: V rows {past}..{past + T - 1}")
    assert_layer_close(y[ROWS_4096], ref, f"layer {layer}: output rows")
    assert gm.get_seq_len(0) == past + T
    gm.check_error()
    gm.close()
