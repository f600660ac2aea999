"""The row-parallel oracle layer of tests/layer_ref.py is the oracle model's
layer: bit-identical outputs, K/V caches, logits and next token on small
models (fp32 and bf16), whole prompts and a second chunk at an offset with
sampled rows.  CPU only."""

import dataclasses

import pytest
import torch

import layer_ref
import oracle
import synth

SMALL_BF16 = dataclasses.replace(synth.QWEN2_1P5B, n_layers=2, hidden=256, n_heads=4, n_kv_heads=2,
                                 head_dim=64, intermediate=512, vocab=1000)


@pytest.fixture(scope="module")
def pool():
    p = layer_ref.make_pool(4)
    yield p
    p.shutdown()


@pytest.mark.parametrize("shape", [synth.TINY_F32, SMALL_BF16], ids=["tiny-f32", "small-bf16"])
def test_prefill_equals_the_oracle_model(pool, shape):
    w = synth.model_weights(shape, 31)
    ids = synth.prompt_ids(shape, 19, 32)
    om = oracle.OracleModel(shape, max_seq=32)
    om.load(w)
    nxt_ref, lg_ref = om.forward(0, ids)
    nxt, lg, _, caches, _ = layer_ref.prefill(pool, shape, w, ids, max_seq=32)
    assert nxt == nxt_ref
    assert torch.equal(lg, lg_ref)
    for l, (kc, vc) in enumerate(caches):
        k_ref, v_ref = om.kv(l, 0)
        assert torch.equal(kc[:19], k_ref[:19]) and torch.equal(vc[:19], v_ref[:19])


def test_second_chunk_sampled_rows_equal_the_oracle_model(pool):
    """A chunk at pos0 > 0 over a cache holding the earlier positions: the
    sampled output rows and the chunk's K/V rows equal the oracle model's."""
    shape = dataclasses.replace(SMALL_BF16, n_layers=1)
    w = synth.model_weights(shape, 41)
    lw = layer_ref.layer_weights(w, 0)
    x1 = synth.hidden_input(shape, 13, 42)
    x2 = synth.hidden_input(shape, 11, 43)
    om = oracle.OracleModel(shape, max_seq=40)
    om.load(w)
    om.forward_hidden(0, x1)
    y2_ref = om.forward_hidden(0, x2)
    kc = torch.zeros((40, shape.n_kv_heads, shape.head_dim), dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    layer_ref.layer_prefill(pool, shape, lw, x1, 0, kc, vc)
    rows = [0, 4, 10]
    y2 = layer_ref.layer_prefill(pool, shape, lw, x2, 13, kc, vc, rows=rows)
    assert torch.equal(y2, y2_ref[rows])
    k_ref, v_ref = om.kv(0, 0)
    assert torch.equal(kc[:24], k_ref[:24]) and torch.equal(vc[:24], v_ref[:24])


def test_single_row_linear_split_over_weight_rows(pool):
    x = synth.normal((1, 96), 1.0, 5, "bf16")
    w = synth.normal((301, 96), 0.02, 6, "bf16")
    b = synth.normal((301,), 0.01, 7, "bf16")
    assert torch.equal(layer_ref.linear(pool, x, w, b), oracle.linear(x, w, b))
    assert torch.equal(layer_ref.linear(pool, x, w, None, out_dtype=torch.float32),
                       oracle.linear(x, w, None, out_dtype=torch.float32))
