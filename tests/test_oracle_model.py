"""Pins of the oracle's whole-model forward against HF's Qwen2 in float64 (a
library implementation of the same architecture), plus self-consistency.
CPU only."""

import dataclasses

import pytest
import torch

import oracle
import synth
from hf_ref import build_hf, hf_greedy, hf_logits

SHAPE = synth.TINY_F32
SEED = 1001


@pytest.fixture(scope="module")
def tiny():
    w = synth.model_weights(SHAPE, SEED)
    prompt = synth.prompt_ids(SHAPE, 16, SEED)
    return w, prompt


def _oracle(shape, w, max_seq=64, max_batch=1):
    om = oracle.OracleModel(shape, max_seq=max_seq, max_batch=max_batch)
    om.load(w)
    return om


def test_prompt_logits_match_hf_float64(tiny):
    w, prompt = tiny
    om = _oracle(SHAPE, w)
    _, _, allg = om.forward(0, prompt, all_logits=True)
    ref = hf_logits(build_hf(SHAPE, w), prompt)
    err = (allg.double() - ref).abs().max().item()
    # the oracle rounds to fp32 between operators; HF stays in fp64
    assert err <= 1e-5 * ref.abs().max().item(), err


def test_greedy_tokens_match_hf_untethered(tiny):
    w, prompt = tiny
    om = _oracle(SHAPE, w)
    ours, our_logits = om.generate(0, prompt, 16)
    theirs, their_logits = hf_greedy(build_hf(SHAPE, w), prompt, 16)
    assert ours == theirs
    for a, b in zip(our_logits, their_logits):
        assert (a.double() - b).abs().max().item() <= 1e-5 * b.abs().max().item()


def test_kv_cache_matches_hf_past_keys(tiny):
    w, prompt = tiny
    om = _oracle(SHAPE, w)
    om.forward(0, prompt)
    model = build_hf(SHAPE, w)
    with torch.no_grad():
        out = model(prompt.reshape(1, -1), use_cache=True)
    pkv = out.past_key_values
    for l in range(SHAPE.n_layers):
        k_ref, v_ref = pkv.layers[l].keys[0], pkv.layers[l].values[0]  # [nkv, T, hd]
        k, v = om.kv(l, 0)
        T = prompt.numel()
        assert torch.allclose(k[:T].permute(1, 0, 2).double(), k_ref, rtol=1e-6, atol=1e-7)
        assert torch.allclose(v[:T].permute(1, 0, 2).double(), v_ref, rtol=1e-6, atol=1e-7)


def test_decoder_layer_on_hidden_input_matches_hf(tiny):
    w, prompt = tiny
    one = dataclasses.replace(SHAPE, n_layers=1)
    om = _oracle(one, w)
    x = synth.hidden_input(one, 6, SEED)
    got = om.forward_hidden(0, x).double()
    model = build_hf(one, w)
    with torch.no_grad():
        layer = model.model.layers[0]
        pos = torch.arange(6).reshape(1, -1)
        cos_sin = model.model.rotary_emb(x.double().reshape(1, 6, -1), pos)
        mask = torch.full((6, 6), float("-inf"), dtype=torch.float64).triu(1).reshape(1, 1, 6, 6)
        ref = layer(x.double().reshape(1, 6, -1), attention_mask=mask, position_ids=pos,
                    position_embeddings=cos_sin)
        ref = ref[0] if isinstance(ref, tuple) else ref
    assert torch.allclose(got, ref[0], rtol=1e-5, atol=1e-6)


def test_bf16_model_tracks_float64_hf():
    shape = dataclasses.replace(SHAPE, dtype="bf16")
    w = synth.model_weights(shape, SEED)
    prompt = synth.prompt_ids(shape, 16, SEED)
    om = _oracle(shape, w)
    _, _, allg = om.forward(0, prompt, all_logits=True)
    ref = hf_logits(build_hf(shape, w), prompt)
    cos = torch.nn.functional.cosine_similarity(allg.double(), ref, dim=1)
    assert (cos > 0.999).all(), cos.min()
    assert (allg.double() - ref).abs().max() < 5e-2


def test_prefill_then_decode_equals_longer_prefill(tiny):
    w, prompt = tiny
    a = _oracle(SHAPE, w)
    nxt_a, lg_a = a.forward(0, prompt)
    _, lg_a2 = a.forward(0, torch.tensor([nxt_a]))
    b = _oracle(SHAPE, w)
    _, lg_b = b.forward(0, torch.cat([prompt, torch.tensor([nxt_a])]))
    assert torch.allclose(lg_a2, lg_b, rtol=1e-5, atol=1e-6)
    assert a.get_len(0) == b.get_len(0) == 17


def test_sequences_are_independent(tiny):
    w, prompt = tiny
    om = _oracle(SHAPE, w, max_batch=2)
    other = synth.prompt_ids(SHAPE, 9, SEED, seq=1)
    om.forward(1, other)
    n0, lg0 = om.forward(0, prompt)
    solo = _oracle(SHAPE, w)
    n1, lg1 = solo.forward(0, prompt)
    assert n0 == n1 and torch.equal(lg0, lg1)


def test_capacity_and_range_errors(tiny):
    w, prompt = tiny
    om = _oracle(SHAPE, w, max_seq=16)
    om.forward(0, prompt)
    with pytest.raises(oracle.OracleError):
        om.forward(0, torch.tensor([1]))  # would exceed max_seq
    om2 = _oracle(SHAPE, w)
    with pytest.raises(oracle.OracleError):
        om2.forward(0, torch.tensor([SHAPE.vocab]))  # id out of range


def test_oracle_reproduces_frozen_greedy_fixture():
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_f32_greedy.json")
    ref = json.load(open(path))
    wl = synth.WORKLOADS[ref["workload"]]
    w = synth.model_weights(wl["shape"], wl["seed"])
    prompt = synth.prompt_ids(wl["shape"], wl["prompt"], wl["seed"])
    assert prompt.tolist() == ref["prompt"]
    om = _oracle(wl["shape"], w)
    tokens, logits = om.generate(0, prompt, wl["decode"])
    assert tokens == ref["greedy_tokens"]
    assert [float(x) for x in logits[0][:8]] == ref["first_logits_head"]
