"""The batch-64 workload (Qwen2-1.5B shape, bf16, 64 sequences at 4096
cached positions, N(0,1) cache) at full size, in the launch configuration
the bench times: tcgen05 linears with M = 64 tokens (split-K for the 1536-
and 2048-row projections) and the tensor-core decode attention (two splits
per sequence and kv head).

The oracle decodes sampled sequences one by one over the same cache:
* layer by layer with teacher forcing (each layer's sampled rows fed the
  oracle's input for that layer; rows are independent sequences), within the
  per-layer bound, then the head (final RMSNorm, lm_head, argmax) on the
  oracle's final state: logits within the bf16 bound, the token bit-exact
  against the oracle's argmax of the same fp32 logits (and equal to the
  oracle's own token when its top two logits are further apart than the
  logit bound);
* the whole step free-running for sampled sequences, within the long-context
  free-running bound (twice the oracle's own fp32-accumulation drift at
  32768 positions, an upper bound for 4096).
"""
import dataclasses

import pytest

import oracle
import qwen2_decode_step_b200 as q2
import synth
import torch
from tol import assert_bf16_logits, assert_bf16_logits_long_context, assert_layer_close

pytestmark = pytest.mark.gpu

WL = synth.WORKLOADS["qwen2-1.5b-b64-ctx4096-decode32"]
SAMPLED = (0, 37, 63)


@pytest.fixture(autouse=True)
def _gpu(cuda_ok):
    pass


@pytest.fixture(scope="module")
def b64():
    shape = synth.QWEN2_1P5B
    seed, past, B = WL["seed"], WL["past"], WL["batch"]
    w = synth.model_weights(shape, seed, device="cuda")
    wc = {k: t.cpu() for k, t in w.items()}
    ids = synth.uniform_ids(B, shape.vocab, seed + 7)
    return shape, seed, past, B, w, wc, ids


def _fill_cache(model, shape, seed, past, B, layers, dst_layer=None):
    """The N(0,1) cache of the workload for `layers`, written into `model`
    (at dst_layer when given); returns the sampled sequences' K/V on the host."""
    host = {}
    for l in layers:
        for b in range(B):
            k, v = synth.kv_fill(shape, past, seed, l, b, device="cuda")
            gk, gv = model.kv_cache(l if dst_layer is None else dst_layer, b)
            gk[:, :past] = k.permute(1, 0, 2)
            gv[:, :past] = v.permute(1, 0, 2)
            if b in SAMPLED:
                host[(l, b)] = (k.cpu(), v.cpu())
    for b in range(B):
        model.set_seq_len(b, past)
    return host


def test_batch64_decode_layerwise_teacher_forced(b64):
    shape, seed, past, B, w, wc, ids = b64
    one = dataclasses.replace(shape, n_layers=1)
    g1 = q2.Model(one, max_seq=past + 8, max_batch=B)
    g1.load({k: t for k, t in w.items() if k[1] == -1})
    emb = wc[("embed", -1)]
    x_ref = {b: oracle.embedding(ids[b:b + 1], emb) for b in SAMPLED}
    x = oracle.embedding(ids, emb).cuda()  # all 64 rows (rows are independent sequences)
    for l in range(shape.n_layers):
        g1.load({(n, 0): t for (n, ll), t in w.items() if ll == l})
        host = _fill_cache(g1, shape, seed, past, B, [l], dst_layer=0)
        for b in SAMPLED:
            x[b] = x_ref[b][0].cuda()
        y = g1.forward_hidden(x)
        om = oracle.OracleModel(one, max_seq=past + 8)
        om.load({(n, 0): t for (n, ll), t in wc.items() if ll == l})
        for b in SAMPLED:
            ok, ov = om.kv(0, 0)
            ok[:past] = host[(l, b)][0]
            ov[:past] = host[(l, b)][1]
            om.set_len(0, past)
            y_ref = om.forward_hidden(0, x_ref[b])
            assert_layer_close(y[b:b + 1], y_ref, f"layer {l} sequence {b}")
            x_ref[b] = y_ref
        del om
        x = y
    # the head on the oracle's final state of each sampled sequence
    for b in SAMPLED:
        h = oracle.rms_norm(x_ref[b], wc[("final_norm", -1)], shape.eps)
        lg_ref = oracle.linear(h, wc[("lm_head", -1)], None, out_dtype=torch.float32)[0]
        nxt_ref = int(oracle.argmax(lg_ref)[0][0])
        nxt, lg = g1.head(x_ref[b].cuda())
        lg = lg[0].cpu()
        assert_bf16_logits(lg, lg_ref, f"head, sequence {b}")
        assert int(nxt[0]) == int(oracle.argmax(lg)[0][0]), f"sequence {b}: argmax of the GPU's logits"
        top2 = torch.topk(lg_ref, 2).values
        if float(top2[0] - top2[1]) > 5e-2:
            assert int(nxt[0]) == nxt_ref, f"sequence {b}: token"
    g1.check_error()


def test_batch64_decode_step_free_running(b64):
    shape, seed, past, B, w, wc, ids = b64
    gm = q2.Model(shape, max_seq=past + 8, max_batch=B)
    gm.load(w)
    host = _fill_cache(gm, shape, seed, past, B, range(shape.n_layers))
    nxt, lg = gm.decode_step(ids.cuda(), want_logits=True)
    for b in SAMPLED:
        om = oracle.OracleModel(shape, max_seq=past + 8)
        om.load(wc)
        for l in range(shape.n_layers):
            ok, ov = om.kv(l, 0)
            ok[:past] = host[(l, b)][0]
            ov[:past] = host[(l, b)][1]
        om.set_len(0, past)
        _, lg_ref = om.forward(0, ids[b:b + 1])
        assert_bf16_logits_long_context(lg[b], lg_ref, f"sequence {b}")
        del om
    for b in range(B):
        assert gm.get_seq_len(b) == past + 1
