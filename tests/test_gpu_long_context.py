"""The 32768-token workload (Qwen2-1.5B shape, bf16) at full size.

The oracle cannot run a 32768-token prefill in a test's time (about 1.6
TFLOP per layer of attention alone in fp64), so these tests check what it
can compute exactly at full size:

* the prefill attention kernel in the launch configuration of the model's
  last prefill chunk (4096 query rows over 32768 keys), on sampled rows that
  the oracle computes one by one (first and last rows, rows on both sides of
  a 64-row block and a 64-key tile boundary);
* a decode step at 32768 context over the GPU's own prefilled cache (the
  oracle is given that cache): layer by layer with teacher forcing (each
  layer fed the oracle's input; the stated bounds), and free-running through
  all 28 layers (a bound derived from the oracle's own fp32-accumulation
  drift at this context).
"""
import math

import pytest
import torch

import oracle
import qwen2_decode_step_b200 as q2
import synth
from synth import normal
from tol import assert_bf16_logits_long_context, assert_op_close

pytestmark = pytest.mark.gpu

WL = synth.WORKLOADS["qwen2-1.5b-b1-prompt32768-decode64"]


@pytest.fixture(autouse=True)
def _gpu(cuda_ok):
    pass


def test_prefill_attention_last_chunk_of_32768_sampled_rows():
    S, T, nh, nkv, hd = 4096, 32768, 12, 2, 128
    seed = WL["seed"]
    q = normal((S, nh, hd), 1.0, seed + 11, "bf16")
    k = normal((T, nkv, hd), 1.0, seed + 12, "bf16")
    v = normal((T, nkv, hd), 1.0, seed + 13, "bf16")
    out = torch.empty((S, nh, hd), dtype=torch.bfloat16, device="cuda")
    scale = 1.0 / math.sqrt(hd)
    q2.q2_self_attention(out, q.cuda(), k.cuda(), v.cuda(), scale)
    got = out.cpu()
    for i in (0, 1, 63, 64, 65, 2047, 4031, 4032, 4095):
        p = T - S + i  # absolute position of row i: it sees keys 0..p
        ref = oracle.self_attention(q[i:i + 1], k[:p + 1], v[:p + 1], scale)
        assert_op_close(got[i:i + 1], ref, f"row {i} (position {p})")


@pytest.fixture(scope="module")
def long_ctx():
    """The GPU prefilled with the 32768-token prompt, its cache copied out, and
    the oracle-side weights (same bits)."""
    shape = synth.QWEN2_1P5B
    seed, prompt_len = WL["seed"], WL["prompt"]
    w = synth.model_weights(shape, seed, device="cuda")
    gm = q2.Model(shape, max_seq=prompt_len + 8, max_batch=1)
    gm.load(w)
    ids = synth.prompt_ids(shape, prompt_len, seed)
    first = gm.prefill(ids.cuda(), [prompt_len])
    torch.cuda.synchronize()
    cache = []
    for l in range(shape.n_layers):
        gk, gv = gm.kv_cache(l, 0)
        cache.append((gk[:, :prompt_len].permute(1, 0, 2).cpu(), gv[:, :prompt_len].permute(1, 0, 2).cpu()))
    wc = {k_: t.cpu() for k_, t in w.items()}
    del w
    return shape, prompt_len, gm, first, cache, wc


def test_decode_at_32768_context_layerwise_teacher_forced(long_ctx):
    """Every layer fed the oracle's input for that layer, over the GPU's cache:
    each within the per-layer bound, the head on the oracle's final state within
    the stated logits bound."""
    import dataclasses
    from tol import assert_bf16_logits, assert_layer_close
    shape, P, _, first, cache, wc = long_ctx
    one = dataclasses.replace(shape, n_layers=1)
    g1 = q2.Model(one, max_seq=P + 8, max_batch=1)
    g1.load({k_: t for k_, t in wc.items() if k_[1] == -1})
    x = oracle.embedding(first.cpu(), wc[("embed", -1)])
    errs = []
    for l in range(shape.n_layers):
        lw = {(n, 0): t for (n, ll), t in wc.items() if ll == l}
        om = oracle.OracleModel(one, max_seq=P + 8)
        om.load(lw)
        ok, ov = om.kv(0, 0)
        ok[:P] = cache[l][0]
        ov[:P] = cache[l][1]
        om.set_len(0, P)
        y_ref = om.forward_hidden(0, x)
        g1.load(lw)
        gk, gv = g1.kv_cache(0, 0)
        gk[:, :P] = cache[l][0].permute(1, 0, 2).cuda()
        gv[:, :P] = cache[l][1].permute(1, 0, 2).cuda()
        g1.set_seq_len(0, P)
        y = g1.forward_hidden(x.cuda())
        errs.append(assert_layer_close(y, y_ref, f"layer {l} at 32768 context"))
        x = y_ref
        del om
    h = oracle.rms_norm(x, wc[("final_norm", -1)], shape.eps)
    ref_logits = oracle.linear(h, wc[("lm_head", -1)], None, out_dtype=torch.float32)[0]
    nxt, lg = g1.head(x.cuda())
    assert_bf16_logits(lg[0].cpu(), ref_logits, "head at 32768 context")
    assert max(errs) <= 1e-2, errs


def test_decode_step_at_32768_context_free_running(long_ctx):
    """The whole decode step (all layers, the GPU's own hidden states) against
    the oracle decoding the same token over the GPU's cache."""
    shape, P, gm, first, cache, wc = long_ctx
    om = oracle.OracleModel(shape, max_seq=P + 8)
    om.load(wc)
    for l in range(shape.n_layers):
        ok, ov = om.kv(l, 0)
        ok[:P] = cache[l][0]
        ov[:P] = cache[l][1]
    om.set_len(0, P)
    nxt_ref, lg_ref = om.forward(0, first.cpu())
    nxt, lg = gm.decode_step(first, want_logits=True)
    assert_bf16_logits_long_context(lg[0], lg_ref, "decode logits at 32768 context")
    assert gm.get_seq_len(0) == P + 1
    gk, gv = gm.kv_cache(0, 0)
    ok, ov = om.kv(0, 0)
    assert_op_close(gk[:, P].cpu(), ok[P], "k appended at 32768")
    assert_op_close(gv[:, P].cpu(), ov[P], "v appended at 32768")
