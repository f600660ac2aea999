"""Model-level parity: the CUDA decoder (prefill + greedy decode steps,
through the C ABI) against the CPU oracle on the same seeded weights and
inputs, plus GPU self-consistency and error paths.  GPU only."""

import dataclasses

import pytest
import torch

import oracle
import qwen2_decode_step_b200 as q2
import synth
from tol import (assert_bf16_logits, assert_bf16_logits_free_running, assert_close,
                 assert_layer_close, assert_op_close, bits_equal)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu(cuda_ok):
    yield
    torch.cuda.synchronize()


def layer_weights(shape, seed, device="cpu"):
    """All weights except the two [vocab, hidden] tables."""
    return {k: synth.weight(shape, k[0], k[1], seed, device) for k in shape.weight_shapes()
            if k[0] not in ("embed", "lm_head")}


def pair(shape, w, max_seq, max_batch=1, **kw):
    om = oracle.OracleModel(shape, max_seq=max_seq, max_batch=max_batch)
    om.load(w)
    gm = q2.Model(shape, max_seq=max_seq, max_batch=max_batch, **kw)
    gm.load(w)
    return om, gm


# ------------------------------------------------------------ tiny fp32

TINY = synth.WORKLOADS["tiny-2l-f32-prompt16-decode16"]


@pytest.fixture(scope="module")
def tiny_w():
    return synth.model_weights(TINY["shape"], TINY["seed"])


def gpu_generate(gm, prompt, n_decode, teacher=None):
    nxt, lg = gm.prefill(prompt.cuda(), [prompt.numel()], want_logits=True)
    toks, logits = [int(nxt[0])], [lg[0].cpu()]
    for i in range(n_decode):
        feed = nxt if teacher is None else torch.tensor([teacher[i]], device="cuda")
        nxt, lg = gm.decode_step(feed, want_logits=True)
        toks.append(int(nxt[0]))
        logits.append(lg[0].cpu())
    return toks, logits


def test_tiny_f32_greedy_untethered(tiny_w):
    shape = TINY["shape"]
    prompt = synth.prompt_ids(shape, TINY["prompt"], TINY["seed"])
    om, gm = pair(shape, tiny_w, max_seq=64)
    ref_toks, ref_logits = om.generate(0, prompt, TINY["decode"])
    toks, logits = gpu_generate(gm, prompt, TINY["decode"])
    assert toks == ref_toks
    for i, (a, b) in enumerate(zip(logits, ref_logits)):
        assert_close(a, b, 1e-4, f"logits step {i}")
    gm.check_error()


def test_tiny_f32_chunked_prefill_and_eager_match(tiny_w):
    shape = TINY["shape"]
    prompt = synth.prompt_ids(shape, TINY["prompt"], TINY["seed"])
    om, gm = pair(shape, tiny_w, max_seq=64, max_prefill_tokens=5)  # chunks 5+5+5+1
    ref_toks, ref_logits = om.generate(0, prompt, 4)
    gm.set_graphs(False)
    toks, logits = gpu_generate(gm, prompt, 4)
    assert toks == ref_toks
    for a, b in zip(logits, ref_logits):
        assert_close(a, b, 1e-4, "chunked/eager logits")


def test_tiny_f32_batched_decode_matches_each_sequence_alone(tiny_w):
    shape = TINY["shape"]
    lens = [5, 16, 9]
    prompts = [synth.prompt_ids(shape, n, TINY["seed"], seq=b) for b, n in enumerate(lens)]
    _, gm = pair(shape, tiny_w, max_seq=64, max_batch=3)
    nxt = gm.prefill(torch.cat(prompts).cuda(), lens)
    got = [[int(t)] for t in nxt.cpu()]
    for _ in range(8):
        nxt = gm.decode_step(nxt)
        for b, t in enumerate(nxt.cpu().tolist()):
            got[b].append(t)
    for b in range(3):
        om = oracle.OracleModel(shape, max_seq=64)
        om.load(tiny_w)
        ref, _ = om.generate(0, prompts[b], 8)
        assert got[b] == ref, b
        assert gm.get_seq_len(b) == lens[b] + 8


# ------------------------------------------- one Qwen2-1.5B layer, decode

def test_one_layer_decode_at_4096_context():
    wl = synth.WORKLOADS["qwen2-1.5b-layer-decode-ctx4096"]
    shape, seed, past = wl["shape"], wl["seed"], wl["past"]
    w = layer_weights(shape, seed)
    om, gm = pair(shape, w, max_seq=past + 1)
    k, v = synth.kv_fill(shape, past, seed, layer=0, seq=0)
    ok, ov = om.kv(0, 0)
    ok[:past] = k
    ov[:past] = v
    om.set_len(0, past)
    gk, gv = gm.kv_cache(0, 0)
    gk[:, :past] = k.permute(1, 0, 2).cuda()
    gv[:, :past] = v.permute(1, 0, 2).cuda()
    gm.set_seq_len(0, past)
    x = synth.hidden_input(shape, 1, seed)
    ref = om.forward_hidden(0, x)
    got = gm.forward_hidden(x.cuda())
    assert_layer_close(got, ref, "layer output")
    # the appended K/V row (k after RoPE) at position 4095
    assert_op_close(gk[:, past].cpu(), ok[past], "k appended")
    assert_op_close(gv[:, past].cpu(), ov[past], "v appended")
    assert gm.get_seq_len(0) == past + 1


# --------------------------------------------- full Qwen2-1.5B shape, bf16

@pytest.fixture(scope="module")
def full_w():
    shape = synth.QWEN2_1P5B
    seed = synth.WORKLOADS["qwen2-1.5b-b1-prompt512-decode128"]["seed"]
    w = synth.model_weights(shape, seed, device="cuda")  # drawn on the GPU (fast) ...
    return {k: t.cpu() for k, t in w.items()}           # ... same bits on both sides


def test_full_model_layerwise_teacher_forced(full_w):
    """All 28 full-size layers, each fed the oracle's own input for that layer
    (per-layer teacher forcing): a 6-position prefill then one decode position
    through every layer within the per-op tolerance, and the head on the
    oracle's final hidden state within the logits bound."""
    shape = synth.QWEN2_1P5B
    one = dataclasses.replace(shape, n_layers=1)
    prompt = synth.prompt_ids(shape, 6, 2003)
    tok = synth.uniform_ids(1, shape.vocab, 2005)
    emb = full_w[("embed", -1)]
    xp, xd = oracle.embedding(prompt, emb), oracle.embedding(tok, emb)
    gm = q2.Model(one, max_seq=16)
    gm.load({k: t for k, t in full_w.items() if k[1] == -1})
    errs = []
    for l in range(shape.n_layers):
        lw = {(n, 0): t for (n, ll), t in full_w.items() if ll == l}
        om = oracle.OracleModel(one, max_seq=16)
        om.load(lw)
        yp_ref = om.forward_hidden(0, xp)
        yd_ref = om.forward_hidden(0, xd)
        gm.reset_kv()
        gm.load(lw)
        yp = gm.prefill_hidden(0, xp.cuda())
        yd = gm.forward_hidden(xd.cuda())
        errs.append(max(assert_layer_close(yp, yp_ref, f"layer {l} prefill"),
                        assert_layer_close(yd, yd_ref, f"layer {l} decode")))
        xp, xd = yp_ref, yd_ref
    # the head on the oracle's final hidden state of the decode position
    h = oracle.rms_norm(xd, full_w[("final_norm", -1)], shape.eps)
    ref_logits = oracle.linear(h, full_w[("lm_head", -1)], None, out_dtype=torch.float32)[0]
    nxt, lg = gm.head(xd.cuda())
    assert_bf16_logits(lg[0].cpu(), ref_logits, "head")
    top2 = torch.topk(ref_logits, 2).values
    if float(top2[0] - top2[1]) > 1e-2:
        assert int(nxt[0]) == int(torch.argmax(ref_logits))
    # the per-layer (norm) error does not grow with depth
    assert max(errs) <= 1e-2 and max(errs[-7:]) <= 2 * max(errs[:7]) + 1e-3, errs


def test_full_model_free_running_teacher_forced_tokens(full_w):
    shape = synth.QWEN2_1P5B
    prompt = synth.prompt_ids(shape, 6, 2003)
    om, gm = pair(shape, full_w, max_seq=64)
    ref_toks, ref_logits = om.generate(0, prompt, 3)
    toks, logits = gpu_generate(gm, prompt, 3, teacher=ref_toks)
    for i, (a, b) in enumerate(zip(logits, ref_logits)):
        assert_bf16_logits_free_running(a, b, f"step {i}")
    agree = sum(int(a == b) for a, b in zip(toks, ref_toks))
    assert agree >= len(toks) - 1, (toks, ref_toks)


def test_full_model_batched_decode_rows_match_oracle(full_w):
    """Batch of 4 sequences with different lengths; rows 0 and 3 against the oracle."""
    shape = synth.QWEN2_1P5B
    lens = [4, 7, 3, 5]
    prompts = [synth.prompt_ids(shape, n, 2004, seq=b) for b, n in enumerate(lens)]
    gm = q2.Model(shape, max_seq=32, max_batch=4)
    gm.load(full_w)
    nxt, lg = gm.prefill(torch.cat(prompts).cuda(), lens, want_logits=True)
    for b in (0, 3):
        om = oracle.OracleModel(shape, max_seq=32)
        om.load(full_w)
        t, l0 = om.forward(0, prompts[b])
        assert_bf16_logits_free_running(lg[b].cpu(), l0, f"prefill row {b}")
        feed = torch.tensor([t])
        _, l1 = om.forward(0, feed)
        ids = nxt.clone()
        ids[b] = t
        n2, lg2 = gm.decode_step(ids, want_logits=True)
        assert_bf16_logits_free_running(lg2[b].cpu(), l1, f"decode row {b}")
        for s in range(4):  # rewind all rows for the next sampled sequence
            gm.set_seq_len(s, lens[s])


# ------------------------------------------------- GPU self-consistency

@pytest.fixture(scope="module")
def mid():
    shape = dataclasses.replace(synth.QWEN2_1P5B, n_layers=4, vocab=32000)
    return shape, synth.model_weights(shape, 77, device="cuda")


def test_batched_prefill_matches_each_sequence_alone(mid):
    """Prefill of several sequences in one call: each sequence's attention
    reads its own K/V cache (sequence 1 has enough rows for the tensor-core
    attention, sequence 2 too few), so its logits match a prefill of that
    sequence alone."""
    shape, w = mid
    gm = q2.Model(shape, max_seq=128, max_batch=4)
    gm.load(w)
    lens = [20, 33, 7]
    prompts = [synth.prompt_ids(shape, n, 40 + b, seq=b) for b, n in enumerate(lens)]
    _, lg = gm.prefill(torch.cat(prompts).cuda(), lens, want_logits=True)
    lg = lg.cpu()
    for b, pr in enumerate(prompts):
        gm.reset_kv()
        _, one = gm.prefill(pr.cuda(), [lens[b]], want_logits=True)
        assert_bf16_logits(one[0].cpu(), lg[b], f"sequence {b} alone vs batched")
    gm.check_error()


def test_prefill_plus_decode_equals_longer_prefill(mid):
    shape, w = mid
    gm = q2.Model(shape, max_seq=128)
    gm.load(w)
    prompt = synth.prompt_ids(shape, 40, 5).cuda()
    n1 = gm.prefill(prompt, [40])
    _, la = gm.decode_step(n1, want_logits=True)
    gm.reset_kv()
    _, lb = gm.prefill(torch.cat([prompt, n1]), [41], want_logits=True)
    assert_bf16_logits(la[0].cpu(), lb[0].cpu(), "S+1 vs S+decode")


def test_reset_and_rerun_is_bit_identical_and_graphs_match_eager(mid):
    shape, w = mid
    gm = q2.Model(shape, max_seq=128, max_batch=2)
    gm.load(w)
    prompt = synth.prompt_ids(shape, 30, 6).cuda()

    def run(graphs):
        gm.reset_kv()
        gm.set_graphs(graphs)
        nxt = gm.prefill(torch.cat([prompt, prompt]), [30, 30])
        outs = []
        for _ in range(5):
            nxt, lg = gm.decode_step(nxt, want_logits=True)
            outs.append(lg.clone())
        return outs

    a, b, c = run(True), run(True), run(False)
    for x, y, z in zip(a, b, c):
        assert bits_equal(x, y) and bits_equal(x, z)
        assert bits_equal(x[0], x[1])  # identical sequences in one batch


# ---------------------------------------------------------- error paths

def test_capacity_and_index_errors(tiny_w):
    shape = TINY["shape"]
    gm = q2.Model(shape, max_seq=8)
    gm.load(tiny_w)
    with pytest.raises(q2.Q2Error) as e:
        gm.prefill(synth.prompt_ids(shape, 9, 1).cuda(), [9])
    assert e.value.status == "Q2_ERR_CAPACITY"
    nxt = gm.prefill(synth.prompt_ids(shape, 8, 1).cuda(), [8])
    with pytest.raises(q2.Q2Error) as e:
        gm.decode_step(nxt)
    assert e.value.status == "Q2_ERR_CAPACITY"
    gm.reset_kv()
    gm.decode_step(torch.tensor([shape.vocab + 5], device="cuda"))
    with pytest.raises(q2.Q2Error) as e:
        gm.check_error()
    assert e.value.status == "Q2_ERR_INDEX"
    gm.check_error()  # cleared
    with pytest.raises(q2.Q2Error) as e:
        gm.decode_step(torch.zeros(2, dtype=torch.int64, device="cuda"))  # batch > max_batch
    assert e.value.status == "Q2_ERR_CAPACITY"


def test_error_words_map_bits_to_statuses(tiny_w):
    """Each bit of a device error word has its own status: 1 (a token id
    outside the vocabulary) -> Q2_ERR_INDEX, 2 (a bounded wait ran out) ->
    Q2_ERR_TIMEOUT, which takes precedence; reading clears the word."""
    shape = TINY["shape"]
    gm = q2.Model(shape, max_seq=8)
    gm.load(tiny_w)
    for bits, status in ((1, "Q2_ERR_INDEX"), (2, "Q2_ERR_TIMEOUT"), (3, "Q2_ERR_TIMEOUT")):
        gm.test_raise_error(bits)
        with pytest.raises(q2.Q2Error) as e:
            gm.check_error()
        assert e.value.status == status
        if bits == 3:
            assert "token id" in str(e.value)
        gm.check_error()  # cleared
        q2.q2_test_raise_device_error(bits)
        with pytest.raises(q2.Q2Error) as e:
            q2.q2_check_device_error()
        assert e.value.status == status
        q2.q2_check_device_error()


def test_stream_step_wait_that_runs_out_is_reported_and_recoverable(mid):
    """A grid-phase counter of the streaming step that never completes (test
    hook: one arrival more than the grid makes): every wait on it gives up at
    its deadline, the step returns promptly, q2_model_check_error reports
    Q2_ERR_TIMEOUT, and after the hook is cleared the model decodes exactly as
    before."""
    import time

    shape, w = mid
    gm = q2.Model(shape, max_seq=64)
    gm.load(w)
    gm.set_decode_path("stream")
    prompt = synth.prompt_ids(shape, 12, 8).cuda()

    def run(n):
        gm.reset_kv()
        nxt = gm.prefill(prompt, [12])
        out = []
        for _ in range(n):
            nxt, lg = gm.decode_step(nxt, want_logits=True)
            out.append(lg.clone())
        return nxt, out

    _, ref = run(3)
    gm.check_error()
    gm.reset_kv()
    nxt = gm.prefill(prompt, [12])
    gm.test_set_wait_fault(5 * 1 + 2, 2_000_000)  # layer 1's o phase; 2 ms deadline
    gm.set_graphs(False)  # an eager launch: the time is the step's own
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    gm.decode_step(nxt)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    gm.set_graphs(True)
    with pytest.raises(q2.Q2Error) as e:
        gm.check_error()
    assert e.value.status == "Q2_ERR_TIMEOUT"
    assert dt < 0.15, dt  # one 2 ms deadline, not one per phase (nor the 200 ms default)
    gm.test_set_wait_fault(-1)
    _, again = run(3)
    gm.check_error()
    assert all(bits_equal(a, b) for a, b in zip(ref, again))


def test_decode_step_host_matches_device_path(tiny_w):
    shape = TINY["shape"]
    prompt = synth.prompt_ids(shape, 10, 3)
    _, gm = pair(shape, tiny_w, max_seq=64)
    nxt = gm.prefill(prompt.cuda(), [10])
    ids_h = torch.empty(1, dtype=torch.int64).pin_memory()
    out_h = torch.empty(1, dtype=torch.int64).pin_memory()
    ids_h[0] = int(nxt[0])
    dev = []
    host = []
    gm2 = q2.Model(shape, max_seq=64)
    gm2.load(tiny_w)
    n2 = gm2.prefill(prompt.cuda(), [10])
    for _ in range(5):
        gm.decode_step_host(ids_h, out_h)
        host.append(int(out_h[0]))
        ids_h[0] = out_h[0]
        n2 = gm2.decode_step(n2)
        dev.append(int(n2[0]))
    assert host == dev


# ------------------------------------------------ decode implementations

@pytest.mark.parametrize("B", [1, 3])
def test_decode_paths_agree_with_each_other_and_the_oracle(mid, B):
    """The streaming step (batch 1), the persistent step, the five-kernel fused
    path and the per-operator path compute the same decode steps
    (teacher-forced ids, B sequences)."""
    shape, w = mid
    lens = [20, 33, 7][:B]
    prompts = [synth.prompt_ids(shape, n, 40 + b, seq=b) for b, n in enumerate(lens)]
    feeds = [synth.uniform_ids(B, shape.vocab, 90 + i) for i in range(4)]
    gm = q2.Model(shape, max_seq=128, max_batch=4)
    gm.load(w)
    out = {}
    paths = ("stream", "persistent", "kernels", "generic") if B == 1 else ("persistent", "kernels", "generic")
    for path in paths:
        gm.set_decode_path(path)
        gm.reset_kv()
        gm.prefill(torch.cat(prompts).cuda(), lens)
        lg = []
        for f in feeds:
            _, l = gm.decode_step(f.cuda(), want_logits=True)
            lg.append(l.cpu())
        gm.check_error()
        out[path] = lg
    for path in paths[:-1]:
        for a, b in zip(out[path], out["generic"]):
            for r in range(B):
                assert_bf16_logits(a[r], b[r], f"{path} vs generic, row {r}")
    # and the first decode step of sequence 0 against the oracle
    om = oracle.OracleModel(shape, max_seq=128)
    om.load({k: t.cpu() for k, t in w.items()})
    om.forward(0, prompts[0])
    _, ref = om.forward(0, feeds[0][:1])
    for path in paths[:2]:
        assert_bf16_logits(out[path][0][0], ref, f"{path} vs oracle")


def test_persistent_step_is_deterministic_and_graph_safe(mid):
    shape, w = mid
    gm = q2.Model(shape, max_seq=64, max_batch=2)
    gm.load(w)
    gm.set_decode_path("persistent")
    prompt = synth.prompt_ids(shape, 12, 8).cuda()
    runs = []
    for graphs in (True, False, True):
        gm.reset_kv()
        gm.set_graphs(graphs)
        nxt = gm.prefill(torch.cat([prompt, prompt]), [12, 12])
        lgs = []
        for _ in range(6):
            nxt, lg = gm.decode_step(nxt, want_logits=True)
            lgs.append(lg.clone())
        runs.append(lgs)
        gm.check_error()
    for x, y, z in zip(*runs):
        assert bits_equal(x, y) and bits_equal(x, z)
    assert gm.get_seq_len(0) == gm.get_seq_len(1) == 18


def test_stream_step_is_deterministic_and_graph_safe(mid):
    """The batch-1 streaming step: graphs and eager launches, reruns after
    reset_kv, all bit-identical (fixed summation orders everywhere); the
    length advances once per step."""
    shape, w = mid
    gm = q2.Model(shape, max_seq=300, max_batch=1)
    gm.load(w)
    gm.set_decode_path("stream")
    prompt = synth.prompt_ids(shape, 150, 9).cuda()
    runs = []
    for graphs in (True, False, True):
        gm.reset_kv()
        gm.set_graphs(graphs)
        nxt = gm.prefill(prompt, [150])
        lgs, toks = [], []
        for _ in range(6):
            nxt, lg = gm.decode_step(nxt, want_logits=True)
            lgs.append(lg.clone())
            toks.append(int(nxt[0]))
        runs.append((lgs, toks))
        gm.check_error()
    for (x, tx), (y, ty) in zip(runs, runs[1:]):
        assert tx == ty
        assert all(bits_equal(a, b) for a, b in zip(x, y))
    assert gm.get_seq_len(0) == 156
    # the token is the argmax of the step's own logits (lowest index on ties)
    assert toks_match_argmax(runs[0][0], runs[0][1])


def toks_match_argmax(logits, toks):
    return all(int(torch.argmax(l[0]).item()) == t for l, t in zip(logits, toks))
