"""How far fp32 accumulation alone moves the model's logits.

Tolerance-derivation tool (test infrastructure, like the rest of oracle/):
runs the same forward through the oracle and through its fp32-accumulating
copy (built from the same source with -DORACLE_FP32_ACCUMULATION: the linear
and attention's weighted sum of V accumulate in float), on the same weights
and inputs, and prints the difference of the final logits.  A GPU path that
accumulates in fp32 cannot be expected to sit closer to the oracle than this;
the free-running tolerances of the tests are derived from it.

    python -m oracle.drift prompt  [--tokens 6]          # prefill of a short prompt
    python -m oracle.drift cache   [--context 32768]     # one token over an N(0,1) cache
    python -m oracle.drift layer   [--tokens 128] [--layer 0]
        # one decoder layer on the prompt's layer input (the embedding rows for
        # layer 0): the elementwise scaled error max |a - b| / max(|b|, rms(b))
        # and the relative norm error of the layer output (the layer bound's
        # two measures)
    python -m oracle.drift prefill-layers [--tokens 512]
        # every one of the 28 layers, each on its own seeded N(0,1) input of
        # `tokens` rows (the 512-token per-layer prefill check's inputs), the
        # output compared on the check's sampled rows: both measures per
        # layer and their maxima

Each side runs in its own process (the library variant is chosen at import).
"""
import argparse
import json
import os
import subprocess
import sys

_ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


# the rows the per-layer prefill check compares (both sides of the 64-row
# attention block and the 128/256-token GEMM tile edges, first and last row)
PREFILL_ROWS = [0, 1, 2, 63, 64, 65, 127, 128, 191, 192, 255, 256, 257, 319, 320, 383, 384, 447, 448, 449,
                500, 509, 510, 511]


def _prefill_layers(n: int) -> list:
    """The outputs of every layer on its own N(0,1) input, on PREFILL_ROWS."""
    sys.path.insert(0, os.path.join(_ROOT, "tests"))
    import dataclasses
    import torch
    import synth
    import layer_ref
    shape = synth.QWEN2_1P5B
    one = dataclasses.replace(shape, n_layers=1)
    seed = synth.WORKLOADS["qwen2-1.5b-b1-prompt512-decode128"]["seed"]
    w = synth.model_weights(shape, seed)
    rows = [r for r in PREFILL_ROWS if r < n]
    pool = layer_ref.make_pool()
    out = []
    for l in range(shape.n_layers):
        lw = layer_ref.layer_weights({(k, 0): t for (k, ll), t in w.items() if ll == l}, 0)
        x = synth.normal((n, shape.hidden), 1.0, synth.tensor_seed(seed, "prefill-input", l), "bf16")
        kc = torch.zeros((n, shape.n_kv_heads, shape.head_dim), dtype=torch.bfloat16)
        vc = torch.zeros_like(kc)
        y = layer_ref.layer_prefill(pool, one, lw, x, 0, kc, vc, rows=rows)
        out.append(y.double().reshape(-1).tolist())
    pool.shutdown()
    return out


def _logits(mode: str, n: int, layer: int = 0) -> list:
    sys.path.insert(0, _ROOT)
    import dataclasses
    import synth
    import oracle
    if mode == "prefill-layers":
        return _prefill_layers(n)
    shape = synth.QWEN2_1P5B
    if mode == "layer":
        w = synth.model_weights(shape, 1003)
        x = oracle.embedding(synth.prompt_ids(shape, n, 1003 + 500), w[("embed", -1)])
        for l in range(layer + 1):
            one = dataclasses.replace(shape, n_layers=1)
            om = oracle.OracleModel(one, max_seq=n)
            om.load({(k, 0): t for (k, ll), t in w.items() if ll == l})
            x = om.forward_hidden(0, x)
        return x.double().reshape(-1).tolist()
    if mode == "prompt":
        w = synth.model_weights(shape, 1003)
        om = oracle.OracleModel(shape, max_seq=n + 8)
        om.load(w)
        _, lg = om.forward(0, synth.prompt_ids(shape, n, 2003))
    else:
        w = synth.model_weights(shape, 1005)
        om = oracle.OracleModel(shape, max_seq=n + 8)
        om.load(w)
        for l in range(shape.n_layers):
            k, v = synth.kv_fill(shape, n, 1005, layer=l, seq=0)
            ok, ov = om.kv(l, 0)
            ok[:n] = k
            ov[:n] = v
        om.set_len(0, n)
        _, lg = om.forward(0, synth.uniform_ids(1, shape.vocab, 77))
    return lg.double().tolist()


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("mode", choices=["prompt", "cache", "layer", "prefill-layers"])
    ap.add_argument("--tokens", type=int, default=6)
    ap.add_argument("--context", type=int, default=32768)
    ap.add_argument("--layer", type=int, default=0)
    ap.add_argument("--child", action="store_true", help=argparse.SUPPRESS)
    a = ap.parse_args()
    n = a.context if a.mode == "cache" else a.tokens
    if a.child:
        json.dump(_logits(a.mode, n, a.layer), sys.stdout)
        return
    procs = []
    for f32 in ("0", "1"):  # the two builds side by side
        env = dict(os.environ, ORACLE_FP32_ACCUMULATION=f32)
        procs.append(subprocess.Popen([sys.executable, "-m", "oracle.drift", a.mode, "--tokens", str(a.tokens),
                                       "--context", str(a.context), "--layer", str(a.layer), "--child"],
                                      cwd=_ROOT, env=env, stdout=subprocess.PIPE, text=True))
    out = []
    for p in procs:
        o, _ = p.communicate()
        if p.returncode != 0:
            raise SystemExit(p.returncode)
        out.append(json.loads(o))
    import torch
    if a.mode == "prefill-layers":
        per = []
        for rl, gl in zip(out[0], out[1]):
            r, g = torch.tensor(rl, dtype=torch.float64), torch.tensor(gl, dtype=torch.float64)
            scale = torch.maximum(r.abs(), r.pow(2).mean().sqrt().expand_as(r))
            per.append((float(((g - r).abs() / scale).max()), float((g - r).norm() / r.norm())))
        print(json.dumps({"mode": a.mode, "n": n, "max_scaled": max(p[0] for p in per),
                          "rel_norm": max(p[1] for p in per),
                          "per_layer_max_scaled": [round(p[0], 5) for p in per],
                          "per_layer_rel_norm": [round(p[1], 5) for p in per]}))
        return
    r, g = torch.tensor(out[0], dtype=torch.float64), torch.tensor(out[1], dtype=torch.float64)
    res = {"mode": a.mode, "n": n, "max_abs": float((g - r).abs().max()),
           "cosine": float(torch.nn.functional.cosine_similarity(g, r, dim=0))}
    if a.mode == "layer":
        scale = torch.maximum(r.abs(), r.pow(2).mean().sqrt().expand_as(r))
        res["layer"] = a.layer
        res["max_scaled"] = float(((g - r).abs() / scale).max())
        res["rel_norm"] = float((g - r).norm() / r.norm())
    print(json.dumps(res))


if __name__ == "__main__":
    main()
