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

Each side runs in its own process (the library variant is chosen at import).
"""
import argparse
import json
import os
import subprocess
import sys

_ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _logits(mode: str, n: int) -> list:
    sys.path.insert(0, _ROOT)
    import synth
    import oracle
    shape = synth.QWEN2_1P5B
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
    ap.add_argument("mode", choices=["prompt", "cache"])
    ap.add_argument("--tokens", type=int, default=6)
    ap.add_argument("--context", type=int, default=32768)
    ap.add_argument("--child", action="store_true", help=argparse.SUPPRESS)
    a = ap.parse_args()
    n = a.tokens if a.mode == "prompt" else a.context
    if a.child:
        json.dump(_logits(a.mode, n), sys.stdout)
        return
    out = []
    for f32 in ("0", "1"):
        env = dict(os.environ, ORACLE_FP32_ACCUMULATION=f32)
        p = subprocess.run([sys.executable, "-m", "oracle.drift", a.mode, "--tokens", str(a.tokens),
                            "--context", str(a.context), "--child"], cwd=_ROOT, env=env,
                           capture_output=True, text=True, check=True)
        out.append(json.loads(p.stdout))
    import torch
    r, g = torch.tensor(out[0], dtype=torch.float64), torch.tensor(out[1], dtype=torch.float64)
    res = {"mode": a.mode, "n": n, "max_abs": float((g - r).abs().max()),
           "cosine": float(torch.nn.functional.cosine_similarity(g, r, dim=0))}
    print(json.dumps(res))


if __name__ == "__main__":
    main()
