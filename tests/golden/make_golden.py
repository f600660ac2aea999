"""Write tiny_f32_greedy.json from the oracle alone (regression fixture).

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402

WORKLOAD = "tiny-2l-f32-prompt16-decode16"


def main():
    wl = synth.WORKLOADS[WORKLOAD]
    shape, seed = wl["shape"], wl["seed"]
    w = synth.model_weights(shape, seed)
    prompt = synth.prompt_ids(shape, wl["prompt"], seed)
    om = oracle.OracleModel(shape, max_seq=64)
    om.load(w)
    tokens, logits = om.generate(0, prompt, wl["decode"])
    out = {
        "workload": WORKLOAD,
        "source": "oracle/ only (make_golden.py)",
        "prompt": prompt.tolist(),
        "greedy_tokens": tokens,
        "first_logits_head": [float(x) for x in logits[0][:8]],
        "last_logits_head": [float(x) for x in logits[-1][:8]],
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_f32_greedy.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(path)


if __name__ == "__main__":
    main()
