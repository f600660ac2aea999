"""Hugging Face's Qwen2 (transformers, a library implementation) run in float64
on the CPU, as an independent pin of the oracle's model.  Test helper only."""

import torch

_NAMES = {
    "in_norm": "input_layernorm.weight",
    "q_w": "self_attn.q_proj.weight", "q_b": "self_attn.q_proj.bias",
    "k_w": "self_attn.k_proj.weight", "k_b": "self_attn.k_proj.bias",
    "v_w": "self_attn.v_proj.weight", "v_b": "self_attn.v_proj.bias",
    "o_w": "self_attn.o_proj.weight",
    "post_norm": "post_attention_layernorm.weight",
    "gate_w": "mlp.gate_proj.weight", "up_w": "mlp.up_proj.weight", "down_w": "mlp.down_proj.weight",
}


def build_hf(shape, weights, max_pos=4096):
    from transformers import Qwen2Config, Qwen2ForCausalLM
    cfg = Qwen2Config(vocab_size=shape.vocab, hidden_size=shape.hidden,
                      intermediate_size=shape.intermediate, num_hidden_layers=shape.n_layers,
                      num_attention_heads=shape.n_heads, num_key_value_heads=shape.n_kv_heads,
                      rms_norm_eps=shape.eps, rope_theta=shape.theta, tie_word_embeddings=False,
                      max_position_embeddings=max_pos, attn_implementation="eager")
    model = Qwen2ForCausalLM(cfg).double().eval()
    sd = {}
    for (name, layer), t in weights.items():
        if name == "embed":
            sd["model.embed_tokens.weight"] = t
        elif name == "lm_head":
            sd["lm_head.weight"] = t
        elif name == "final_norm":
            sd["model.norm.weight"] = t
        elif layer < shape.n_layers:
            sd[f"model.layers.{layer}.{_NAMES[name]}"] = t
    sd = {k: v.double() for k, v in sd.items()}
    missing, unexpected = model.load_state_dict(sd, strict=False)
    assert not unexpected, unexpected
    assert all("rotary" in m for m in missing), missing
    return model


@torch.no_grad()
def hf_logits(model, ids):
    """fp64 logits for every position of a 1-D id sequence."""
    return model(ids.reshape(1, -1)).logits[0]


@torch.no_grad()
def hf_greedy(model, prompt, n_decode):
    """Greedy decoding by re-running the whole sequence each step (no cache)."""
    ids = prompt.clone()
    chosen, logits = [], []
    for _ in range(n_decode + 1):
        lg = model(ids.reshape(1, -1)).logits[0, -1]
        nxt = int(torch.argmax(lg))
        chosen.append(nxt)
        logits.append(lg)
        ids = torch.cat([ids, torch.tensor([nxt])])
    return chosen, logits
