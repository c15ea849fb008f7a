"""Pins of the oracle's model variants (CPU only): the Llama-3.x RoPE frequency scaling
against Hugging Face's own implementation and its closed-form bands, and the Qwen3
QK-norm step against the Hugging Face Qwen3 model in float64.  Planted mistakes in
either must fail a pin."""
import math

import pytest
import torch

import oracle
import synth
from oracle import decode as od

F64 = torch.float64

SCALINGS = [(32.0, 1.0, 4.0, 8192), (8.0, 1.0, 4.0, 8192), (8.0, 1.0, 4.0, 64)]


def _hf_llama3_inv_freq(hd, theta, scaling):
    from transformers import LlamaConfig
    from transformers.modeling_rope_utils import ROPE_INIT_FUNCTIONS

    f, lo, hi, n = scaling
    cfg = LlamaConfig(hidden_size=4 * hd, num_attention_heads=4, head_dim=hd, rope_theta=theta,
                      max_position_embeddings=int(n * f),
                      rope_scaling={"rope_type": "llama3", "factor": f, "low_freq_factor": lo,
                                    "high_freq_factor": hi, "original_max_position_embeddings": n})
    inv, attention_factor = ROPE_INIT_FUNCTIONS["llama3"](cfg, "cpu")
    assert attention_factor == 1.0
    return inv.to(F64)


@pytest.mark.parametrize("hd, theta", [(64, 5e5), (128, 5e5), (64, 1e4)])
@pytest.mark.parametrize("scaling", SCALINGS)
def test_rope_scaling_matches_huggingface_llama3(hd, theta, scaling):
    ours = od.rope_inv_freq(hd, theta, scaling)
    ref = _hf_llama3_inv_freq(hd, theta, scaling)  # computed in float32 there
    assert torch.allclose(ours, ref, rtol=2e-6, atol=0)


@pytest.mark.parametrize("scaling", SCALINGS)
def test_rope_scaling_bands(scaling):
    factor, low, high, n = scaling
    base = od.rope_inv_freq(128, 5e5)
    out = od.rope_inv_freq(128, 5e5, scaling)
    seen = set()
    for b, o in zip(base.tolist(), out.tolist()):
        w = 2 * math.pi / b
        if w < n / high:
            assert o == b
            seen.add("high")
        elif w > n / low:
            assert o == b / factor
            seen.add("low")
        else:
            assert b / factor <= o <= b
            seen.add("mid")
    assert "low" in seen and "high" in seen
    assert od.rope_inv_freq(128, 5e5, (1.0, low, high, n)).equal(base)  # factor 1: no scaling


def test_scaled_rope_is_still_a_rotation():
    v = torch.randn(128, dtype=F64, generator=torch.Generator().manual_seed(3))
    for pos in (0, 7, 5000):
        r = od.rope(v, pos, 5e5, SCALINGS[0])
        assert abs(float(r.norm() - v.norm())) < 1e-12
    assert torch.equal(od.rope(v, 0, 5e5, SCALINGS[0]), v)


def _swapped_bands(hd, theta, scaling):
    f, lo, hi, n = scaling
    return _ORIG_INV(hd, theta, (f, hi, lo, n)) if scaling else _ORIG_INV(hd, theta)


def _all_divided(hd, theta, scaling):
    base = _ORIG_INV(hd, theta)
    return base / scaling[0] if scaling else base


_ORIG_INV = od.rope_inv_freq


@pytest.mark.parametrize("mutant", [_swapped_bands, _all_divided])
def test_planted_scaling_mistakes_are_caught(mutant):
    ours = mutant(128, 5e5, SCALINGS[0])
    ref = _hf_llama3_inv_freq(128, 5e5, SCALINGS[0])
    assert not torch.allclose(ours, ref, rtol=2e-6, atol=0)


# --- Qwen3 QK-norm -------------------------------------------------------------------------

QWEN_TINY = synth.scaled_model(synth.QWEN3_0_6B, name="qwen3-tiny", n_layers=2, hidden=256, n_heads=4,
                               n_kv_heads=2, head_dim=128, ffn=512, vocab=1000)


def _hf_qwen3_reference(m, wts, kv, toks, lens):
    """Logits, per-layer hidden states and new K/V from the Hugging Face Qwen3 model in float64."""
    from transformers import Qwen3Config, Qwen3ForCausalLM
    from transformers.cache_utils import DynamicCache

    cfg = Qwen3Config(vocab_size=m.vocab, hidden_size=m.hidden, intermediate_size=m.ffn,
                      num_hidden_layers=m.n_layers, num_attention_heads=m.n_heads,
                      num_key_value_heads=m.n_kv_heads, head_dim=m.head_dim, rms_norm_eps=m.rms_eps,
                      rope_theta=m.rope_theta, tie_word_embeddings=m.tied, max_position_embeddings=8192,
                      attention_bias=False, use_sliding_window=False)
    cfg._attn_implementation = "sdpa"
    model = Qwen3ForCausalLM(cfg).to(F64).eval()
    hd = m.head_dim
    inv64 = 1.0 / (m.rope_theta ** (torch.arange(0, hd, 2, dtype=F64) / hd))

    def _rot64(x, position_ids):
        freqs = position_ids[:, :, None].to(F64) * inv64[None, None, :]
        emb = torch.cat((freqs, freqs), dim=-1)
        return emb.cos().to(x.dtype), emb.sin().to(x.dtype)

    model.model.rotary_emb.forward = _rot64
    for mod in model.modules():
        if type(mod).__name__ == "Qwen3RMSNorm":
            mod.forward = (lambda mm: (lambda h: torch.nn.functional.rms_norm(
                h, (h.shape[-1],), weight=mm.weight, eps=mm.variance_epsilon)))(mod)
    sd = {"model.embed_tokens.weight": wts["embed"], "model.norm.weight": wts["final_norm"],
          "lm_head.weight": wts["lm_head"]}
    names = {"wq": "self_attn.q_proj", "wk": "self_attn.k_proj", "wv": "self_attn.v_proj",
             "wo": "self_attn.o_proj", "w_gate": "mlp.gate_proj", "w_up": "mlp.up_proj",
             "w_down": "mlp.down_proj", "attn_norm": "input_layernorm",
             "mlp_norm": "post_attention_layernorm", "q_norm": "self_attn.q_norm", "k_norm": "self_attn.k_norm"}
    for li, lw in enumerate(wts["layers"]):
        for k, v in lw.items():
            sd[f"model.layers.{li}.{names[k]}.weight"] = v
    missing, unexpected = model.load_state_dict({k: v.to(F64) for k, v in sd.items()}, strict=False)
    assert not unexpected and all("rotary" in k for k in missing), (missing, unexpected)
    res = []
    P = m.page_size
    for t, p in zip(toks, lens):
        cache = DynamicCache()
        for li in range(m.n_layers):
            Ks = od._gather_prior(kv.k_pool[li], kv.page_table[len(res)], p, P)[None]
            Vs = od._gather_prior(kv.v_pool[li], kv.page_table[len(res)], p, P)[None]
            cache.update(Ks, Vs, li)
        with torch.no_grad():
            o = model(input_ids=torch.tensor([[t]]), position_ids=torch.tensor([[p]]),
                      cache_position=torch.tensor([p]), past_key_values=cache, use_cache=True,
                      output_hidden_states=True)
        knew = torch.stack([cache.layers[li].keys[0, :, p, :] for li in range(m.n_layers)])
        vnew = torch.stack([cache.layers[li].values[0, :, p, :] for li in range(m.n_layers)])
        hs = torch.stack([h[0, 0] for h in o.hidden_states[:-1]])
        res.append((o.logits[0, 0], hs, knew, vnew))
    return res


def _worst(out, ref):
    worst = 0.0
    for i, (logits, hs, knew, vnew) in enumerate(ref):
        worst = max(worst, float((out["logits"][i] - logits).abs().max()))
        worst = max(worst, float((out["hidden"][:hs.shape[0], i] - hs).abs().max()))
        worst = max(worst, float((out["k_new_exact"][:, i] - knew).abs().max()))
        worst = max(worst, float((out["v_new_exact"][:, i] - vnew).abs().max()))
    return worst


@pytest.fixture(scope="module")
def hf_qwen():
    m = QWEN_TINY
    lens = [0, 15, 16, 47]
    wts = synth.make_weights(m, gain_std=0.2)
    kv = synth.make_kv_cache(m, lens)
    toks = synth.token_ids(m, len(lens), tag="pins")
    return m, wts, kv, toks, lens, _hf_qwen3_reference(m, wts, kv, toks, lens)


def test_qk_norm_step_matches_huggingface_qwen3_float64(hf_qwen):
    m, wts, kv, toks, lens, ref = hf_qwen
    assert m.head_dim * m.n_heads != m.hidden  # q_dim != hidden, as in Qwen3-0.6B
    out = oracle.decode_step(m, wts, kv.k_pool, kv.v_pool, kv.page_table, toks, lens, round_new_kv=False)
    assert _worst(out, ref) < 1e-10


def _rmsnorm_skipping_heads(orig):
    return lambda x, g, e: x if x.shape[-1] == QWEN_TINY.head_dim else orig(x, g, e)


def _rmsnorm_heads_without_gain(orig):
    return lambda x, g, e: orig(x, torch.ones_like(g) if x.shape[-1] == QWEN_TINY.head_dim else g, e)


def _rmsnorm_heads_over_all_heads(orig):
    def f(x, g, e):
        if x.shape[-1] != QWEN_TINY.head_dim:
            return orig(x, g, e)
        flat = x.reshape(x.shape[0], -1)
        ms = (flat * flat).mean(-1, keepdim=True)[:, :, None]
        return x / torch.sqrt(ms + e) * g
    return f


@pytest.mark.parametrize("make", [_rmsnorm_skipping_heads, _rmsnorm_heads_without_gain,
                                  _rmsnorm_heads_over_all_heads])
def test_planted_qk_norm_mistakes_are_caught(make, hf_qwen, monkeypatch):
    m, wts, kv, toks, lens, ref = hf_qwen
    monkeypatch.setattr(od, "rmsnorm", make(od.rmsnorm))
    out = oracle.decode_step(m, wts, kv.k_pool, kv.v_pool, kv.page_table, toks, lens, round_new_kv=False)
    assert _worst(out, ref) > 1e-6
