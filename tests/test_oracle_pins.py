"""Pins of the float64 oracle to things other than itself (CPU only).

Each pin is a closed form, an invariant, a brute-force loop on tiny inputs, or a
special case that reduces to an independent library routine (torch's
scaled-dot-product attention, rms_norm and silu; the Hugging Face Llama model in
float64).  ``test_planted_mistakes_are_caught`` plants plausible mistakes in the
oracle and checks that the pins reject every one of them.
"""
import math

import pytest
import torch

import oracle
import synth
from oracle import decode as od

F64 = torch.float64


def _gen(seed):
    g = torch.Generator()
    g.manual_seed(seed)
    return g


# --- RMSNorm -------------------------------------------------------------------------------

def test_rmsnorm_unit_rms_closed_form():
    g = _gen(0)
    for d in (8, 256, 4096):
        x = torch.randn(3, d, generator=g, dtype=F64) * 3.0
        eps = 1e-5
        y = oracle.rmsnorm(x, torch.ones(d, dtype=F64), eps)
        m = (x * x).mean(-1)
        rms_y = torch.sqrt((y * y).mean(-1))
        assert torch.allclose(rms_y, torch.sqrt(m / (m + eps)), rtol=1e-13, atol=0)


def test_rmsnorm_matches_torch_rms_norm():
    g = _gen(1)
    x = torch.randn(4, 576, generator=g, dtype=F64)
    gain = 1.0 + 0.1 * torch.randn(576, generator=g, dtype=F64)
    ref = torch.nn.functional.rms_norm(x, (576,), weight=gain, eps=1e-5)
    assert torch.allclose(oracle.rmsnorm(x, gain, 1e-5), ref, rtol=1e-13, atol=1e-15)


# --- RoPE --------------------------------------------------------------------------------

def test_rope_basis_vectors_rotate_half_pairing():
    # hd = 4, theta = 10^4: inv_freq = (1, 10^-2).  Dimension j pairs with j + 2.
    e = torch.eye(4, dtype=F64)
    c1, s1 = math.cos(1.0), math.sin(1.0)
    assert torch.allclose(oracle.rope(e[0], 1, 1e4), torch.tensor([c1, 0, s1, 0], dtype=F64), atol=1e-15)
    assert torch.allclose(oracle.rope(e[2], 1, 1e4), torch.tensor([-s1, 0, c1, 0], dtype=F64), atol=1e-15)
    c, s = math.cos(0.03), math.sin(0.03)
    assert torch.allclose(oracle.rope(e[1], 3, 1e4), torch.tensor([0, c, 0, s], dtype=F64), atol=1e-15)
    assert torch.allclose(oracle.rope(e[3], 3, 1e4), torch.tensor([0, -s, 0, c], dtype=F64), atol=1e-15)


def test_rope_identity_at_zero_and_norm_preservation():
    g = _gen(2)
    for hd in (64, 128):
        v = torch.randn(5, hd, generator=g, dtype=F64)
        assert torch.equal(oracle.rope(v, 0, 5e5), v)
        for pos in (1, 17, 4095):
            r = oracle.rope(v, pos, 5e5)
            half = hd // 2
            pair_in = v[:, :half] ** 2 + v[:, half:] ** 2
            pair_out = r[:, :half] ** 2 + r[:, half:] ** 2
            assert torch.allclose(pair_in, pair_out, rtol=1e-12, atol=1e-14)


def test_rope_relative_position_identity():
    g = _gen(3)
    for hd, theta in ((64, 1e4), (128, 5e5)):
        q = torch.randn(hd, generator=g, dtype=F64)
        k = torch.randn(hd, generator=g, dtype=F64)
        for m_, n_ in ((0, 5), (7, 300), (1000, 4000), (33, 33)):
            lhs = torch.dot(oracle.rope(q, m_, theta), oracle.rope(k, n_, theta))
            rhs = torch.dot(q, oracle.rope(k, n_ - m_, theta)) if n_ >= m_ else \
                torch.dot(oracle.rope(q, m_ - n_, theta), k)
            assert abs(float(lhs - rhs)) < 1e-9 * (1 + abs(float(lhs)))


def test_rope_inv_freq_closed_form():
    f = oracle.rope_inv_freq(128, 5e5)
    assert f[0] == 1.0
    assert math.isclose(float(f[32]), 5e5 ** -0.5, rel_tol=1e-14)
    assert math.isclose(float(f[63]), 5e5 ** (-126 / 128), rel_tol=1e-14)


# --- attention ---------------------------------------------------------------------------

def test_attention_single_key_returns_value_exactly():
    g = _gen(4)
    q = torch.randn(4, 64, generator=g, dtype=F64)
    K = torch.randn(1, 64, generator=g, dtype=F64)
    V = torch.randn(1, 64, generator=g, dtype=F64)
    assert torch.equal(oracle.attention(q, K, V), V.expand(4, 64))


def test_attention_equal_keys_give_mean_value():
    g = _gen(5)
    q = torch.randn(2, 32, generator=g, dtype=F64)
    K = torch.randn(1, 32, generator=g, dtype=F64).expand(9, 32)
    V = torch.randn(9, 32, generator=g, dtype=F64)
    assert torch.allclose(oracle.attention(q, K, V), V.mean(0).expand(2, 32), rtol=1e-13, atol=1e-14)


def _brute_attention(q, K, V):
    """Explicit scalar loops: scores, max, exponentials, weighted sum."""
    g_, hd = q.shape
    n = K.shape[0]
    out = [[0.0] * hd for _ in range(g_)]
    for h in range(g_):
        s = []
        for t in range(n):
            acc = 0.0
            for j in range(hd):
                acc += float(q[h, j]) * float(K[t, j])
            s.append(acc / math.sqrt(hd))
        mx = max(s)
        e = [math.exp(v - mx) for v in s]
        tot = sum(e)
        for j in range(hd):
            out[h][j] = sum(e[t] * float(V[t, j]) for t in range(n)) / tot
    return torch.tensor(out, dtype=F64)


def test_attention_matches_brute_force_loops():
    g = _gen(6)
    for n in (1, 2, 7, 20):
        q = torch.randn(3, 8, generator=g, dtype=F64) * 2
        K = torch.randn(n, 8, generator=g, dtype=F64)
        V = torch.randn(n, 8, generator=g, dtype=F64)
        assert torch.allclose(oracle.attention(q, K, V), _brute_attention(q, K, V), rtol=1e-12, atol=1e-12)


def test_attention_matches_sdpa():
    g = _gen(7)
    q = torch.randn(4, 128, generator=g, dtype=F64)
    K = torch.randn(300, 128, generator=g, dtype=F64)
    V = torch.randn(300, 128, generator=g, dtype=F64)
    ref = torch.nn.functional.scaled_dot_product_attention(q[None, :, None, :].transpose(1, 2),
                                                           K[None, None], V[None, None])
    ref = ref[0, 0]  # [g][hd]
    assert torch.allclose(oracle.attention(q, K, V), ref, rtol=1e-12, atol=1e-13)


def test_split_k_combine_equals_unsplit_for_every_split():
    g = _gen(8)
    n = 13
    q = torch.randn(4, 16, generator=g, dtype=F64) * 3
    K = torch.randn(n, 16, generator=g, dtype=F64)
    V = torch.randn(n, 16, generator=g, dtype=F64)
    full = oracle.attention(q, K, V)
    for cut1 in range(1, n):
        for cut2 in range(cut1 + 1, n + 1):
            spans = [(0, cut1), (cut1, cut2)] + ([(cut2, n)] if cut2 < n else [])
            parts = [oracle.attention_partial(q, K[a:b], V[a:b]) for a, b in spans]
            assert torch.allclose(oracle.combine_partials(parts), full, rtol=1e-12, atol=1e-13)


def test_gqa_mapping():
    assert [oracle.kv_head_of(h, 32, 8) for h in range(8)] == [0, 0, 0, 0, 1, 1, 1, 1]
    assert [oracle.kv_head_of(h, 9, 3) for h in range(9)] == [0, 0, 0, 1, 1, 1, 2, 2, 2]
    assert [oracle.kv_head_of(h, 40, 40) for h in range(40)] == list(range(40))  # MHA


# --- small helpers -----------------------------------------------------------------------

def test_silu_matches_torch():
    z = torch.linspace(-30, 30, 1001, dtype=F64)
    assert torch.allclose(oracle.silu(z), torch.nn.functional.silu(z), rtol=1e-14, atol=1e-300)


def test_bf16_rne_is_nearest_with_ties_to_even():
    g = _gen(9)
    x = torch.randn(20000, generator=g, dtype=F64) * torch.exp(torch.randn(20000, generator=g, dtype=F64) * 4)
    r = oracle.bf16_rne(x)
    # r must be representable in bf16 ...
    assert torch.equal(r.to(torch.float32).to(torch.bfloat16).to(F64), r)
    # ... and nearest: both bf16 neighbours of x are no closer (brute force on the bit grid).
    bits = r.to(torch.float32).view(torch.int32)
    up = (bits + (1 << 16)).view(torch.float32).to(F64)
    dn = (bits - (1 << 16)).view(torch.float32).to(F64)
    d0 = (x - r).abs()
    assert bool((d0 <= (x - up).abs()).all()) and bool((d0 <= (x - dn).abs()).all())
    # exact halfway points go to the even mantissa
    one = torch.tensor([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8)], dtype=F64)
    assert oracle.bf16_rne(one).tolist() == [1.0, 1.0 + 4 * 2.0 ** -8, -1.0]


def test_bf16_rne_agrees_with_torch_on_float32_inputs():
    g = _gen(10)
    x32 = torch.randn(50000, generator=g, dtype=torch.float32) * 10
    assert torch.equal(oracle.bf16_rne(x32.to(F64)), x32.to(torch.bfloat16).to(F64))


def test_argmax_lowest_index_on_ties():
    v = torch.tensor([0.5, 2.0, -1.0, 2.0, 2.0], dtype=F64)
    assert oracle.argmax_lowest(v) == 1


# --- byte count (§2.2) ---------------------------------------------------------------------

@pytest.mark.parametrize("wname", ["tiny-b1", "smollm2-135m-b1"])
def test_model_bytes_equals_tensor_nbytes(wname):
    w = synth.WORKLOADS[wname]
    m = w.model
    lens = w.context_lengths()
    wts = synth.make_weights(m)
    nb = sum(t.numel() * t.element_size() for lw in wts["layers"] for t in lw.values())
    nb += wts["final_norm"].numel() * 2 + wts["lm_head"].numel() * 2
    nb += w.batch * m.hidden * 2  # gathered embedding rows
    kv = synth.make_kv_cache(m, lens)
    per_tok = kv.k_pool[0, 0, :, 0, :].numel() * 2 * 2 * m.n_layers
    nb += sum(lens) * per_tok
    assert oracle.model_bytes(m, lens) == nb


def test_model_bytes_closed_forms():
    # tiny: 2 layers; weight elements 2*(2*256 + 3*256*256 ... ) spelled out by hand.
    d, q, kv, F, V, L = 256, 256, 128, 688, 2048, 2
    layer = 2 * d + q * d + 2 * kv * d + d * q + 3 * F * d
    tiny = 2 * (L * layer + d + V * d + 1 * d + 64 * L * 2 * kv)
    assert oracle.model_bytes(synth.TINY, [64]) == tiny
    # Llama-3-8B b1 at 2048 prior entries: 15.28 GB, b8: 17.16 GB
    assert round(oracle.model_bytes(synth.LLAMA3_8B, [2048]) / 1e9, 2) == 15.28
    assert round(oracle.model_bytes(synth.LLAMA3_8B, [2048] * 8) / 1e9, 2) == 17.16


# --- the whole step ----------------------------------------------------------------------

def _tiny_inputs(gain_std=0.1, lens=(5, 64, 16, 33)):
    m = synth.TINY
    wts = synth.make_weights(m, gain_std=gain_std)
    kv = synth.make_kv_cache(m, list(lens))
    toks = synth.token_ids(m, len(lens), tag="pins")
    return m, wts, kv, toks, list(lens)


def test_embedding_gather_is_exact():
    m, wts, kv, toks, lens = _tiny_inputs()
    out = oracle.decode_step(m, wts, kv.k_pool, kv.v_pool, kv.page_table, toks, lens, layers=0)
    for i, t in enumerate(toks):
        assert torch.equal(out["hidden"][0, i], wts["embed"][t].to(F64))


def test_zero_output_projections_make_layer_identity():
    m, wts, kv, toks, lens = _tiny_inputs()
    for lw in wts["layers"]:
        lw["wo"] = torch.zeros_like(lw["wo"])
        lw["w_down"] = torch.zeros_like(lw["w_down"])
    out = oracle.decode_step(m, wts, kv.k_pool, kv.v_pool, kv.page_table, toks, lens)
    for li in range(m.n_layers + 1):
        assert torch.equal(out["hidden"][li], out["hidden"][0])


def test_sequences_are_independent_in_a_ragged_batch():
    m, wts, kv, toks, lens = _tiny_inputs()
    full = oracle.decode_step(m, wts, kv.k_pool, kv.v_pool, kv.page_table, toks, lens)
    for i in range(len(toks)):
        one = oracle.decode_step(m, wts, kv.k_pool, kv.v_pool, kv.page_table[i:i + 1], toks[i:i + 1],
                                 lens[i:i + 1])
        # BLAS may block a batched product differently: equal up to float64 rounding
        assert torch.allclose(one["logits"][0], full["logits"][i], rtol=1e-12, atol=1e-13)
        assert torch.allclose(one["hidden"][:, 0], full["hidden"][:, i], rtol=1e-12, atol=1e-13)


def test_physical_page_placement_does_not_matter():
    m, wts, kv, toks, lens = _tiny_inputs()
    base = oracle.decode_step(m, wts, kv.k_pool, kv.v_pool, kv.page_table, toks, lens)
    perm = torch.randperm(kv.num_pages, generator=_gen(11))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(kv.num_pages)
    k2 = torch.empty_like(kv.k_pool)
    v2 = torch.empty_like(kv.v_pool)
    k2[:, perm] = kv.k_pool
    v2[:, perm] = kv.v_pool
    t2 = kv.page_table.clone()
    t2[t2 >= 0] = perm[t2[t2 >= 0].long()].to(torch.int32)
    moved = oracle.decode_step(m, wts, k2, v2, t2, toks, lens)
    assert torch.equal(moved["logits"], base["logits"])
    assert [perm[p].item() for p, _ in base["slots"]] == [p for p, _ in moved["slots"]]


def test_new_entry_slot_addresses():
    m, wts, kv, toks, lens = _tiny_inputs()
    out = oracle.decode_step(m, wts, kv.k_pool, kv.v_pool, kv.page_table, toks, lens, layers=1)
    for i, s in enumerate(lens):
        assert out["slots"][i] == (int(kv.page_table[i, s // 16]), s % 16)


def _hf_reference(m, wts, kv, toks, lens, gains=True):
    """Logits, per-layer hidden states and new K/V from the Hugging Face Llama model in float64."""
    from transformers import LlamaConfig, LlamaForCausalLM
    from transformers.cache_utils import DynamicCache

    cfg = LlamaConfig(vocab_size=m.vocab, hidden_size=m.hidden, intermediate_size=m.ffn,
                      num_hidden_layers=m.n_layers, num_attention_heads=m.n_heads,
                      num_key_value_heads=m.n_kv_heads, head_dim=m.head_dim, rms_norm_eps=m.rms_eps,
                      rope_theta=m.rope_theta, tie_word_embeddings=m.tied,
                      max_position_embeddings=8192, attention_bias=False, mlp_bias=False)
    cfg._attn_implementation = "sdpa"  # the eager path takes its softmax in float32
    model = LlamaForCausalLM(cfg).to(F64).eval()
    # The HF rotary module forces float32 cos/sin; give it the same angles in float64 so
    # the comparison is float64 throughout (its rotate-half application is unchanged).
    rot = model.model.rotary_emb
    hd = m.head_dim
    inv64 = 1.0 / (m.rope_theta ** (torch.arange(0, hd, 2, dtype=F64) / hd))

    def _rot64(x, position_ids):
        freqs = position_ids[:, :, None].to(F64) * inv64[None, None, :]
        emb = torch.cat((freqs, freqs), dim=-1)
        return emb.cos().to(x.dtype), emb.sin().to(x.dtype)

    rot.forward = _rot64
    # Likewise the HF RMSNorm computes in float32; run it as torch's rms_norm in float64.
    for mod in model.modules():
        if type(mod).__name__ == "LlamaRMSNorm":
            mod.forward = (lambda mm: (lambda h: torch.nn.functional.rms_norm(
                h, (h.shape[-1],), weight=mm.weight, eps=mm.variance_epsilon)))(mod)
    sd = {"model.embed_tokens.weight": wts["embed"], "model.norm.weight": wts["final_norm"],
          "lm_head.weight": wts["lm_head"]}
    names = {"wq": "self_attn.q_proj", "wk": "self_attn.k_proj", "wv": "self_attn.v_proj",
             "wo": "self_attn.o_proj", "w_gate": "mlp.gate_proj", "w_up": "mlp.up_proj",
             "w_down": "mlp.down_proj", "attn_norm": "input_layernorm",
             "mlp_norm": "post_attention_layernorm"}
    for li, lw in enumerate(wts["layers"]):
        for k, v in lw.items():
            sd[f"model.layers.{li}.{names[k]}.weight"] = v
    model.load_state_dict({k: v.to(F64) for k, v in sd.items()}, strict=False)
    res = []
    P = m.page_size
    for i, (t, p) in enumerate(zip(toks, lens)):
        cache = DynamicCache()
        for li in range(m.n_layers):
            Ks = od._gather_prior(kv.k_pool[li], kv.page_table[i], p, P)[None]
            Vs = od._gather_prior(kv.v_pool[li], kv.page_table[i], p, P)[None]
            cache.update(Ks, Vs, li)
        with torch.no_grad():
            o = model(input_ids=torch.tensor([[t]]), position_ids=torch.tensor([[p]]),
                      cache_position=torch.tensor([p]), past_key_values=cache, use_cache=True,
                      output_hidden_states=True)
        knew = torch.stack([cache.layers[li].keys[0, :, p, :] for li in range(m.n_layers)])
        vnew = torch.stack([cache.layers[li].values[0, :, p, :] for li in range(m.n_layers)])
        hs = torch.stack([h[0, 0] for h in o.hidden_states[:-1]])  # last entry is after the final norm
        res.append((o.logits[0, 0], hs, knew, vnew))
    return res


def _compare_to_hf(out, ref):
    worst = 0.0
    for i, (logits, hs, knew, vnew) in enumerate(ref):
        worst = max(worst, float((out["logits"][i] - logits).abs().max()))
        worst = max(worst, float((out["hidden"][:hs.shape[0], i] - hs).abs().max()))
        worst = max(worst, float((out["k_new_exact"][:, i] - knew).abs().max()))
        worst = max(worst, float((out["v_new_exact"][:, i] - vnew).abs().max()))
    return worst


@pytest.fixture(scope="module")
def hf_tiny():
    m, wts, kv, toks, lens = _tiny_inputs(gain_std=0.1)
    return m, wts, kv, toks, lens, _hf_reference(m, wts, kv, toks, lens)


def test_decode_step_matches_huggingface_llama_float64(hf_tiny):
    m, wts, kv, toks, lens, ref = hf_tiny
    out = oracle.decode_step(m, wts, kv.k_pool, kv.v_pool, kv.page_table, toks, lens, round_new_kv=False)
    assert _compare_to_hf(out, ref) < 1e-10


def test_rounding_the_new_entry_is_a_small_perturbation(hf_tiny):
    m, wts, kv, toks, lens, ref = hf_tiny
    out = oracle.decode_step(m, wts, kv.k_pool, kv.v_pool, kv.page_table, toks, lens)
    err = _compare_to_hf(out, ref)
    assert 0 < err < 5e-2


def _interleaved_rope(v, pos, theta, scaling=None):
    hd = v.shape[-1]
    ang = float(pos) * od.rope_inv_freq(hd, theta, scaling)
    c, s = torch.cos(ang), torch.sin(ang)
    x1, x2 = v[..., 0::2], v[..., 1::2]
    out = torch.empty_like(v)
    out[..., 0::2] = x1 * c - x2 * s
    out[..., 1::2] = x2 * c + x1 * s
    return out


MUTANTS = {
    "rope-interleaved": ("rope", lambda orig: _interleaved_rope),
    "rope-pos-plus-one": ("rope", lambda orig: (lambda v, p, t, s=None: orig(v, p + 1, t, s))),
    "rope-sign": ("rope", lambda orig: (lambda v, p, t, s=None: orig(v, -p, t, s))),
    "gqa-modulo": ("kv_head_of", lambda orig: (lambda h, nq, nkv: h % nkv)),
    "no-score-scale": ("attention", lambda orig: (lambda q, K, V: orig(q * math.sqrt(q.shape[-1]), K, V))),
    "eps-outside-sqrt": ("rmsnorm", lambda orig: (lambda x, g, e: x / (torch.sqrt((x * x).mean(-1, keepdim=True)) + e) * g)),
    "norm-no-gain": ("rmsnorm", lambda orig: (lambda x, g, e: orig(x, torch.ones_like(g), e))),
    "silu-as-sigmoid": ("silu", lambda orig: (lambda z: 1.0 / (1.0 + torch.exp(-z)))),
    "new-token-not-attended": ("attention", lambda orig: (lambda q, K, V: orig(q, K[:-1], V[:-1]) if K.shape[0] > 1 else orig(q, K, V))),
    "transposed-kv-gather": ("_gather_prior", lambda orig: (lambda pool_l, row, n, P: orig(pool_l, row, n, P).flip(0))),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes_are_caught(name, hf_tiny, monkeypatch):
    m, wts, kv, toks, lens, ref = hf_tiny
    attr, make = MUTANTS[name]
    monkeypatch.setattr(od, attr, make(getattr(od, attr)))
    out = oracle.decode_step(m, wts, kv.k_pool, kv.v_pool, kv.page_table, toks, lens, round_new_kv=False)
    assert _compare_to_hf(out, ref) > 1e-6, f"mutant {name} slipped past the Hugging Face pin"


SMALL_SHAPES = {
    # multi-head (n_kv == n_heads) with head_dim 128, like the 13B shape
    "mha-hd128": synth.scaled_model(synth.LLAMA2_13B, name="mha-hd128", n_layers=2, hidden=256,
                                    n_heads=2, n_kv_heads=2, ffn=512, vocab=1000),
    # tied embeddings with 3 query heads per KV head, like the SmolLM2 shape
    "tied-g3": synth.scaled_model(synth.SMOLLM2_135M, name="tied-g3", n_layers=3, hidden=192,
                                  n_heads=3, n_kv_heads=1, ffn=384, vocab=1000),
}


@pytest.mark.parametrize("shape", sorted(SMALL_SHAPES))
def test_other_shapes_match_huggingface_llama_float64(shape):
    m = SMALL_SHAPES[shape]
    lens = [0, 15, 16, 47]
    wts = synth.make_weights(m, gain_std=0.1)
    kv = synth.make_kv_cache(m, lens)
    toks = synth.token_ids(m, len(lens), tag="pins")
    ref = _hf_reference(m, wts, kv, toks, lens)
    out = oracle.decode_step(m, wts, kv.k_pool, kv.v_pool, kv.page_table, toks, lens, round_new_kv=False)
    assert _compare_to_hf(out, ref) < 1e-10


def test_layer_by_layer_run_from_its_own_states_reproduces_the_step():
    """The re-anchored comparison of the GPU parity tests runs each oracle layer from a given
    residual stream.  Fed the oracle's own states it must reproduce the whole step exactly."""
    from parity import Case, run_oracle

    m, wts, kv, toks, lens = _tiny_inputs()
    c = Case(m, list(lens), toks, 0.1, len(lens), max(lens) + 1, wts, kv)
    whole = oracle.decode_step(m, wts, kv.k_pool, kv.v_pool, kv.page_table, toks, lens)
    out = run_oracle(c, kv.k_pool, kv.v_pool, anchor=whole["hidden"])
    for key in ("k_new", "v_new", "k_new_exact", "v_new_exact"):
        assert torch.equal(out[key], whole[key])
        assert torch.equal(out["anchored"][key], whole[key])
    assert torch.equal(out["hidden"], whole["hidden"])
    assert torch.equal(out["logits"], whole["logits"])
    assert out["argmax"] == whole["argmax"] and out["slots"] == whole["slots"]
