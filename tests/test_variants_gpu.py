"""GPU parity of the model variants the pages evaluate ("ForgeMegakernel" §5.3 and
Appendix A: Qwen3 with QK-norm; the Llama 3 family, whose 3.x models scale the RoPE
frequencies) against the float64 oracle: per-layer residual stream, new K/V (re-anchored on
the GPU's own layer input, 1 bf16 ulp), logits and argmax, on ragged batches."""
import gc

import pytest
import torch

import bandwidth_bound_b200 as mk
import synth
from parity import check_step, gpu_step, make_case, run_oracle

pytestmark = pytest.mark.gpu

TINY_QK = synth.scaled_model(synth.TINY, name="tiny-qk", qk_norm=True)
# head_dim 128 with q_dim (512) != hidden (256), as in Qwen3-0.6B
QWEN_SMALL = synth.scaled_model(synth.QWEN3_0_6B, name="qwen3-small", n_layers=2, hidden=256, n_heads=4,
                                n_kv_heads=2, head_dim=128, ffn=512, vocab=4096)
# original context 64: all three frequency bands occur at head_dim 64 and theta 1e4
TINY_SCALED = synth.scaled_model(synth.TINY, name="tiny-scaled", rope_scaling=(8.0, 1.0, 4.0, 64))


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device (deselect with -m 'not gpu')")
    yield
    gc.collect()
    torch.cuda.empty_cache()


def _run(c, batch=None, **kw):
    kb, vb = c.kv.k_pool.cpu(), c.kv.v_pool.cpu()
    out, h = gpu_step(c, batch=batch)
    ref = run_oracle(c, kb, vb, batch=batch, anchor=out["hidden"])
    errs = check_step(c, out, ref, kb, vb, batch=batch, **kw)
    print(c.m.name, errs)
    return out, h


@pytest.mark.parametrize("m", [TINY_QK, QWEN_SMALL], ids=lambda m: m.name)
def test_qk_norm_ragged(m):
    c = make_case(m, [0, 15, 16, 130, 7], gain_std=0.2, max_ctx=256, tag="qk")
    _run(c)


@pytest.mark.parametrize("b", [1, 8, 9])
def test_qk_norm_batch_sizes(b):
    g = torch.Generator().manual_seed(300 + b)
    lens = [int(v) for v in torch.randint(0, 300, (b,), generator=g)]
    c = make_case(QWEN_SMALL, lens, gain_std=0.2, max_ctx=320, tag=f"qk-b{b}")
    _run(c)


def test_rope_scaling_ragged():
    c = make_case(TINY_SCALED, [0, 17, 63, 64, 200, 511], gain_std=0.1, max_ctx=512, tag="scaled")
    _run(c)


def test_rope_scaling_changes_the_step():
    """The scaled table is in use: the same inputs without the scaling give other logits."""
    c = make_case(TINY_SCALED, [200, 300], gain_std=0.1, max_ctx=512, tag="scaled-vs-plain")
    out, h = gpu_step(c, debug=False)
    h.close()
    plain = type(c)(synth.TINY, c.lens, c.tokens, c.gain_std, c.max_batch, c.max_ctx, c.weights, c.kv)
    out2, h2 = gpu_step(plain, debug=False)
    h2.close()
    assert (out["logits"] - out2["logits"]).abs().max() > 1e-3


def test_qwen3_0_6b_b1_ctx128():
    """The configuration the pages' milestone ablation forges (Qwen3-0.6B, batch 1, 128
    tokens), at full size."""
    w = synth.WORKLOADS["qwen3-0.6b-b1"]
    c = make_case(w.model, w.context_lengths(), gain_std=0.1, max_ctx=256, tag=w.name)
    _run(c)


def test_llama32_1b_scaled_rope_full_size_b2():
    c = make_case(synth.LLAMA32_1B, [3000, 77], gain_std=0.1, max_ctx=4096, tag="l32-scaled")
    assert synth.LLAMA32_1B.rope_scaling is not None
    _run(c)


def test_qk_norm_multistep_matches_single_steps():
    """The new key is normalised and stored by the attention task holding its position;
    later steps must read it back exactly as one-step calls leave it."""
    n = 4
    c = make_case(QWEN_SMALL, [14, 40, 0], gain_std=0.2, max_ctx=64, tag="qk-multi", kv_room=n)
    kv2 = synth.KVCache(c.kv.k_pool.clone(), c.kv.v_pool.clone(), c.kv.page_table.clone(), c.kv.num_pages,
                        c.kv.max_pages_per_seq, list(c.kv.ctx_lens))
    h = mk.Megakernel(c.m, c.weights, c.max_batch, c.max_ctx)
    b = len(c.lens)
    toks = torch.full((n, b), -1, dtype=torch.int32, device="cuda")
    h.steps(n, torch.tensor(c.tokens, dtype=torch.int32, device="cuda"),
            torch.tensor(c.lens, dtype=torch.int32, device="cuda"), c.kv, toks)
    torch.cuda.synchronize()
    tok = torch.tensor(c.tokens, dtype=torch.int32, device="cuda")
    pos = torch.tensor(c.lens, dtype=torch.int32, device="cuda")
    lg = torch.empty((b, c.m.vocab), dtype=torch.float32, device="cuda")
    am = torch.empty((b,), dtype=torch.int32, device="cuda")
    for k in range(n):
        h.step(tok, pos, pos + 1, kv2, lg, am)
        torch.cuda.synchronize()
        assert torch.equal(am.cpu(), toks[k].cpu())
        tok, pos = am.clone(), pos + 1
    assert torch.equal(kv2.k_pool.view(torch.int16), c.kv.k_pool.view(torch.int16))
    # and the last step against the oracle, from the cache the run left
    last = type(c)(c.m, [s + n - 1 for s in c.lens], [int(t) for t in toks[n - 2].cpu()], c.gain_std,
                   c.max_batch, c.max_ctx, c.weights, c.kv)
    kb, vb = c.kv.k_pool.cpu(), c.kv.v_pool.cpu()
    out, h2 = gpu_step(last, handle=h)
    ref = run_oracle(last, kb, vb, anchor=out["hidden"])
    check_step(last, out, ref, kb, vb)
    h.close()
