"""The allocation-free entry point (mk_decode_step_static) against mk_decode_step.

Two decode steps in a row (the second feeds the first's greedy tokens at the next
positions) run through both entry points on separate copies of the same KV cache;
logits must agree within the parity tolerance, argmax exactly, and every KV entry
within 1 bf16 ulp.  The file is named to be collected last: the static scratch is
process-wide, and the test must hold after every other test has run in the process.
"""
import gc

import pytest
import torch

import bandwidth_bound_b200 as mk
import synth
from parity import KV_ULP, LOGIT_ABS, bf16_ulp_error, make_case

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device (deselect with -m 'not gpu')")
    yield
    gc.collect()
    torch.cuda.empty_cache()


def _clone_kv(kv):
    return synth.KVCache(kv.k_pool.clone(), kv.v_pool.clone(), kv.page_table.clone(), kv.num_pages,
                         kv.max_pages_per_seq, list(kv.ctx_lens))


def _two_steps(c, run):
    """Steps at positions p and p+1 (greedy token of the first); returns both results."""
    b = len(c.lens)
    tok = torch.tensor(c.tokens, dtype=torch.int32, device="cuda")
    pos = torch.tensor(c.lens, dtype=torch.int32, device="cuda")
    outs = []
    for _ in range(2):
        logits = torch.full((b, c.m.vocab), float("nan"), dtype=torch.float32, device="cuda")
        am = torch.full((b,), -1, dtype=torch.int32, device="cuda")
        run(tok, pos, pos + 1, logits, am)
        torch.cuda.synchronize()
        outs.append((logits.cpu(), am.cpu()))
        tok = am.clone()
        pos = pos + 1
    return outs


def _compare(c, kv_ref, kv_static, ref, got):
    for (l_ref, a_ref), (l_got, a_got) in zip(ref, got):
        assert torch.isfinite(l_got).all()
        dl = (l_got.to(torch.float64) - l_ref.to(torch.float64)).abs().max().item()
        assert dl <= LOGIT_ABS, f"max |dlogit| {dl}"
        assert torch.equal(a_got, a_ref)
    for pool_ref, pool_got in ((kv_ref.k_pool, kv_static.k_pool), (kv_ref.v_pool, kv_static.v_pool)):
        r = pool_ref.cpu().to(torch.float64)
        g = pool_got.cpu().to(torch.float64)
        finite = torch.isfinite(r)
        # canary (NaN) slots must be untouched by both, bit for bit
        assert torch.equal(pool_ref.cpu().view(torch.int16)[~finite], pool_got.cpu().view(torch.int16)[~finite])
        e = bf16_ulp_error(torch.where(finite, g, 0.0), torch.where(finite, r, 0.0))
        assert float(e.max()) <= KV_ULP


@pytest.mark.parametrize("name, lens, max_ctx", [("tiny", [5, 70, 130], 256),
                                                  ("smollm2", [1000], 2048)])
def test_static_entry_point_matches_handle_entry_point(name, lens, max_ctx):
    m = synth.TINY if name == "tiny" else synth.SMOLLM2_135M
    c = make_case(m, lens, gain_std=0.1, max_ctx=max_ctx, tag="static-" + name)
    kv_static = _clone_kv(c.kv)
    h = mk.Megakernel(c.m, c.weights, c.max_batch, c.max_ctx)
    ref = _two_steps(c, lambda t, p, n, lo, am: h.step(t, p, n, c.kv, lo, am))
    got = _two_steps(c, lambda t, p, n, lo, am: mk.decode_step_static(c.m, c.weights, c.max_batch, c.max_ctx,
                                                                      t, p, n, kv_static, lo, am))
    _compare(c, c.kv, kv_static, ref, got)
    h.close()


def test_static_entry_point_rejects_scratch_beyond_its_limit():
    c = make_case(synth.TINY, [9], max_ctx=64, tag="static-limit")
    tok = torch.tensor(c.tokens, dtype=torch.int32, device="cuda")
    pos = torch.tensor(c.lens, dtype=torch.int32, device="cuda")
    logits = torch.empty((1, c.m.vocab), dtype=torch.float32, device="cuda")
    # at head_dim 64 a RoPE table of 2^16 positions alone fills the 16 MiB
    with pytest.raises(mk.MkError) as ei:
        mk.decode_step_static(c.m, c.weights, 1, 1 << 16, tok, pos, pos + 1, c.kv, logits)
    assert ei.value.code == mk.MK_ERR_INVALID_ARG and "static area" in str(ei.value)
    # the entry point still works afterwards
    kv_ref = _clone_kv(c.kv)
    h = mk.Megakernel(c.m, c.weights, 1, c.max_ctx)
    ref = _two_steps(c, lambda t, p, n, lo, am: h.step(t, p, n, kv_ref, lo, am))
    got = _two_steps(c, lambda t, p, n, lo, am: mk.decode_step_static(c.m, c.weights, 1, c.max_ctx, t, p, n,
                                                                      c.kv, lo, am))
    _compare(c, kv_ref, c.kv, ref, got)
    h.close()
