"""The allocation-free entry point (mk_decode_step_static).

Some callers cannot call cudaMalloc: a process whose device memory belongs to another
allocator (a caching allocator that has reserved the free memory), or a serving loop in
which an allocation would synchronise the device.  mk_decode_step_static runs the same
step on a fixed device array instead of a handle's arena.  These tests check that it:
  * matches the float64 oracle (logits, argmax, appended K/V) on its first step;
  * matches mk_decode_step on two steps in a row (the second feeds the first's greedy
    tokens at the next positions), on separate copies of the same KV cache;
  * reports an out-of-range token as MK_ERR_BOUNDS and then, on the next good call,
    starts from a clean state again;
  * allocates no device memory, including when a changed max_ctx redoes its set-up;
  * rejects a model whose scratch exceeds the array.
The file is collected last, so that a run that stops at its first failure has run every
other test first.  Nothing here depends on that order: every test either builds the
state it needs (the entry point redoes its set-up whenever cfg or weights change) or
only reads it.
"""
import gc

import pytest
import torch

import bandwidth_bound_b200 as mk
import synth
from parity import KV_ULP, LOGIT_ABS, bf16_ulp_error, check_step, make_case, run_oracle

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


def _dev(v):
    return torch.tensor(v, dtype=torch.int32, device="cuda")


def _two_steps(c, run):
    """Steps at positions p and p+1 (greedy token of the first); returns both results."""
    b = len(c.lens)
    tok = _dev(c.tokens)
    pos = _dev(c.lens)
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


def _compare(kv_ref, kv_static, ref, got):
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


def _static_step(c, tok, pos, logits, am=None, max_batch=None, max_ctx=None, check=True, lens=None):
    lens = pos + 1 if lens is None else lens
    return mk.decode_step_static(c.m, c.weights, max_batch or c.max_batch, max_ctx or c.max_ctx, tok, pos, lens,
                                 c.kv, logits, am, check=check)


QWEN_SMALL = synth.scaled_model(synth.QWEN3_0_6B, name="qwen3-small", n_layers=2, hidden=256, n_heads=4,
                                n_kv_heads=2, head_dim=128, ffn=512, vocab=4096)
MODELS = {"tiny": synth.TINY, "smollm2": synth.SMOLLM2_135M, "qwen3-small": QWEN_SMALL}


@pytest.mark.parametrize("name, lens, max_ctx", [("tiny", [5, 70, 130], 256),
                                                  ("smollm2", [1000], 2048),
                                                  ("qwen3-small", [40, 0, 17], 64)])
def test_static_entry_point_matches_oracle_and_handle_entry_point(name, lens, max_ctx):
    m = MODELS[name]
    c = make_case(m, lens, gain_std=0.1, max_ctx=max_ctx, tag="static-" + name)
    kv_handle = _clone_kv(c.kv)
    kb, vb = c.kv.k_pool.cpu(), c.kv.v_pool.cpu()

    # first step against the oracle (the static path has no mid-state capture: logits,
    # argmax and the appended K/V end to end)
    b = len(c.lens)
    logits = torch.full((b, m.vocab), float("nan"), dtype=torch.float32, device="cuda")
    am = torch.full((b,), -1, dtype=torch.int32, device="cuda")
    assert _static_step(c, _dev(c.tokens), _dev(c.lens), logits, am) == mk.MK_OK
    torch.cuda.synchronize()
    out = {"status": mk.MK_OK, "logits": logits.cpu(), "argmax": am.cpu(), "hidden": None}
    ref = run_oracle(c, kb, vb)
    check_step(c, out, ref, kb, vb)

    # two steps through both entry points on separate copies of the cache (the first step
    # above rewrote the same slot with the same bits, so the copies still agree)
    kv_static = c.kv
    c.kv = kv_handle
    h = mk.Megakernel(c.m, c.weights, c.max_batch, c.max_ctx)
    want = _two_steps(c, lambda t, p, n, lo, a: h.step(t, p, n, kv_handle, lo, a))
    c.kv = kv_static
    got = _two_steps(c, lambda t, p, n, lo, a: _static_step(c, t, p, lo, a))
    _compare(kv_handle, kv_static, want, got)
    h.close()


def test_static_entry_point_reports_bounds_and_recovers():
    c = make_case(synth.TINY, [10, 20], gain_std=0.1, max_ctx=128, tag="static-bounds")
    kb, vb = c.kv.k_pool.cpu(), c.kv.v_pool.cpu()
    logits = torch.empty((2, c.m.vocab), dtype=torch.float32, device="cuda")
    am = torch.empty((2,), dtype=torch.int32, device="cuda")
    bad = list(c.tokens)
    bad[1] = c.m.vocab  # checked on the device before any access
    rc = _static_step(c, _dev(bad), _dev(c.lens), logits, am, check=False)
    assert rc == mk.MK_ERR_BOUNDS
    # nothing was written to the cache
    assert torch.equal(c.kv.k_pool.cpu().view(torch.int16), kb.view(torch.int16))
    # the next good call clears the counters and the status first
    logits.fill_(float("nan"))
    assert _static_step(c, _dev(c.tokens), _dev(c.lens), logits, am) == mk.MK_OK
    torch.cuda.synchronize()
    out = {"status": mk.MK_OK, "logits": logits.cpu(), "argmax": am.cpu(), "hidden": None}
    check_step(c, out, run_oracle(c, kb, vb), kb, vb)


def test_static_entry_point_allocates_no_device_memory():
    c = make_case(synth.TINY, [9, 33], gain_std=0.1, max_ctx=128, tag="static-noalloc")
    tok, pos = _dev(c.tokens), _dev(c.lens)
    lens = pos + 1  # every device tensor the calls use exists before the measurement
    logits = torch.empty((2, c.m.vocab), dtype=torch.float32, device="cuda")
    am = torch.empty((2,), dtype=torch.int32, device="cuda")
    _static_step(c, tok, pos, logits, am, lens=lens)  # loads the library's module and sets up
    _static_step(c, tok, pos, logits, am, lens=lens, max_ctx=256)
    _static_step(c, tok, pos, logits, am, lens=lens)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for k in range(4):
        _static_step(c, tok, pos, logits, am, lens=lens)
    _static_step(c, tok, pos, logits, am, lens=lens, max_ctx=256)  # another cfg: the set-up runs again
    _static_step(c, tok, pos, logits, am, lens=lens)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0


def test_static_entry_point_rejects_scratch_beyond_its_limit():
    c = make_case(synth.TINY, [9], max_ctx=64, tag="static-limit")
    tok = _dev(c.tokens)
    pos = _dev(c.lens)
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
    _compare(kv_ref, c.kv, ref, got)
    h.close()
