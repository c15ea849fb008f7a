"""The on-device multi-step greedy loop (mk_decode_steps) against the float64 oracle.

n steps run as n stream-ordered launches with no host round trip: step k takes the
greedy token of step k-1 at every position k further on ("ForgeMegakernel" §4.3, the
engine's generation loop behind the launch).  Checked here:
  * each step k against the oracle's step from the same cache state: the oracle runs
    with the tokens the GPU fed in, at positions + k, over the GPU's own cache (the
    entries steps 0..k-1 appended are read back from the pool after the run); its
    greedy token must equal tokens_out[k], its new K/V the entries at positions + k
    (1 bf16 ulp), and for the last step its logits;
  * the run is bit-identical to the same steps made one call at a time;
  * runs that cross a page boundary and that start at position 0;
  * a step whose position has no page stops the run with MK_ERR_BOUNDS: the steps
    before it stand, the later rows of tokens_out are untouched.
"""
import gc

import pytest
import torch

import bandwidth_bound_b200 as mk
import oracle
import synth
from parity import LOGIT_ABS, check_step, make_case, run_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device (deselect with -m 'not gpu')")
    yield
    gc.collect()
    torch.cuda.empty_cache()


def _dev(v):
    return torch.tensor(v, dtype=torch.int32, device="cuda")


def _clone_kv(kv):
    return synth.KVCache(kv.k_pool.clone(), kv.v_pool.clone(), kv.page_table.clone(), kv.num_pages,
                         kv.max_pages_per_seq, list(kv.ctx_lens))


def _one_call(c, h, kv, n, **smp):
    """The run as one call of n steps (mid-state capture off, as a server runs it)."""
    b = len(c.lens)
    toks = torch.full((n, b), -1, dtype=torch.int32, device="cuda")
    logits = torch.full((b, c.m.vocab), float("nan"), dtype=torch.float32, device="cuda")
    h.set_debug(None)
    h.steps(n, _dev(c.tokens), _dev(c.lens), kv, toks, logits, **smp)
    torch.cuda.synchronize()
    return toks.cpu(), logits.cpu()


def _one_call_per_step(c, h, n, top_k=1, temperature=1.0, u=None):
    """The same run made one step per call (n_steps = 1) with the mid-state capture on:
    tokens [n][b], and per step the logits and the captured residual stream [L+1][b][d]."""
    b = len(c.lens)
    tok = _dev(c.tokens)
    toks, logits, hidden = [], [], []
    for k in range(n):
        dbg = torch.full((c.m.n_layers + 1, c.max_batch, c.m.hidden), float("nan"), dtype=torch.float32,
                         device="cuda")
        h.set_debug(dbg)
        out = torch.full((1, b), -1, dtype=torch.int32, device="cuda")
        lg = torch.full((b, c.m.vocab), float("nan"), dtype=torch.float32, device="cuda")
        h.steps(1, tok, _dev([s + k for s in c.lens]), c.kv, out, lg, top_k=top_k, temperature=temperature,
                uniforms=None if u is None else u[k:k + 1].cuda())
        torch.cuda.synchronize()
        toks.append(out[0].cpu())
        logits.append(lg.cpu())
        hidden.append(dbg[:, :b].cpu())
        tok = out[0].clone()
    h.set_debug(None)
    return torch.stack(toks), logits, hidden


def _check_against_oracle(c, toks, logits, hidden, k0, v0, greedy=True):
    """Step k against the oracle's step from the same cache state: the oracle runs with the
    tokens the GPU fed in, at positions + k, over the GPU's own cache (the entries of steps
    0..k-1 are read back from the pool after the run: the oracle gathers prior positions
    only, so the final pool serves as every step's "before" state), each layer also re-run
    from the GPU's captured input to it.  The re-anchored comparison gates the new K/V (the
    end-to-end one, which carries earlier layers' drift, is reported)."""
    n = toks.shape[0]
    k_after, v_after = c.kv.k_pool.cpu(), c.kv.v_pool.cpu()
    tokens, lens = list(c.tokens), list(c.lens)
    for k in range(n):
        sc = type(c)(c.m, [s + k for s in lens], tokens, c.gain_std, c.max_batch, c.max_ctx, c.weights, c.kv)
        ref = run_oracle(sc, k_after, v_after, anchor=hidden[k])
        out = {"status": mk.MK_OK, "logits": logits[k], "argmax": toks[k] if greedy else None, "hidden": hidden[k]}
        check_step(sc, out, ref, k0, v0, check_pool=False, e2e_kv_gate=False)
        tokens = [int(t) for t in toks[k]]
    # nothing outside the n new slots per (layer, sequence, kv head) changed
    P = c.m.page_size
    mask = torch.ones(k_after.shape[1:4], dtype=torch.bool)
    for i, s in enumerate(lens):
        for k in range(n):
            mask[int(c.kv.page_table[i, (s + k) // P]), :, (s + k) % P] = False
    mm = mask[None, :, :, :, None].expand_as(k_after)
    assert torch.equal(k_after.view(torch.int16)[mm], k0.view(torch.int16)[mm])
    assert torch.equal(v_after.view(torch.int16)[mm], v0.view(torch.int16)[mm])


def _same_run(c, kv_one, toks_one, lg_one, toks, logits):
    """The one-call run equals the step-per-call run bit for bit (tokens, last logits, cache)."""
    assert torch.equal(toks_one, toks)
    assert torch.equal(lg_one.view(torch.int32), logits[-1].view(torch.int32))
    assert torch.equal(kv_one.k_pool.view(torch.int16), c.kv.k_pool.view(torch.int16))
    assert torch.equal(kv_one.v_pool.view(torch.int16), c.kv.v_pool.view(torch.int16))


@pytest.mark.parametrize("name, lens, n", [("tiny", [0, 14, 130], 5), ("tiny", [45], 3),
                                           ("smollm2", [1000, 31], 3), ("smollm2", [700, 5], 3)])
def test_multistep_matches_oracle_step_by_step(name, lens, n):
    m = synth.TINY if name == "tiny" else synth.SMOLLM2_135M
    c = make_case(m, lens, gain_std=0.1, max_ctx=max(lens) + n + 1, tag=f"multi-{name}-{n}", kv_room=n)
    kv_one = _clone_kv(c.kv)
    k0, v0 = c.kv.k_pool.cpu(), c.kv.v_pool.cpu()
    h = mk.Megakernel(c.m, c.weights, c.max_batch, c.max_ctx)
    toks_one, lg_one = _one_call(c, h, kv_one, n)
    toks, logits, hidden = _one_call_per_step(c, h, n)
    assert h.status() == mk.MK_OK
    _same_run(c, kv_one, toks_one, lg_one, toks, logits)
    _check_against_oracle(c, toks, logits, hidden, k0, v0)
    h.close()


def test_multistep_equals_single_steps_bit_for_bit():
    n = 4
    c = make_case(synth.TINY, [3, 15, 77, 200], gain_std=0.1, max_ctx=256, tag="multi-vs-single", kv_room=n)
    kv_single = _clone_kv(c.kv)
    h = mk.Megakernel(c.m, c.weights, c.max_batch, c.max_ctx)
    toks, logits = _one_call(c, h, c.kv, n)
    b = len(c.lens)
    tok = _dev(c.tokens)
    pos = _dev(c.lens)
    lg = torch.empty((b, c.m.vocab), dtype=torch.float32, device="cuda")
    am = torch.empty((b,), dtype=torch.int32, device="cuda")
    for k in range(n):
        h.step(tok, pos, pos + 1, kv_single, lg, am)
        torch.cuda.synchronize()
        assert torch.equal(am.cpu(), toks[k]), f"step {k}"
        tok = am.clone()
        pos = pos + 1
    assert torch.equal(lg.cpu().view(torch.int32), logits.view(torch.int32))
    assert torch.equal(kv_single.k_pool.view(torch.int16), c.kv.k_pool.view(torch.int16))
    assert torch.equal(kv_single.v_pool.view(torch.int16), c.kv.v_pool.view(torch.int16))
    h.close()


def _check_greedy(k, got, ref):
    """Step k's greedy tokens against the oracle's: equal, except where the oracle's top two
    logits are closer than the logit tolerance (a numerical tie), where the GPU's token must
    be within that tolerance of the oracle's maximum."""
    for i, g in enumerate(int(x) for x in got):
        want = ref["argmax"][i]
        if g != want:
            top = ref["logits"][i].max()
            assert float(top - ref["logits"][i, g]) <= LOGIT_ABS, f"step {k} sequence {i}: {g} vs oracle {want}"


def test_multistep_stops_at_a_position_without_a_page():
    # pages for 2 more tokens only (positions 30, 31); the third step (position 32) has no page
    c = make_case(synth.TINY, [30], gain_std=0.1, max_ctx=64, tag="multi-bounds", kv_room=2)
    assert int(c.kv.page_table[0, 32 // c.m.page_size]) == -1
    k0, v0 = c.kv.k_pool.cpu(), c.kv.v_pool.cpu()
    h = mk.Megakernel(c.m, c.weights, c.max_batch, c.max_ctx)
    toks = torch.full((4, 1), -1, dtype=torch.int32, device="cuda")
    h.steps(4, _dev(c.tokens), _dev(c.lens), c.kv, toks, None, check=False)
    torch.cuda.synchronize()
    assert h.status() == mk.MK_ERR_BOUNDS
    t = toks.cpu()
    assert (t[2:] == -1).all(), "steps after the failing one must not run"
    # the two steps that had pages ran to the end, and match the oracle
    tokens, lens = list(c.tokens), list(c.lens)
    k_after, v_after = c.kv.k_pool.cpu(), c.kv.v_pool.cpu()
    for k in range(2):
        sc = type(c)(c.m, [s + k for s in lens], tokens, c.gain_std, c.max_batch, c.max_ctx, c.weights, c.kv)
        ref = run_oracle(sc, k_after, v_after)
        _check_greedy(k, t[k], ref)
        tokens = [int(x) for x in t[k]]
    h.reset()
    assert h.status() == mk.MK_OK
    h.close()


def _uniforms(n, b, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.rand((n, b), generator=g, dtype=torch.float32)


def _check_draws(toks, logits, top_k, temp, u):
    """Each drawn token against the oracle's sampler on the device's own float32 logits."""
    near = 0
    for k in range(toks.shape[0]):
        for i in range(toks.shape[1]):
            row = logits[k][i].numpy()
            want = oracle.sample_top_k(row, top_k, temp, float(u[k, i]))
            got = int(toks[k, i])
            if got != want:
                # only a draw within rounding of a running-sum boundary may go either way
                assert oracle.boundary_margin(row, top_k, temp, float(u[k, i])) < 1e-5, (k, i, got, want)
                ranked = oracle.top_k_ranked(row, top_k)
                assert abs(ranked.index(got) - ranked.index(want)) == 1
                near += 1
    return near


@pytest.mark.parametrize("name, lens, top_k, temp", [("tiny", [0, 14, 130], 2, 0.7), ("tiny", [0, 14, 130], 50, 1.3),
                                                     ("tiny", [33], 256, 1.0), ("smollm2", [700, 5], 64, 0.8),
                                                     ("smollm2", [700, 5], 256, 2.0)])
def test_top_k_sampling_matches_oracle_sampler(name, lens, top_k, temp):
    n = 3
    m = synth.TINY if name == "tiny" else synth.SMOLLM2_135M
    c = make_case(m, lens, gain_std=0.1, max_ctx=max(lens) + n + 1, tag=f"sample-{name}", kv_room=n)
    kv_one = _clone_kv(c.kv)
    k0, v0 = c.kv.k_pool.cpu(), c.kv.v_pool.cpu()
    u = _uniforms(n, len(lens), seed=top_k)
    h = mk.Megakernel(c.m, c.weights, c.max_batch, c.max_ctx)
    toks_one, lg_one = _one_call(c, h, kv_one, n, top_k=top_k, temperature=temp, uniforms=u.cuda())
    toks, logits, hidden = _one_call_per_step(c, h, n, top_k, temp, u)
    assert h.status() == mk.MK_OK
    _same_run(c, kv_one, toks_one, lg_one, toks, logits)
    near = _check_draws(toks, logits, top_k, temp, u)
    print("draws within rounding of a boundary:", near)
    _check_against_oracle(c, toks, logits, hidden, k0, v0, greedy=False)
    h.close()


@pytest.mark.parametrize("name, top_k", [("tiny", 3), ("tiny", 256), ("smollm2", 64), ("smollm2", 256)])
def test_top_k_sampling_all_logits_equal(name, top_k):
    """A zero LM head makes every logit 0: the top k are vocabulary indices 0..k-1 with equal
    weights, so the draw is floor(u * k) exactly.  Every logit of the k tasks with the lowest
    indices is then a candidate: with SmolLM2's 768 LM-head tasks and k >= 64 that is more
    than shared memory holds, and the selection reads them from global memory instead."""
    n = 2
    m = synth.TINY if name == "tiny" else synth.SMOLLM2_135M
    c = make_case(m, [7, 40], gain_std=0.1, max_ctx=64, tag="sample-flat", kv_room=n)
    c.weights["lm_head"].zero_()  # tied models: the embedding too, which keeps every logit 0
    u = _uniforms(n, 2, seed=5 + top_k)
    h = mk.Megakernel(c.m, c.weights, c.max_batch, c.max_ctx)
    toks = torch.full((n, 2), -1, dtype=torch.int32, device="cuda")
    h.steps(n, _dev(c.tokens), _dev(c.lens), c.kv, toks, None, top_k=top_k, temperature=0.9, uniforms=u.cuda())
    torch.cuda.synchronize()
    assert h.status() == mk.MK_OK
    want = torch.floor(u * torch.tensor(top_k, dtype=torch.float32)).to(torch.int32)
    assert torch.equal(toks.cpu(), want), (toks.cpu(), want)
    h.close()


def test_sampling_arguments_are_checked_on_the_host():
    c = make_case(synth.TINY, [5], max_ctx=16, tag="sample-args", kv_room=1)
    h = mk.Megakernel(c.m, c.weights, 1, c.max_ctx)
    toks = torch.empty((1, 1), dtype=torch.int32, device="cuda")
    u = torch.zeros((1, 1), dtype=torch.float32, device="cuda")
    for kw in ({"top_k": mk.MAX_TOP_K + 1, "temperature": 1.0, "uniforms": u},
               {"top_k": 5, "temperature": 0.0, "uniforms": u},
               {"top_k": 5, "temperature": float("inf"), "uniforms": u},
               {"top_k": 5, "temperature": 1.0, "uniforms": None}):
        rc = h.steps(1, _dev(c.tokens), _dev(c.lens), c.kv, toks, None, check=False, **kw)
        assert rc == mk.MK_ERR_INVALID_ARG, kw
    assert h.status() == mk.MK_OK
    h.close()
