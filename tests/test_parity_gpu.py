"""GPU parity: one decode step through the C ABI against the float64 oracle.

Every case checks, per mid-state: the residual stream after each layer (relative
L2 <= 1e-2, whole batch and per sequence), each new K/V entry (within 1 bf16 ulp
of the oracle's rounded value) and bit-identity of every other KV slot (canary
NaN patterns included), the logits (max |d| <= 5e-2) and the argmax (exact up to
true numerical ties).  Ragged batches use distinct positions, the failure mode
of "ForgeMegakernel" §3.2.
"""
import gc

import pytest
import torch

import bandwidth_bound_b200 as mk
import synth
from parity import check_step, gpu_step, make_case, run_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device (deselect with -m 'not gpu')")
    yield
    gc.collect()
    torch.cuda.empty_cache()


def _run(c, batch=None, handle=None, **kw):
    kb, vb = c.kv.k_pool.cpu(), c.kv.v_pool.cpu()
    out, h = gpu_step(c, handle=handle, batch=batch)
    ref = run_oracle(c, kb, vb, batch=batch, anchor=out["hidden"])
    errs = check_step(c, out, ref, kb, vb, batch=batch, **kw)
    print(c.m.name, len(c.lens) if batch is None else batch, errs)
    return out, ref, h, errs


def _new_entries(c, b):
    """The K and V entries the step appended (bit patterns), [L][b][n_kv][hd] each."""
    P = c.m.page_size
    pages = [int(c.kv.page_table[i, c.lens[i] // P]) for i in range(b)]
    slots = [c.lens[i] % P for i in range(b)]
    k = torch.stack([c.kv.k_pool[:, pages[i], :, slots[i], :] for i in range(b)], 1)
    v = torch.stack([c.kv.v_pool[:, pages[i], :, slots[i], :] for i in range(b)], 1)
    return k.view(torch.int16).cpu(), v.view(torch.int16).cpu()


def _run_capture_off_then_on(c):
    """The step as bench.py times it (no mid-state capture) against the oracle, then the same
    step with capture on: logits, argmax and the appended K/V must be bit-identical, and the
    captured run adds the per-layer hidden and re-anchored K/V checks."""
    b = len(c.lens)
    kb, vb = c.kv.k_pool.cpu(), c.kv.v_pool.cpu()
    off, h = gpu_step(c, debug=False)
    assert off["hidden"] is None
    k_off, v_off = _new_entries(c, b)
    on, _ = gpu_step(c, handle=h, debug=True)
    k_on, v_on = _new_entries(c, b)
    assert torch.equal(off["logits"], on["logits"])
    assert torch.equal(off["argmax"], on["argmax"])
    assert torch.equal(k_off, k_on) and torch.equal(v_off, v_on)
    ref = run_oracle(c, kb, vb, anchor=on["hidden"])
    errs_off = check_step(c, off, ref, kb, vb, check_pool=False)
    errs_on = check_step(c, on, ref, kb, vb, check_pool=False)
    print(c.m.name, b, "capture off:", errs_off)
    print(c.m.name, b, "capture on:", errs_on)
    h.close()


def test_tiny_config_b1_position_64():
    c = make_case(synth.TINY, [64])
    _run(c)


def test_tiny_ragged_with_gains_and_page_edges():
    # positions 0 (no prior entries), 15/16 (page boundary), 33, 64
    c = make_case(synth.TINY, [0, 15, 16, 33, 64], gain_std=0.1, max_ctx=128, tag="edges")
    _run(c)


@pytest.mark.parametrize("b", [2, 3, 8, 9, 16])
def test_tiny_batch_sizes(b):
    g = torch.Generator().manual_seed(100 + b)
    lens = [int(v) for v in torch.randint(0, 200, (b,), generator=g)]
    c = make_case(synth.TINY, lens, gain_std=0.1, max_ctx=256, tag=f"b{b}")
    _run(c)


def test_max_position_and_long_chunks():
    # one sequence at the last position the handle allows, beside short ones
    m = synth.scaled_model(synth.LLAMA3_8B, name="wide-tiny", n_layers=2, hidden=512, n_heads=8,
                           n_kv_heads=2, ffn=1024, vocab=4096)
    c = make_case(m, [4095, 3, 700], gain_std=0.1, max_ctx=4096, tag="maxpos")
    _run(c)


def test_mha_head_dim_128_shape():
    m = synth.scaled_model(synth.LLAMA2_13B, name="mha-small", n_layers=2, hidden=512, n_heads=4,
                           n_kv_heads=4, ffn=1024, vocab=4096)
    c = make_case(m, [100, 1000, 17, 1], gain_std=0.1, max_ctx=1024, tag="mha")
    _run(c)


def test_g3_tied_shape():
    m = synth.scaled_model(synth.SMOLLM2_135M, name="tied-g3-small", n_layers=3)
    c = make_case(m, [1024], tag="g3")
    _run(c)


def test_repeated_step_is_deterministic_and_idempotent():
    c = make_case(synth.TINY, [5, 70, 130], gain_std=0.1, max_ctx=256, tag="det")
    out1, h = gpu_step(c)
    k1 = c.kv.k_pool.clone()
    out2, _ = gpu_step(c, handle=h)
    assert torch.equal(out1["logits"], out2["logits"])
    assert torch.equal(out1["hidden"], out2["hidden"])
    assert torch.equal(k1.view(torch.int16), c.kv.k_pool.view(torch.int16))


def test_host_buffer_entry_point_matches_device_entry_point():
    c = make_case(synth.TINY, [3, 64, 99], gain_std=0.1, max_ctx=128, tag="host")
    out, h = gpu_step(c)
    b = len(c.lens)
    tok = torch.tensor(c.tokens, dtype=torch.int32).pin_memory()
    pos = torch.tensor(c.lens, dtype=torch.int32).pin_memory()
    lens = (pos + 1).pin_memory()
    logits = torch.empty((b, c.m.vocab), dtype=torch.float32).pin_memory()
    am = torch.empty((b,), dtype=torch.int32).pin_memory()
    h.step_host(tok, pos, lens, c.kv, logits, am)
    assert torch.equal(logits, out["logits"])
    assert torch.equal(am, out["argmax"])


def test_smollm2_config_b1_ctx1024():
    w = synth.WORKLOADS["smollm2-135m-b1"]
    c = make_case(w.model, w.context_lengths(), max_ctx=2048, tag=w.name)
    _run(c)


def test_llama32_1b_late_arrival_same_handle():
    """Batch of 8, then a 9th sequence joins on the same handle (configs' 8+1)."""
    w = synth.WORKLOADS["llama3.2-1b-b9"]
    c = make_case(w.model, w.context_lengths(), max_batch=9, max_ctx=4097, tag=w.name)
    kb, vb = c.kv.k_pool.cpu(), c.kv.v_pool.cpu()
    out8, h = gpu_step(c, batch=8)
    ref8 = run_oracle(c, kb, vb, batch=8, anchor=out8["hidden"])
    print("b8", check_step(c, out8, ref8, kb, vb, batch=8))
    kb2, vb2 = c.kv.k_pool.cpu(), c.kv.v_pool.cpu()
    out9, _ = gpu_step(c, handle=h, batch=9)
    ref9 = run_oracle(c, kb2, vb2, batch=9, anchor=out9["hidden"])
    print("b9", check_step(c, out9, ref9, kb2, vb2, batch=9))


@pytest.mark.slow
@pytest.mark.parametrize("b", [1, 8])
def test_llama3_8b_ctx2048(b):
    """Full size, in the handle configuration bench.py times (max_batch = b, capture off)."""
    w = synth.WORKLOADS[f"llama3-8b-b{b}"]
    c = make_case(w.model, w.context_lengths(), max_ctx=max(w.context_lengths()) + 2, tag=w.name)
    _run_capture_off_then_on(c)


@pytest.mark.slow
def test_llama2_13b_ragged_b4():
    w = synth.WORKLOADS["llama2-13b-b4"]
    c = make_case(w.model, w.context_lengths(), max_ctx=max(w.context_lengths()) + 2, tag=w.name)
    _run_capture_off_then_on(c)


# --- errors -----------------------------------------------------------------------------

def _small_handle(max_batch=4, max_ctx=128):
    c = make_case(synth.TINY, [10, 20], max_batch=max_batch, max_ctx=max_ctx, tag="err")
    return c, mk.Megakernel(c.m, c.weights, c.max_batch, c.max_ctx)


def _dev(v):
    return torch.tensor(v, dtype=torch.int32, device="cuda")


def test_host_side_argument_errors():
    c, h = _small_handle()
    logits = torch.empty((2, c.m.vocab), device="cuda")
    pos = _dev(c.lens)
    for bad_batch in (0, 5):
        tok = _dev([1] * max(bad_batch, 1))
        assert h.step(tok[:bad_batch] if bad_batch else tok[:0], pos, pos + 1, c.kv, logits,
                      check=False) == mk.MK_ERR_INVALID_ARG
    kvs = mk.Megakernel.kv_struct(c.kv)
    rc = h.lib.mk_decode_step(h.handle, 0, 0, 0, 2, None, 0, 0, None)
    assert rc == mk.MK_ERR_INVALID_ARG
    assert "null" in h.last_error()
    del kvs


@pytest.mark.parametrize("what", ["token", "position", "length", "page"])
def test_device_bounds_errors_are_reported_and_sticky(what):
    c, h = _small_handle()
    tok, pos = list(c.tokens), list(c.lens)
    lens = [p + 1 for p in pos]
    if what == "token":
        tok[1] = c.m.vocab
    elif what == "position":
        pos[0] = c.max_ctx
        lens[0] = pos[0] + 1
    elif what == "length":
        lens[1] = pos[1] + 2
    else:
        c.kv.page_table[0, 0] = -1  # a prior page of sequence 0
    logits = torch.empty((2, c.m.vocab), device="cuda")
    h.step(_dev(tok), _dev(pos), _dev(lens), c.kv, logits, check=False)
    torch.cuda.synchronize()
    assert h.status() == mk.MK_ERR_BOUNDS
    # sticky until reset
    assert h.step(_dev(c.tokens), _dev(c.lens), _dev([p + 1 for p in c.lens]), c.kv, logits,
                  check=False) == mk.MK_ERR_BOUNDS
    if what == "page":
        return
    h.reset()
    h.step(_dev(c.tokens), _dev(c.lens), _dev([p + 1 for p in c.lens]), c.kv, logits)
    torch.cuda.synchronize()
    assert h.status() == mk.MK_OK


def test_unreachable_wait_times_out_and_context_survives():
    """A schedule whose LM-head wait can never be met (validator bypassed) must come back
    as a device timeout within the limit; the context stays usable."""
    c = make_case(synth.TINY, [10, 20], max_ctx=128, tag="timeout")
    plan = mk.Plan(mk.model_cfg(c.m, c.max_batch, c.max_ctx), num_sms=torch.cuda.get_device_properties(0).multi_processor_count)
    assert plan.inject_fault(mk.MK_FAULT_RAISE_TARGET) == mk.MK_OK
    assert plan.validate()[0] == mk.MK_ERR_SCHEDULE_INVALID
    with pytest.raises(mk.MkError):
        mk.Megakernel(c.m, c.weights, c.max_batch, c.max_ctx, plan=plan)
    h = mk.Megakernel(c.m, c.weights, c.max_batch, c.max_ctx, plan=plan, skip_validate=True)
    h.set_timeout_ns(50_000_000)
    logits = torch.empty((2, c.m.vocab), device="cuda")
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    h.step(_dev(c.tokens), _dev(c.lens), _dev([p + 1 for p in c.lens]), c.kv, logits)
    ev1.record()
    torch.cuda.synchronize()
    assert h.status() == mk.MK_ERR_DEVICE_TIMEOUT
    assert ev0.elapsed_time(ev1) < 2000.0
    h.close()
    # a fresh handle on the same context still works
    out, h2 = gpu_step(c)
    assert out["status"] == mk.MK_OK
