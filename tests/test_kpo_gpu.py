"""The kernel-per-op step (mk_kpo_*: one launch per operation, replayed as a CUDA graph with
programmatic dependent launch) against the float64 oracle: logits, argmax, the appended K/V
and every other cache slot, on ragged batches; its launch modes agree bit for bit; its launch
count is 10 per layer plus 4."""
import gc

import pytest
import torch

import bandwidth_bound_b200 as mk
import synth
from parity import check_step, make_case, run_oracle

pytestmark = pytest.mark.gpu

MHA_SMALL = synth.scaled_model(synth.LLAMA2_13B, name="mha-small", n_layers=2, hidden=512, n_heads=4, n_kv_heads=4,
                               ffn=1024, vocab=4096)


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device (deselect with -m 'not gpu')")
    yield
    gc.collect()
    torch.cuda.empty_cache()


def _dev(v):
    return torch.tensor(v, dtype=torch.int32, device="cuda")


def _kpo_step(c, k, mode=mk.KPO_GRAPH):
    b = len(c.lens)
    logits = torch.full((b, c.m.vocab), float("nan"), dtype=torch.float32, device="cuda")
    am = torch.full((b,), -1, dtype=torch.int32, device="cuda")
    pos = _dev(c.lens)
    busy = k.step(_dev(c.tokens), pos, pos + 1, c.kv, logits, am, mode=mode)
    torch.cuda.synchronize()
    return {"status": mk.MK_OK, "logits": logits.cpu(), "argmax": am.cpu(), "hidden": None}, busy


@pytest.mark.parametrize("name, lens, max_ctx", [("tiny", [0, 15, 16, 130, 77], 256), ("smollm2", [1000], 1100),
                                                 ("mha-small", [100, 7, 600], 700), ("llama3.2-1b", [3000, 40], 3100)])
def test_kernel_per_op_matches_oracle(name, lens, max_ctx):
    m = {"tiny": synth.TINY, "smollm2": synth.SMOLLM2_135M, "mha-small": MHA_SMALL,
         "llama3.2-1b": synth.LLAMA32_1B}[name]
    c = make_case(m, lens, gain_std=0.1, max_ctx=max_ctx, tag="kpo-" + name)
    kb, vb = c.kv.k_pool.cpu(), c.kv.v_pool.cpu()
    k = mk.KernelPerOp(c.m, c.weights, len(lens), c.max_ctx)
    out, _ = _kpo_step(c, k)
    errs = check_step(c, out, run_oracle(c, kb, vb), kb, vb)
    print(name, errs)
    k.close()


def test_kernel_per_op_modes_agree_and_count_launches():
    c = make_case(synth.TINY, [5, 70, 130], gain_std=0.1, max_ctx=256, tag="kpo-modes")
    k = mk.KernelPerOp(c.m, c.weights, 4, c.max_ctx)
    assert k.launches_per_step() == 10 * c.m.n_layers + 4
    outs = []
    for mode in (mk.KPO_GRAPH, mk.KPO_STREAM, mk.KPO_TIMED, mk.KPO_GRAPH):
        out, busy = _kpo_step(c, k, mode)
        if mode == mk.KPO_TIMED:
            assert busy > 0.0
        outs.append(out)
    for o in outs[1:]:
        assert torch.equal(o["logits"].view(torch.int32), outs[0]["logits"].view(torch.int32))
        assert torch.equal(o["argmax"], outs[0]["argmax"])
    # the launches alone: same grids, kernels that do nothing; no results are written
    before = outs[-1]["logits"].clone()
    lg = torch.full((3, c.m.vocab), 7.0, dtype=torch.float32, device="cuda")
    pos = _dev(c.lens)
    k.step(_dev(c.tokens), pos, pos + 1, c.kv, lg, None, mode=mk.KPO_EMPTY)
    torch.cuda.synchronize()
    assert bool((lg == 7.0).all())
    out, _ = _kpo_step(c, k)
    assert torch.equal(out["logits"].view(torch.int32), before.view(torch.int32))
    k.close()


def test_kernel_per_op_rejects_what_it_does_not_cover():
    qk = synth.scaled_model(synth.TINY, name="tiny-qk", qk_norm=True)
    for m, mb in ((qk, 2), (synth.TINY, 9)):
        wts = synth.make_weights(m, device="cuda")
        with pytest.raises(mk.MkError) as ei:
            mk.KernelPerOp(m, wts, mb, 128)
        assert ei.value.code == mk.MK_ERR_UNSUPPORTED_CFG
