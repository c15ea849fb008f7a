"""The multi-token step (mk_verify_step) against the float64 oracle.

Several new tokens of a sequence run as consecutive batch rows over one page-table row
(repeated per row), at consecutive positions; row r attends to the sequence's prior
entries and to the new tokens of the rows before it.  The oracle runs the same batch -
one decode step per row, each row's prior entries gathered from the cache the GPU step
left (so the earlier rows' new K/V are the GPU's own, re-anchored per layer as in the
single-token tests).  Also: one-token rows give the decode step bit for bit, and a
malformed grouping is rejected on the device."""
import gc

import pytest
import torch

import bandwidth_bound_b200 as mk
import synth
from parity import check_step, make_case, run_oracle

pytestmark = pytest.mark.gpu

QWEN_SMALL = synth.scaled_model(synth.QWEN3_0_6B, name="qwen3-small", n_layers=2, hidden=256, n_heads=4,
                                n_kv_heads=2, head_dim=128, ffn=512, vocab=4096)


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device (deselect with -m 'not gpu')")
    yield
    gc.collect()
    torch.cuda.empty_cache()


def _dev(v):
    return torch.tensor(v, dtype=torch.int32, device="cuda")


def _grouped_case(m, prior, counts, tag):
    """Sequences with `prior` entries each and counts[s] new tokens: the batch rows, their
    positions, group_first, and a cache whose page table repeats each sequence's row."""
    seq = make_case(m, prior, gain_std=0.2, max_ctx=max(p + n for p, n in zip(prior, counts)) + 1, tag=tag,
                    kv_room=max(counts))
    rows, pos, first = [], [], []
    for s, (p, n) in enumerate(zip(prior, counts)):
        f = len(rows)
        for j in range(n):
            rows.append(s)
            pos.append(p + j)
            first.append(f)
    kv = seq.kv
    table = kv.page_table[torch.tensor(rows, device=kv.page_table.device)].contiguous()
    gkv = synth.KVCache(kv.k_pool, kv.v_pool, table, kv.num_pages, kv.max_pages_per_seq, pos)
    toks = synth.token_ids(m, len(rows), tag=tag + "-rows")
    c = type(seq)(m, pos, toks, seq.gain_std, len(rows), seq.max_ctx, seq.weights, gkv)
    return c, first


def _verify(c, first, h, capture=True):
    b = len(c.lens)
    dbg = None
    if capture:
        dbg = torch.full((c.m.n_layers + 1, c.max_batch, c.m.hidden), float("nan"), dtype=torch.float32,
                         device="cuda")
    h.set_debug(dbg)
    logits = torch.full((b, c.m.vocab), float("nan"), dtype=torch.float32, device="cuda")
    am = torch.full((b,), -1, dtype=torch.int32, device="cuda")
    pos = _dev(c.lens)
    rc = h.verify(_dev(c.tokens), pos, pos + 1, _dev(first), c.kv, logits, am, check=False)
    torch.cuda.synchronize()
    h.set_debug(None)
    return rc, {"status": h.status(), "logits": logits.cpu(), "argmax": am.cpu(),
                "hidden": dbg[:, :b].cpu() if capture else None}


@pytest.mark.parametrize("m", [synth.TINY, QWEN_SMALL], ids=lambda m: m.name)
def test_verify_step_matches_oracle(m):
    # 4 draft tokens at 30..33, a plain decode row at 100, 3 tokens across a page edge
    # (15, 16, 17) and 5 tokens of a sequence with no prior entries (0..4)
    c, first = _grouped_case(m, [30, 100, 15, 0], [4, 1, 3, 5], tag="verify-" + m.name)
    k0, v0 = c.kv.k_pool.cpu(), c.kv.v_pool.cpu()
    h = mk.Megakernel(c.m, c.weights, c.max_batch, c.max_ctx)
    rc, out = _verify(c, first, h)
    assert rc == mk.MK_OK and out["status"] == mk.MK_OK
    # the oracle reads each row's prior entries from the cache the step left: positions
    # below a row's own, which hold the earlier rows' new entries
    ka, va = c.kv.k_pool.cpu(), c.kv.v_pool.cpu()
    ref = run_oracle(c, ka, va, anchor=out["hidden"])
    errs = check_step(c, out, ref, k0, v0, e2e_kv_gate=False)
    print(m.name, errs)
    h.close()


def test_one_token_groups_equal_the_decode_step():
    c = make_case(synth.TINY, [5, 70, 130], gain_std=0.1, max_ctx=256, tag="verify-plain")
    kv2 = synth.KVCache(c.kv.k_pool.clone(), c.kv.v_pool.clone(), c.kv.page_table.clone(), c.kv.num_pages,
                        c.kv.max_pages_per_seq, list(c.kv.ctx_lens))
    h = mk.Megakernel(c.m, c.weights, c.max_batch, c.max_ctx)
    rc, out = _verify(c, [0, 1, 2], h, capture=False)
    assert rc == mk.MK_OK and out["status"] == mk.MK_OK
    b = len(c.lens)
    lg = torch.empty((b, c.m.vocab), dtype=torch.float32, device="cuda")
    am = torch.empty((b,), dtype=torch.int32, device="cuda")
    pos = _dev(c.lens)
    h.step(_dev(c.tokens), pos, pos + 1, kv2, lg, am)
    torch.cuda.synchronize()
    assert torch.equal(lg.cpu().view(torch.int32), out["logits"].view(torch.int32))
    assert torch.equal(am.cpu(), out["argmax"])
    assert torch.equal(kv2.k_pool.view(torch.int16), c.kv.k_pool.view(torch.int16))
    h.close()


@pytest.mark.parametrize("bad", ["first-after-row", "gap-in-positions", "first-not-a-head"])
def test_malformed_groups_are_rejected_on_the_device(bad):
    c, first = _grouped_case(synth.TINY, [30, 10], [3, 2], tag="verify-bad")
    k0 = c.kv.k_pool.clone()
    if bad == "first-after-row":
        first = [0, 2, 0, 3, 3]
    elif bad == "gap-in-positions":
        c.lens[2] += 1
    else:  # row 3 joins row 0's group without following it, and row 4 names row 3 as its first
        first = [0, 0, 0, 0, 3]
    h = mk.Megakernel(c.m, c.weights, c.max_batch, c.max_ctx)
    rc, out = _verify(c, first, h, capture=False)
    assert out["status"] == mk.MK_ERR_BOUNDS
    assert torch.equal(k0.view(torch.int16), c.kv.k_pool.view(torch.int16))  # nothing written
    h.reset()
    h.close()
