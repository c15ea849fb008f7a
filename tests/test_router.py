"""Routing among handles built for different bounds: the pick rule on the host (no GPU),
and a routed step equal, bit for bit, to the same step on the picked handle (GPU)."""
import gc

import pytest
import torch

import bandwidth_bound_b200 as mk
import synth
from parity import make_case

BOUNDS = [(8, 4096), (1, 4096), (1, 512), (16, 8192), (8, 4096)]


@pytest.mark.parametrize("batch, pos, want", [
    (1, 100, 2),     # the batch-1 handle with the shortest context that holds position 100
    (1, 511, 2),     # max_ctx 512 holds positions up to 511
    (1, 512, 1),
    (3, 10, 0),      # batch 3: a batch-8 handle; the first of two equal ones
    (8, 4095, 0),
    (9, 0, 3),
    (2, 5000, 3),
])
def test_pick_rule(batch, pos, want):
    assert mk.route_pick(BOUNDS, batch, pos) == want


@pytest.mark.parametrize("batch, pos", [(17, 0), (1, 8192), (0, 5), (1, -1)])
def test_no_handle_fits(batch, pos):
    assert mk.route_pick(BOUNDS, batch, pos) == mk.MK_ERR_INVALID_ARG


@pytest.mark.gpu
def test_routed_step_equals_the_picked_handle():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device (deselect with -m 'not gpu')")
    c = make_case(synth.TINY, [40, 9, 77], gain_std=0.1, max_ctx=128, tag="router")
    h8 = mk.Megakernel(c.m, c.weights, 8, 128)
    h1 = mk.Megakernel(c.m, c.weights, 1, 128)
    r = mk.Router([h8, h1])
    for b, want in ((1, 1), (3, 0)):
        kv2 = synth.KVCache(c.kv.k_pool.clone(), c.kv.v_pool.clone(), c.kv.page_table.clone(), c.kv.num_pages,
                            c.kv.max_pages_per_seq, list(c.kv.ctx_lens))
        tok = torch.tensor(c.tokens[:b], dtype=torch.int32, device="cuda")
        pos = torch.tensor(c.lens[:b], dtype=torch.int32, device="cuda")
        lg = torch.empty((b, c.m.vocab), dtype=torch.float32, device="cuda")
        am = torch.empty((b,), dtype=torch.int32, device="cuda")
        rc, picked = r.step(tok, pos, pos + 1, max(c.lens[:b]), c.kv, lg, am)
        assert rc == mk.MK_OK and picked == want
        lg2 = torch.empty_like(lg)
        am2 = torch.empty_like(am)
        (h1 if want == 1 else h8).step(tok, pos, pos + 1, kv2, lg2, am2)
        torch.cuda.synchronize()
        assert torch.equal(lg.cpu().view(torch.int32), lg2.cpu().view(torch.int32))
        assert torch.equal(am.cpu(), am2.cpu())
    r.close()
    h8.close()
    h1.close()
    gc.collect()
    torch.cuda.empty_cache()
