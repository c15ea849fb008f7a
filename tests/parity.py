"""Helpers shared by the GPU parity tests: run one step on the device through the
C ABI, run the float64 oracle on the same inputs, compare mid-states."""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

import bandwidth_bound_b200 as mk
import oracle
import synth

# Tolerances (stated on the decode path: hidden-state relative L2 per layer, max |dlogit|,
# 1 bf16 ulp on stored KV entries; integer state bit-exact).
HIDDEN_REL_L2 = 1e-2
LOGIT_ABS = 5e-2
KV_ULP = 1.0


@dataclass
class Case:
    m: synth.ModelConfig
    lens: list            # prior entries S_i per sequence (= positions)
    tokens: list
    gain_std: float = 0.0
    max_batch: int = 0
    max_ctx: int = 0
    weights: dict = None
    kv: synth.KVCache = None
    extra: dict = field(default_factory=dict)


def make_case(m, lens, gain_std=0.0, max_batch=0, max_ctx=0, tag="", weights=None, kv_spare=3,
              kv_room=1) -> Case:
    b = len(lens)
    max_batch = max_batch or b
    max_ctx = max_ctx or (max(lens) + 1)
    wts = weights if weights is not None else synth.make_weights(m, device="cuda", gain_std=gain_std)
    kv = synth.make_kv_cache(m, list(lens), device="cuda", max_ctx=max_ctx, spare_pages=kv_spare,
                             batch_cap=max_batch, tag=tag, room=kv_room)
    toks = synth.token_ids(m, b, tag=tag or m.name)
    return Case(m, list(lens), toks, gain_std, max_batch, max_ctx, wts, kv)


def gpu_step(c: Case, handle=None, batch=None, debug=True, argmax=True):
    """Run one step; returns dict of device results (CPU copies) and the handle."""
    b = len(c.lens) if batch is None else batch
    if handle is None:
        handle = mk.Megakernel(c.m, c.weights, c.max_batch, c.max_ctx)
    dev = "cuda"
    tok = torch.tensor(c.tokens[:b], dtype=torch.int32, device=dev)
    pos = torch.tensor(c.lens[:b], dtype=torch.int32, device=dev)
    lens = pos + 1
    logits = torch.full((b, c.m.vocab), float("nan"), dtype=torch.float32, device=dev)
    am = torch.full((b,), -1, dtype=torch.int32, device=dev) if argmax else None
    dbg = None
    if debug:
        dbg = torch.full((c.m.n_layers + 1, c.max_batch, c.m.hidden), float("nan"), dtype=torch.float32,
                         device=dev)
    handle.set_debug(dbg)  # None: the configuration a server (and bench.py) runs, no mid-state stores
    handle.step(tok, pos, lens, c.kv, logits, am)
    torch.cuda.synchronize()
    st = handle.status()
    out = {"status": st, "logits": logits.cpu(), "argmax": am.cpu() if am is not None else None,
           "hidden": dbg[:, :b].cpu() if dbg is not None else None}
    return out, handle


def run_oracle(c: Case, k_before, v_before, batch=None, layers=None, anchor=None):
    """The float64 oracle on the case's inputs.

    With ``anchor`` (the GPU's captured residual stream [L+1][b][d]) each layer is also
    run from the GPU's own input to that layer: "anchored" then holds, per layer, the
    oracle's new K/V for exactly the hidden state the GPU's layer started from, so the
    stored K/V are judged by that layer's arithmetic alone, without the drift that earlier
    layers' rounding carries into an unanchored comparison.  One float64 copy of each
    layer's weights serves both passes.
    """
    b = len(c.lens) if batch is None else batch
    table = c.kv.page_table[:b].cpu()
    if anchor is None:
        return oracle.decode_step(c.m, c.weights, k_before, v_before, table, c.tokens[:b], c.lens[:b],
                                  layers=layers)
    m = c.m
    L = m.n_layers if layers is None else layers
    ref = oracle.decode_step(c.m, c.weights, k_before, v_before, table, c.tokens[:b], c.lens[:b], layers=0)
    x = ref["hidden"][0]
    hidden = [x.clone()]
    keys = ("k_new", "v_new", "k_new_exact", "v_new_exact")
    e2e = {k: [] for k in keys}
    anch = {k: [] for k in keys}
    for li in range(L):
        lw = oracle.layer_weights_f64(c.weights, li)
        r = oracle.decode_layer(m, lw, x, k_before[li], v_before[li], table, c.lens[:b])
        ra = oracle.decode_layer(m, lw, anchor[li].to(torch.float64), k_before[li], v_before[li], table,
                                 c.lens[:b])
        x = r["x"]
        hidden.append(x.clone())
        for k in keys:
            e2e[k].append(r[k])
            anch[k].append(ra[k])
        del lw
    out = {"hidden": torch.stack(hidden), "slots": ref["slots"],
           "anchored": {k: torch.stack(v) for k, v in anch.items()}}
    out.update({k: torch.stack(v) for k, v in e2e.items()})
    if L == m.n_layers:
        out["logits"] = oracle.lm_head(m, c.weights, x)
        out["argmax"] = [oracle.argmax_lowest(out["logits"][i]) for i in range(b)]
    return out


def rel_l2(a: torch.Tensor, b: torch.Tensor) -> float:
    a = a.to(torch.float64)
    b = b.to(torch.float64)
    return float((a - b).norm() / b.norm().clamp_min(1e-300))


# Entries smaller than this fraction of their head vector's RMS are measured in ulps of
# the floor: drift from earlier layers is relative to the vector's scale, not to each
# entry.  A sequence at position 0 attends only to its own bf16-rounded V, so one
# legitimate rounding flip there moves the residual by ~2e-5 of its scale and the next
# layer's small entries by that much in absolute terms.
KV_FLOOR = 2.0 ** -5
# The re-anchored check (each layer run from the GPU's own input) needs no allowance for
# drift: only entries below 2^-8 of their head's RMS are measured at that floor.
KV_FLOOR_ANCHORED = 2.0 ** -8


def bf16_ulp_error(gpu: torch.Tensor, ref: torch.Tensor, floor: float = KV_FLOOR) -> torch.Tensor:
    """|gpu - ref| in units of the bf16 spacing at |ref|, per element.

    ref: float64 values already rounded to bf16 (oracle), shape [..., hd].  The
    magnitude is floored at ``floor`` times the RMS of its head vector, so that
    entries near zero are not counted in ulps of a tiny number.
    """
    g = gpu.to(torch.float64)
    r = ref.to(torch.float64)
    rms = torch.sqrt((r * r).mean(-1, keepdim=True))
    mag = torch.maximum(r.abs(), rms * floor).clamp_min(1e-30)
    ulp = torch.exp2(torch.floor(torch.log2(mag)) - 7)
    return (g - r).abs() / ulp


def check_step(c: Case, out: dict, ref: dict, k_before, v_before, batch=None, check_pool=True,
               logit_tol=LOGIT_ABS, e2e_kv_gate=True) -> dict:
    """Compare one GPU step with the oracle; returns the measured errors.

    e2e_kv_gate=False reports the end-to-end KV comparison without gating on it; it needs the
    re-anchored comparison (``ref`` from run_oracle with ``anchor``), which then decides."""
    b = len(c.lens) if batch is None else batch
    m = c.m
    P = m.page_size
    errs = {}
    assert out["status"] == mk.MK_OK, f"device status {out['status']}"
    # per-layer hidden states, whole batch and per sequence
    if out["hidden"] is not None:
        worst = 0.0
        hidden_fail = None
        for li in range(m.n_layers + 1):
            e = rel_l2(out["hidden"][li], ref["hidden"][li])
            worst = max(worst, e)
            for i in range(b):
                ei = rel_l2(out["hidden"][li, i], ref["hidden"][li, i])
                worst = max(worst, ei)
                if ei > HIDDEN_REL_L2 and hidden_fail is None:
                    hidden_fail = f"sequence {i} hidden after layer {li - 1}: rel L2 {ei}"
        errs["hidden_rel_l2"] = worst
        errs["hidden_rel_l2_per_layer"] = [round(rel_l2(out["hidden"][li], ref["hidden"][li]), 8)
                                           for li in range(m.n_layers + 1)]
    # KV: new entries within 1 ulp; everything else bit-identical (canaries included)
    k_after = c.kv.k_pool
    v_after = c.kv.v_pool
    worst_ulp = 0.0
    strict_fail = 0
    for i in range(b):
        page, slot = ref["slots"][i]
        assert page == int(c.kv.page_table[i, c.lens[i] // P]) and slot == c.lens[i] % P
        kg = k_after[:, page, :, slot, :].cpu()
        vg = v_after[:, page, :, slot, :].cpu()
        ek = bf16_ulp_error(kg, ref["k_new"][:, i])
        ev = bf16_ulp_error(vg, ref["v_new"][:, i])
        for name, e, gv, rv, ex in (("k", ek, kg, ref["k_new"][:, i], ref["k_new_exact"][:, i]),
                                    ("v", ev, vg, ref["v_new"][:, i], ref["v_new_exact"][:, i])):
            if float(e.max()) > worst_ulp:
                worst_ulp = float(e.max())
                at = [int(v) for v in torch.nonzero(e == e.max())[0]]
                errs["kv_worst"] = {"which": name, "seq": i, "layer_head_dim": at,
                                    "gpu": float(gv[tuple(at)]), "oracle_bf16": float(rv[tuple(at)]),
                                    "oracle_exact": float(ex[tuple(at)]),
                                    "head_rms": float(ex[at[0], at[1]].pow(2).mean().sqrt())}
        strict_fail += int((kg.to(torch.float64) != ref["k_new"][:, i]).sum())
        strict = max(float(bf16_ulp_error(kg, ref["k_new"][:, i], 0.0).max()),
                     float(bf16_ulp_error(vg, ref["v_new"][:, i], 0.0).max()))
        errs["kv_max_ulp_unfloored"] = max(errs.get("kv_max_ulp_unfloored", 0.0), strict)
    errs["kv_max_ulp"] = worst_ulp
    errs["kv_entries_not_bit_equal"] = strict_fail
    errs["kv_entries"] = 2 * b * ref["k_new"][:, 0].numel()
    # entries the end-to-end comparison lets through only because of its 2^-5 floor
    floor_only = 0
    anchored_worst, anchored_unfloored, anchored_over = 0.0, 0.0, 0
    for i in range(b):
        page, slot = ref["slots"][i]
        for pool, key in ((k_after, "k_new"), (v_after, "v_new")):
            gv = pool[:, page, :, slot, :].cpu()
            floored = bf16_ulp_error(gv, ref[key][:, i])
            plain = bf16_ulp_error(gv, ref[key][:, i], 0.0)
            floor_only += int(((plain > KV_ULP) & (floored <= KV_ULP)).sum())
            if "anchored" in ref:
                ra = ref["anchored"][key][:, i]
                ea = bf16_ulp_error(gv, ra, KV_FLOOR_ANCHORED)
                anchored_worst = max(anchored_worst, float(ea.max()))
                anchored_unfloored = max(anchored_unfloored, float(bf16_ulp_error(gv, ra, 0.0).max()))
                anchored_over += int((ea > KV_ULP).sum())
    errs["kv_pass_only_by_e2e_floor"] = floor_only
    if "anchored" in ref:
        errs["kv_anchored_max_ulp"] = anchored_worst
        errs["kv_anchored_max_ulp_unfloored"] = anchored_unfloored
    if "logits" in ref:
        errs["logit_max_abs"] = (out["logits"].to(torch.float64) - ref["logits"]).abs().max().item()
    print("parity:", errs)
    if out["hidden"] is not None:
        assert hidden_fail is None, hidden_fail
    if e2e_kv_gate:
        assert worst_ulp <= KV_ULP, f"new KV entry off by {worst_ulp} bf16 ulp"
    else:
        assert "anchored" in ref, "without the end-to-end KV gate the re-anchored check is required"
    if "anchored" in ref:
        assert anchored_worst <= KV_ULP, \
            f"{anchored_over} new KV entries off by up to {anchored_worst} bf16 ulp from the oracle's layer run " \
            f"from the GPU's own input (floor 2^-8 of the head RMS)"
    if check_pool:
        mask = torch.ones(k_after.shape[1:4], dtype=torch.bool)  # [P][nkv][page]
        for i in range(b):
            page, slot = ref["slots"][i]
            mask[page, :, slot] = False
        kb = k_before.view(torch.int16)
        vb = v_before.view(torch.int16)
        ka = k_after.cpu().view(torch.int16)
        va = v_after.cpu().view(torch.int16)
        mm = mask[None, :, :, :, None].expand_as(ka)
        assert torch.equal(ka[mm], kb[mm]), "the step wrote KV outside the new slots"
        assert torch.equal(va[mm], vb[mm]), "the step wrote KV outside the new slots"
    # logits and argmax
    if "logits" in ref:
        dl = (out["logits"].to(torch.float64) - ref["logits"]).abs().max().item()
        errs["logit_max_abs"] = dl
        assert math.isfinite(dl) and dl <= logit_tol, f"max |dlogit| {dl}"
        # mean log-prob error of the greedy token (reported, not gated)
        lp_g = torch.log_softmax(out["logits"].to(torch.float64), -1)
        lp_r = torch.log_softmax(ref["logits"], -1)
        idx = torch.tensor(ref["argmax"])
        errs["logprob_err"] = float((lp_g.gather(1, idx[:, None]) - lp_r.gather(1, idx[:, None])).abs().mean())
        if out["argmax"] is not None:
            for i in range(b):
                got, want = int(out["argmax"][i]), ref["argmax"][i]
                if got != want:
                    # only a true numerical tie may differ: the oracle's top-2 gap below the error
                    top = torch.topk(ref["logits"][i], 2).values
                    gap = float(top[0] - top[1])
                    assert gap < dl and abs(float(ref["logits"][i, got]) - float(top[0])) <= 2 * dl, \
                        f"sequence {i}: argmax {got} != oracle {want} (gap {gap})"
                    errs.setdefault("argmax_ties", 0)
                    errs["argmax_ties"] += 1
            # the device argmax is the argmax of the device logits
            assert [int(v) for v in out["argmax"]] == [oracle.argmax_lowest(out["logits"][i].to(torch.float64))
                                                       for i in range(b)]
    return errs
