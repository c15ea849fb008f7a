"""Summaries of the per-task timeline the megakernel records (mk_set_trace).

Each record is {t_wait_start, t_wait_end, t_end, meta, compute, reduce, epilogue,
signal}: the three timestamps in globaltimer ns (comparable across SMs), meta = op |
layer << 8 | sm << 24 | slot_wait << 40, and the durations in SM clock cycles (the
globaltimer is too coarse for sub-microsecond intervals), converted here with the SM
clock.  The summary answers where a step's time goes: waiting on dependency counters
(another SM's work not done), waiting on pool slots (HBM bytes not yet landed), or
computing.  The in-task durations (compute, reduce, epilogue, slot_wait) are recorded only
by a library built with MK_TRACE_DETAIL=1 (`build.py --trace-detail`); the default build
leaves them 0 and records the timestamps and the signal time.
"""
from __future__ import annotations

import numpy as np

OPS = {1: "embed", 2: "qkv", 3: "attn", 4: "oproj", 5: "gateup", 6: "down", 7: "lmhead"}


def decode(records, sm_mhz: float = 1965.0) -> dict:
    """Fields of the records; durations converted from SM cycles to ns at sm_mhz."""
    r = np.asarray(records, dtype=np.uint64).reshape(-1, 8)
    meta = r[:, 3]
    ns = 1e3 / sm_mhz
    cyc = lambda a: (a.astype(np.float64) * ns).astype(np.int64)  # noqa: E731
    return {
        "compute": cyc(r[:, 4]), "reduce": cyc(r[:, 5]),
        "epilogue": cyc(r[:, 6]), "signal": cyc(r[:, 7]),
        "t0": r[:, 0].astype(np.int64), "t1": r[:, 1].astype(np.int64), "t2": r[:, 2].astype(np.int64),
        "op": (meta & np.uint64(0xFF)).astype(np.int64),
        "layer": ((meta >> np.uint64(8)) & np.uint64(0xFFFF)).astype(np.int64),
        "sm": ((meta >> np.uint64(24)) & np.uint64(0xFFFF)).astype(np.int64),
        "slot_wait": cyc(meta >> np.uint64(40)),
    }


def summarize(records, n_layers: int, sm_mhz: float = 1965.0) -> str:
    d = decode(records, sm_mhz)
    base = int(d["t0"].min())
    end = int(d["t2"].max())
    step_us = (end - base) / 1e3
    nsm = int(d["sm"].max()) + 1
    lines = [f"step {step_us:.1f} us over {nsm} SMs, {len(d['op'])} tasks"]
    lines.append(f"{'op':8s} {'tasks':>6s} {'dep-wait':>9s} {'work':>8s} {'slot-wait':>10s} {'compute':>8s} "
                 f"{'reduce':>7s} {'epilog':>7s} {'signal':>7s}   (us per SM over the step)")
    for op, name in OPS.items():
        m = d["op"] == op
        if not m.any():
            continue
        dep = (d["t1"][m] - d["t0"][m]).sum() / 1e3 / nsm
        work = (d["t2"][m] - d["t1"][m]).sum() / 1e3 / nsm
        sw = d["slot_wait"][m].sum() / 1e3 / nsm
        part = [d[k][m].sum() / 1e3 / nsm for k in ("compute", "reduce", "epilogue", "signal")]
        lines.append(f"{name:8s} {int(m.sum()):6d} {dep:9.1f} {work:8.1f} {sw:10.1f} {part[0]:8.1f} {part[1]:7.1f} "
                     f"{part[2]:7.1f} {part[3]:7.1f}")
    # per-layer phase windows (first work start -> last end), relative to the step start
    lines.append("phase windows (us from step start: first start .. last end) for a few layers")
    for l in sorted({0, 1, n_layers // 2, n_layers - 1}):
        parts = []
        for op in (2, 3, 4, 5, 6):
            m = (d["op"] == op) & (d["layer"] == l)
            if m.any():
                parts.append(f"{OPS[op]} {(d['t1'][m].min() - base) / 1e3:.1f}..{(d['t2'][m].max() - base) / 1e3:.1f}")
        lines.append(f"  layer {l}: " + ", ".join(parts))
    m = d["op"] == 7
    if m.any():
        lines.append(f"  lmhead {(d['t1'][m].min() - base) / 1e3:.1f}..{(d['t2'][m].max() - base) / 1e3:.1f}")
    busy = np.zeros(nsm)
    dep = np.zeros(nsm)
    for s in range(nsm):
        m = d["sm"] == s
        busy[s] = (d["t2"][m] - d["t1"][m]).sum() / 1e3
        dep[s] = (d["t1"][m] - d["t0"][m]).sum() / 1e3
    lines.append(f"per-SM work us: min {busy.min():.1f} median {np.median(busy):.1f} max {busy.max():.1f}; "
                 f"dep-wait us: min {dep.min():.1f} median {np.median(dep):.1f} max {dep.max():.1f}")
    return "\n".join(lines)
