"""Decode-step benchmark: tokens/s and model bandwidth utilisation on B200.

One step = one call of mk_decode_step: the whole decode step (embedding gather,
all layers, final norm, LM head, argmax) for one batch, as one kernel launch.
The metric follows "ForgeMegakernel" §2.2: MBU = B(b, S) / (t_step * peak HBM),
B counting every weight byte, the gathered embedding rows (not the table) and
the prior KV entries; decode tokens/s = b / t_step.

  python bench.py [--gpus N --steps K --warmup W --workload NAME --impl mk|reference]

Under torchrun (N > 1) every rank runs an independent replica of the workload on
its own GPU (the step has no data-parallel exchange); value = tokens of all
ranks / the slowest rank's time.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "decode tokens/s"
NOMINAL_HBM_GBS = 8000.0  # the pages' "~8 TB/s" B200 peak used for MBU
MULTI_STEPS = 32  # steps per call of the on-device greedy loop line


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="llama3-8b-b8", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="mk", choices=["mk", "reference"])
    ap.add_argument("--no-secondary", action="store_true", help="skip the batch-1 line of the same model")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-all-configs", action="store_true", help="skip timing the other named shapes")
    ap.add_argument("--no-kernel-per-op", action="store_true", help="skip timing the kernel-per-op comparison step")
    ap.add_argument("--no-multi-step", action="store_true",
                    help="skip timing the on-device multi-step loop, its sampling variant and the multi-token step")
    ap.add_argument("--max-blocks", type=int, default=0, help="schedule option: 8-row blocks per GEMV task")
    ap.add_argument("--attn-slots", type=int, default=0, help="schedule option: attention slots per SM")
    ap.add_argument("--trace", default="", help="write a per-task timeline summary of one step to this file")
    ap.add_argument("--layers", type=int, default=0,
                    help="profiling aid: run a model shortened to this many layers (not a bench line)")
    return ap.parse_args()


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "source": "fallback"}


def workload_desc(w: synth.Workload, lens) -> dict:
    m = w.model
    return {
        "workload": w.name,
        "shape": (f"{m.n_layers}L d{m.hidden} {m.n_heads}/{m.n_kv_heads} heads hd{m.head_dim} "
                  f"F{m.ffn} V{m.vocab} {'tied' if m.tied else 'untied'}"),
        "batch": w.batch,
        "context": w.ctx[1] if w.ctx[0] == "fixed" else f"U[{w.ctx[1]},{w.ctx[2]}] seeded: {lens}",
        "kv": "paged bf16, 16-token pages, shuffled page table",
    }


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 7:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": float(rows[0][1]),
                "power_w_max": max(float(r[2]) for r in rows), "samples": len(rows), "reasons": sorted(reasons)}


def setup_dist(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(world, v: float) -> float:
    if world == 1:
        return v
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, total_ms_this_rank: float, steps: int, batch: int) -> tuple[float, float]:
    """(ms per step, tokens/s of the whole job): the slowest rank's device time over
    `steps` steps, every rank decoding its own batch of `batch` sequences."""
    ms = max_over_ranks(world, total_ms_this_rank) / steps
    return ms, world * batch / (ms / 1e3)


def kernel_source_hash(root: str = ROOT) -> str:
    """Hash of the kernel's source code, comments and layout left out: a summary taken on a
    kernel stays valid through edits of its comments, and no longer after any code change."""
    import hashlib
    import re

    code = ""
    for f in ("mk_kernel.cu", "mk_common.h", "mk_kernel.h"):
        with open(os.path.join(root, "bandwidth_bound_b200", "csrc", f)) as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        code += " ".join(text.split()) + "\n"
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def traffic_from_profile(workload: str):
    """Per-launch DRAM bytes recorded by the committed ncu summary, if it covers this
    workload and the kernel code it was taken on is unchanged."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    h = kernel_source_hash()
    with open(p) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 3 and parts[0] == workload and parts[1] == h:
                return float(parts[2])
    return None


def cpu_baseline(w: synth.Workload, wts, kv, toks, lens, budget_s: float = 12.0) -> dict:
    """The float64 oracle on the host cores, on a bounded sample of the same step:
    whole layers (repeated until ~budget_s of CPU time) and a slice of the LM head,
    scaled to one full step."""
    import oracle

    m = w.model
    cores = torch.get_num_threads()
    pt = kv.page_table.cpu()
    kp = kv.k_pool[:1].cpu()
    vp = kv.v_pool[:1].cpu()
    one = {"embed": wts["embed"], "final_norm": wts["final_norm"], "lm_head": wts["lm_head"],
           "layers": [{k: v.cpu() for k, v in wts["layers"][0].items()}]}
    cfg1 = synth.scaled_model(m, n_layers=1)
    t_layers = []
    t0 = time.perf_counter()
    while True:
        a = time.perf_counter()
        oracle.decode_step(cfg1, one, kp, vp, pt, toks, lens, want_logits=False)
        t_layers.append(time.perf_counter() - a)
        if time.perf_counter() - t0 > budget_s * 0.8:
            break
    rows = min(m.vocab, 16384)
    head = wts["lm_head"][:rows].cpu()
    x = torch.randn(len(toks), m.hidden, dtype=torch.float64)
    a = time.perf_counter()
    _ = x @ head.to(torch.float64).T
    t_head = (time.perf_counter() - a) * m.vocab / rows
    t_step = statistics.median(t_layers) * m.n_layers + t_head
    return {"value": len(toks) / t_step, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": (f"{len(t_layers)} runs of layer 0 (embedding gather + 1 layer, float64) x {m.n_layers} "
                       f"layers + {rows} of {m.vocab} LM-head rows scaled; same seeded inputs"),
            "seconds_per_step": t_step}


def run_reference(args, world, rank):
    """The oracle itself, timed as the reference arm."""
    if rank != 0:
        return
    w = synth.WORKLOADS[args.workload]
    lens = w.context_lengths()
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    m = w.model
    wts = synth.make_weights(m, device=dev, layers=[0])
    kv = synth.make_kv_cache(m, lens, device=dev)
    toks = synth.token_ids(m, w.batch, tag=w.name)
    per = []
    for k in range(args.warmup + args.steps):
        cb = cpu_baseline(w, wts, kv, toks, lens, budget_s=0.5)
        if k >= args.warmup:
            per.append(cb["seconds_per_step"])
    t = statistics.median(per)
    value = w.batch / t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
            "ms_per_step_kind": "projected: median over samples of (one layer x layers + an LM-head slice scaled "
                                "to the vocabulary), not a timed full step",
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_desc(w, lens),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cb["cores"], "kind": "oracle",
                             "sample": cb["sample"]},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def time_steps(fn, steps, stream, flush=None):
    """CUDA-event time of `steps` calls of fn on `stream` (ms total, per-step list)."""
    per = []
    torch.cuda.nvtx.range_push("timed")  # lets ncu --nvtx-include "timed/" select these launches
    try:
        return _time_steps(fn, steps, stream, flush, per)
    finally:
        torch.cuda.nvtx.range_pop()


def _time_steps(fn, steps, stream, flush, per):
    if flush is None:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        e0.record(stream)
        ev[0].record(stream)
        for k in range(steps):
            fn()
            ev[k + 1].record(stream)
        e1.record(stream)
        torch.cuda.synchronize()
        per = [ev[k].elapsed_time(ev[k + 1]) for k in range(steps)]
        return e0.elapsed_time(e1), per
    total = 0.0
    for _ in range(steps):
        flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        per.append(a.elapsed_time(b))
        total += per[-1]
    return total, per


def run_mk(args, world, rank, local):
    import bandwidth_bound_b200 as mk

    w = synth.WORKLOADS[args.workload]
    if args.layers:
        w = synth.Workload(w.name + f"-first{args.layers}layers", synth.scaled_model(w.model, n_layers=args.layers),
                           w.batch, w.ctx)
    m = w.model
    lens = w.context_lengths() if not args.layers else synth.WORKLOADS[args.workload].context_lengths()
    b = w.batch
    max_ctx = max(lens) + MULTI_STEPS + 1
    wts = synth.make_weights(m, device="cuda")
    # pages for the multi-step line's positions too (lens .. lens + MULTI_STEPS - 1)
    kv = synth.make_kv_cache(m, lens, device="cuda", max_ctx=max_ctx, batch_cap=max(b, 8), room=MULTI_STEPS)
    toks = synth.token_ids(m, b, tag=w.name)
    plan = None
    if args.max_blocks or args.attn_slots:
        plan = mk.Plan(mk.model_cfg(m, b, max_ctx), num_sms=torch.cuda.get_device_properties(local).multi_processor_count,
                       attn_slots_per_sm=args.attn_slots, max_blocks=args.max_blocks)
    h = mk.Megakernel(m, wts, b, max_ctx, plan=plan)
    stream = torch.cuda.current_stream()
    tok_d = torch.tensor(toks, dtype=torch.int32, device="cuda")
    pos_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
    len_d = pos_d + 1
    logits = torch.empty((b, m.vocab), dtype=torch.float32, device="cuda")
    am = torch.empty((b,), dtype=torch.int32, device="cuda")
    B = mk.step_bytes(m, lens)
    l2 = torch.cuda.get_device_properties(local).L2_cache_size
    flush = None
    l2_note = f"inputs larger than L2 ({B / 1e9:.2f} GB read per step vs {l2 / 1e6:.0f} MB L2)"
    if B < 4 * l2:
        scrub = torch.empty(2 * l2 // 4, dtype=torch.float32, device="cuda")
        flush = lambda: scrub.zero_()  # noqa: E731
        l2_note = "L2 flushed between steps (2x L2 buffer written, untimed)"

    def step():
        h.step(tok_d, pos_d, len_d, kv, logits, am, stream=stream, check=False)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert h.status() == mk.MK_OK, f"device status {h.status()}"
    if args.trace:
        from bandwidth_bound_b200 import trace as mktrace

        rec = torch.zeros((h.num_tasks(), 8), dtype=torch.int64, device="cuda")
        h.set_trace(rec)
        step()
        torch.cuda.synchronize()
        h.set_trace(None)
        raw = rec.cpu().numpy().view("uint64")
        with open(args.trace, "w") as f:
            f.write(mktrace.summarize(raw, m.n_layers) + "\n")
        import numpy as np

        np.save(os.path.splitext(args.trace)[0] + ".npy", raw)
        if not args.no_secondary and b > 1:
            h1t = mk.Megakernel(m, wts, 1, max_ctx)  # the batch-1 handle of the secondary line
            for _ in range(args.warmup):
                h1t.step(tok_d[:1], pos_d[:1], len_d[:1], kv, logits[:1], am[:1], stream=stream, check=False)
            rec1 = torch.zeros((h1t.num_tasks(), 8), dtype=torch.int64, device="cuda")
            h1t.set_trace(rec1)
            h1t.step(tok_d[:1], pos_d[:1], len_d[:1], kv, logits[:1], am[:1], stream=stream, check=False)
            torch.cuda.synchronize()
            h1t.set_trace(None)
            h1t.close()
            raw1 = rec1.cpu().numpy().view("uint64")
            with open(args.trace, "a") as f:
                f.write("--- batch 1 ---\n" + mktrace.summarize(raw1, m.n_layers) + "\n")
            np.save(os.path.splitext(args.trace)[0] + "_b1.npy", raw1)
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    total_ms, per = time_steps(step, args.steps, stream, flush)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    assert h.status() == mk.MK_OK, f"device status {h.status()}"
    ms, value = job_throughput(world, total_ms, args.steps, b)
    peaks = measured_peaks()
    achieved = B / (ms / 1e3) / 1e9
    traffic = traffic_from_profile(w.name)

    # end to end through the host-buffer entry point (pinned host memory)
    tok_h = torch.tensor(toks, dtype=torch.int32).pin_memory()
    pos_h = torch.tensor(lens, dtype=torch.int32).pin_memory()
    len_h = (pos_h + 1).pin_memory()
    logits_h = torch.empty((b, m.vocab), dtype=torch.float32).pin_memory()
    am_h = torch.empty((b,), dtype=torch.int32).pin_memory()

    def step_host():
        h.step_host(tok_h, pos_h, len_h, kv, logits_h, am_h, stream=stream, check=False)

    for _ in range(3):
        step_host()
    barrier(world)
    e2e_total, _ = time_steps(step_host, min(args.steps, 100), stream, flush)
    e2e_ms = max_over_ranks(world, e2e_total) / min(args.steps, 100)
    h2d = 3 * 4 * b
    d2h = b * m.vocab * 4 + b * 4

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_desc(w, lens), l2=l2_note, parallelism=f"replicas x{world}"),
        "mbu": B / (ms / 1e3) / (NOMINAL_HBM_GBS * 1e9),
        "mbu_vs_measured_copy": achieved / peaks["hbm_gbs"],
        "bytes_per_step": B,
        "step_ms": {"median": statistics.median(per), "p10": sorted(per)[len(per) // 10],
                    "p90": sorted(per)[(9 * len(per)) // 10]},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                     "peak_source": peaks["source"], "kernel": "mk_decode_kernel (the whole step)"},
        "clocks": clk,
        "e2e": {"value": world * b / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": args.steps * h.launches_per_step(),
    }
    if not args.no_secondary and b > 1:
        # batch 1 of the same model, weights and KV cache (first sequence) on a handle built for
        # batch 1, as a batch-1 server would create it: its stages carry one fp32 operand row,
        # so each 50 KB stage holds 384 weight columns of a 64-row task instead of 320
        h1 = mk.Megakernel(m, wts, 1, max_ctx)
        b1 = lambda: h1.step(tok_d[:1], pos_d[:1], len_d[:1], kv, logits[:1], am[:1], stream=stream,  # noqa: E731
                             check=False)
        for _ in range(args.warmup):
            b1()
        barrier(world)
        t1, _ = time_steps(b1, min(args.steps, 200), stream, flush)
        ms1 = max_over_ranks(world, t1) / min(args.steps, 200)
        B1 = mk.step_bytes(m, lens[:1])
        h1.close()
        line["secondary"] = {"workload": f"{m.name}-b1 (batch-1 handle, context {lens[0]})", "ms_per_step": ms1,
                             "tokens_per_s": world / (ms1 / 1e3), "mbu": B1 / (ms1 / 1e3) / (NOMINAL_HBM_GBS * 1e9),
                             "achieved_gbs": B1 / (ms1 / 1e3) / 1e9}
    if not args.no_multi_step:
        line["multi_step"] = time_multi_step(mk, h, m, tok_d, pos_d, kv, lens, logits, stream, world, ms, flush)
        line["multi_step_top_k"] = time_multi_step(mk, h, m, tok_d, pos_d, kv, lens, logits, stream, world, ms, flush,
                                                   top_k=50)
        if world == 1 and not args.layers:
            line["verify"] = [time_verify(mk, m, wts, kv, lens[0], t, stream, flush) for t in (4, 8)]
    if world == 1 and not args.layers and not args.no_kernel_per_op:
        line["kernel_per_op"] = [time_kernel_per_op(mk, m, wts, kv, lens, bb, max_ctx, stream, flush, steps)
                                 for bb, steps in ((b, ms), (1, line.get("secondary", {}).get("ms_per_step")))]
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = {k: v for k, v in cpu_baseline(w, wts, kv, toks, lens).items()
                                if k != "seconds_per_step"}
    h.close()
    if world == 1 and not args.no_all_configs and not args.layers and args.workload == "llama3-8b-b8":
        # every named shape, each on a handle built for its own batch; the Llama-3-8B lines are
        # the headline's and the batch-1 line's own measurements
        rows = [{"workload": w.name, "batch": b, "ms_per_step": ms, "tokens_per_s": value,
                 "mbu": line["mbu"], "frac_of_measured_copy": line["mbu_vs_measured_copy"], "l2": l2_note}]
        if "secondary" in line:
            sec = line["secondary"]
            rows.append({"workload": "llama3-8b-b1", "batch": 1, "ms_per_step": sec["ms_per_step"],
                         "tokens_per_s": sec["tokens_per_s"], "mbu": sec["mbu"],
                         "frac_of_measured_copy": sec["achieved_gbs"] / peaks["hbm_gbs"], "l2": l2_note})
        del wts, kv
        torch.cuda.empty_cache()
        for name in ("tiny-b1", "smollm2-135m-b1", "llama3.2-1b-b9", "llama2-13b-b4", "qwen3-0.6b-b1", "qwen3-8b-b1"):
            rows.extend(time_config(mk, name, stream, min(args.steps, 200), args.warmup, peaks))
        line["all_configs"] = rows
    if rank == 0:
        print(json.dumps(line), flush=True)


def time_multi_step(mk, h, m, tok_d, pos_d, kv, lens, logits, stream, world, single_ms, flush, top_k=1) -> dict:
    """The on-device loop: MULTI_STEPS steps per call (each step's token is the next step's
    input, at the next position), the host waiting once per call; greedy, or top-k sampling
    (temperature 0.8, seeded uniforms) fused into the step.  Per call the context of every
    sequence grows by MULTI_STEPS, so the bytes are summed step by step."""
    n, runs = MULTI_STEPS, 5
    b = len(lens)
    toks_out = torch.empty((n, b), dtype=torch.int32, device="cuda")
    g = torch.Generator(device="cpu").manual_seed(11)
    uni = torch.rand((n, b), generator=g).to("cuda")

    def run():
        h.steps(n, tok_d, pos_d, kv, toks_out, logits, stream=stream, check=False, top_k=top_k, temperature=0.8,
                uniforms=uni)

    for _ in range(2):
        run()
    torch.cuda.synchronize()
    barrier(world)
    total, _ = time_steps(run, runs, stream, flush)
    assert h.status() == mk.MK_OK, f"device status {h.status()}"
    ms = max_over_ranks(world, total) / (runs * n)
    B = sum(mk.step_bytes(m, [s + k for s in lens]) for k in range(n)) / n
    return {"n_steps_per_call": n, "calls": runs, "top_k": top_k, "ms_per_step": ms,
            "tokens_per_s": world * b / (ms / 1e3),
            "mbu": B / (ms / 1e3) / (NOMINAL_HBM_GBS * 1e9), "single_step_ms": single_ms,
            "launches_per_call": n, "host_waits_per_call": 1,
            "l2": "no flush between the steps of one call" + ("; L2 flushed between calls" if flush else "")}


def time_verify(mk, m, wts, kv, prior: int, t: int, stream, flush, runs: int = 50) -> dict:
    """A multi-token step: one sequence with `prior` cached entries and t new (draft) tokens
    as t rows of one launch on a handle built for t rows; the rows share the sequence's
    page-table row.  Against t single-token steps, which read every weight t times."""
    h = mk.Megakernel(m, wts, t, prior + t + 1)
    table = kv.page_table[torch.zeros(t, dtype=torch.long, device=kv.page_table.device)].contiguous()
    gkv = synth.KVCache(kv.k_pool, kv.v_pool, table, kv.num_pages, kv.max_pages_per_seq, [prior + j for j in range(t)])
    tok = torch.tensor(synth.token_ids(m, t, tag="verify"), dtype=torch.int32, device="cuda")
    pos = torch.arange(prior, prior + t, dtype=torch.int32, device="cuda")
    first = torch.zeros(t, dtype=torch.int32, device="cuda")
    lg = torch.empty((t, m.vocab), dtype=torch.float32, device="cuda")
    am = torch.empty((t,), dtype=torch.int32, device="cuda")

    def run():
        h.verify(tok, pos, pos + 1, first, gkv, lg, am, stream=stream, check=False)

    for _ in range(3):
        run()
    torch.cuda.synchronize()
    total, _ = time_steps(run, runs, stream, flush)
    assert h.status() == mk.MK_OK, f"device status {h.status()}"
    h.close()
    ms = total / runs
    return {"workload": f"{m.name}: 1 sequence, {prior} cached entries, {t} new tokens in one launch",
            "tokens": t, "ms_per_step": ms, "tokens_per_s": t / (ms / 1e3)}


def time_kernel_per_op(mk, m, wts, kv, lens, b, max_ctx, stream, flush, mk_ms, runs: int = 30) -> dict:
    """The same step as one kernel per operation (10 per layer + 4), on the same weights and
    cache: replayed as a CUDA graph with programmatic dependent launch, launched on the
    stream, and the same launches with kernels that do nothing: that graph's time is what
    the 10 L + 4 kernel boundaries cost by themselves."""
    k = mk.KernelPerOp(m, wts, b, max_ctx)
    tok = torch.tensor(synth.token_ids(m, b, tag="kpo"), dtype=torch.int32, device="cuda")
    pos = torch.tensor(lens[:b], dtype=torch.int32, device="cuda")
    lg = torch.empty((b, m.vocab), dtype=torch.float32, device="cuda")
    am = torch.empty((b,), dtype=torch.int32, device="cuda")
    out = {"workload": f"{m.name} b{b}", "launches_per_step": k.launches_per_step()}
    for name, mode in (("graph_pdl", mk.KPO_GRAPH), ("stream_pdl", mk.KPO_STREAM)):
        run = lambda: k.step(tok, pos, pos + 1, kv, lg, am, mode=mode, stream=stream)  # noqa: E731
        for _ in range(3):
            run()
        torch.cuda.synchronize()
        total, _ = time_steps(run, runs, stream, flush)
        out[f"ms_per_step_{name}"] = total / runs
    run = lambda: k.step(tok, pos, pos + 1, kv, lg, am, mode=mk.KPO_EMPTY, stream=stream)  # noqa: E731
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    total, _ = time_steps(run, runs, stream, None)
    out["ms_per_step_launches_only"] = total / runs
    out["us_per_launch"] = 1e3 * out["ms_per_step_launches_only"] / out["launches_per_step"]
    if mk_ms:
        out["megakernel_ms_per_step"] = mk_ms
        out["graph_vs_megakernel"] = out["ms_per_step_graph_pdl"] / mk_ms
    k.close()
    return out


def time_config(mk, name: str, stream, steps: int, warmup: int, peaks: dict) -> list:
    """ms/step, tokens/s and MBU of one named workload on a handle built for its batch.  The
    ragged Llama-3.2-1B batch is timed as its 8 first sequences and then with the 9th joined,
    on the same handle (max_batch 9), as a server would run a late arrival."""
    w = synth.WORKLOADS[name]
    m = w.model
    lens = w.context_lengths()
    max_ctx = max(lens) + 2
    wts = synth.make_weights(m, device="cuda")
    kv = synth.make_kv_cache(m, lens, device="cuda", max_ctx=max_ctx, batch_cap=w.batch)
    toks = synth.token_ids(m, w.batch, tag=w.name)
    tok_d = torch.tensor(toks, dtype=torch.int32, device="cuda")
    pos_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
    len_d = pos_d + 1
    logits = torch.empty((w.batch, m.vocab), dtype=torch.float32, device="cuda")
    am = torch.empty((w.batch,), dtype=torch.int32, device="cuda")
    h = mk.Megakernel(m, wts, w.batch, max_ctx)
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    scrub = torch.empty(2 * l2 // 4, dtype=torch.float32, device="cuda")
    out = []
    batches = [8, 9] if name == "llama3.2-1b-b9" else [w.batch]
    for b in batches:
        B = mk.step_bytes(m, lens[:b])
        flush = (lambda: scrub.zero_()) if B < 4 * l2 else None
        fn = lambda: h.step(tok_d[:b], pos_d[:b], len_d[:b], kv, logits[:b], am[:b], stream=stream,  # noqa: E731
                            check=False)
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        total, per = time_steps(fn, steps, stream, flush)
        assert h.status() == mk.MK_OK, f"{name}: device status {h.status()}"
        ms = total / steps
        out.append({"workload": name if len(batches) == 1 else f"{name} (first {b} of 9 on one handle)",
                    "batch": b, "ms_per_step": ms, "tokens_per_s": b / (ms / 1e3),
                    "mbu": B / (ms / 1e3) / (NOMINAL_HBM_GBS * 1e9),
                    "frac_of_measured_copy": B / (ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                    "l2": ("L2 flushed between steps (2x L2 buffer written, untimed)" if flush is not None
                           else f"inputs larger than L2 ({B / 1e9:.2f} GB read per step)")})
    if len(out) == 2:
        out[1]["tokens_per_s_vs_batch_8"] = out[1]["tokens_per_s"] / out[0]["tokens_per_s"]
    h.close()
    del wts, kv, scrub
    torch.cuda.empty_cache()
    return out


def main():
    args = parse()
    world, rank, local = setup_dist(args) if args.impl == "mk" else (
        int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_mk(args, world, rank, local)
    finally:
        if world > 1 and args.impl == "mk":
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
