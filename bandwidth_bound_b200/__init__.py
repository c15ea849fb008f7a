"""Python binding of libmk.so, the B200 decode-step megakernel.

Argument marshalling only: every step of the decode path runs inside the CUDA
kernel behind the C ABI declared in include/mk.h.  torch is used for device
memory and streams.  There is no CPU fallback: if libmk.so is missing or cannot
be loaded, importing the binding's entry points raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmk.so")

MK_OK = 0
MK_ERR_INVALID_ARG = -1
MK_ERR_UNSUPPORTED_CFG = -2
MK_ERR_SCHEDULE_INVALID = -3
MK_ERR_CUDA = -4
MK_ERR_DEVICE_TIMEOUT = -5
MK_ERR_BOUNDS = -6
MK_ERR_NO_DEVICE = -7

MK_CREATE_SKIP_VALIDATE = 1

MK_FAULT_DROP_WAIT = 1
MK_FAULT_RAISE_TARGET = 2
MK_FAULT_REORDER = 3
MK_FAULT_DUP_UNIT = 4
MK_FAULT_OVERSIZE_STAGE = 5


class MkError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"mk error {code}: {msg}")
        self.code = code


class ModelCfg(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("hidden", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("ffn", ctypes.c_int32),
                ("vocab", ctypes.c_int32), ("tied", ctypes.c_int32), ("rope_theta", ctypes.c_float),
                ("rms_eps", ctypes.c_float), ("max_batch", ctypes.c_int32), ("max_ctx", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("rope_scale_factor", ctypes.c_float),
                ("rope_low_freq_factor", ctypes.c_float), ("rope_high_freq_factor", ctypes.c_float),
                ("rope_original_max_pos", ctypes.c_int32), ("qk_norm", ctypes.c_int32)]


_PP = ctypes.POINTER(ctypes.c_void_p)


class WeightPtrs(ctypes.Structure):
    _fields_ = [("embed", ctypes.c_void_p), ("final_norm", ctypes.c_void_p), ("lm_head", ctypes.c_void_p),
                ("attn_norm", _PP), ("wq", _PP), ("wk", _PP), ("wv", _PP), ("wo", _PP),
                ("mlp_norm", _PP), ("w_gate", _PP), ("w_up", _PP), ("w_down", _PP),
                ("q_norm", _PP), ("k_norm", _PP)]


class KvCache(ctypes.Structure):
    _fields_ = [("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p), ("page_table", ctypes.c_void_p),
                ("num_pages", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32)]


class PlanOpts(ctypes.Structure):
    _fields_ = [("num_sms", ctypes.c_int32), ("attn_slots_per_sm", ctypes.c_int32),
                ("max_blocks", ctypes.c_int32)]


class PlanInfo(ctypes.Structure):
    _fields_ = [("n_tasks", ctypes.c_int64), ("n_stages", ctypes.c_int64), ("max_tasks_per_sm", ctypes.c_int64),
                ("weight_bytes_min_sm", ctypes.c_int64), ("weight_bytes_max_sm", ctypes.c_int64),
                ("attn_slots", ctypes.c_int64), ("n_counters", ctypes.c_int64)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmk.so (built by bandwidth_bound_b200/build.py); raises if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python bandwidth_bound_b200/build.py`")
    lib = ctypes.CDLL(path)
    vp, i32, u64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint64
    sig = {
        "mk_create": (ctypes.c_int, [ctypes.POINTER(ModelCfg), ctypes.POINTER(WeightPtrs), ctypes.POINTER(vp)]),
        "mk_create_from_plan": (ctypes.c_int, [vp, ctypes.POINTER(WeightPtrs), i32, ctypes.POINTER(vp)]),
        "mk_decode_step": (ctypes.c_int, [vp, vp, vp, vp, i32, ctypes.POINTER(KvCache), vp, vp, vp]),
        "mk_decode_step_host": (ctypes.c_int, [vp, vp, vp, vp, i32, ctypes.POINTER(KvCache), vp, vp, vp]),
        "mk_verify_step": (ctypes.c_int, [vp, vp, vp, vp, vp, i32, ctypes.POINTER(KvCache), vp, vp, vp]),
        "mk_decode_steps": (ctypes.c_int, [vp, i32, vp, vp, i32, ctypes.POINTER(KvCache), ctypes.POINTER(Sampling),
                                           vp, vp, vp]),
        "mk_decode_step_static": (ctypes.c_int, [ctypes.POINTER(ModelCfg), ctypes.POINTER(WeightPtrs), vp, vp, vp,
                                                 i32, ctypes.POINTER(KvCache), vp, vp, vp]),
        "mk_route_pick": (ctypes.c_int, [ctypes.POINTER(i32), ctypes.POINTER(i32), i32, i32, i32]),
        "mk_router_create": (ctypes.c_int, [ctypes.POINTER(vp), i32, ctypes.POINTER(vp)]),
        "mk_router_step": (ctypes.c_int, [vp, vp, vp, vp, i32, i32, ctypes.POINTER(KvCache), vp, vp,
                                          ctypes.POINTER(i32), vp]),
        "mk_router_destroy": (ctypes.c_int, [vp]),
        "mk_kpo_create": (ctypes.c_int, [ctypes.POINTER(ModelCfg), ctypes.POINTER(WeightPtrs), ctypes.POINTER(vp)]),
        "mk_kpo_step": (ctypes.c_int, [vp, vp, vp, vp, i32, ctypes.POINTER(KvCache), vp, vp, i32,
                                       ctypes.POINTER(ctypes.c_float), vp]),
        "mk_kpo_launches_per_step": (ctypes.c_int, [vp]),
        "mk_kpo_destroy": (ctypes.c_int, [vp]),
        "mk_kpo_last_error": (ctypes.c_char_p, [vp]),
        "mk_get_status": (ctypes.c_int, [vp]),
        "mk_reset": (ctypes.c_int, [vp]),
        "mk_set_debug": (ctypes.c_int, [vp, vp]),
        "mk_set_timeout_ns": (ctypes.c_int, [vp, u64]),
        "mk_set_trace": (ctypes.c_int, [vp, vp, ctypes.c_int64]),
        "mk_num_tasks": (ctypes.c_int64, [vp]),
        "mk_launches_per_step": (ctypes.c_int, [vp]),
        "mk_destroy": (ctypes.c_int, [vp]),
        "mk_last_error": (ctypes.c_char_p, [vp]),
        "mk_plan_create": (ctypes.c_int, [ctypes.POINTER(ModelCfg), ctypes.POINTER(PlanOpts), ctypes.POINTER(vp)]),
        "mk_plan_validate": (ctypes.c_int, [vp, ctypes.c_char_p, ctypes.c_size_t]),
        "mk_plan_stats": (ctypes.c_int, [vp, ctypes.POINTER(PlanInfo)]),
        "mk_plan_inject_fault": (ctypes.c_int, [vp, i32, i32]),
        "mk_plan_destroy": (None, [vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def model_cfg(m, max_batch: int, max_ctx: int) -> ModelCfg:
    """ModelCfg from any object with the synth.ModelConfig fields (rope_scaling: None or
    (factor, low_freq_factor, high_freq_factor, original_max_pos); qk_norm: bool)."""
    sc = getattr(m, "rope_scaling", None) or (1.0, 0.0, 0.0, 0)
    return ModelCfg(m.n_layers, m.hidden, m.n_heads, m.n_kv_heads, m.head_dim, m.ffn, m.vocab, int(m.tied),
                    float(m.rope_theta), float(m.rms_eps), int(max_batch), int(max_ctx), int(m.page_size),
                    float(sc[0]), float(sc[1]), float(sc[2]), int(sc[3]), int(bool(getattr(m, "qk_norm", False))))


_PER_LAYER = ("attn_norm", "wq", "wk", "wv", "wo", "mlp_norm", "w_gate", "w_up", "w_down")


def weight_struct(m, weights: dict):
    """(WeightPtrs, the host pointer arrays it points into - keep them alive) for a weights
    dict as built by synth.make_weights."""
    L = m.n_layers
    names = _PER_LAYER + (("q_norm", "k_norm") if getattr(m, "qk_norm", False) else ())
    arr = {n: (ctypes.c_void_p * L)(*[_ptr(weights["layers"][i][n]) for i in range(L)]) for n in names}
    per = [ctypes.cast(arr[n], _PP) if n in arr else None for n in _PER_LAYER + ("q_norm", "k_norm")]
    return WeightPtrs(_ptr(weights["embed"]), _ptr(weights["final_norm"]), _ptr(weights["lm_head"]), *per), arr


def step_bytes(m, ctx_lens: Sequence[int]) -> int:
    """Bytes one decode step must read from HBM, the numerator of model bandwidth
    utilisation ("Inside the megakernel serving engine", the MBU definition): every
    layer's projection weights and its two norm gains, the final norm gain, the whole
    LM-head matrix (counted even when tied to the embedding), the gathered embedding
    row of each sequence and the prior K and V entries of every layer, all bf16.
    Writes and the new token's own K/V, produced on chip, are not counted."""
    d, L = m.hidden, m.n_layers
    q_out = m.n_heads * m.head_dim
    kv_out = m.n_kv_heads * m.head_dim
    per_layer = d * q_out + 2 * d * kv_out + q_out * d + 3 * d * m.ffn + 2 * d
    if getattr(m, "qk_norm", False):
        per_layer += 2 * m.head_dim  # the q_norm and k_norm gains
    elements = L * per_layer + d + m.vocab * d + len(ctx_lens) * d
    elements += 2 * L * kv_out * sum(int(s) for s in ctx_lens)
    return 2 * elements


def _check(rc: int, handle=None, what: str = ""):
    if rc != MK_OK:
        lib = load_library()
        msg = lib.mk_last_error(handle)
        raise MkError(rc, f"{what}: {msg.decode() if msg else ''}")


class Plan:
    """The per-SM task schedule (host only)."""

    def __init__(self, cfg: ModelCfg, num_sms: int = 0, attn_slots_per_sm: int = 0, max_blocks: int = 0):
        self.lib = load_library()
        self.ptr = ctypes.c_void_p()
        opts = PlanOpts(num_sms, attn_slots_per_sm, max_blocks)
        _check(self.lib.mk_plan_create(ctypes.byref(cfg), ctypes.byref(opts), ctypes.byref(self.ptr)),
               None, "mk_plan_create")

    def validate(self) -> tuple[int, str]:
        buf = ctypes.create_string_buffer(512)
        rc = self.lib.mk_plan_validate(self.ptr, buf, 512)
        return rc, buf.value.decode()

    def stats(self) -> dict:
        info = PlanInfo()
        _check(self.lib.mk_plan_stats(self.ptr, ctypes.byref(info)), None, "mk_plan_stats")
        return {k: getattr(info, k) for k, _ in PlanInfo._fields_}

    def inject_fault(self, kind: int, arg: int = 0) -> int:
        return self.lib.mk_plan_inject_fault(self.ptr, kind, arg)

    def close(self):
        if self.ptr:
            self.lib.mk_plan_destroy(self.ptr)
            self.ptr = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


class Sampling(ctypes.Structure):
    """mk_sampling: top-k sampling of the next token (top_k <= 1: greedy)."""
    _fields_ = [("top_k", ctypes.c_int32), ("temperature", ctypes.c_float), ("uniforms", ctypes.c_void_p)]


MAX_TOP_K = 256


class Megakernel:
    """A handle of the decode megakernel bound to one model's device weights.

    ``weights`` is a dict as built by ``synth.make_weights`` (bf16 CUDA tensors);
    the tensors must stay alive while the handle is used.
    """

    def __init__(self, m, weights: dict, max_batch: int, max_ctx: int, plan: Optional[Plan] = None,
                 skip_validate: bool = False):
        import torch  # plumbing only: device pointers and streams

        self.lib = load_library()
        self.m = m
        self.cfg = model_cfg(m, max_batch, max_ctx)
        self.weights = weights
        w, self._arrays = weight_struct(m, weights)
        self.handle = ctypes.c_void_p()
        if plan is None:
            rc = self.lib.mk_create(ctypes.byref(self.cfg), ctypes.byref(w), ctypes.byref(self.handle))
        else:
            rc = self.lib.mk_create_from_plan(plan.ptr, ctypes.byref(w),
                                              MK_CREATE_SKIP_VALIDATE if skip_validate else 0,
                                              ctypes.byref(self.handle))
        _check(rc, None, "mk_create")
        self._torch = torch

    @staticmethod
    def kv_struct(kv) -> KvCache:
        return KvCache(_ptr(kv.k_pool), _ptr(kv.v_pool), _ptr(kv.page_table), int(kv.num_pages),
                       int(kv.max_pages_per_seq))

    def step(self, token_ids, positions, seq_lens, kv, logits, argmax=None, stream=None, check: bool = True) -> int:
        """One decode step on device tensors (int32 token_ids/positions/seq_lens, fp32 logits)."""
        if stream is None:
            stream = self._torch.cuda.current_stream()
        kvs = self.kv_struct(kv)
        rc = self.lib.mk_decode_step(self.handle, _ptr(token_ids), _ptr(positions), _ptr(seq_lens),
                                     int(token_ids.numel()), ctypes.byref(kvs), _ptr(logits), _ptr(argmax),
                                     ctypes.c_void_p(stream.cuda_stream))
        if check:
            _check(rc, self.handle, "mk_decode_step")
        return rc

    def verify(self, token_ids, positions, seq_lens, group_first, kv, logits, argmax=None, stream=None,
               check: bool = True) -> int:
        """A multi-token step: rows of one sequence (group_first) at consecutive positions,
        attending causally to each other's new tokens."""
        if stream is None:
            stream = self._torch.cuda.current_stream()
        kvs = self.kv_struct(kv)
        rc = self.lib.mk_verify_step(self.handle, _ptr(token_ids), _ptr(positions), _ptr(seq_lens), _ptr(group_first),
                                     int(token_ids.numel()), ctypes.byref(kvs), _ptr(logits), _ptr(argmax),
                                     ctypes.c_void_p(stream.cuda_stream))
        if check:
            _check(rc, self.handle, "mk_verify_step")
        return rc

    def steps(self, n_steps: int, token_ids, positions, kv, tokens_out, logits=None, stream=None,
              check: bool = True, top_k: int = 1, temperature: float = 1.0, uniforms=None) -> int:
        """n_steps steps in one call: step k feeds the token step k-1 chose at positions + k.
        tokens_out: device int32 [n_steps][batch]; logits (optional): the last step's.
        top_k > 1 samples among the top_k logits at `temperature` with the device fp32
        uniforms [n_steps][batch]; otherwise the choice is greedy."""
        if stream is None:
            stream = self._torch.cuda.current_stream()
        kvs = self.kv_struct(kv)
        smp = Sampling(int(top_k), float(temperature), _ptr(uniforms))
        rc = self.lib.mk_decode_steps(self.handle, int(n_steps), _ptr(token_ids), _ptr(positions),
                                      int(token_ids.numel()), ctypes.byref(kvs), ctypes.byref(smp), _ptr(tokens_out),
                                      _ptr(logits), ctypes.c_void_p(stream.cuda_stream))
        if check:
            _check(rc, self.handle, "mk_decode_steps")
        return rc

    def step_host(self, token_ids, positions, seq_lens, kv, logits_host=None, argmax_host=None, stream=None,
                  check: bool = True) -> int:
        """One decode step from host (CPU, ideally pinned) tensors; synchronises the stream."""
        if stream is None:
            stream = self._torch.cuda.current_stream()
        kvs = self.kv_struct(kv)
        rc = self.lib.mk_decode_step_host(self.handle, _ptr(token_ids), _ptr(positions), _ptr(seq_lens),
                                          int(token_ids.numel()), ctypes.byref(kvs), _ptr(logits_host),
                                          _ptr(argmax_host), ctypes.c_void_p(stream.cuda_stream))
        if check:
            _check(rc, self.handle, "mk_decode_step_host")
        return rc

    def status(self) -> int:
        return self.lib.mk_get_status(self.handle)

    def reset(self):
        _check(self.lib.mk_reset(self.handle), self.handle, "mk_reset")

    def set_debug(self, layer_hidden):
        _check(self.lib.mk_set_debug(self.handle, _ptr(layer_hidden)), self.handle, "mk_set_debug")

    def num_tasks(self) -> int:
        return int(self.lib.mk_num_tasks(self.handle))

    def set_trace(self, records):
        """records: device uint64 tensor [>= num_tasks()][8], or None."""
        n = 0 if records is None else records.shape[0]
        _check(self.lib.mk_set_trace(self.handle, _ptr(records), n), self.handle, "mk_set_trace")

    def set_timeout_ns(self, ns: int):
        _check(self.lib.mk_set_timeout_ns(self.handle, int(ns)), self.handle, "mk_set_timeout_ns")

    def launches_per_step(self) -> int:
        return self.lib.mk_launches_per_step(self.handle)

    def last_error(self) -> str:
        msg = self.lib.mk_last_error(self.handle)
        return msg.decode() if msg else ""

    def close(self):
        if self.handle:
            self.lib.mk_destroy(self.handle)
            self.handle = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def route_pick(bounds, batch: int, max_position: int) -> int:
    """The router's rule on [(max_batch, max_ctx), ...]: index of the handle a step goes to,
    or a negative status when none covers it."""
    lib = load_library()
    n = len(bounds)
    mb = (ctypes.c_int32 * n)(*[int(b) for b, _ in bounds])
    mc = (ctypes.c_int32 * n)(*[int(c) for _, c in bounds])
    return lib.mk_route_pick(mb, mc, n, int(batch), int(max_position))


class Router:
    """Steps routed among handles of one model built for different bounds (mk_router_*)."""

    def __init__(self, handles):
        import torch

        self.lib = load_library()
        self._torch = torch
        self.handles = list(handles)
        arr = (ctypes.c_void_p * len(self.handles))(*[h.handle.value for h in self.handles])
        self.ptr = ctypes.c_void_p()
        _check(self.lib.mk_router_create(arr, len(self.handles), ctypes.byref(self.ptr)), None, "mk_router_create")

    def step(self, token_ids, positions, seq_lens, max_position: int, kv, logits, argmax=None, stream=None,
             check: bool = True):
        """One step on the picked handle; returns (status, picked index)."""
        if stream is None:
            stream = self._torch.cuda.current_stream()
        picked = ctypes.c_int32(-1)
        kvs = Megakernel.kv_struct(kv)
        rc = self.lib.mk_router_step(self.ptr, _ptr(token_ids), _ptr(positions), _ptr(seq_lens),
                                     int(token_ids.numel()), int(max_position), ctypes.byref(kvs), _ptr(logits),
                                     _ptr(argmax), ctypes.byref(picked), ctypes.c_void_p(stream.cuda_stream))
        if check:
            _check(rc, None, "mk_router_step")
        return rc, picked.value

    def close(self):
        if self.ptr:
            self.lib.mk_router_destroy(self.ptr)
            self.ptr = ctypes.c_void_p()


KPO_GRAPH, KPO_STREAM, KPO_TIMED, KPO_EMPTY = 0, 1, 2, 3


class KernelPerOp:
    """The same decode step as one kernel per operation (mk_kpo_*): a comparison for the
    single-launch step.  mode: KPO_GRAPH (CUDA graph replay), KPO_STREAM (launches on the
    stream), KPO_TIMED (no overlap; step() then returns the summed kernel time in ms),
    KPO_EMPTY (the same launches doing nothing: the cost of the launches alone)."""

    def __init__(self, m, weights: dict, max_batch: int, max_ctx: int):
        import torch

        self.lib = load_library()
        self._torch = torch
        self.cfg = model_cfg(m, max_batch, max_ctx)
        w, self._arrays = weight_struct(m, weights)
        self.weights = weights
        self.ptr = ctypes.c_void_p()
        rc = self.lib.mk_kpo_create(ctypes.byref(self.cfg), ctypes.byref(w), ctypes.byref(self.ptr))
        if rc != MK_OK:
            raise MkError(rc, "mk_kpo_create: " + (self.lib.mk_kpo_last_error(None) or b"").decode())

    def step(self, token_ids, positions, seq_lens, kv, logits, argmax=None, mode: int = KPO_GRAPH, stream=None):
        if stream is None:
            stream = self._torch.cuda.current_stream()
        busy = ctypes.c_float(0.0)
        kvs = Megakernel.kv_struct(kv)
        rc = self.lib.mk_kpo_step(self.ptr, _ptr(token_ids), _ptr(positions), _ptr(seq_lens), int(token_ids.numel()),
                                  ctypes.byref(kvs), _ptr(logits), _ptr(argmax), int(mode), ctypes.byref(busy),
                                  ctypes.c_void_p(stream.cuda_stream))
        if rc != MK_OK:
            raise MkError(rc, "mk_kpo_step: " + (self.lib.mk_kpo_last_error(self.ptr) or b"").decode())
        return busy.value

    def launches_per_step(self) -> int:
        return self.lib.mk_kpo_launches_per_step(self.ptr)

    def close(self):
        if self.ptr:
            self.lib.mk_kpo_destroy(self.ptr)
            self.ptr = ctypes.c_void_p()


def decode_step_static(m, weights: dict, max_batch: int, max_ctx: int, token_ids, positions, seq_lens, kv,
                       logits, argmax=None, stream=None, check: bool = True) -> int:
    """One decode step through mk_decode_step_static: no handle, no device allocation.

    The scratch is the library's fixed 16 MiB device array; the call returns after the
    step has finished with its device status.
    """
    import torch

    lib = load_library()
    if stream is None:
        stream = torch.cuda.current_stream()
    cfg = model_cfg(m, max_batch, max_ctx)
    w, arr = weight_struct(m, weights)  # noqa: F841 (arr keeps the pointer arrays alive)
    kvs = Megakernel.kv_struct(kv)
    rc = lib.mk_decode_step_static(ctypes.byref(cfg), ctypes.byref(w), _ptr(token_ids), _ptr(positions),
                                   _ptr(seq_lens), int(token_ids.numel()), ctypes.byref(kvs), _ptr(logits),
                                   _ptr(argmax), ctypes.c_void_p(stream.cuda_stream))
    if check:
        _check(rc, None, "mk_decode_step_static")
    return rc


def header_functions(header: Optional[str] = None) -> list[str]:
    """Names of the entry points include/mk.h declares (MK_API lines)."""
    import re

    header = header or os.path.join(os.path.dirname(HERE), "include", "mk.h")
    src = open(header).read()
    return re.findall(r"MK_API\s+[\w\s\*]*?\b(mk_\w+)\s*\(", src)
