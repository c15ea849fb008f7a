"""The C ABI loads and exports what include/mk.h declares; the host schedule and
its static validator (CPU only, no GPU calls)."""
import ctypes
import subprocess

import pytest

import bandwidth_bound_b200 as mk
import synth
from bandwidth_bound_b200 import build


@pytest.fixture(scope="module")
def lib():
    build.build()
    return mk.load_library()


def test_library_exports_every_declared_entry_point(lib):
    declared = mk.header_functions()
    assert len(declared) >= 16
    out = subprocess.run(["nm", "-D", "--defined-only", mk.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [f for f in declared if f not in exported]
    assert not missing, f"declared in mk.h but not exported: {missing}"
    for f in declared:
        assert hasattr(lib, f)
    # nothing else leaks out of the library
    extra = [f for f in exported if f.startswith("mk_") and f not in declared]
    assert not extra, f"exported but not declared: {extra}"


def test_cfg_struct_sizes_match_header():
    assert ctypes.sizeof(mk.ModelCfg) == 18 * 4
    assert ctypes.sizeof(mk.KvCache) == 3 * 8 + 2 * 4
    assert ctypes.sizeof(mk.WeightPtrs) == 14 * 8
    assert ctypes.sizeof(mk.Sampling) == 2 * 4 + 8


ALL_MODELS = [synth.TINY, synth.SMOLLM2_135M, synth.LLAMA32_1B, synth.LLAMA3_8B, synth.LLAMA2_13B, synth.QWEN3_0_6B,
              synth.QWEN3_8B]


@pytest.mark.parametrize("m", ALL_MODELS, ids=lambda m: m.name)
@pytest.mark.parametrize("max_batch", [1, 9, 16])
def test_default_plans_validate(lib, m, max_batch):
    plan = mk.Plan(mk.model_cfg(m, max_batch, 4097))
    rc, msg = plan.validate()
    assert rc == mk.MK_OK, msg
    st = plan.stats()
    # one attention range per SM and layer: ranges split the concatenated KV token lines
    # of all (sequence, kv head) pairs evenly, whatever the batch
    assert st["attn_slots"] == 148
    assert st["n_counters"] == 2 + 5 * m.n_layers


@pytest.mark.parametrize("m", [synth.LLAMA3_8B, synth.LLAMA32_1B, synth.LLAMA2_13B], ids=lambda m: m.name)
def test_weight_bytes_balanced_across_sms(lib, m):
    st = mk.Plan(mk.model_cfg(m, 8, 4097)).stats()
    lo, hi = st["weight_bytes_min_sm"], st["weight_bytes_max_sm"]
    # each GEMV phase takes the cheaper of equal ranges of (task group, 64-column chunk) work
    # and one task per SM (row groups within one unit of each other, cut into equal K pieces);
    # either way the larger shares go to the SMs with the fewest bytes so far, so over the
    # step the SMs stay within one unit plus one chunk per phase
    chunk = 64 * 64 * 2
    unit = max(8 * m.ffn * 2, 16 * m.hidden * 2)
    assert hi - lo <= unit + chunk * (4 * m.n_layers + 1), (lo, hi)


def test_plan_for_other_sm_counts(lib):
    for nsm in (1, 7, 132, 148, 160):
        plan = mk.Plan(mk.model_cfg(synth.TINY, 4, 256), num_sms=nsm)
        assert plan.validate()[0] == mk.MK_OK


@pytest.mark.parametrize("kind,arg,needle", [
    (mk.MK_FAULT_DROP_WAIT, 1, "race"),
    (mk.MK_FAULT_RAISE_TARGET, 0, "waits for"),
    (mk.MK_FAULT_REORDER, 1, "deadlock"),
    (mk.MK_FAULT_DUP_UNIT, 0, "covered"),
    (mk.MK_FAULT_OVERSIZE_STAGE, 0, "slot"),
])
def test_validator_rejects_injected_faults(lib, kind, arg, needle):
    plan = mk.Plan(mk.model_cfg(synth.TINY, 4, 256))
    assert plan.validate()[0] == mk.MK_OK
    assert plan.inject_fault(kind, arg) == mk.MK_OK
    rc, msg = plan.validate()
    assert rc == mk.MK_ERR_SCHEDULE_INVALID
    assert needle in msg, msg


@pytest.mark.parametrize("field,value,code", [
    ("head_dim", 96, mk.MK_ERR_UNSUPPORTED_CFG),
    ("page_size", 32, mk.MK_ERR_UNSUPPORTED_CFG),
    ("max_batch", 17, mk.MK_ERR_UNSUPPORTED_CFG),
    ("n_kv_heads", 3, mk.MK_ERR_UNSUPPORTED_CFG),
    ("hidden", 0, mk.MK_ERR_INVALID_ARG),
    ("rms_eps", 0.0, mk.MK_ERR_INVALID_ARG),
])
def test_unsupported_configs_are_rejected(lib, field, value, code):
    cfg = mk.model_cfg(synth.TINY, 4, 256)
    setattr(cfg, field, value)
    with pytest.raises(mk.MkError) as ei:
        mk.Plan(cfg)
    assert ei.value.code == code


def test_create_without_gpu_fails_cleanly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    cfg = mk.model_cfg(synth.TINY, 1, 256)
    w = mk.WeightPtrs()
    h = ctypes.c_void_p()
    rc = lib.mk_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h))
    assert rc in (mk.MK_ERR_INVALID_ARG, mk.MK_ERR_NO_DEVICE)
    assert not h.value
    assert lib.mk_decode_step(None, None, None, None, 1, None, None, None, None) == mk.MK_ERR_INVALID_ARG


def test_operand_room_follows_the_handles_batch(lib):
    # A stage reserves operand room for the handle's largest batch: 4 bytes per fp32 row
    # for batches the FMA path takes (1 or 2 rows), else 32 bytes per 8-row bf16 tile of
    # activation parts.  Less room leaves more weight columns per 50 KB stage, so fewer stages.
    m = synth.LLAMA3_8B
    n = {mb: mk.Plan(mk.model_cfg(m, mb, 2050)).stats()["n_stages"] for mb in (1, 2, 4, 8)}
    assert n[1] < n[2] < n[4] == n[8]
    for mb in (1, 2, 4, 8):
        rc, msg = mk.Plan(mk.model_cfg(m, mb, 2050)).validate()
        assert rc == mk.MK_OK, msg
