"""Seeded synthetic inputs for the decode step: shapes, weights, KV cache, tokens.

This module is shared by the GPU path's tests/bench and by the float64 oracle.
It holds no arithmetic of the decode step itself: it only draws random numbers,
lays them out in the boundary's formats and builds page tables.

Recipe (all seeded):
  * weights: seed 0, one derived generator per tensor, N(0, std=0.02) drawn in
    fp32 and rounded to bf16 by torch; RMSNorm gains are 1 (or 1 + N(0, gain_std)
    when a test asks for non-trivial gains);
  * KV cache: seed 1, prior entries N(0, 1) rounded to bf16; every slot that is
    not a prior entry holds a canary NaN bit pattern;
  * token ids, context lengths and the page permutation: seed 2 (CPU generator,
    so they are identical on every device).

Layouts (the boundary's):
  * weights bf16 row-major [out, in] (Hugging Face ``nn.Linear`` layout);
  * K and V pools bf16 [n_layers][num_pages][n_kv_heads][page_size][head_dim];
  * page table int32 [batch][max_pages_per_seq], unused entries -1.
"""
from __future__ import annotations

import dataclasses
import hashlib
from dataclasses import dataclass
from typing import Optional

import torch

CANARY_BF16_BITS = 0x7FC1  # a quiet-NaN bf16 pattern that no arithmetic produces by chance


@dataclass(frozen=True)
class ModelConfig:
    name: str
    n_layers: int
    hidden: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    tied: bool
    rope_theta: float
    rms_eps: float = 1e-5
    page_size: int = 16
    # Llama-3.x RoPE frequency scaling: (factor, low_freq_factor, high_freq_factor,
    # original_max_position), or None
    rope_scaling: Optional[tuple] = None
    qk_norm: bool = False  # Qwen3-style RMSNorm of each query and key head before RoPE

    @property
    def group(self) -> int:
        return self.n_heads // self.n_kv_heads

    @property
    def q_dim(self) -> int:
        return self.n_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim


@dataclass(frozen=True)
class Workload:
    """A model plus a batch: ``ctx`` is ("fixed", S) or ("uniform", lo, hi).

    S_i is the number of prior cache entries of sequence i; its new token sits
    at position S_i and attends to S_i + 1 keys.
    """
    name: str
    model: ModelConfig
    batch: int
    ctx: tuple

    def context_lengths(self, seed: int = 2) -> list[int]:
        return context_lengths(self, seed)


# --- the five shapes named for this decode path -------------------------------------------

TINY = ModelConfig("tiny", 2, 256, 4, 2, 64, 688, 2048, False, 10000.0)
SMOLLM2_135M = ModelConfig("smollm2-135m", 30, 576, 9, 3, 64, 1536, 49152, True, 100000.0)
LLAMA32_1B = ModelConfig("llama3.2-1b", 16, 2048, 32, 8, 64, 8192, 128256, True, 500000.0,
                         rope_scaling=(32.0, 1.0, 4.0, 8192))
LLAMA3_8B = ModelConfig("llama3-8b", 32, 4096, 32, 8, 128, 14336, 128256, False, 500000.0)
LLAMA2_13B = ModelConfig("llama2-13b", 40, 5120, 40, 40, 128, 13824, 32000, False, 10000.0)

# the Qwen3 shapes the pages evaluate (QK-norm, head_dim 128 with q_dim != hidden at 0.6B)
QWEN3_0_6B = ModelConfig("qwen3-0.6b", 28, 1024, 16, 8, 128, 3072, 151936, True, 1000000.0, rms_eps=1e-6,
                         qk_norm=True)
QWEN3_8B = ModelConfig("qwen3-8b", 36, 4096, 32, 8, 128, 12288, 151936, False, 1000000.0, rms_eps=1e-6,
                       qk_norm=True)

MODELS = {m.name: m for m in (TINY, SMOLLM2_135M, LLAMA32_1B, LLAMA3_8B, LLAMA2_13B, QWEN3_0_6B, QWEN3_8B)}

WORKLOADS = {
    w.name: w
    for w in (
        Workload("tiny-b1", TINY, 1, ("fixed", 64)),
        Workload("smollm2-135m-b1", SMOLLM2_135M, 1, ("fixed", 1024)),
        Workload("llama3.2-1b-b9", LLAMA32_1B, 9, ("uniform", 128, 4096)),
        Workload("llama3-8b-b1", LLAMA3_8B, 1, ("fixed", 2048)),
        Workload("llama3-8b-b8", LLAMA3_8B, 8, ("fixed", 2048)),
        Workload("llama2-13b-b4", LLAMA2_13B, 4, ("uniform", 1024, 4096)),
        Workload("qwen3-0.6b-b1", QWEN3_0_6B, 1, ("fixed", 128)),
        Workload("qwen3-8b-b1", QWEN3_8B, 1, ("fixed", 2048)),
    )
}


def scaled_model(base: ModelConfig, **changes) -> ModelConfig:
    """A copy of ``base`` with some fields replaced (used for small test shapes)."""
    return dataclasses.replace(base, **changes)


# --- integer inputs (device independent) ----------------------------------------------------

def _cpu_gen(seed: int, tag: str) -> torch.Generator:
    h = hashlib.sha256(f"{seed}:{tag}".encode()).digest()
    g = torch.Generator(device="cpu")
    g.manual_seed(int.from_bytes(h[:8], "little") & ((1 << 63) - 1))
    return g


def context_lengths(w: Workload, seed: int = 2) -> list[int]:
    kind = w.ctx[0]
    if kind == "fixed":
        return [int(w.ctx[1])] * w.batch
    if kind == "uniform":
        lo, hi = int(w.ctx[1]), int(w.ctx[2])
        g = _cpu_gen(seed, f"{w.name}:ctx")
        return [int(v) for v in torch.randint(lo, hi + 1, (w.batch,), generator=g)]
    raise ValueError(f"unknown context spec {w.ctx}")


def token_ids(model: ModelConfig, batch: int, seed: int = 2, tag: str = "") -> list[int]:
    g = _cpu_gen(seed, f"{model.name}:tokens:{tag}")
    return [int(v) for v in torch.randint(0, model.vocab, (batch,), generator=g)]


# --- weights ---------------------------------------------------------------------------------

LAYER_TENSORS = ("attn_norm", "wq", "wk", "wv", "wo", "mlp_norm", "w_gate", "w_up", "w_down")


def layer_shapes(m: ModelConfig) -> dict[str, tuple]:
    d = m.hidden
    return {
        "attn_norm": (d,),
        "wq": (m.q_dim, d),
        "wk": (m.kv_dim, d),
        "wv": (m.kv_dim, d),
        "wo": (d, m.q_dim),
        "mlp_norm": (d,),
        "w_gate": (m.ffn, d),
        "w_up": (m.ffn, d),
        "w_down": (d, m.ffn),
    }


def _tensor_gen(seed: int, name: str, device) -> torch.Generator:
    h = hashlib.sha256(f"{seed}:{name}".encode()).digest()
    g = torch.Generator(device=device)
    g.manual_seed(int.from_bytes(h[:8], "little") & ((1 << 63) - 1))
    return g


def _normal_bf16(shape, std, mean, seed, name, device) -> torch.Tensor:
    g = _tensor_gen(seed, name, device)
    t = torch.empty(shape, dtype=torch.float32, device=device)
    t.normal_(mean=mean, std=std, generator=g)
    return t.to(torch.bfloat16)


def make_weights(m: ModelConfig, device="cpu", seed: int = 0, std: float = 0.02,
                 gain_std: float = 0.0, layers: Optional[list[int]] = None) -> dict:
    """All weights of ``m`` as bf16 tensors on ``device``.

    Returns {"embed", "final_norm", "lm_head", "layers": [dict per layer]}; when the
    model is tied, "lm_head" is the same tensor object as "embed". ``layers``
    restricts generation to some layer indices (others are None).
    """
    def gain(name, n=m.hidden):
        if gain_std == 0.0:
            return torch.ones((n,), dtype=torch.bfloat16, device=device)
        return _normal_bf16((n,), gain_std, 1.0, seed, name, device)

    out = {"embed": _normal_bf16((m.vocab, m.hidden), std, 0.0, seed, "embed", device),
           "final_norm": gain("final_norm")}
    out["lm_head"] = out["embed"] if m.tied else _normal_bf16((m.vocab, m.hidden), std, 0.0, seed,
                                                              "lm_head", device)
    shapes = layer_shapes(m)
    want = set(range(m.n_layers)) if layers is None else set(layers)
    out["layers"] = []
    for li in range(m.n_layers):
        if li not in want:
            out["layers"].append(None)
            continue
        lw = {}
        for name in LAYER_TENSORS:
            if name.endswith("norm"):
                lw[name] = gain(f"L{li}.{name}")
            else:
                lw[name] = _normal_bf16(shapes[name], std, 0.0, seed, f"L{li}.{name}", device)
        if m.qk_norm:
            for name in ("q_norm", "k_norm"):
                lw[name] = gain(f"L{li}.{name}", m.head_dim)
        out["layers"].append(lw)
    return out


# --- paged KV cache --------------------------------------------------------------------------

@dataclass
class KVCache:
    k_pool: torch.Tensor          # bf16 [L][P][nkv][page][hd]
    v_pool: torch.Tensor
    page_table: torch.Tensor      # int32 [batch_cap][max_pages_per_seq], -1 where unused
    num_pages: int
    max_pages_per_seq: int
    ctx_lens: list[int]           # prior entries S_i per sequence


def pages_needed(n_tokens: int, page: int) -> int:
    return (n_tokens + page - 1) // page


def make_kv_cache(m: ModelConfig, ctx_lens: list[int], device="cpu", seed: int = 1,
                  max_ctx: Optional[int] = None, spare_pages: int = 3, batch_cap: Optional[int] = None,
                  tag: str = "", room: int = 1) -> KVCache:
    """A paged cache holding ``ctx_lens[i]`` prior entries per sequence.

    Each sequence owns ceil((S_i + room) / page) pages (room for the new token, or for the
    ``room`` tokens of a multi-step run), the
    physical pages are a random permutation (so contiguity is never implied),
    ``spare_pages`` pages belong to nobody, and every slot that is not a prior
    entry holds the canary pattern.
    """
    P = m.page_size
    b = len(ctx_lens)
    batch_cap = b if batch_cap is None else batch_cap
    if max_ctx is None:
        max_ctx = max(ctx_lens) + 1
    mpps = pages_needed(max_ctx, P)
    need = [pages_needed(s + room, P) for s in ctx_lens]
    num_pages = sum(need) + spare_pages
    g = _cpu_gen(2, f"{m.name}:pages:{tag}:{num_pages}")
    perm = torch.randperm(num_pages, generator=g)
    table = torch.full((batch_cap, mpps), -1, dtype=torch.int32)
    prior = torch.zeros((num_pages, P), dtype=torch.bool)
    pos = 0
    for i, (s, n) in enumerate(zip(ctx_lens, need)):
        ids = perm[pos:pos + n]
        pos += n
        table[i, :n] = ids.to(torch.int32)
        for j in range(n):
            lo = j * P
            cnt = max(0, min(P, s - lo))
            prior[int(ids[j]), :cnt] = True
    shape = (m.n_layers, num_pages, m.n_kv_heads, P, m.head_dim)
    k = torch.empty(shape, dtype=torch.bfloat16, device=device)
    v = torch.empty(shape, dtype=torch.bfloat16, device=device)
    gk = _tensor_gen(seed, f"{m.name}:k:{tag}", device)
    gv = _tensor_gen(seed, f"{m.name}:v:{tag}", device)
    mask = prior.to(device).view(1, num_pages, 1, P, 1)
    canary = torch.tensor(CANARY_BF16_BITS, dtype=torch.int16).view(torch.bfloat16).to(device)
    for li in range(m.n_layers):
        for pool, gen in ((k, gk), (v, gv)):
            t = torch.empty(shape[1:], dtype=torch.float32, device=device)
            t.normal_(0.0, 1.0, generator=gen)
            tb = t.to(torch.bfloat16)
            pool[li] = torch.where(mask[0], tb, canary)
    return KVCache(k, v, table.to(device), num_pages, mpps, list(ctx_lens))


def workload_inputs(w: Workload, device="cpu", gain_std: float = 0.0, batch: Optional[int] = None):
    """(weights, kv cache, token ids, positions) for a workload.

    ``batch`` < w.batch takes the first sequences only (the cache still holds all
    of them, so a later call with the full batch finds the others in place).
    """
    m = w.model
    lens = context_lengths(w)
    wts = make_weights(m, device=device, gain_std=gain_std)
    kv = make_kv_cache(m, lens, device=device)
    toks = token_ids(m, w.batch, tag=w.name)
    b = w.batch if batch is None else batch
    return wts, kv, toks[:b], lens[:b]
