"""The decode step written out plainly, in float64, on the CPU.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Nothing here is tuned:
every step is the definition, applied per sequence, with library primitives
(matmul, exp, sqrt, cos/sin) as its only building blocks.

What is computed follows "ForgeMegakernel: A General Framework for Efficient
Auto-Regressive Model Decode Megakernels" (paperlayer.ai digest of arXiv
2609.12379v1):
  * §2.1 "The decode step": per layer RMSNorm, projections, RoPE, attention over
    the cached prior positions, an MLP; then a final RMSNorm and the LM head;
  * §2.2 "Model bandwidth utilization": the byte count B(b, S) (reads only,
    gathered embedding rows instead of the whole table);
  * §4.2 "The mid-state test oracle": intermediate KV-cache states and logits
    are checked against float64 references;
  * §3.2 "Unverifiable correctness of kernel fusing": each sequence of a ragged
    batch decodes at its own position.

Readings where the pages are silent:
  * Llama conventions: RMSNorm with eps inside the square root and the gain
    applied afterwards; RoPE in the Hugging Face rotate-half pairing (j, j+hd/2)
    with inv_freq_j = theta^(-2j/hd), slowed by the Llama-3.x frequency scaling where
    the model has one (rope_inv_freq); keys are cached after RoPE; query head h reads
    KV head h // (n_heads / n_kv_heads); SiLU-gated MLP; scores scaled by
    1/sqrt(head_dim).
  * Qwen3 models (QK-norm): each query and key head is RMS-normalised over head_dim
    with the layer's q_norm / k_norm gain (same epsilon) between the projection and
    RoPE; the cached key is the normalised, rotated one.
  * The new token sits at position p_i = number of prior entries and attends to
    p_i + 1 keys; its own key and value enter attention as the bf16 values that
    are stored into the cache (round-to-nearest-even of the float64 result).
  * Argmax takes the lowest index among equal maxima.
"""
from __future__ import annotations

import math
from typing import Optional

import torch

F64 = torch.float64


def to_f64(t: torch.Tensor) -> torch.Tensor:
    """bf16 (or any) tensor -> float64 on the CPU; exact for bf16 inputs."""
    return t.detach().to("cpu").to(F64)


def bf16_rne(x: torch.Tensor) -> torch.Tensor:
    """Round float64 values to the nearest bf16 value, ties to even (8 significant bits).

    Written from the definition: x = m * 2^e with 0.5 <= |m| < 1, keep 8 bits of m
    with round-half-to-even.  Values below the bf16 normal range are not handled.
    """
    m, e = torch.frexp(x)
    r = torch.round(m * 256.0)  # torch.round rounds halves to even
    return torch.ldexp(r, (e - 8).to(F64))


def rmsnorm(x: torch.Tensor, gain: torch.Tensor, eps: float) -> torch.Tensor:
    """y = x / sqrt(mean(x^2) + eps) * gain over the last axis (§2.1, Llama RMSNorm)."""
    ms = (x * x).mean(dim=-1, keepdim=True)
    return x / torch.sqrt(ms + eps) * gain


def rope_inv_freq(head_dim: int, theta: float, scaling=None) -> torch.Tensor:
    """inv_freq_j = theta^(-2j/head_dim), j < head_dim/2 (§2.1 RoPE; HF convention).

    scaling = (factor, low_freq_factor, high_freq_factor, original_max_position), the
    Llama-3.x frequency scaling (the Llama 3 models the pages evaluate; the pages do not
    spell it out, so this follows the published model configuration): with wavelength
    w_j = 2 pi / inv_freq_j and N the original context, components with w_j < N / high
    keep their frequency, those with w_j > N / low are slowed by the factor, and those in
    between blend the two linearly in s = (N / w_j - low) / (high - low).
    """
    j = torch.arange(head_dim // 2, dtype=F64)
    inv = torch.pow(torch.tensor(theta, dtype=F64), -2.0 * j / head_dim)
    if scaling is None or scaling[0] <= 1.0:
        return inv
    factor, low, high, n_orig = (float(s) for s in scaling)
    out = inv.clone()
    for i in range(len(inv)):
        wavelen = 2.0 * math.pi / float(inv[i])
        if wavelen > n_orig / low:
            out[i] = inv[i] / factor
        elif wavelen >= n_orig / high:
            s = (n_orig / wavelen - low) / (high - low)
            out[i] = (1.0 - s) * inv[i] / factor + s * inv[i]
    return out


def rope(v: torch.Tensor, pos: int, theta: float, scaling=None) -> torch.Tensor:
    """Rotate pairs (j, j + hd/2) of ``v[..., hd]`` by angle pos * inv_freq_j."""
    hd = v.shape[-1]
    half = hd // 2
    ang = float(pos) * rope_inv_freq(hd, theta, scaling)
    c, s = torch.cos(ang), torch.sin(ang)
    x1, x2 = v[..., :half], v[..., half:]
    return torch.cat([x1 * c - x2 * s, x2 * c + x1 * s], dim=-1)


def kv_head_of(q_head: int, n_heads: int, n_kv_heads: int) -> int:
    """Grouped-query mapping: query head h reads KV head h // (n_heads / n_kv_heads)."""
    return q_head // (n_heads // n_kv_heads)


def attention(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor) -> torch.Tensor:
    """softmax(q K^T / sqrt(hd)) V for q [g, hd], K, V [n, hd] -> [g, hd] (§2.1)."""
    hd = q.shape[-1]
    s = (q @ K.T) / math.sqrt(hd)
    s = s - s.max(dim=-1, keepdim=True).values
    p = torch.exp(s)
    p = p / p.sum(dim=-1, keepdim=True)
    return p @ V


def attention_partial(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor):
    """Unnormalised softmax state over one span of keys: (m, l, acc).

    m = max score, l = sum exp(s - m), acc = sum exp(s - m) v.  Used to state the
    split-K (flash-decode) reading; the decode step itself uses ``attention``.
    """
    hd = q.shape[-1]
    s = (q @ K.T) / math.sqrt(hd)
    m = s.max(dim=-1).values
    p = torch.exp(s - m[:, None])
    return m, p.sum(dim=-1), p @ V


def combine_partials(parts) -> torch.Tensor:
    """Merge (m, l, acc) states of disjoint key spans: sum_c e^{m_c-M} acc_c / sum_c e^{m_c-M} l_c."""
    M = torch.stack([p[0] for p in parts]).max(dim=0).values
    num = sum(torch.exp(p[0] - M)[:, None] * p[2] for p in parts)
    den = sum(torch.exp(p[0] - M) * p[1] for p in parts)
    return num / den[:, None]


def silu(z: torch.Tensor) -> torch.Tensor:
    """z * sigmoid(z) = z / (1 + e^{-z})."""
    return z / (1.0 + torch.exp(-z))


def argmax_lowest(v: torch.Tensor) -> int:
    """Index of the maximum, lowest index among ties."""
    mx = v.max()
    return int(torch.nonzero(v == mx)[0, 0])


def _gather_prior(pool_l: torch.Tensor, table_row, n_prior: int, page: int) -> torch.Tensor:
    """Prior entries 0..n_prior-1 of one sequence from a paged pool layer.

    pool_l: [num_pages][n_kv][page][hd] (any dtype) -> float64 [n_kv][n_prior][hd].
    Entry t lives in physical page table_row[t // page], slot t % page.
    """
    n_kv, hd = pool_l.shape[1], pool_l.shape[3]
    if n_prior == 0:
        return torch.zeros((n_kv, 0, hd), dtype=F64)
    npg = (n_prior + page - 1) // page
    ids = torch.as_tensor([int(table_row[j]) for j in range(npg)], dtype=torch.long)
    blk = pool_l.index_select(0, ids)                  # [npg][n_kv][page][hd]
    blk = blk.permute(1, 0, 2, 3).reshape(n_kv, npg * page, hd)
    return to_f64(blk[:, :n_prior, :])


def layer_weights_f64(weights: dict, layer: int) -> dict:
    """The bf16 weights of one layer as float64 CPU tensors (exact)."""
    return {k: to_f64(t) for k, t in weights["layers"][layer].items()}


def decode_layer(cfg, lw: dict, x: torch.Tensor, k_pool_l: torch.Tensor, v_pool_l: torch.Tensor,
                 page_table, positions, *, round_new_kv: bool = True) -> dict:
    """One transformer layer of the decode step (§2.1) for a ragged batch.

    lw: float64 weights of the layer (``layer_weights_f64``); x: float64 [b][d] residual
    stream entering the layer; k_pool_l/v_pool_l: that layer's pools [P][n_kv][page][hd]
    holding the prior entries; positions[i] = prior entries of sequence i = its new
    token's position.  Per sequence: RMSNorm, the three projections, RoPE at the
    sequence's position, the new K/V rounded to bf16 as stored, attention of every
    query head over the prior keys plus the new one, the O projection and residual,
    RMSNorm, the SwiGLU MLP and residual.

    Returns {"x": [b][d] after the layer, "k_new"/"v_new" [b][n_kv][hd] (bf16-rounded),
    "k_new_exact"/"v_new_exact" (before rounding)}.
    """
    b = x.shape[0]
    nq, nkv, hd = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    P = cfg.page_size
    xn = rmsnorm(x, lw["attn_norm"], cfg.rms_eps)
    q = (xn @ lw["wq"].T).view(b, nq, hd)
    k = (xn @ lw["wk"].T).view(b, nkv, hd)
    v = (xn @ lw["wv"].T).view(b, nkv, hd)
    if getattr(cfg, "qk_norm", False):
        # Qwen3 QK-norm: each query and key head vector RMS-normalised over head_dim with
        # its own gain, before RoPE (the Qwen3 models of §5.3 and Appendix A)
        q = rmsnorm(q, lw["q_norm"], cfg.rms_eps)
        k = rmsnorm(k, lw["k_norm"], cfg.rms_eps)
    scaling = getattr(cfg, "rope_scaling", None)
    attn = torch.zeros((b, nq, hd), dtype=F64)
    k_new = torch.zeros((b, nkv, hd), dtype=F64)
    v_new = torch.zeros_like(k_new)
    k_exact = torch.zeros_like(k_new)
    v_exact = torch.zeros_like(k_new)
    for i in range(b):
        p = int(positions[i])
        qi = rope(q[i], p, cfg.rope_theta, scaling)
        ki = rope(k[i], p, cfg.rope_theta, scaling)
        vi = v[i]
        k_exact[i], v_exact[i] = ki, vi
        kr, vr = bf16_rne(ki), bf16_rne(vi)
        k_new[i], v_new[i] = kr, vr
        kin, vin = (kr, vr) if round_new_kv else (ki, vi)
        Kp = _gather_prior(k_pool_l, page_table[i], p, P)        # [nkv][p][hd]
        Vp = _gather_prior(v_pool_l, page_table[i], p, P)
        for h in range(nq):
            kvh = kv_head_of(h, nq, nkv)
            Kh = torch.cat([Kp[kvh], kin[kvh][None, :]], dim=0)
            Vh = torch.cat([Vp[kvh], vin[kvh][None, :]], dim=0)
            attn[i, h] = attention(qi[h][None, :], Kh, Vh)[0]
    x = x + attn.reshape(b, nq * hd) @ lw["wo"].T
    xn = rmsnorm(x, lw["mlp_norm"], cfg.rms_eps)
    hmid = silu(xn @ lw["w_gate"].T) * (xn @ lw["w_up"].T)
    x = x + hmid @ lw["w_down"].T
    return {"x": x, "k_new": k_new, "v_new": v_new, "k_new_exact": k_exact, "v_new_exact": v_exact}


def lm_head(cfg, weights: dict, x: torch.Tensor) -> torch.Tensor:
    """logits = W_lm (rmsnorm(x) * g_final) for x float64 [b][d] -> float64 [b][V]."""
    xf = rmsnorm(x, to_f64(weights["final_norm"]), cfg.rms_eps)
    head = weights["lm_head"]
    V = head.shape[0]
    logits = torch.empty((x.shape[0], V), dtype=F64)
    step = 16384
    for r0 in range(0, V, step):
        logits[:, r0:r0 + step] = xf @ to_f64(head[r0:r0 + step]).T
    return logits


def decode_step(cfg, weights: dict, k_pool: torch.Tensor, v_pool: torch.Tensor,
                page_table, token_ids, positions, *, round_new_kv: bool = True,
                layers: Optional[int] = None, want_logits: bool = True) -> dict:
    """One decode step for a ragged batch (§2.1), every sequence on its own.

    cfg: object with n_layers, hidden, n_heads, n_kv_heads, head_dim, ffn, vocab,
    rope_theta, rms_eps, page_size.  weights: bf16 tensors as built by
    ``synth.make_weights`` (any device; copied to float64 on the CPU one layer at
    a time).  k_pool/v_pool: [L][P][n_kv][page][hd]; page_table[i][j]: physical
    page of sequence i's entries j*page .. j*page+page-1; positions[i]: number of
    prior entries of sequence i, which is also its new token's position.

    Returns float64 mid-states: "hidden" [L+1][b][d] (after the embedding gather
    and after each layer), "k_new"/"v_new" [L][b][n_kv][hd] (bf16-rounded values
    the step stores), "k_new_exact"/"v_new_exact" (before rounding), "slots"
    [b] = (physical page, slot) of the new entry, "logits" [b][V] and "argmax".
    ``round_new_kv=False`` lets the new token attend to its unrounded k, v.
    ``layers`` stops after that many layers (no logits then).
    """
    L = cfg.n_layers if layers is None else layers
    b = len(token_ids)
    d, nkv, hd = cfg.hidden, cfg.n_kv_heads, cfg.head_dim
    P = cfg.page_size
    kp = k_pool.detach().to("cpu")
    vp = v_pool.detach().to("cpu")
    table = page_table.detach().to("cpu") if torch.is_tensor(page_table) else page_table

    emb = weights["embed"]
    x = torch.stack([to_f64(emb[int(t)]) for t in token_ids])        # [b][d]
    hidden = [x.clone()]
    k_new = torch.zeros((L, b, nkv, hd), dtype=F64)
    v_new = torch.zeros_like(k_new)
    k_exact = torch.zeros_like(k_new)
    v_exact = torch.zeros_like(k_new)
    slots = []
    for i in range(b):
        p = int(positions[i])
        slots.append((int(table[i][p // P]), p % P))

    for li in range(L):
        lw = layer_weights_f64(weights, li)
        r = decode_layer(cfg, lw, x, kp[li], vp[li], table, positions, round_new_kv=round_new_kv)
        x = r["x"]
        k_new[li], v_new[li] = r["k_new"], r["v_new"]
        k_exact[li], v_exact[li] = r["k_new_exact"], r["v_new_exact"]
        hidden.append(x.clone())
        del lw

    out = {"hidden": torch.stack(hidden), "k_new": k_new, "v_new": v_new,
           "k_new_exact": k_exact, "v_new_exact": v_exact, "slots": slots}
    if L == cfg.n_layers and want_logits:
        logits = lm_head(cfg, weights, x)
        out["logits"] = logits
        out["argmax"] = [argmax_lowest(logits[i]) for i in range(b)]
    return out


def model_bytes(cfg, ctx_lens) -> int:
    """B(b, S) of §2.2: bytes the step must read from HBM, reads only.

    All layer weights (norm gains included), the final norm, the full LM-head
    matrix, the b gathered embedding rows (counted even when the head is tied to
    the embedding) and the prior KV entries sum_i S_i * L * 2 * n_kv * hd, all bf16.
    The new token's K/V (produced on chip), KV writes, logits, page table and
    scratch are not counted.
    """
    d, hd, L = cfg.hidden, cfg.head_dim, cfg.n_layers
    qd, kvd, F, V = cfg.n_heads * hd, cfg.n_kv_heads * hd, cfg.ffn, cfg.vocab
    per_layer = 2 * d + qd * d + 2 * kvd * d + d * qd + 3 * F * d
    if getattr(cfg, "qk_norm", False):
        per_layer += 2 * hd  # the q_norm and k_norm gains
    elems = L * per_layer + d + V * d + len(ctx_lens) * d
    elems += sum(int(s) for s in ctx_lens) * L * 2 * kvd
    return 2 * elems
