"""Top-k sampling of the next token, written out plainly on the CPU.

TEST INFRASTRUCTURE ONLY (see the package docstring).

What is computed: the engine's sampler that sits behind the decode launch
("ForgeMegakernel: A General Framework for Efficient Auto-Regressive Model Decode
Megakernels", paperlayer.ai digest of arXiv 2609.12379v1, §4.3 "generation framework
/ serving integration").  The pages name the sampler but do not define it; the
reading taken is the usual top-k sampling of a language model:
  * keep the k largest logits (equal logits: the lower vocabulary index first);
  * weight each by exp((logit - largest) / temperature), the softmax over the kept
    logits up to its normalisation;
  * draw by inverting the cumulative weight in rank order with a uniform u in [0, 1)
    that the caller supplies: the first rank whose running sum exceeds u times the total.

The draw turns floating point into an integer, so it is taken in the precision the
device takes it in: float32 throughout (the subtraction, the division by the
temperature, exp, the running sum in rank order and the product u * total).
"""
from __future__ import annotations

import numpy as np


def top_k_ranked(logits: np.ndarray, k: int) -> list[int]:
    """Vocabulary indices of the k largest logits, largest first, ties by lower index."""
    order = sorted(range(len(logits)), key=lambda i: (-float(logits[i]), i))
    return order[:k]


def sample_top_k(logits: np.ndarray, k: int, temperature: float, u: float) -> int:
    """The token drawn from a float32 logit row (the reading in the module docstring)."""
    if k <= 1:
        return top_k_ranked(logits, 1)[0]
    row = np.asarray(logits, dtype=np.float32)
    ranked = top_k_ranked(row, min(k, len(row)))
    t = np.float32(temperature)
    v0 = row[ranked[0]]
    w = [np.float32(np.exp(np.float32(np.float32(row[i] - v0) / t))) for i in ranked]
    total = np.float32(0.0)
    for x in w:
        total = np.float32(total + x)
    thr = np.float32(np.float32(u) * total)
    cum = np.float32(0.0)
    for r, x in enumerate(w):
        cum = np.float32(cum + x)
        if cum > thr:
            return ranked[r]
    return ranked[-1]


def boundary_margin(logits: np.ndarray, k: int, temperature: float, u: float) -> float:
    """How far u * total lies from the nearest running-sum boundary, relative to the total:
    a draw this close to a boundary may go either way under one-ulp differences in exp."""
    row = np.asarray(logits, dtype=np.float32)
    ranked = top_k_ranked(row, min(k, len(row)))
    v0 = float(row[ranked[0]])
    w = np.array([np.exp((float(row[i]) - v0) / temperature) for i in ranked])
    c = np.cumsum(w)
    return float(np.min(np.abs(c - u * c[-1])) / c[-1])
