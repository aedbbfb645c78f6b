"""Dense float64 attention over the visible tokens.

Test infrastructure only (see the package docstring).

What is computed ([P1] "FlashInfer Kernel Execution": the kernel attends only
to the listed pages; [P1] "Memory Efficiency Analysis": the validation path
gathers the paged K/V into dense tensors and runs scaled dot-product
attention): for each head h and query row i of the new frame,

    O[i, h] = sum_j softmax_j( q[i, h] . k[j, h] / sqrt(D) ) v[j, h]

over every visible token j, with no mask: all cached tokens precede the frame
and the frame's own tokens attend to each other in both directions. The pages
state no soft-cap, bias or other scale, so none is applied; Q and K arrive
after any rotary embedding.

Inputs are the 16-bit values the GPU reads (bf16 or fp16), converted exactly
to float64; everything after that is float64.
"""
from __future__ import annotations

import math

import numpy as np


def decode(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 value of 16-bit floating-point bit patterns."""
    bits = np.asarray(bits, dtype=np.uint16)
    if dtype == "bf16":
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if dtype == "fp16":
        return bits.view(np.float16).astype(np.float64)
    raise ValueError(dtype)


def scores(q: np.ndarray, k: np.ndarray) -> np.ndarray:
    """[H, T, L] scaled dot products q.k / sqrt(D)."""
    D = q.shape[-1]
    return np.einsum("thd,lhd->htl", q, k) / math.sqrt(D)


def probs(q: np.ndarray, k: np.ndarray) -> np.ndarray:
    """[H, T, L] softmax over the visible tokens (max-subtracted exponent)."""
    s = scores(q, k)
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    return p / p.sum(axis=-1, keepdims=True)


def dense(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """O [T, H, D] for q [T, H, D] over k, v [L, H, D]."""
    return np.einsum("htl,lhd->thd", probs(q, k), v)


def brute(q, k, v) -> np.ndarray:
    """The same result by explicit loops, for tiny inputs only."""
    T, H, D = q.shape
    L = k.shape[0]
    out = np.zeros((T, H, D))
    for h in range(H):
        for i in range(T):
            s = []
            for j in range(L):
                acc = 0.0
                for d in range(D):
                    acc += q[i, h, d] * k[j, h, d]
                s.append(acc / math.sqrt(D))
            m = max(s)
            e = [math.exp(x - m) for x in s]
            z = sum(e)
            for d in range(D):
                out[i, h, d] = sum(e[j] * v[j, h, d] for j in range(L)) / z
    return out


def partial(q, k, v):
    """Attention over one chunk of the visible tokens: the chunk-normalised
    output [T, H, D] and its natural-log sum-exp [T, H]."""
    s = scores(q, k)
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=-1, keepdims=True)
    o = np.einsum("htl,lhd->thd", e / z, v)
    lse = (m + np.log(z))[..., 0].transpose(1, 0)
    return o, lse


def merge(parts) -> np.ndarray:
    """Combine chunk partials [(o_c, lse_c)] into the full-softmax output:
    O = sum_c exp(lse_c - lse*) o_c / sum_c exp(lse_c - lse*)."""
    lse = np.stack([p[1] for p in parts])          # [C, T, H]
    top = lse.max(axis=0, keepdims=True)
    w = np.exp(lse - top)                           # [C, T, H]
    o = sum(w[c][..., None] * parts[c][0] for c in range(len(parts)))
    return o / w.sum(axis=0)[..., None]
