"""Contiguous-cache attention in numpy, fp64 -- the brute-force cross-check.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

This restates, for contiguous per-sequence caches, what "Inference
optimization" (AI Engineering from Scratch, Phase 10 / 12) builds in
"Build it -- Step 1: a KV cache from scratch" and "Step 2: attention with the
KV cache": keys and values of one sequence are stored in one contiguous
[heads, seq, d] buffer, new rows are written at the current length, and
attention is softmax(q K^T / sqrt(d) + mask) V with the causal mask of a
query block that sits at the END of the keys (query row i sees keys
j <= i + Lk - Lq).  The mask is applied the way the page does it -- an additive
-1e9 on the strictly-upper part -- which in fp64 makes those weights exactly 0.
It never sees a block table; it exists to pin the paged oracle.
"""
from __future__ import annotations

import numpy as np


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 is the upper half of a binary32: widen exactly."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def sdpa_bottom_right(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """q [Lq, d], k/v [Lk, d] (fp64) -> [Lq, d]; mask aligned to the bottom right."""
    lq, lk = q.shape[0], k.shape[0]
    scores = (q @ k.T) * scale
    if lq > 1:
        upper = np.triu(np.ones((lq, lk)), k=lk - lq + 1)
        scores = scores + upper * (-1e9)
    scores = scores - scores.max(axis=-1, keepdims=True)
    w = np.exp(scores)
    w = w / w.sum(axis=-1, keepdims=True)
    return w @ v


def contiguous_attention(q_rows, k_seq, v_seq, num_q_heads, scale):
    """One sequence: q_rows [Lq, Hq, d] (fp64), k_seq/v_seq [Lk, Hkv, d] (fp64),
    the Lq query rows being the last Lq positions.  Query head h uses KV head
    h // (Hq // Hkv).  Returns [Lq, Hq, d]."""
    lq, hq, d = q_rows.shape
    lk, hkv, _ = k_seq.shape
    group = hq // hkv
    out = np.zeros((lq, hq, d))
    if lk == 0 or lq == 0:
        return out
    for h in range(hq):
        out[:, h, :] = sdpa_bottom_right(q_rows[:, h, :], k_seq[:, h // group, :], v_seq[:, h // group, :], scale)
    return out
