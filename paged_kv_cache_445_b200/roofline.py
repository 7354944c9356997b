"""Byte and FLOP counts of the paged-attention path, and roofline fractions.

``kv_cache_bytes`` is the KV-cache size formula of "Inference optimization"
(AI Engineering from Scratch, Phase 10 / 12, section "KV cache"):
2 (K and V) x layers x KV heads x head_dim x tokens x bytes per element.
The per-step counts below apply it to one layer and add the other tensors a
kernel must touch at least once (q, out, block-table entries, lengths).
"""
from __future__ import annotations

import numpy as np

BF16 = 2


def kv_cache_bytes(num_layers: int, num_kv_heads: int, head_dim: int, seq_len: int,
                   bytes_per_elem: int = BF16) -> int:
    return 2 * num_layers * num_kv_heads * head_dim * seq_len * bytes_per_elem


def decode_kv_bytes(context_lens, num_kv_heads: int, head_dim: int) -> int:
    """KV bytes one decode step must read: every cached token once, K and V."""
    return kv_cache_bytes(1, num_kv_heads, head_dim, int(np.sum(np.asarray(context_lens, dtype=np.int64))))


def unique_kv_bytes(block_tables, context_lens, block_size: int, num_kv_heads: int, head_dim: int) -> int:
    """KV bytes of the distinct physical token rows referenced by the batch
    (shared prefix blocks counted once)."""
    seen = {}
    bt = np.asarray(block_tables)
    for s, n in enumerate(np.asarray(context_lens)):
        for lb in range(-(-int(n) // block_size)):
            rows = min(block_size, int(n) - lb * block_size)
            b = int(bt[s, lb])
            seen[b] = max(seen.get(b, 0), rows)
    return kv_cache_bytes(1, num_kv_heads, head_dim, sum(seen.values()))


def attention_algorithmic_bytes(context_lens, query_start, num_q_heads: int, num_kv_heads: int,
                                head_dim: int, block_size: int) -> int:
    """Minimum HBM bytes of one attention launch: KV of every context once,
    q and out once (bf16), the block-table entries and the length arrays."""
    cl = np.asarray(context_lens, dtype=np.int64)
    tq = int(np.asarray(query_start)[-1])
    kv = decode_kv_bytes(cl, num_kv_heads, head_dim)
    qo = 2 * tq * num_q_heads * head_dim * BF16
    tables = 4 * int(np.sum(-(-cl // block_size)))
    meta = 4 * (len(cl) + len(np.asarray(query_start)))
    return kv + qo + tables + meta


def append_algorithmic_bytes(num_tokens: int, num_kv_heads: int, head_dim: int) -> int:
    """Cache append: read k_new, v_new, write the same bytes, read the slots."""
    return 2 * 2 * num_tokens * num_kv_heads * head_dim * BF16 + 4 * num_tokens


def prefill_flops(context_lens, query_start, num_q_heads: int, head_dim: int) -> int:
    """Useful FLOPs (QK^T and PV, 2 per multiply-add) of the causal rows:
    row i of a sequence with ctx tokens and qlen rows sees ctx - qlen + i + 1 keys."""
    total = 0
    qs = np.asarray(query_start)
    for s, n in enumerate(np.asarray(context_lens, dtype=np.int64)):
        qlen = int(qs[s + 1] - qs[s])
        keys = int(n) - qlen + 1 + np.arange(qlen, dtype=np.int64)
        total += int(keys.sum())
    return 4 * head_dim * num_q_heads * total


def ridge_point(peak_flops_per_s: float, peak_bytes_per_s: float) -> float:
    """FLOP per byte at which a kernel stops being bound by memory bandwidth
    and becomes bound by arithmetic: peak FLOP/s over peak bytes/s.  The
    section on the ops:byte framework of "Inference optimization" (AI
    Engineering from Scratch, Phase 10 / 12) puts A100's crossover near 156
    this way, and its table of scenarios reads the bound off that point."""
    return peak_flops_per_s / peak_bytes_per_s


def stream_time_s(nbytes: float, bytes_per_s: float) -> float:
    """Least time to read nbytes once at bytes_per_s: the floor that page's
    section "Prefill vs decode" gives one decode step, every weight streamed
    from HBM per token."""
    return nbytes / bytes_per_s


def bound(flops: float, nbytes: float, peak_flops_per_s: float, peak_bytes_per_s: float) -> str:
    """"hbm" below the ridge point, "tensor" at or above it."""
    return "hbm" if flops < ridge_point(peak_flops_per_s, peak_bytes_per_s) * nbytes else "tensor"
