"""Test-only helpers: scatter contiguous per-sequence K/V into a paged pool.

The scatter here is written independently of the oracle and of the product
(plain index arithmetic in a loop) so that "paged oracle == contiguous brute
force" pins the oracle's gather.
"""
from __future__ import annotations

import numpy as np

from paged_kv_cache_445_b200.workloads import BF16_NAN, f32_to_bf16_bits


def rand_bf16(rng, shape, std=1.0):
    return f32_to_bf16_bits((rng.standard_normal(size=shape) * std).astype(np.float32))


def to_bf16(x):
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def scatter_to_pool(k_seqs, v_seqs, block_size, num_blocks, perm, fill=BF16_NAN):
    """k_seqs[s]: uint16 [L_s, Hkv, d].  Sequence s takes the next
    ceil(L_s / bs) IDs of ``perm``.  Returns k_cache, v_cache, block_tables."""
    hkv, d = k_seqs[0].shape[1], k_seqs[0].shape[2]
    k_cache = np.full((num_blocks, hkv, block_size, d), fill, dtype=np.uint16)
    v_cache = np.full((num_blocks, hkv, block_size, d), fill, dtype=np.uint16)
    nblk = [-(-len(k) // block_size) for k in k_seqs]
    tables = np.full((len(k_seqs), max(nblk + [1])), -1, dtype=np.int32)
    it = iter(int(p) for p in perm)
    for s, (ks, vs) in enumerate(zip(k_seqs, v_seqs)):
        for lb in range(nblk[s]):
            tables[s, lb] = next(it)
        for pos in range(len(ks)):
            b = tables[s, pos // block_size]
            for h in range(hkv):
                k_cache[b, h, pos % block_size, :] = ks[pos, h]
                v_cache[b, h, pos % block_size, :] = vs[pos, h]
    return k_cache, v_cache, tables
