"""Seeded synthetic inputs for the paged-attention path.

This module is the one source of inputs for both the CUDA path and the fp64
oracle.  It holds no attention arithmetic: it draws lengths and bf16 values
from a seeded numpy PCG64 stream and asks the host block allocator for block
tables and slots.  No public dataset is involved; the shapes follow the
workloads the pages discuss (Llama-3-8B / Llama-3.3-70B attention layers with
GQA, GRPO rollouts sharing a prompt, a 512-token prefill chunk of a 32k prompt
mixed with decodes -- "vLLM serving internals" and "Inference optimization",
AI Engineering from Scratch; "How vLLM gets real throughput on H100s").

A workload is the state of ONE attention layer at one engine step:

* ``k_cache`` / ``v_cache`` hold the pool BEFORE this step's append
  (bf16 bits, uint16, [num_blocks, Hkv, block_size, d]).  Every slot holds a
  draw; with ``poison=True`` every slot that is not a valid earlier token holds
  a NaN pattern instead, so a kernel that reads past a context shows it.
* ``k_new`` / ``v_new`` are this step's rows, ``slot_mapping`` their slots.
* ``q`` has one row per query token; ``query_start`` delimits sequences.
* ``context_lens`` count tokens INCLUDING this step's new ones.
"""
from __future__ import annotations

import dataclasses
import math
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from .allocator import BlockAllocator

BF16_NAN = np.uint16(0x7FC0)
_CHUNK = 1 << 24


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round binary32 to bf16 (nearest, ties to even) and return the bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).copy()
    lsb = (u >> 16) & 1
    u += lsb + 0x7FFF
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(seed: int, stream: int, shape, std: float = 1.0) -> np.ndarray:
    """bf16 bits of N(0, std^2) draws; chunk i of the output comes from
    PCG64(seed) jumped (stream * 4096 + i) times, so the result does not depend
    on how many threads fill it."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    nchunks = max(1, -(-n // _CHUNK))

    def fill(i):
        lo, hi = i * _CHUNK, min(n, (i + 1) * _CHUNK)
        g = np.random.Generator(np.random.PCG64(seed).jumped(stream * 4096 + i))
        x = g.standard_normal(hi - lo, dtype=np.float32)
        if std != 1.0:
            x *= np.float32(std)
        out[lo:hi] = f32_to_bf16_bits(x)

    if nchunks == 1:
        fill(0)
    else:
        with ThreadPoolExecutor(max_workers=min(16, nchunks)) as ex:
            list(ex.map(fill, range(nchunks)))
    return out.reshape(shape)


@dataclasses.dataclass
class Workload:
    name: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    scale: float
    q: np.ndarray
    k_new: np.ndarray
    v_new: np.ndarray
    k_cache: np.ndarray
    v_cache: np.ndarray
    block_tables: np.ndarray
    context_lens: np.ndarray
    query_start: np.ndarray
    slot_mapping: np.ndarray
    shared_prefix_tokens: int = 0
    shared_groups: tuple = ()  # (first sequence, end sequence) of each copy-on-write group

    @property
    def num_seqs(self) -> int:
        return len(self.context_lens)

    @property
    def num_query_tokens(self) -> int:
        return int(self.query_start[-1])

    @property
    def query_lens(self) -> np.ndarray:
        return np.diff(self.query_start).astype(np.int32)

    @property
    def is_decode(self) -> bool:
        return bool(np.all(self.query_lens == 1))

    def prefix_groups(self):
        """(group_start int32 [G + 1], group_prefix int32 [G]) describing the
        shared-prefix groups as consecutive sequence ranges (gaps between
        groups become groups with prefix 0), or None when nothing is shared."""
        if not self.shared_groups or self.shared_prefix_tokens <= 0:
            return None
        start, prefix, pos = [], [], None
        for lo, hi in sorted(self.shared_groups):
            if pos is not None and lo > pos:  # sequences between two groups share nothing
                start.append(pos)
                prefix.append(0)
            start.append(lo)
            prefix.append(self.shared_prefix_tokens)
            pos = hi
        start.append(pos)
        return np.asarray(start, dtype=np.int32), np.asarray(prefix, dtype=np.int32)


@dataclasses.dataclass(frozen=True)
class Spec:
    """Shape of one workload.  ``prefix`` / ``new`` give, per sequence, the
    tokens stored before this step and the tokens this step appends (= its
    query rows).  ``share`` lists groups of sequences whose first
    ``share_tokens`` tokens are one stored prefix (copy-on-write)."""
    name: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    prefix: tuple
    new: tuple
    pool_factor: float = 1.25
    num_blocks: int | None = None
    q_std: float = 1.0
    share: tuple = ()
    share_tokens: int = 0


def _lengths(cfg: int, rng: np.random.Generator):
    """Draw the per-sequence lengths of one of the five standard workloads."""
    if cfg == 1:
        ctx = np.array([5, 17, 33, 64])
        return tuple(ctx - 1), (1,) * 4
    if cfg == 2:
        ctx = rng.integers(512, 4096, size=64, endpoint=True)
        return tuple(ctx - 1), (1,) * 64
    if cfg == 3:
        ctx = np.clip(np.round(rng.lognormal(math.log(1500.0), 0.8, size=128)), 16, 8192).astype(np.int64)
        return tuple(ctx - 1), (1,) * 128
    if cfg == 4:
        tails = rng.integers(0, 1024, size=32, endpoint=True)
        return tuple(2048 + tails), (1,) * 32
    if cfg == 5:
        ctx = rng.integers(256, 8192, size=127, endpoint=True)
        return (16384,) + tuple(ctx - 1), (512,) + (1,) * 127
    if cfg == 6:  # the 70B-like length mix, each sequence verifying 4 draft tokens
        ctx = np.clip(np.round(rng.lognormal(math.log(1500.0), 0.8, size=128)), 16, 8192).astype(np.int64)
        return tuple(ctx - 4), (4,) * 128
    if cfg == 7:  # GRPO with long prompts: 8 prompts x 16 rollouts, 8192-token shared prefixes
        tails = rng.integers(0, 1024, size=128, endpoint=True)
        return tuple(8192 + tails), (1,) * 128
    raise ValueError(f"unknown workload {cfg}")


def standard_spec(cfg: int, seed: int | None = None) -> Spec:
    """The standard workloads (1 tiny decode, 2 Llama-3-8B-like decode,
    3 Llama-3.3-70B-like decode at concurrency 128, 4 GRPO shared-prefix decode,
    5 mixed 512-token prefill chunk + 127 decodes, 6 the workload-3 layer
    verifying 4 draft tokens per sequence, as speculative decoding does --
    "Inference optimization", section "Speculative decoding"; 7 the GRPO
    shape with 8 prompts of 8192 tokens x 16 rollouts, whose shared prefixes
    (268 MB of KV) no longer fit in the 126 MB L2)."""
    seed = 445 + cfg if seed is None else seed
    rng = np.random.Generator(np.random.PCG64(seed))
    prefix, new = _lengths(cfg, rng)
    if cfg == 1:
        return Spec("tiny-decode", 2, 1, 64, 16, prefix, new, num_blocks=16)
    if cfg == 2:
        return Spec("llama3-8b-layer-decode-b64", 32, 8, 128, 16, prefix, new)
    if cfg == 3:
        return Spec("llama3.3-70b-layer-decode-b128", 64, 8, 128, 16, prefix, new, q_std=0.5)
    if cfg == 4:
        groups = (tuple(range(16)), tuple(range(16, 32)))
        return Spec("grpo-shared-prefix-decode-2x16", 24, 4, 256, 32, prefix, new,
                    share=groups, share_tokens=2048)
    if cfg == 5:
        return Spec("mixed-prefill512-plus-127-decodes", 64, 8, 128, 16, prefix, new)
    if cfg == 7:
        groups = tuple(tuple(range(16 * g, 16 * g + 16)) for g in range(8))
        return Spec("grpo-long-prefix-decode-8x16", 24, 4, 256, 32, prefix, new, share=groups, share_tokens=8192)
    return Spec("llama3.3-70b-layer-verify4-b128", 64, 8, 128, 16, prefix, new, q_std=0.5)


def build(spec: Spec, seed: int, poison: bool = False, max_blocks: int | None = None) -> Workload:
    """Materialise a workload: allocator state, tables, slots and bf16 data."""
    prefix = np.asarray(spec.prefix, dtype=np.int64)
    new = np.asarray(spec.new, dtype=np.int64)
    b = len(prefix)
    bs = spec.block_size
    blocks = lambda n: -(-int(n) // bs)  # noqa: E731

    # pool size: pool_factor x the blocks the batch needs (shared prefixes once)
    shared_members = {s for g in spec.share for s in g}
    need = sum(blocks(prefix[s] + new[s]) for s in range(b) if s not in shared_members)
    for g in spec.share:
        pblk = blocks(spec.share_tokens)
        need += pblk + sum(blocks(prefix[s] + new[s]) - spec.share_tokens // bs for s in g)
    nb = spec.num_blocks if spec.num_blocks is not None else max(1, int(math.ceil(spec.pool_factor * need)))

    alloc = BlockAllocator(nb, bs, seed=seed)
    seq_ids = list(range(b))
    in_group = {}
    for gi, g in enumerate(spec.share):
        root = -1 - gi
        alloc.add_sequence(root, spec.share_tokens)
        for s in g:
            in_group[s] = root
    for s in seq_ids:
        if s in in_group:
            alloc.fork(in_group[s], s)
            alloc.append_slots(s, int(prefix[s]) - spec.share_tokens)
        else:
            alloc.add_sequence(s, int(prefix[s]))
    slot_chunks = [alloc.append_slots(s, int(new[s])) for s in seq_ids]
    slot_mapping = np.concatenate(slot_chunks).astype(np.int32) if slot_chunks else np.zeros(0, np.int32)
    if alloc.pending_copies:
        raise AssertionError("standard workloads keep shared prefixes block-aligned")
    context_lens = alloc.context_lens(seq_ids)
    block_tables = alloc.block_table(seq_ids, max_blocks)
    query_start = np.concatenate([[0], np.cumsum(new)]).astype(np.int32)

    hkv, d, hq = spec.num_kv_heads, spec.head_dim, spec.num_q_heads
    tq = int(query_start[-1])
    k_cache = normal_bf16(seed, 1, (nb, hkv, bs, d))
    v_cache = normal_bf16(seed, 2, (nb, hkv, bs, d))
    k_new = normal_bf16(seed, 3, (tq, hkv, d))
    v_new = normal_bf16(seed, 4, (tq, hkv, d))
    q = normal_bf16(seed, 5, (tq, hq, d), std=spec.q_std)

    if poison:
        valid = np.zeros((nb, bs), dtype=bool)
        for s in seq_ids:
            pos = np.arange(int(prefix[s]), dtype=np.int64)
            valid[block_tables[s, pos // bs], pos % bs] = True
        bad = ~valid
        k_cache.transpose(0, 2, 1, 3)[bad] = BF16_NAN  # views: writes land in the caches
        v_cache.transpose(0, 2, 1, 3)[bad] = BF16_NAN

    groups = []
    for g in spec.share:
        members = sorted(g)
        if members != list(range(members[0], members[-1] + 1)):
            raise AssertionError("copy-on-write groups are consecutive sequences")
        groups.append((members[0], members[-1] + 1))
    return Workload(spec.name, hq, hkv, d, bs, nb, 1.0 / math.sqrt(d), q, k_new, v_new,
                    k_cache, v_cache, block_tables, context_lens, query_start, slot_mapping,
                    spec.share_tokens, tuple(groups))


E4M3_NAN = np.uint8(0x7F)


def fp8_caches(w: Workload, seed: int, poison: bool = False):
    """Synthetic contents of an FP8 (E4M3 code) cache of w's shape: codes with
    a random sign, exponent field 3..9 and mantissa (values 2^-4 .. 3.75 before
    the scale), and the per-tensor scales (0.5 for K, 0.25 for V).  With
    ``poison`` every slot that does not hold a valid earlier token holds the
    NaN code.  Returns (k_codes, v_codes, k_scale, v_scale)."""
    out = []
    for stream in (11, 12):
        g = np.random.Generator(np.random.PCG64(seed).jumped(stream))
        shape = w.k_cache.shape
        sign = g.integers(0, 2, size=shape, dtype=np.uint8) << 7
        exp = g.integers(3, 10, size=shape, dtype=np.uint8) << 3
        man = g.integers(0, 8, size=shape, dtype=np.uint8)
        out.append((sign | exp | man).astype(np.uint8))
    kc, vc = out
    if poison:
        bad = np.ones((w.num_blocks, w.block_size), dtype=bool)
        qs = w.query_start
        for s in range(w.num_seqs):
            prefix = int(w.context_lens[s]) - int(qs[s + 1] - qs[s])
            pos = np.arange(prefix, dtype=np.int64)
            bad[w.block_tables[s, pos // w.block_size], pos % w.block_size] = False
        kc.transpose(0, 2, 1, 3)[bad] = E4M3_NAN
        vc.transpose(0, 2, 1, 3)[bad] = E4M3_NAN
    return kc, vc, 0.5, 0.25


def standard(cfg: int, seed: int | None = None, poison: bool = False) -> Workload:
    seed = 445 + cfg if seed is None else seed
    return build(standard_spec(cfg, seed), seed, poison=poison)


def custom(prefix, new, num_q_heads, num_kv_heads, head_dim, block_size, seed=0,
           poison=False, pool_factor=1.25, num_blocks=None, share=(), share_tokens=0,
           q_std=1.0, max_blocks=None) -> Workload:
    """A workload of any shape (tests use small ones that still span tiles)."""
    spec = Spec("custom", num_q_heads, num_kv_heads, head_dim, block_size, tuple(int(x) for x in prefix),
                tuple(int(x) for x in new), pool_factor=pool_factor, num_blocks=num_blocks,
                q_std=q_std, share=share, share_tokens=share_tokens)
    return build(spec, seed, poison=poison, max_blocks=max_blocks)
