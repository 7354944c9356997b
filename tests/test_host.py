"""Host-side logic: block allocator, workloads, byte counts (CPU only)."""
from __future__ import annotations

import json
import math
import os

import numpy as np
import pytest

from paged_kv_cache_445_b200 import roofline, workloads
from paged_kv_cache_445_b200.allocator import BlockAllocator, OutOfBlocks, static_reservation_waste

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- allocator

def test_blocks_per_sequence_is_ceil():
    a = BlockAllocator(100, 16, seed=1)
    for sid, n in enumerate([1, 15, 16, 17, 64, 65, 0]):
        a.add_sequence(sid, n)
        assert len(a.table(sid)) == -(-n // 16)
    assert a.used_blocks() == sum(-(-n // 16) for n in [1, 15, 16, 17, 64, 65, 0])


def test_no_block_is_double_owned_and_free_returns_everything():
    rng = np.random.default_rng(0)
    a = BlockAllocator(200, 16, seed=2)
    lens = rng.integers(1, 300, size=12)
    for sid, n in enumerate(lens):
        a.add_sequence(sid, int(n))
    owned = [b for sid in range(12) for b in a.table(sid)]
    assert len(owned) == len(set(owned))
    assert all(a.refcount(b) == 1 for b in owned)
    for sid in range(12):
        a.free(sid)
    assert a.num_free == 200 and a.used_blocks() == 0


def test_growth_takes_a_block_only_at_a_boundary():
    a = BlockAllocator(10, 4, seed=3)
    a.add_sequence(0, 3)
    assert len(a.table(0)) == 1
    s = a.append_slots(0, 1)  # position 3 fills block 0
    assert len(a.table(0)) == 1 and s[0] == a.table(0)[0] * 4 + 3
    s = a.append_slots(0, 1)  # position 4 starts block 1
    assert len(a.table(0)) == 2 and s[0] == a.table(0)[1] * 4 + 0


def test_fork_shares_and_copy_on_write_happens_only_on_a_shared_partial_block():
    a = BlockAllocator(20, 4, seed=4)
    a.add_sequence(0, 6)  # blocks: full, half
    a.fork(0, 1)
    a.fork(0, 2)
    shared = a.table(0)
    assert all(a.refcount(b) == 3 for b in shared)
    # child 1 writes position 6: the half block is shared -> copy on write
    s = a.append_slots(1, 1)
    assert len(a.pending_copies) == 1
    src, dst = a.pending_copies[0]
    assert src == shared[1] and dst == a.table(1)[1] and dst not in shared
    assert s[0] == dst * 4 + 2
    assert a.refcount(shared[1]) == 2 and a.refcount(shared[0]) == 3
    # child 2 writes at position 6 too -> another copy; parent keeps the original
    a.append_slots(2, 2)
    assert len(a.pending_copies) == 2 and a.refcount(shared[1]) == 1
    # parent now owns its half block alone: no copy
    a.append_slots(0, 1)
    assert len(a.pending_copies) == 2
    for sid in (0, 1, 2):
        a.free(sid)
    assert a.num_free == 20


def test_block_aligned_prefix_never_copies():
    a = BlockAllocator(128, 32, seed=5)
    a.add_sequence(-1, 2048)  # 64 full blocks
    for r in range(16):
        a.fork(-1, r)
        a.append_slots(r, 1 + r)
    assert a.pending_copies == []


def test_out_of_blocks_raises():
    a = BlockAllocator(2, 16)
    a.add_sequence(0, 32)
    with pytest.raises(OutOfBlocks):
        a.append_slots(0, 1)


def test_block_table_padding_and_width():
    a = BlockAllocator(10, 16, seed=6)
    a.add_sequence(0, 40)
    a.add_sequence(1, 1)
    bt = a.block_table([0, 1], 4)
    assert bt.shape == (2, 4) and bt.dtype == np.int32
    assert (bt[0, 3] == -1) and (bt[1, 1:] == -1).all()
    with pytest.raises(ValueError):
        a.block_table([0], 2)


def test_fragmentation_matches_the_pages():
    g = json.load(open(os.path.join(GOLDEN, "fragmentation.json")))
    # static reservation: 1 - 1500 / 8192 printed as ~82%
    w = static_reservation_waste([g["static_mean_tokens"]], g["static_reserved"])
    assert round(w, g["static_waste_printed_digits"]) == g["static_waste_printed"]
    # the exercise: 1000 requests, mean 1500, std 600
    rng = np.random.default_rng(445)
    lens = np.clip(np.round(rng.normal(g["exercise_mean"], g["exercise_std"], g["exercise_requests"])), 1, 8192).astype(int)
    static = static_reservation_waste(lens, g["static_reserved"])
    a = BlockAllocator(int(sum(-(-n // 16) for n in lens)), g["paged_block_size"], seed=1)
    for sid, n in enumerate(lens):
        a.add_sequence(sid, int(n))
    paged = a.internal_waste()
    assert 0.79 < static < 0.84
    assert paged < g["paged_waste_bound"]
    # closed form: expected waste per sequence is about (bs - 1) / 2 slots
    expect = (16 - 1) / 2 * len(lens) / (a.used_blocks() * 16)
    assert abs(paged - expect) < 0.003


# ---------------------------------------------------------------- byte formula

def test_kv_bytes_match_the_printed_numbers():
    g = json.load(open(os.path.join(GOLDEN, "kv_bytes.json")))
    for c in g["cases"]:
        b = roofline.kv_cache_bytes(c["layers"], c["kv_heads"], c["head_dim"], c["tokens"], c["bytes"])
        if "expect_bytes" in c:
            assert b == c["expect_bytes"], c["what"]
        else:
            assert round(b / c["printed_unit_bytes"], c["printed_digits"]) == c["expect_printed_value"], c["what"]


def test_decode_bytes_and_unique_bytes():
    w = workloads.custom([31, 15], [1, 1], 4, 2, 16, 16, seed=1)
    assert roofline.decode_kv_bytes(w.context_lens, 2, 16) == (32 + 16) * 2 * 2 * 16 * 2
    # shared prefix counted once
    w = workloads.custom([64, 70, 65], [1, 1, 1], 4, 2, 16, 32, seed=2, share=((0, 1, 2),), share_tokens=64)
    u = roofline.unique_kv_bytes(w.block_tables, w.context_lens, 32, 2, 16)
    assert u == (64 + 1 + 7 + 2) * 2 * 2 * 16 * 2


def test_prefill_flops_closed_form():
    # one sequence: 4 rows at the end of 10 keys -> 7 + 8 + 9 + 10 keys
    assert roofline.prefill_flops([10], [0, 4], 2, 8) == 4 * 8 * 2 * (7 + 8 + 9 + 10)


# ---------------------------------------------------------------- workloads

def test_standard_tiny_workload_shape():
    w = workloads.standard(1)
    assert w.context_lens.tolist() == [5, 17, 33, 64]
    assert w.num_blocks == 16 and w.block_tables.shape[1] == 4
    used = [b for s in range(4) for b in w.block_tables[s] if b >= 0]
    assert len(used) == 10 and len(set(used)) == 10
    assert w.is_decode and w.num_query_tokens == 4
    assert w.k_cache.shape == (16, 1, 16, 64) and w.q.shape == (4, 2, 64)
    assert w.scale == pytest.approx(1 / 8)


@pytest.mark.parametrize("cfg", [2, 3, 4, 5, 6])
def test_standard_workload_specs(cfg):
    spec = workloads.standard_spec(cfg)
    ctx = np.array(spec.prefix) + np.array(spec.new)
    if cfg == 2:
        assert len(ctx) == 64 and ctx.min() >= 512 and ctx.max() <= 4096
    if cfg == 3:
        assert len(ctx) == 128 and ctx.min() >= 16 and ctx.max() <= 8192
        assert 1000 < np.median(ctx) < 2200
    if cfg == 4:
        assert len(ctx) == 32 and (ctx >= 2049).all() and (ctx <= 2048 + 1025).all()
        assert spec.share_tokens == 2048 and len(spec.share) == 2
    if cfg == 5:
        assert spec.new[0] == 512 and spec.prefix[0] == 16384 and len(ctx) == 128
        assert (ctx[1:] >= 256).all() and (ctx[1:] <= 8192).all()
    if cfg == 6:
        assert len(ctx) == 128 and set(spec.new) == {4} and ctx.min() >= 16 and ctx.max() <= 8192


def test_poisoned_workload_marks_every_invalid_slot():
    w = workloads.custom([20, 3], [1, 1], 2, 1, 8, 16, seed=4, poison=True)
    nan = workloads.BF16_NAN
    valid = set()
    for s, n in enumerate([20, 3]):
        for pos in range(n):
            valid.add((int(w.block_tables[s, pos // 16]), pos % 16))
    for b in range(w.num_blocks):
        for off in range(16):
            isnan = bool((w.k_cache[b, 0, off] == nan).all())
            assert isnan == ((b, off) not in valid)


def test_normal_bf16_is_deterministic_and_thread_count_free():
    a = workloads.normal_bf16(9, 1, (3, 1 << 23))  # spans two chunks
    b = workloads.normal_bf16(9, 1, (3, 1 << 23))
    assert np.array_equal(a, b)
    x = workloads.bf16_bits_to_f32(a[:, :100000]).astype(np.float64)
    assert abs(x.mean()) < 0.02 and abs(x.std() - 1) < 0.02


def test_bf16_rounding_ties_to_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5], dtype=np.float32)
    bits = workloads.f32_to_bf16_bits(x)
    back = workloads.bf16_bits_to_f32(bits)
    assert back.tolist() == [1.0, 1.0, 1.0 + 2 ** -6, -2.5]
    assert math.isclose(float(workloads.bf16_bits_to_f32(workloads.f32_to_bf16_bits(np.float32([3.14159])))[0]), 3.140625)


def test_roofline_points_match_the_printed_numbers():
    fx = json.load(open(os.path.join(GOLDEN, "roofline_points.json")))
    r = fx["ridge"]
    assert roofline.ridge_point(r["peak_flops_per_s"], r["peak_bytes_per_s"]) == pytest.approx(r["printed"])
    f = fx["floor"]
    assert roofline.stream_time_s(f["bytes"], f["bytes_per_s"]) * 1e3 == pytest.approx(f["printed_ms"])
    for row in fx["table"]:  # the page's bound column, from the ridge point ("batch 256" sits on the edge: left out)
        got = roofline.bound(row["ops_per_byte"] * 1e9, 1e9, r["peak_flops_per_s"], r["peak_bytes_per_s"])
        assert got == row["expect"], row["scenario"]
