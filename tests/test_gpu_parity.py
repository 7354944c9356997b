"""GPU parity: libpa.so (through the C-ABI binding) against the fp64 oracle.

Append and slot indexing must be bit-exact; attention outputs must be within
1e-2 max-abs and 5e-3 relative-L2 error of the oracle (bf16 inputs, fp32
accumulation, bf16 output).  Caches are poisoned: every slot that does not
hold a valid token holds NaN, so reading past a context shows up.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_445_b200 import workloads
from tests.gpu_helpers import DeviceStep, compare, dev_to_bits, i32, load_library, oracle_after_append

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    load_library()


def _attend_ref(w, kc, vc, only=None):
    return oracle.paged_attention(w.q, kc, vc, w.block_tables, w.context_lens, w.query_start, w.scale, only=only)


# ------------------------------------------------------------------ append

@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5, 6])
def test_append_is_bit_exact_on_the_standard_workloads(cfg):
    w = workloads.standard(cfg, poison=True)
    ds = DeviceStep(w)
    ds.append()
    torch.cuda.synchronize()
    kc, vc = oracle_after_append(w)
    assert np.array_equal(dev_to_bits(ds.k_cache), kc)
    assert np.array_equal(dev_to_bits(ds.v_cache), vc)
    assert int(ds.status.item()) == 0


def test_append_skips_padding_and_reports_out_of_range_slots():
    import paged_kv_cache_445_b200 as pa
    w = workloads.custom([10, 40, 3], [1, 1, 1], 4, 2, 128, 16, seed=21)
    ds = DeviceStep(w)
    slots = w.slot_mapping.copy()
    slots[1] = -1
    slots[2] = w.num_blocks * w.block_size + 7  # outside the pool
    ds.slot_mapping = i32(slots)
    before_k = dev_to_bits(ds.k_cache)
    ds.append()
    torch.cuda.synchronize()
    got = dev_to_bits(ds.k_cache)
    want = before_k.copy()
    s0 = int(slots[0])
    want[s0 // 16, :, s0 % 16, :] = w.k_new[0]
    assert np.array_equal(got, want)
    assert int(ds.status.item()) == pa.status_bit(pa._binding.PA_ERR_RANGE)


# ------------------------------------------------------------------ decode

@pytest.mark.parametrize("cfg", [1, 2, 3, 4])
def test_decode_matches_oracle_on_the_standard_workloads(cfg):
    w = workloads.standard(cfg, poison=True)
    ds = DeviceStep(w)
    got = ds.step()
    kc, vc = oracle_after_append(w)
    compare(got, _attend_ref(w, kc, vc), f"config {cfg}")
    assert int(ds.status.item()) == 0


def test_mixed_chunk_and_decodes_match_oracle():
    # every row of the batch: all 512 chunk tokens x 64 heads (so every
    # (M-tile pair, KV head) item of the tensor-core chunk kernel) and all 127
    # decode rows, element by element
    w = workloads.standard(5, poison=True)
    ds = DeviceStep(w)
    got = ds.step()
    assert int(ds.status.item()) == 0
    kc, vc = oracle_after_append(w)
    ref = _attend_ref(w, kc, vc)
    compare(got[:512], ref[:512], "config 5, the 512-token chunk")
    compare(got[512:], ref[512:], "config 5, the 127 decode rows")
    compare(got, ref, "config 5, whole batch")


def test_verify4_batch_matches_oracle_on_every_row():
    # 128 sequences of the 70B-like mix, 4 query rows each (speculative
    # verification): all 512 rows x 64 heads
    w = workloads.standard(6, poison=True)
    ds = DeviceStep(w)
    got = ds.step()
    assert int(ds.status.item()) == 0
    kc, vc = oracle_after_append(w)
    compare(got, _attend_ref(w, kc, vc), "verify-4, every row")


SMALL = [  # ctx list, qlen list, Hq, Hkv, d, bs
    ([1, 15, 16, 17, 33, 100, 257], [1] * 7, 8, 1, 128, 16),
    ([1, 31, 32, 33, 65, 300], [1] * 6, 8, 4, 64, 32),
    ([5, 16, 40, 129, 700], [1] * 5, 12, 2, 256, 16),
    ([3, 32, 64, 500], [1] * 4, 16, 1, 128, 32),
    ([17, 90, 1000], [1] * 3, 32, 2, 128, 16),
    ([2, 77, 400, 1300], [1] * 4, 4, 4, 64, 16),
    ([64, 200], [40, 1], 8, 2, 128, 16),
    ([50, 9, 300, 1], [50, 3, 17, 1], 6, 3, 64, 32),
    ([600], [77], 24, 4, 256, 32),
    # prefill chunks on the tcgen05 path (head_dim 128, G in {1, 2, 4, 8, 16})
    ([300], [300], 8, 1, 128, 16),               # whole prompt from position 0, partial last token block
    ([1000, 40], [130, 1], 16, 2, 128, 32),      # G 8, 32-token blocks, chunk deep in the context
    ([700], [200], 4, 4, 128, 16),               # G 1: 128 tokens per tile
    ([500, 77], [50, 1], 32, 2, 128, 16),        # G 16: 8 tokens per tile
    ([260, 129, 1], [5, 129, 1], 8, 4, 128, 16), # G 2, several chunks and a decode in one batch
    # the same on the tcgen05 path at head_dim 64 (one 64-column panel per row)
    ([300], [300], 8, 1, 64, 16),
    ([1000, 40], [130, 1], 16, 2, 64, 32),
    ([700], [200], 4, 4, 64, 16),
    ([500, 77], [50, 1], 32, 2, 64, 16),
    ([260, 129, 1], [5, 129, 1], 8, 4, 64, 16),
    # groups that do not divide 128 rows: G 6 and 12 (120-row M-tiles, 8 rows of padding)
    ([900, 40], [300, 1], 24, 4, 128, 32),       # G 6, the GRPO shape's group
    ([500, 77, 9], [161, 1, 3], 24, 4, 64, 16),  # G 6 at head_dim 64, a 3-row sequence on the chunk path
    ([700], [90], 24, 2, 128, 16),               # G 12
    ([333, 20], [333, 2], 12, 1, 64, 16),        # G 12 at head_dim 64, whole prompt from position 0
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"Hq{c[2]}-Hkv{c[3]}-d{c[4]}-bs{c[5]}-q{max(c[1])}")
def test_small_shapes_match_oracle(case):
    ctx, qlen, hq, hkv, d, bs = case
    prefix = [c - q for c, q in zip(ctx, qlen)]
    w = workloads.custom(prefix, qlen, hq, hkv, d, bs, seed=sum(ctx), poison=True)
    ds = DeviceStep(w)
    got = ds.step()
    kc, vc = oracle_after_append(w)
    compare(got, _attend_ref(w, kc, vc), str(case))
    assert int(ds.status.item()) == 0


def test_late_large_scores_rescale_some_rows_of_a_tile():
    # one key deep in the prefix gets 40x the usual magnitude: for about half
    # the query rows its score raises the running maximum far above the
    # earlier tiles' (the others see a very negative score), so the rescale of
    # O runs for some rows of a tile and not for others -- on the tensor-core
    # chunk path (G 8, head_dim 128 and 64) and on the rows path (G 6, head_dim 64)
    from paged_kv_cache_445_b200.workloads import bf16_bits_to_f32, f32_to_bf16_bits
    for prefix, qlen, hq, hkv, d, bs in (([870, 39], [130, 1], 16, 2, 128, 32), ([870, 39], [130, 1], 16, 2, 64, 32),
                                         ([500, 20], [60, 1], 12, 2, 64, 16)):
        w = workloads.custom(prefix, qlen, hq, hkv, d, bs, seed=12, poison=True)
        pos = 300
        blk, off = int(w.block_tables[0, pos // bs]), pos % bs
        row = bf16_bits_to_f32(w.k_cache[blk, :, off, :]) * 40.0
        w.k_cache[blk, :, off, :] = f32_to_bf16_bits(row)
        ds = DeviceStep(w)
        got = ds.step()
        kc, vc = oracle_after_append(w)
        compare(got, _attend_ref(w, kc, vc), f"large late score, d{d}")
        assert int(ds.status.item()) == 0


@pytest.mark.parametrize("cfg", [1, 2, 3, 4])
def test_fused_append_decode_equals_the_two_calls_bit_for_bit(cfg):
    import paged_kv_cache_445_b200 as pa
    w = workloads.standard(cfg, poison=True)
    two = DeviceStep(w)
    two.step()
    one = DeviceStep(w)
    pa.pa_decode_append(one.out, one.q, one.k_new, one.v_new, one.k_cache, one.v_cache, one.block_tables,
                        one.context_lens, w.scale, one.workspace, one.status)
    torch.cuda.synchronize()
    assert int(one.status.item()) == 0
    assert torch.equal(one.out.view(torch.int16), two.out.view(torch.int16))
    assert torch.equal(one.k_cache.view(torch.int16), two.k_cache.view(torch.int16))
    assert torch.equal(one.v_cache.view(torch.int16), two.v_cache.view(torch.int16))
    if cfg == 1:
        kc, vc = oracle_after_append(w)
        compare(one.out.float().cpu().numpy(), _attend_ref(w, kc, vc), "fused append, tiny")


def test_fused_append_reports_a_bad_block_and_keeps_going():
    import paged_kv_cache_445_b200 as pa
    w = workloads.custom([40, 60, 7], [1, 1, 1], 8, 2, 128, 16, seed=13)
    ds = DeviceStep(w)
    bt = w.block_tables.copy()
    bt[1, 60 // 16] = w.num_blocks + 3  # the newest token's block is outside the pool
    ds.block_tables = i32(bt)
    pa.pa_decode_append(ds.out, ds.q, ds.k_new, ds.v_new, ds.k_cache, ds.v_cache, ds.block_tables,
                        ds.context_lens, w.scale, ds.workspace, ds.status)
    torch.cuda.synchronize()
    assert int(ds.status.item()) & pa.status_bit(pa._binding.PA_ERR_RANGE)


def test_varlen_entry_on_a_pure_decode_batch_matches_decode_entry():
    w = workloads.custom([30, 700, 4000], [1, 1, 1], 16, 2, 128, 16, seed=3, poison=True)
    a = DeviceStep(w).step()
    b = DeviceStep(w).step(force_varlen=True)
    kc, vc = oracle_after_append(w)
    ref = _attend_ref(w, kc, vc)
    compare(a, ref, "decode entry")
    assert np.array_equal(a, b)  # same batch, same partition of the work: the same bits


def test_long_segments_split_over_many_warps_merge_exactly():
    # two very long contexts: each (row, head) segment spans dozens of warps
    w = workloads.custom([32000, 24999], [1, 1], 16, 2, 128, 16, seed=4, poison=True)
    ds = DeviceStep(w)
    got = ds.step()
    kc, vc = oracle_after_append(w)
    compare(got, _attend_ref(w, kc, vc), "long contexts")


def test_results_are_deterministic_and_workspace_is_reusable():
    w = workloads.custom([100, 2000, 5000, 9], [1, 1, 1, 1], 8, 1, 128, 16, seed=6)
    ds = DeviceStep(w)
    ds.append()
    kc, vc = oracle_after_append(w)
    ref = _attend_ref(w, kc, vc)
    outs = []
    for _ in range(4):
        ds.attend()
        torch.cuda.synchronize()
        outs.append(ds.out.float().cpu().numpy())
        compare(outs[-1], ref, "repeated call")
        assert int(ds.status.item()) == 0
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_large_batch_with_claimed_tail_chunks_is_exact_and_deterministic():
    # at least 16 tiles per launched warp: the last 3/16 of the tiles are
    # handed out at run time in fixed chunks; whichever warp takes a chunk,
    # the pieces and therefore the bits must be the same
    ctx = [5000, 7000, 3000, 6000, 4500, 8000, 2500, 6500, 1, 17]
    w = workloads.custom([c - 1 for c in ctx], [1] * len(ctx), 64, 8, 128, 16, seed=11, poison=True)
    ds = DeviceStep(w)
    ds.append()
    kc, vc = oracle_after_append(w)
    ref = _attend_ref(w, kc, vc)
    outs = []
    for _ in range(3):
        ds.attend()
        torch.cuda.synchronize()
        assert int(ds.status.item()) == 0
        outs.append(ds.out.float().cpu().numpy())
    compare(outs[0], ref, "tail chunks")
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_empty_context_gives_zeros():
    w = workloads.custom([0, 40, 0], [1, 1, 1], 8, 2, 128, 16, seed=7)
    ds = DeviceStep(w)
    ds.append()
    cl = w.context_lens.copy()
    cl[0] = 0  # sequence 0 has no key at all
    ds.context_lens = i32(cl)
    ds.out.fill_(7.0)
    ds.attend()
    torch.cuda.synchronize()
    got = ds.out.float().cpu().numpy()
    assert np.all(got[0] == 0)
    kc, vc = oracle_after_append(w)
    ref = oracle.paged_attention(w.q, kc, vc, w.block_tables, cl, w.query_start, w.scale)
    compare(got, ref, "empty context")


def test_guard_regions_are_untouched():
    w = workloads.custom([33, 200, 5], [1, 1, 1], 8, 2, 128, 16, seed=8)
    ds = DeviceStep(w)
    big = torch.full((w.num_query_tokens + 4, w.num_q_heads, w.head_dim), 3.0, dtype=torch.bfloat16, device="cuda")
    ds.out = big[2:-2]
    ds.step()
    assert torch.all(big[:2] == 3.0) and torch.all(big[-2:] == 3.0)


def test_bad_block_ids_and_long_contexts_are_reported_not_faulted():
    import paged_kv_cache_445_b200 as pa
    w = workloads.custom([40, 60], [1, 1], 8, 2, 128, 16, seed=9)
    ds = DeviceStep(w)
    ds.append()
    bt = w.block_tables.copy()
    bt[0, 1] = w.num_blocks + 1000  # outside the pool
    ds.block_tables = i32(bt)
    ds.attend()
    torch.cuda.synchronize()
    assert int(ds.status.item()) & pa.status_bit(pa._binding.PA_ERR_RANGE)
    ds.status.zero_()
    cl = w.context_lens.copy()
    cl[1] = bt.shape[1] * w.block_size + 50  # longer than its table
    ds.context_lens = i32(cl)
    ds.block_tables = i32(w.block_tables)
    ds.workspace.zero_()
    ds.attend()
    torch.cuda.synchronize()
    assert int(ds.status.item()) & pa.status_bit(pa._binding.PA_ERR_RANGE)
    # the context stays usable
    ds.status.zero_()
    ds.context_lens = i32(w.context_lens)
    ds.workspace.zero_()
    ds.attend()
    torch.cuda.synchronize()
    assert int(ds.status.item()) == 0


def test_small_workspace_is_rejected():
    import paged_kv_cache_445_b200 as pa
    w = workloads.custom([40], [1], 8, 2, 128, 16, seed=10)
    ds = DeviceStep(w)
    ds.workspace = torch.zeros(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(pa.PAError) as e:
        ds.attend()
    assert e.value.code == pa._binding.PA_ERR_WORKSPACE


@pytest.mark.parametrize("cfg", [3, 5])
def test_a_captured_step_replays_bit_identically(cfg):
    # the step's launches (cooperative, programmatic dependent launch) captured
    # in a CUDA graph: replays give the eager result, bit for bit
    import paged_kv_cache_445_b200 as pa
    w = workloads.standard(cfg)
    ds = DeviceStep(w)
    kc0, vc0 = ds.k_cache.clone(), ds.v_cache.clone()

    def step():
        if w.is_decode:
            pa.pa_decode_append(ds.out, ds.q, ds.k_new, ds.v_new, ds.k_cache, ds.v_cache, ds.block_tables,
                                ds.context_lens, w.scale, ds.workspace, ds.status)
        else:
            ds.append()
            ds.attend()

    step()
    torch.cuda.synchronize()
    eager = ds.out.clone()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(2):
        ds.out.fill_(0)
        ds.k_cache.copy_(kc0)
        ds.v_cache.copy_(vc0)
        graph.replay()
        torch.cuda.synchronize()
        assert int(ds.status.item()) == 0
        assert torch.equal(ds.out.view(torch.int16), eager.view(torch.int16))


def test_a_wait_that_runs_out_is_reported_and_the_context_stays_usable():
    # The decode kernel's grid barrier waits (bounded, about 2 s) until every
    # warp has arrived on the workspace counter, which the caller zero-fills.
    # A counter left at -1 (the zero-fill skipped) never reaches the target:
    # the wait runs out, the kernel sets the TIMEOUT bit and returns, and
    # nothing faults.  After a zero-fill the next call is exact again.
    import paged_kv_cache_445_b200 as pa
    w = workloads.custom([3000, 40, 1200], [1, 1, 1], 16, 2, 128, 16, seed=14, poison=True)
    ds = DeviceStep(w)
    ds.append()
    kc, vc = oracle_after_append(w)
    ref = _attend_ref(w, kc, vc)
    ds.workspace.view(torch.int32)[0] = -1  # the barrier's arrival counter
    ds.attend()
    torch.cuda.synchronize()
    assert int(ds.status.item()) & pa.status_bit(pa._binding.PA_ERR_TIMEOUT)
    ds.status.zero_()
    ds.workspace.zero_()
    ds.out.fill_(0)
    ds.attend()
    torch.cuda.synchronize()
    assert int(ds.status.item()) == 0
    compare(ds.out.float().cpu().numpy(), ref, "after a timed-out call")
