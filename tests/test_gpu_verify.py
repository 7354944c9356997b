"""GPU parity of the multi-row (verification) path against the fp64 oracle.

Sequences with 2 .. 64/G query rows run on the tcgen05 kernel with the keys
in M; longer ones on the chunk kernel and single rows on the rows kernel, all
inside one pa_prefill_chunk call.  Pools are poisoned (NaN in every slot that
is not a valid earlier token).  Tolerance: 1e-2 max-abs, 5e-3 relative-L2.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_445_b200 import workloads
from tests.gpu_helpers import DeviceStep, compare, load_library, oracle_after_append

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    load_library()


def _ref(w, kc, vc, only=None):
    return oracle.paged_attention(w.q, kc, vc, w.block_tables, w.context_lens, w.query_start, w.scale, only=only)


CASES = [  # prefix (keys before the rows), query rows, Hq, Hkv, bs
    # G 8 (32 columns up to 4 rows): tiny contexts, tile edges 127/128/129, a decode row, several tiles
    ([0, 1, 3, 124, 125, 126, 127, 200, 1000, 2500], [2, 4, 4, 4, 4, 4, 1, 3, 4, 4], 64, 8, 16),
    # G 8, 5 .. 8 rows (the 64-column kernel), 32-token blocks
    ([0, 10, 300, 1500], [5, 8, 6, 8], 64, 8, 32),
    # G 16: 2 rows (32 columns), 3 and 4 rows (64), 5 rows on the chunk kernel
    ([40, 250, 600, 90], [2, 3, 4, 5], 32, 2, 16),
    # G 1: up to 32 rows on the 32-column kernel, 33 .. 64 on the 64-column one, 65 on the chunk kernel
    ([5, 100, 200, 7, 300, 10], [2, 17, 32, 33, 64, 65], 4, 4, 16),
    # G 4, 32-token blocks: 8 rows (32 columns), 9 and 16 (64), 17 on the chunk kernel
    ([129, 1, 1000, 60], [8, 9, 16, 17], 16, 4, 32),
    # G 2: 2, 16 and 32 rows (4, 32 and 64 columns)
    ([700, 33, 64], [2, 16, 32], 8, 4, 16),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"Hq{c[2]}-Hkv{c[3]}-bs{c[4]}-q{max(c[1])}")
def test_multi_row_batches_match_oracle(case):
    prefix, qlen, hq, hkv, bs = case
    w = workloads.custom(prefix, qlen, hq, hkv, 128, bs, seed=sum(prefix) + len(qlen), poison=True)
    ds = DeviceStep(w)
    got = ds.step()
    kc, vc = oracle_after_append(w)
    compare(got, _ref(w, kc, vc), str(case))
    assert int(ds.status.item()) == 0


def test_items_cut_over_many_ctas_merge_exactly_and_deterministically():
    # few units per CTA: a 20,004-key item is cut into about a hundred pieces,
    # the short ones into a few, and some CTAs get no unit at all
    for prefix, qlen, hq, hkv in (([20000, 5000], [4, 4], 8, 1), ([300], [4], 8, 1), ([900, 17], [3, 2], 16, 2)):
        w = workloads.custom(prefix, qlen, hq, hkv, 128, 16, seed=len(prefix) + sum(prefix) % 97, poison=True)
        ds = DeviceStep(w)
        got = ds.step()
        kc, vc = oracle_after_append(w)
        compare(got, _ref(w, kc, vc), f"cut items {prefix}")
        assert int(ds.status.item()) == 0
        first = ds.out.clone()
        for _ in range(3):  # the same bits every time, with the same workspace (its counters went back to zero)
            ds.attend()
            torch.cuda.synchronize()
            assert torch.equal(ds.out.view(torch.int16), first.view(torch.int16))
        assert int(ds.status.item()) == 0


def test_late_large_score_rescales_some_columns():
    # one key far into the context with 40x the usual magnitude: it raises the
    # running maximum of some columns by far more than 2^8 and lowers others
    from paged_kv_cache_445_b200.workloads import bf16_bits_to_f32, f32_to_bf16_bits
    prefix, qlen, hq, hkv, bs = [1500, 600], [4, 8], 64, 8, 16
    w = workloads.custom(prefix, qlen, hq, hkv, 128, bs, seed=31, poison=True)
    for s, pos in ((0, 700), (1, 300)):
        blk, off = int(w.block_tables[s, pos // bs]), pos % bs
        w.k_cache[blk, :, off, :] = f32_to_bf16_bits(bf16_bits_to_f32(w.k_cache[blk, :, off, :]) * 40.0)
    ds = DeviceStep(w)
    got = ds.step()
    kc, vc = oracle_after_append(w)
    compare(got, _ref(w, kc, vc), "late large score")
    assert int(ds.status.item()) == 0


@pytest.mark.parametrize("scale", [0.0, -0.07])
def test_zero_and_negative_scales(scale):
    w = workloads.custom([260, 40, 1000], [4, 2, 8], 64, 8, 128, 16, seed=5, poison=True)
    w.scale = scale
    ds = DeviceStep(w)
    got = ds.step()
    kc, vc = oracle_after_append(w)
    compare(got, _ref(w, kc, vc), f"scale {scale}")
    assert int(ds.status.item()) == 0


def test_sequences_without_rows_between_multi_row_ones():
    # sequences that add no row this step (one with no keys at all) sit between the multi-row ones
    w = workloads.custom([0, 50, 30, 0, 129], [0, 4, 0, 3, 2], 64, 8, 128, 16, seed=9, poison=True)
    ds = DeviceStep(w)
    got = ds.step()
    kc, vc = oracle_after_append(w)
    compare(got, _ref(w, kc, vc), "rowless sequences")
    assert int(ds.status.item()) == 0


def test_groups_the_tensor_core_paths_do_not_take_run_on_the_decode_kernel():
    # G = 6 at head_dim 128: multi-row sequences run row by row on the decode kernel
    w = workloads.custom([300, 41, 1000], [4, 2, 7], 24, 4, 128, 16, seed=17, poison=True)
    ds = DeviceStep(w)
    got = ds.step()
    kc, vc = oracle_after_append(w)
    compare(got, _ref(w, kc, vc), "G 6")
    assert int(ds.status.item()) == 0


def test_batches_past_the_multi_row_kernels_sequence_limit_run_on_the_chunk_kernel():
    # 600 sequences of 4 rows: more than the multi-row kernel's 512, so the chunk kernel takes them
    rng = np.random.default_rng(23)
    prefix = rng.integers(20, 200, 600).tolist()
    w = workloads.custom(prefix, [4] * 600, 16, 2, 128, 16, seed=23, poison=True)
    ds = DeviceStep(w)
    got = ds.step()
    kc, vc = oracle_after_append(w)
    compare(got, _ref(w, kc, vc), "600 sequences, every row")
    assert int(ds.status.item()) == 0
