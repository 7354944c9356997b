"""Decode with the split weighted by per-SM rates (pa_calibrate): each SM
takes a share of the key tiles in proportion to its measured rate.  The
result must still match the oracle, the fused append must still equal the two
calls bit for bit, and repeated calls must give the same bits (the split is a
function of the batch and the recorded rates only)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_445_b200 import workloads
from tests.gpu_helpers import DeviceStep, compare, load_library, oracle_after_append

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _calibrated():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    load_library()
    import paged_kv_cache_445_b200 as pa
    pa.pa_calibrate()
    yield
    pa.pa_calibration_clear()  # the other test modules run with the equal split


def _ref(w):
    kc, vc = oracle_after_append(w)
    return oracle.paged_attention(w.q, kc, vc, w.block_tables, w.context_lens, w.query_start, w.scale)


def test_calibration_records_a_rate_per_sm():
    import paged_kv_cache_445_b200 as pa
    rates = pa.pa_calibration()
    assert len(rates) == torch.cuda.get_device_properties(0).multi_processor_count
    assert min(rates) > 0
    assert max(rates) < 4 * min(rates)  # the same order of magnitude everywhere


def test_weighted_decode_matches_the_oracle_and_the_fused_step_on_the_70b_layer():
    import paged_kv_cache_445_b200 as pa
    w = workloads.standard(3, poison=True)
    two = DeviceStep(w)
    got = two.step()
    assert int(two.status.item()) == 0
    compare(got, _ref(w), "weighted split, 70B layer")
    one = DeviceStep(w)
    for _ in range(2):  # fused append: the same bits as the two calls, on every call
        pa.pa_decode_append(one.out, one.q, one.k_new, one.v_new, one.k_cache, one.v_cache, one.block_tables,
                            one.context_lens, w.scale, one.workspace, one.status)
        torch.cuda.synchronize()
        assert int(one.status.item()) == 0
        assert torch.equal(one.out.view(torch.int16), two.out.view(torch.int16))


@pytest.mark.parametrize("case", [
    ([1, 15, 16, 17, 33, 100, 257], 8, 1, 128, 16),   # few tiles: most SMs get an empty share
    ([31, 32, 33, 65, 300], 8, 4, 64, 32),
    ([5, 16, 40, 129, 700], 12, 2, 256, 16),
    ([32000, 24999, 7], 16, 2, 128, 16),               # long segments cut between SMs
    ([3, 32, 64, 500, 8000], 16, 1, 128, 32),
], ids=lambda c: f"Hq{c[1]}-Hkv{c[2]}-d{c[3]}-bs{c[4]}-n{len(c[0])}")
def test_weighted_decode_small_shapes_match_the_oracle(case):
    prefix, hq, hkv, d, bs = case
    w = workloads.custom(prefix, [1] * len(prefix), hq, hkv, d, bs, seed=len(prefix) + d, poison=True)
    ds = DeviceStep(w)
    ds.append()
    ref = _ref(w)
    outs = []
    for _ in range(2):
        ds.attend()
        torch.cuda.synchronize()
        assert int(ds.status.item()) == 0
        outs.append(ds.out.clone())
    compare(outs[0].float().cpu().numpy(), ref, str(case))
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))


def test_weighted_decode_beside_the_chunk_kernel_matches_the_oracle():
    # the planned mixed batch: the decode CTAs on part of the SMs register
    # their SMs, then split by the rates of those SMs only
    import paged_kv_cache_445_b200 as pa
    w = workloads.standard(5, poison=True)
    ds = DeviceStep(w)
    ds.append()
    plan = pa.pa_plan_batch(w.query_start, w.context_lens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
                            w.block_tables.shape[1])
    assert 0 < list(plan.words)[2] < list(plan.words)[3]
    outs = []
    for _ in range(2):
        pa.pa_prefill_chunk_planned(ds.out, ds.q, ds.query_start, ds.k_cache, ds.v_cache, ds.block_tables,
                                    ds.context_lens, w.scale, ds.workspace, plan, ds.status)
        torch.cuda.synchronize()
        assert int(ds.status.item()) == 0
        outs.append(ds.out.clone())
    compare(outs[0].float().cpu().numpy(), _ref(w), "weighted decode beside the chunk kernel")
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
