"""The mixed batch with a host plan: decode rows streaming on part of the
SMs while the tcgen05 chunk kernel computes on the others, and the chunk
kernel's stream-K pieces (items cut between SMs and merged), all against the
fp64 oracle element by element."""
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


def _ref(w):
    kc, vc = oracle_after_append(w)
    return oracle.paged_attention(w.q, kc, vc, w.block_tables, w.context_lens, w.query_start, w.scale)


def _planned(ds: DeviceStep):
    import paged_kv_cache_445_b200 as pa
    w = ds.w
    plan = pa.pa_plan_batch(w.query_start, w.context_lens, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
                            w.block_tables.shape[1])
    pa.pa_prefill_chunk_planned(ds.out, ds.q, ds.query_start, ds.k_cache, ds.v_cache, ds.block_tables,
                                ds.context_lens, w.scale, ds.workspace, plan, ds.status)
    return plan


def test_planned_mixed_batch_shares_the_gpu_and_matches_the_oracle_on_every_row():
    w = workloads.standard(5, poison=True)
    ds = DeviceStep(w)
    ds.append()
    plan = _planned(ds)
    torch.cuda.synchronize()
    assert int(ds.status.item()) == 0
    words = list(plan.words)
    assert words[1] & 4 and words[1] & 8, "the plan sees the chunk and the decode rows"
    assert 0 < words[2] < words[3], "decode rows on part of the SMs, the chunk on the rest"
    assert words[2] % 2 == 0, "SMs come in pairs: the decode side takes whole pairs"
    got = ds.out.float().cpu().numpy()
    ref = _ref(w)
    compare(got[:512], ref[:512], "planned mixed batch, the chunk")
    compare(got[512:], ref[512:], "planned mixed batch, the decode rows")
    # the same again: the split and the merge order are fixed, so are the bits
    first = ds.out.clone()
    _planned(ds)
    torch.cuda.synchronize()
    assert torch.equal(first.view(torch.int16), ds.out.view(torch.int16))


@pytest.mark.parametrize("d,hq,qlen", [(128, 64, 640), (64, 64, 640), (128, 48, 800)])
def test_chunk_items_cut_between_ctas_merge_exactly(d, hq, qlen):
    # more items than CTAs: 20 pairs of M-tiles x 8 KV heads = 160 items of
    # about 13 key tiles on the whole GPU (G 8: 32-token pairs; G 6: 40-token
    # pairs), split into equal unit ranges, so items are cut at CTA
    # boundaries and merged from their pieces
    w = workloads.custom([1000], [qlen], hq, 8, d, 16, seed=61, poison=True)
    ds = DeviceStep(w)
    ds.append()
    ref = _ref(w)
    outs = []
    for _ in range(3):
        ds.attend()
        torch.cuda.synchronize()
        assert int(ds.status.item()) == 0
        outs.append(ds.out.clone())
    compare(outs[0].float().cpu().numpy(), ref, f"items cut between CTAs, d{d}, Hq {hq}")
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))


def test_fewer_items_than_ctas_run_whole():
    # one or two items over 20,000 keys (157 key tiles): each on one CTA
    for hkv in (1, 2):
        w = workloads.custom([20000 - 128], [128], 8 * hkv, hkv, 128, 16, seed=51 + hkv, poison=True)
        ds = DeviceStep(w)
        ds.append()
        ds.attend()
        torch.cuda.synchronize()
        assert int(ds.status.item()) == 0
        compare(ds.out.float().cpu().numpy(), _ref(w), f"whole items, Hkv {hkv}")


PLANNED = [  # prefix list, qlen list, Hq, Hkv, d, bs
    ([16384] + [300, 4000, 7000], [512, 1, 1, 1], 64, 8, 128, 16),  # a chunk and decodes
    ([64, 200], [40, 1], 8, 2, 128, 16),
    ([260, 129, 1], [5, 129, 1], 8, 4, 128, 16),   # G 2: verification rows, chunks and a decode
    ([900, 33, 500], [300, 4, 1], 16, 1, 128, 32),  # G 16
    ([3000, 2000], [2, 2], 32, 4, 128, 16),         # verification rows only
    ([1000, 40, 77], [1, 1, 1], 16, 2, 128, 16),    # decodes only
    ([0], [700], 4, 4, 128, 16),                    # one prompt from position 0, G 1
    ([16384] + [300, 4000, 7000], [512, 1, 1, 1], 64, 8, 64, 16),  # head_dim 64: a chunk and decodes
]


@pytest.mark.parametrize("case", PLANNED, ids=lambda c: f"Hq{c[2]}-Hkv{c[3]}-d{c[4]}-q{max(c[1])}-n{len(c[0])}")
def test_planned_calls_match_the_oracle(case):
    prefix, qlen, hq, hkv, d, bs = case
    w = workloads.custom(prefix, qlen, hq, hkv, d, bs, seed=sum(prefix) + len(qlen), poison=True)
    ds = DeviceStep(w)
    ds.append()
    _planned(ds)
    torch.cuda.synchronize()
    assert int(ds.status.item()) == 0
    compare(ds.out.float().cpu().numpy(), _ref(w), str(case))


def test_a_plan_for_another_batch_is_rejected():
    import paged_kv_cache_445_b200 as pa
    w = workloads.custom([64, 200], [40, 1], 8, 2, 128, 16, seed=3)
    other = workloads.custom([64, 200, 5], [40, 1, 1], 8, 2, 128, 16, seed=3)
    ds = DeviceStep(w)
    plan = pa.pa_plan_batch(other.query_start, other.context_lens, 8, 2, 128, 16, other.block_tables.shape[1])
    with pytest.raises(pa.PAError) as e:
        pa.pa_prefill_chunk_planned(ds.out, ds.q, ds.query_start, ds.k_cache, ds.v_cache, ds.block_tables,
                                    ds.context_lens, w.scale, ds.workspace, plan, ds.status)
    assert e.value.code == pa._binding.PA_ERR_SHAPE
