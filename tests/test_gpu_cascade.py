"""GPU parity of the shared-prefix (cascade) decode path against the fp64 oracle.

pa_decode_cascade reads a group's shared prefix once for all of its sequences
and heads (tcgen05 pass), attends to each sequence's private keys in the decode
kernel and folds the two together.  The result must match the oracle within
the attention tolerance, and the fused append must leave the caches exactly as
pa_cache_append does.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_445_b200 import workloads
from tests.gpu_helpers import DeviceStep, compare, i32, load_library, oracle_after_append

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    load_library()


def _cascade(ds: DeviceStep, fused: bool):
    import paged_kv_cache_445_b200 as pa
    w = ds.w
    gs, gp = w.prefix_groups()
    ws = pa.make_cascade_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                   w.block_tables.shape[1], w.block_size, "cuda")
    if not fused:
        ds.append()
    pa.pa_decode_cascade(ds.out, ds.q, ds.k_cache, ds.v_cache, ds.block_tables, ds.context_lens, w.scale,
                         i32(gs), i32(gp), ws, k_new=ds.k_new if fused else None,
                         v_new=ds.v_new if fused else None, dev_status=ds.status)
    torch.cuda.synchronize()
    return ws


def _ref(w):
    kc, vc = oracle_after_append(w)
    return oracle.paged_attention(w.q, kc, vc, w.block_tables, w.context_lens, w.query_start, w.scale)


def test_grpo_workload_matches_oracle_and_the_two_calls():
    w = workloads.standard(4, poison=True)
    plain = DeviceStep(w)
    plain.step()
    ds = DeviceStep(w)
    _cascade(ds, fused=True)
    assert int(ds.status.item()) == 0
    got = ds.out.float().cpu().numpy()
    compare(got, _ref(w), "GRPO cascade")
    compare(got, plain.out.float().cpu().numpy().astype(np.float64), "cascade vs plain decode")
    assert torch.equal(ds.k_cache.view(torch.int16), plain.k_cache.view(torch.int16))
    assert torch.equal(ds.v_cache.view(torch.int16), plain.v_cache.view(torch.int16))


CASES = [  # prefix list, Hq, Hkv, d, bs, share groups, shared tokens
    ([2100, 2200, 2100, 2500], 24, 4, 256, 32, ((0, 1, 2, 3),), 2048),
    ([700, 900, 650, 2000, 800, 1000], 16, 2, 128, 16, ((0, 1, 2), (4, 5)), 640),        # a plain sequence between groups
    ([300, 301, 302] * 7, 64, 8, 128, 16, (tuple(range(21)),), 240),                       # G 8: 16 rows per M-tile, 2 M-tiles
    ([1000, 1030], 8, 8, 64, 16, ((0, 1),), 992),                                          # G 1, d 64, span 960 < 992
    ([400] * 9, 32, 2, 128, 32, (tuple(range(9)),), 384),                                  # G 16: 8 sequences per M-tile
    ([5000], 12, 2, 256, 16, ((0,),), 4096),                                               # a group of one, 8 slices
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"Hq{c[1]}-Hkv{c[2]}-d{c[3]}-bs{c[4]}-p{c[6]}")
@pytest.mark.parametrize("fused", [False, True])
def test_small_shared_prefix_batches_match_oracle(case, fused):
    prefix, hq, hkv, d, bs, share, tokens = case
    w = workloads.custom(prefix, [1] * len(prefix), hq, hkv, d, bs, seed=len(prefix) * 7 + d, poison=True,
                         share=share, share_tokens=tokens)
    ds = DeviceStep(w)
    _cascade(ds, fused)
    assert int(ds.status.item()) == 0
    compare(ds.out.float().cpu().numpy(), _ref(w), f"cascade {case}")


def test_cascade_is_deterministic():
    w = workloads.custom([2100, 2300, 2050, 2600, 3000], [1] * 5, 24, 4, 256, 32, seed=5,
                         share=((0, 1, 2, 3, 4),), share_tokens=2048)
    ds = DeviceStep(w)
    ds.append()
    import paged_kv_cache_445_b200 as pa
    gs, gp = w.prefix_groups()
    ws = pa.make_cascade_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                   w.block_tables.shape[1], w.block_size, "cuda")
    outs = []
    for _ in range(3):
        pa.pa_decode_cascade(ds.out, ds.q, ds.k_cache, ds.v_cache, ds.block_tables, ds.context_lens, w.scale,
                             i32(gs), i32(gp), ws, dev_status=ds.status)
        torch.cuda.synchronize()
        outs.append(ds.out.clone())
    assert int(ds.status.item()) == 0
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))


def test_cascade_reports_a_context_inside_the_shared_prefix():
    import paged_kv_cache_445_b200 as pa
    w = workloads.custom([700, 800], [1, 1], 16, 2, 128, 16, seed=9, share=((0, 1),), share_tokens=640)
    ds = DeviceStep(w)
    ds.append()
    gs, gp = w.prefix_groups()
    gp = gp.copy()
    gp[0] = 768  # claims more shared tokens than sequence 0 has (701)
    ws = pa.make_cascade_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                   w.block_tables.shape[1], w.block_size, "cuda")
    pa.pa_decode_cascade(ds.out, ds.q, ds.k_cache, ds.v_cache, ds.block_tables, ds.context_lens, w.scale,
                         i32(gs), i32(gp), ws, dev_status=ds.status)
    torch.cuda.synchronize()
    assert int(ds.status.item()) & pa.status_bit(pa._binding.PA_ERR_RANGE)


def test_long_prefix_grpo_workload_matches_oracle():
    # 8 prompts x 16 rollouts sharing 8192-token prefixes (268 MB of shared
    # KV, more than the L2 holds): every row against the oracle
    w = workloads.standard(7, poison=True)
    ds = DeviceStep(w)
    _cascade(ds, fused=True)
    assert int(ds.status.item()) == 0
    compare(ds.out.float().cpu().numpy(), _ref(w), "long-prefix GRPO cascade")
