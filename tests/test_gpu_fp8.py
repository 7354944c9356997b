"""GPU parity of the FP8 (E4M3) cache path against the fp64 oracle.

The append must write exactly the oracle's codes (the quantisation decision is
taken in binary32 on both sides); decode over the codes must match the oracle
within the attention tolerance; the fused append + decode must equal the two
separate calls bit for bit.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_445_b200 import workloads
from tests.gpu_helpers import DeviceStep, compare, i32, load_library

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    load_library()


class Fp8Step:
    def __init__(self, w, seed, poison=True):
        self.ds = DeviceStep(w)
        kc, vc, self.k_scale, self.v_scale = workloads.fp8_caches(w, seed, poison=poison)
        self.kc_host, self.vc_host = kc, vc
        self.kc = torch.from_numpy(kc).cuda()
        self.vc = torch.from_numpy(vc).cuda()

    def append(self):
        import paged_kv_cache_445_b200 as pa
        d = self.ds
        pa.pa_cache_append_fp8(d.k_new, d.v_new, self.kc, self.vc, d.slot_mapping, self.k_scale, self.v_scale,
                               d.status)

    def decode(self, fused=False):
        import paged_kv_cache_445_b200 as pa
        d = self.ds
        pa.pa_decode_fp8(d.out, d.q, self.kc, self.vc, d.block_tables, d.context_lens, d.w.scale, self.k_scale,
                         self.v_scale, d.workspace, k_new=d.k_new if fused else None,
                         v_new=d.v_new if fused else None, dev_status=d.status)

    def oracle_caches(self):
        kc, vc = self.kc_host.copy(), self.vc_host.copy()
        w = self.ds.w
        slots = oracle.slot_mapping(w.block_tables, w.context_lens, w.query_start, w.block_size, w.num_blocks)
        oracle.cache_append_fp8(w.k_new, w.v_new, kc, vc, slots, self.k_scale, self.v_scale)
        return kc, vc


@pytest.mark.parametrize("cfg", [1, 2, 4])
def test_fp8_append_writes_the_oracles_codes(cfg):
    w = workloads.standard(cfg, poison=True)
    st = Fp8Step(w, seed=cfg)
    st.append()
    torch.cuda.synchronize()
    kc, vc = st.oracle_caches()
    assert np.array_equal(st.kc.cpu().numpy(), kc)
    assert np.array_equal(st.vc.cpu().numpy(), vc)
    assert int(st.ds.status.item()) == 0


FP8_SMALL = [  # prefix list, Hq, Hkv, d, bs
    ([0, 14, 15, 16, 40, 129, 700], 8, 1, 128, 16),
    ([30, 500, 2000], 16, 1, 128, 32),       # 16 heads per KV head: two 8-wide head tiles
    ([5, 300, 1500], 12, 2, 256, 16),
    ([32000, 24999], 16, 2, 128, 16),        # long contexts: segments split over many warps
    ([7, 31, 32, 33, 47, 300, 1000], 8, 2, 128, 32),  # 32-token blocks: both 16-row halves of a tile in one block
]


@pytest.mark.parametrize("case", FP8_SMALL, ids=lambda c: f"Hq{c[1]}-Hkv{c[2]}-d{c[3]}-bs{c[4]}-n{len(c[0])}")
def test_fp8_decode_matches_oracle(case):
    prefix, hq, hkv, d, bs = case
    w = workloads.custom(prefix, [1] * len(prefix), hq, hkv, d, bs, seed=len(prefix) + d, poison=True)
    st = Fp8Step(w, seed=7)
    st.append()
    st.decode()
    torch.cuda.synchronize()
    assert int(st.ds.status.item()) == 0
    kc, vc = st.oracle_caches()
    ref = oracle.paged_attention_fp8(w.q, kc, vc, w.block_tables, w.context_lens, w.query_start, w.scale,
                                     st.k_scale, st.v_scale)
    compare(st.ds.out.float().cpu().numpy(), ref, f"fp8 {case}")


def test_fp8_70b_layer_matches_oracle_on_every_sequence():
    w = workloads.standard(3, poison=True)
    st = Fp8Step(w, seed=3)
    st.append()
    st.decode()
    torch.cuda.synchronize()
    assert int(st.ds.status.item()) == 0
    kc, vc = st.oracle_caches()
    ref = oracle.paged_attention_fp8(w.q, kc, vc, w.block_tables, w.context_lens, w.query_start, w.scale,
                                     st.k_scale, st.v_scale)
    compare(st.ds.out.float().cpu().numpy(), ref, "fp8 70B layer, all 128 sequences")


@pytest.mark.parametrize("cfg", [2, 3])
def test_fp8_fused_append_equals_the_two_calls_bit_for_bit(cfg):
    w = workloads.standard(cfg)
    a = Fp8Step(w, seed=cfg, poison=False)
    a.append()
    a.decode()
    b = Fp8Step(w, seed=cfg, poison=False)
    b.decode(fused=True)
    torch.cuda.synchronize()
    assert int(b.ds.status.item()) == 0
    assert torch.equal(a.ds.out.view(torch.int16), b.ds.out.view(torch.int16))
    assert torch.equal(a.kc, b.kc) and torch.equal(a.vc, b.vc)


def test_fp8_rejects_what_it_does_not_support():
    import paged_kv_cache_445_b200 as pa
    w = workloads.custom([40, 60], [1, 1], 8, 2, 64, 16, seed=1)
    st = Fp8Step(w, seed=1, poison=False)
    with pytest.raises(pa.PAError) as e:
        st.decode()
    assert e.value.code == pa._binding.PA_ERR_UNSUPPORTED  # head_dim 64
    w = workloads.custom([40, 60], [1, 1], 8, 2, 128, 16, seed=1)
    st = Fp8Step(w, seed=1, poison=False)
    st.k_scale = 0.0
    with pytest.raises(pa.PAError) as e:
        st.decode()
    assert e.value.code == pa._binding.PA_ERR_SHAPE


FP8_VARLEN = [  # prefix list, qlen list, Hq, Hkv, d, bs
    ([1000, 40, 300], [130, 1, 4], 16, 2, 128, 16),     # a chunk, a decode and a 4-row verification
    ([0, 500, 17], [200, 1, 2], 8, 1, 128, 32),         # a prompt from position 0
    ([700, 33], [64, 1], 12, 2, 256, 16),               # head_dim 256
    ([64, 2000, 9], [3, 7, 1], 16, 1, 128, 16),         # G 16: two head tiles
]


@pytest.mark.parametrize("case", FP8_VARLEN, ids=lambda c: f"Hq{c[2]}-Hkv{c[3]}-d{c[4]}-q{max(c[1])}")
def test_fp8_varlen_batches_match_the_oracle(case):
    import paged_kv_cache_445_b200 as pa
    prefix, qlen, hq, hkv, d, bs = case
    w = workloads.custom(prefix, qlen, hq, hkv, d, bs, seed=sum(prefix) + d, poison=True)
    st = Fp8Step(w, seed=9)
    st.append()
    d_ = st.ds
    pa.pa_prefill_chunk_fp8(d_.out, d_.q, d_.query_start, st.kc, st.vc, d_.block_tables, d_.context_lens, w.scale,
                            st.k_scale, st.v_scale, d_.workspace, d_.status)
    torch.cuda.synchronize()
    assert int(d_.status.item()) == 0
    kc, vc = st.oracle_caches()
    ref = oracle.paged_attention_fp8(w.q, kc, vc, w.block_tables, w.context_lens, w.query_start, w.scale,
                                     st.k_scale, st.v_scale)
    compare(d_.out.float().cpu().numpy(), ref, f"fp8 varlen {case}")


def test_fp8_verify4_layer_matches_the_oracle_on_every_row():
    import paged_kv_cache_445_b200 as pa
    w = workloads.standard(6, poison=True)
    st = Fp8Step(w, seed=6)
    st.append()
    d_ = st.ds
    pa.pa_prefill_chunk_fp8(d_.out, d_.q, d_.query_start, st.kc, st.vc, d_.block_tables, d_.context_lens, w.scale,
                            st.k_scale, st.v_scale, d_.workspace, d_.status)
    torch.cuda.synchronize()
    assert int(d_.status.item()) == 0
    kc, vc = st.oracle_caches()
    ref = oracle.paged_attention_fp8(w.q, kc, vc, w.block_tables, w.context_lens, w.query_start, w.scale,
                                     st.k_scale, st.v_scale)
    compare(d_.out.float().cpu().numpy(), ref, "fp8 verify-4 layer")
