"""Pins of the fp64 oracle to the pages and to mathematics (CPU only).

Each ``pin_*`` function raises AssertionError when the oracle library it is
given disagrees with a closed form, a brute-force restatement, an invariance
or a value printed on the pages.  The tests run every pin on the real oracle;
``test_mutations_are_caught`` rebuilds the oracle with one planted mistake at a
time and checks that at least one pin fails for each.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle
from oracle import brute
from paged_kv_cache_445_b200 import workloads
from tests.paging_helpers import rand_bf16, scatter_to_pool, to_bf16

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _attend(lib, q, kc, vc, bt, cl, qs, scale):
    return oracle.paged_attention(q, kc, vc, bt, cl, qs, scale, lib=lib)


def _contiguous_case(rng, lens, qlens, hq, hkv, d, bs, extra_blocks=3, std=1.0):
    k_seqs = [rand_bf16(rng, (n, hkv, d)) for n in lens]
    v_seqs = [rand_bf16(rng, (n, hkv, d)) for n in lens]
    q = rand_bf16(rng, (sum(qlens), hq, d), std)
    nb = sum(-(-n // bs) for n in lens) + extra_blocks
    return k_seqs, v_seqs, q, nb


def _brute_all(q, k_seqs, v_seqs, qlens, hq, scale):
    rows, t = [], 0
    for ks, vs, ql in zip(k_seqs, v_seqs, qlens):
        rows.append(brute.contiguous_attention(brute.bf16_bits_to_f64(q[t:t + ql]), brute.bf16_bits_to_f64(ks),
                                               brute.bf16_bits_to_f64(vs), hq, scale))
        t += ql
    return np.concatenate(rows, axis=0)


# --------------------------------------------------------------------------- pins

def pin_golden_powers_of_two(lib):
    g = json.load(open(os.path.join(GOLDEN, "powers_of_two_softmax.json")))
    d = g["head_dim"]
    keys = to_bf16(g["keys"]).reshape(3, 1, d)
    vals = to_bf16(g["values"]).reshape(3, 1, d)
    kc, vc, bt = scatter_to_pool([keys], [vals], 2, 5, [4, 1, 3, 0, 2])
    q1 = to_bf16([[g["q_head0"], g["q_head1"]]])  # [1, 2 heads, d]
    out = _attend(lib, q1, kc, vc, bt, np.array([3]), np.array([0, 1]), g["scale"])
    np.testing.assert_allclose(out[0, 0], g["decode_head0"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(out[0, 1], g["decode_head1"], rtol=0, atol=1e-12)
    q2 = np.concatenate([q1, q1], axis=0)
    out = _attend(lib, q2, kc, vc, bt, np.array([3]), np.array([0, 2]), g["scale"])
    for r in range(2):
        for h in range(2):
            np.testing.assert_allclose(out[r, h], g[f"chunk_row{r}_head{h}"], rtol=0, atol=1e-12)


def pin_paged_equals_contiguous_brute(lib):
    rng = np.random.default_rng(7)
    cases = [  # lens, qlens, hq, hkv, d, bs
        ([5, 17, 33, 64], [1, 1, 1, 1], 2, 1, 64, 16),
        ([1, 16, 31, 48, 50], [1, 3, 16, 1, 50], 8, 2, 16, 16),
        ([70, 3], [9, 3], 6, 3, 8, 32),
        ([40], [40], 4, 4, 8, 8),
    ]
    for lens, qlens, hq, hkv, d, bs in cases:
        k_seqs, v_seqs, q, nb = _contiguous_case(rng, lens, qlens, hq, hkv, d, bs)
        kc, vc, bt = scatter_to_pool(k_seqs, v_seqs, bs, nb, rng.permutation(nb))
        qs = np.concatenate([[0], np.cumsum(qlens)])
        scale = 1.0 / math.sqrt(d)
        got = _attend(lib, q, kc, vc, bt, np.array(lens), qs, scale)
        want = _brute_all(q, k_seqs, v_seqs, qlens, hq, scale)
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-10)


def pin_block_permutation_invariance(lib):
    rng = np.random.default_rng(11)
    lens, qlens, hq, hkv, d, bs = [37, 80, 16], [1, 5, 1], 4, 2, 32, 16
    k_seqs, v_seqs, q, nb = _contiguous_case(rng, lens, qlens, hq, hkv, d, bs, extra_blocks=6)
    qs = np.concatenate([[0], np.cumsum(qlens)])
    outs = []
    for trial in range(3):
        kc, vc, bt = scatter_to_pool(k_seqs, v_seqs, bs, nb, rng.permutation(nb))
        outs.append(_attend(lib, q, kc, vc, bt, np.array(lens), qs, 0.2))
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def pin_identical_keys_give_mean_of_v(lib):
    rng = np.random.default_rng(3)
    n, hkv, d = 45, 2, 16
    k = np.repeat(rand_bf16(rng, (1, hkv, d)), n, axis=0)
    v = rand_bf16(rng, (n, hkv, d))
    kc, vc, bt = scatter_to_pool([k], [v], 16, 4, [2, 0, 3, 1])
    q = rand_bf16(rng, (1, 4, d))
    out = _attend(lib, q, kc, vc, bt, np.array([n]), np.array([0, 1]), 0.7)
    vf = brute.bf16_bits_to_f64(v)
    for h in range(4):
        np.testing.assert_allclose(out[0, h], vf[:, h // 2].mean(axis=0), rtol=0, atol=1e-12)


def pin_scale_zero_gives_mean_of_v(lib):
    rng = np.random.default_rng(4)
    n, d = 29, 8
    k, v = rand_bf16(rng, (n, 1, d)), rand_bf16(rng, (n, 1, d))
    kc, vc, bt = scatter_to_pool([k], [v], 8, 5, [4, 2, 0, 1, 3])
    q = rand_bf16(rng, (1, 1, d))
    out = _attend(lib, q, kc, vc, bt, np.array([n]), np.array([0, 1]), 0.0)
    np.testing.assert_allclose(out[0, 0], brute.bf16_bits_to_f64(v)[:, 0].mean(axis=0), rtol=0, atol=1e-12)


def pin_single_token_returns_its_v_row(lib):
    rng = np.random.default_rng(5)
    d = 64
    k, v = rand_bf16(rng, (1, 1, d)), rand_bf16(rng, (1, 1, d))
    kc, vc, bt = scatter_to_pool([k], [v], 16, 3, [2, 0, 1])
    q = rand_bf16(rng, (1, 2, d))
    out = _attend(lib, q, kc, vc, bt, np.array([1]), np.array([0, 1]), 0.125)
    for h in range(2):
        assert np.array_equal(out[0, h], brute.bf16_bits_to_f64(v)[0, 0])


def pin_dominant_key_selects_its_v_row(lib):
    rng = np.random.default_rng(6)
    n, d, star = 40, 64, 23
    k, v = rand_bf16(rng, (n, 1, d)), rand_bf16(rng, (n, 1, d))
    q = k[star:star + 1].reshape(1, 1, d)
    kc, vc, bt = scatter_to_pool([k], [v], 16, 3, [1, 2, 0])
    out = _attend(lib, q, kc, vc, bt, np.array([n]), np.array([0, 1]), 50.0)
    np.testing.assert_allclose(out[0, 0], brute.bf16_bits_to_f64(v)[star, 0], rtol=0, atol=1e-12)


def pin_gqa_equals_repeated_mha(lib):
    rng = np.random.default_rng(8)
    lens, hq, hkv, d, bs = [21, 50], 6, 2, 16, 16
    k_seqs = [rand_bf16(rng, (n, hkv, d)) for n in lens]
    v_seqs = [rand_bf16(rng, (n, hkv, d)) for n in lens]
    q = rand_bf16(rng, (2, hq, d))
    nb = 8
    perm = rng.permutation(nb)
    kc, vc, bt = scatter_to_pool(k_seqs, v_seqs, bs, nb, perm)
    gqa = _attend(lib, q, kc, vc, bt, np.array(lens), np.array([0, 1, 2]), 0.25)
    rep = [0, 0, 0, 1, 1, 1]
    kc2, vc2, bt2 = scatter_to_pool([k[:, rep] for k in k_seqs], [v[:, rep] for v in v_seqs], bs, nb, perm)
    mha = _attend(lib, q, kc2, vc2, bt2, np.array(lens), np.array([0, 1, 2]), 0.25)
    assert np.array_equal(gqa, mha)


def pin_causal_chunk_from_zero_equals_textbook_sdpa(lib):
    rng = np.random.default_rng(9)
    n, hq, d = 37, 2, 16
    k, v = rand_bf16(rng, (n, 1, d)), rand_bf16(rng, (n, 1, d))
    q = rand_bf16(rng, (n, hq, d))
    kc, vc, bt = scatter_to_pool([k], [v], 8, 6, [5, 3, 1, 0, 4, 2])
    out = _attend(lib, q, kc, vc, bt, np.array([n]), np.array([0, n]), 0.3)
    qf, kf, vf = (brute.bf16_bits_to_f64(x) for x in (q, k, v))
    for h in range(hq):  # the textbook lower-triangular causal softmax, written out here
        s = (qf[:, h] @ kf[:, 0].T) * 0.3
        s[np.triu_indices(n, 1)] = -np.inf
        w = np.exp(s - s.max(axis=1, keepdims=True))
        np.testing.assert_allclose(out[:, h], (w / w.sum(axis=1, keepdims=True)) @ vf[:, 0], rtol=0, atol=1e-12)


def pin_chunk_split_invariance(lib):
    rng = np.random.default_rng(10)
    n, hq, hkv, d, bs = 53, 4, 2, 16, 16
    k, v = rand_bf16(rng, (n, hkv, d)), rand_bf16(rng, (n, hkv, d))
    q = rand_bf16(rng, (n, hq, d))
    kc, vc, bt = scatter_to_pool([k], [v], bs, 6, rng.permutation(6))
    whole = _attend(lib, q, kc, vc, bt, np.array([n]), np.array([0, n]), 0.25)
    pieces, start = [], 0
    for end in (7, 8, 40, 53):  # chunks of 7, 1, 32, 13 rows at growing context
        pieces.append(_attend(lib, q[start:end], kc, vc, bt, np.array([end]), np.array([0, end - start]), 0.25))
        start = end
    assert np.array_equal(np.concatenate(pieces), whole)


def pin_decode_row_equals_prefill_row(lib):
    rng = np.random.default_rng(12)
    n, hq, hkv, d, bs = 33, 4, 1, 32, 16
    k, v = rand_bf16(rng, (n, hkv, d)), rand_bf16(rng, (n, hkv, d))
    q = rand_bf16(rng, (9, hq, d))
    kc, vc, bt = scatter_to_pool([k], [v], bs, 4, [3, 1, 0, 2])
    chunk = _attend(lib, q, kc, vc, bt, np.array([n]), np.array([0, 9]), 0.2)
    dec = _attend(lib, q[-1:], kc, vc, bt, np.array([n]), np.array([0, 1]), 0.2)
    assert np.array_equal(dec[0], chunk[-1])


def pin_shared_prefix_equals_private_copy(lib):
    rng = np.random.default_rng(13)
    hq, hkv, d, bs, pre = 4, 2, 16, 8, 24
    prefix_k, prefix_v = rand_bf16(rng, (pre, hkv, d)), rand_bf16(rng, (pre, hkv, d))
    tails = [5, 0, 11]
    tk = [rand_bf16(rng, (t, hkv, d)) for t in tails]
    tv = [rand_bf16(rng, (t, hkv, d)) for t in tails]
    q = rand_bf16(rng, (3, hq, d))
    lens = np.array([pre + t for t in tails])
    # private copies
    kc, vc, bt = scatter_to_pool([np.concatenate([prefix_k, a]) for a in tk],
                                 [np.concatenate([prefix_v, a]) for a in tv], bs, 20, rng.permutation(20))
    private = _attend(lib, q, kc, vc, bt, lens, np.arange(4), 0.25)
    # one stored prefix: the three tables share its 3 blocks
    kc2, vc2, bt_prefix = scatter_to_pool([prefix_k] + tk, [prefix_v] + tv, bs, 20, rng.permutation(20))
    bt2 = np.full((3, 5), -1, dtype=np.int32)
    for s in range(3):
        bt2[s, :3] = bt_prefix[0, :3]
        nt = -(-tails[s] // bs)
        bt2[s, 3:3 + nt] = bt_prefix[1 + s, :nt]
    shared = _attend(lib, q, kc2, vc2, bt2, lens, np.arange(4), 0.25)
    assert np.array_equal(shared, private)


def pin_empty_context_gives_zeros(lib):
    rng = np.random.default_rng(14)
    kc = rand_bf16(rng, (2, 1, 16, 8))
    vc = rand_bf16(rng, (2, 1, 16, 8))
    q = rand_bf16(rng, (2, 2, 8))
    bt = np.array([[0], [1]], dtype=np.int32)
    out = _attend(lib, q, kc, vc, bt, np.array([0, 3]), np.arange(3), 0.3)
    assert np.all(out[0] == 0) and np.all(np.isfinite(out[1])) and np.any(out[1] != 0)


def pin_append_is_a_byte_copy(lib):
    rng = np.random.default_rng(15)
    nb, hkv, bs, d, t = 7, 3, 16, 8, 10
    kc = np.full((nb, hkv, bs, d), 0xABCD, dtype=np.uint16)
    vc = np.full((nb, hkv, bs, d), 0x1234, dtype=np.uint16)
    kn, vn = rand_bf16(rng, (t, hkv, d)), rand_bf16(rng, (t, hkv, d))
    slots = rng.choice(nb * bs, size=t, replace=False).astype(np.int32)
    slots[[2, 7]] = -1
    k2, v2 = kc.copy(), vc.copy()
    oracle.cache_append(kn, vn, k2, v2, slots, lib=lib)
    kk, vv = kc.copy(), vc.copy()
    for i, s in enumerate(slots):  # written out independently
        if s >= 0:
            kk[s // bs, :, s % bs, :] = kn[i]
            vv[s // bs, :, s % bs, :] = vn[i]
    assert np.array_equal(k2, kk) and np.array_equal(v2, vv)


def pin_append_then_attend_reads_new_row(lib):
    rng = np.random.default_rng(16)
    hq, hkv, d, bs, n = 4, 2, 16, 16, 32  # the new token starts a fresh block
    k, v = rand_bf16(rng, (n, hkv, d)), rand_bf16(rng, (n, hkv, d))
    kc, vc, bt = scatter_to_pool([k], [v], bs, 5, [4, 0, 2, 1, 3])
    bt = np.array([[4, 0, 2]], dtype=np.int32)  # block 2 receives token n
    kn, vn = rand_bf16(rng, (1, hkv, d)), rand_bf16(rng, (1, hkv, d))
    slots = oracle.slot_mapping(bt, np.array([n + 1]), np.array([0, 1]), bs, 5, lib=lib)
    assert slots[0] == 2 * bs + 0
    oracle.cache_append(kn, vn, kc, vc, slots, lib=lib)
    q = rand_bf16(rng, (1, hq, d))
    out = _attend(lib, q, kc, vc, bt, np.array([n + 1]), np.array([0, 1]), 0.25)
    want = brute.contiguous_attention(brute.bf16_bits_to_f64(q), brute.bf16_bits_to_f64(np.concatenate([k, kn])),
                                      brute.bf16_bits_to_f64(np.concatenate([v, vn])), hq, 0.25)
    np.testing.assert_allclose(out, want, rtol=0, atol=1e-12)


def pin_slot_mapping_closed_form(lib):
    # two sequences, block size 4; tables written by hand
    bt = np.array([[9, 2, 5], [7, 0, -1]], dtype=np.int32)
    cl = np.array([10, 6])
    qs = np.array([0, 3, 5])  # seq 0 appends positions 7, 8, 9; seq 1 positions 4, 5
    got = oracle.slot_mapping(bt, cl, qs, 4, 10, lib=lib)
    assert got.tolist() == [2 * 4 + 3, 5 * 4 + 0, 5 * 4 + 1, 0 * 4 + 0, 0 * 4 + 1]


def pin_sampled_rows_equal_full_rows(lib):
    rng = np.random.default_rng(17)
    lens, qlens, hq, hkv, d, bs = [90, 33, 7], [20, 1, 3], 8, 2, 16, 16
    k_seqs, v_seqs, q, nb = _contiguous_case(rng, lens, qlens, hq, hkv, d, bs)
    kc, vc, bt = scatter_to_pool(k_seqs, v_seqs, bs, nb, rng.permutation(nb))
    qs = np.concatenate([[0], np.cumsum(qlens)])
    full = _attend(lib, q, kc, vc, bt, np.array(lens), qs, 0.3)
    only = [(t, h) for t in (0, 5, 19, 20, 22) for h in (0, 3, 3, 7, 0)]  # with duplicates
    part = oracle.paged_attention(q, kc, vc, bt, np.array(lens), qs, 0.3, only=np.array(only * 3), lib=lib)
    for t, h in only:
        assert np.array_equal(part[t, h], full[t, h])


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]


# --------------------------------------------------------------------------- tests

@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__[4:])
def test_pin(pin):
    pin(oracle.load())


def test_allocator_slots_match_oracle():
    for cfg in (1,):
        w = workloads.standard(cfg)
        got = oracle.slot_mapping(w.block_tables, w.context_lens, w.query_start, w.block_size, w.num_blocks)
        assert np.array_equal(got, w.slot_mapping)
    w = workloads.custom([16384 // 64, 100, 0, 31], [512 // 64, 1, 3, 1], 8, 2, 16, 16, seed=3)
    got = oracle.slot_mapping(w.block_tables, w.context_lens, w.query_start, w.block_size, w.num_blocks)
    assert np.array_equal(got, w.slot_mapping)


@pytest.mark.parametrize("mutation", range(1, 9))
def test_mutations_are_caught(mutation):
    lib = oracle.load(mutation=mutation)
    failed = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"mutation {mutation} passed every pin"


@settings(max_examples=40, deadline=None)
@given(st.data())
def test_paged_equals_contiguous_brute_on_random_shapes(data):
    # the brute-force pin over shapes drawn at random: lengths 1..70, rows 1..len, groups 1..4,
    # head dims 8..32, blocks of 4..32 tokens, any physical placement, NaN in every unused slot
    hkv = data.draw(st.integers(1, 3))
    hq = hkv * data.draw(st.integers(1, 4))
    d = data.draw(st.sampled_from([8, 16, 32]))
    bs = data.draw(st.sampled_from([4, 8, 16, 32]))
    lens = data.draw(st.lists(st.integers(1, 70), min_size=1, max_size=4))
    qlens = [data.draw(st.integers(1, n)) for n in lens]
    seed = data.draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    k_seqs, v_seqs, q, nb = _contiguous_case(rng, lens, qlens, hq, hkv, d, bs, extra_blocks=2)
    kc, vc, bt = scatter_to_pool(k_seqs, v_seqs, bs, nb, rng.permutation(nb))
    qs = np.concatenate([[0], np.cumsum(qlens)])
    scale = 1.0 / math.sqrt(d)
    got = _attend(oracle.load(), q, kc, vc, bt, np.array(lens), qs, scale)
    want = _brute_all(q, k_seqs, v_seqs, qlens, hq, scale)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-10)
