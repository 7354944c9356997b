"""Pins of the oracle's FP8 (E4M3) cache functions (CPU only).

The E4M3 format is the OCP 8-bit floating point one ("FN" variant): 1 sign
bit, 4 exponent bits with bias 7, 3 mantissa bits, no infinities, S.1111.111
is NaN.  The pins use what the format fixes (its largest and smallest values,
its value of one, its NaN codes, that it is monotone and symmetric) and
reduce FP8 attention to the already-pinned bf16 oracle on values that both
represent exactly.  Each ``pin_*`` takes the oracle library to check;
``test_fp8_mutations_are_caught`` rebuilds the oracle with one planted FP8
mistake at a time and checks that at least one pin fails for each.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from tests.paging_helpers import rand_bf16, scatter_to_pool


def _all_codes():
    return np.arange(256, dtype=np.uint8)


def pin_e4m3_values_from_the_definition(lib):
    v = oracle.e4m3_to_f64(_all_codes(), lib=lib)
    nan = np.isnan(v)
    assert nan.sum() == 2 and nan[0x7F] and nan[0xFF]            # S.1111.111 only
    assert v[0x7E] == 448.0 and v[0xFE] == -448.0                 # largest finite: 1.75 * 2^8
    assert v[0x08] == 2.0 ** -6                                   # smallest normal
    assert v[0x01] == 2.0 ** -9                                   # smallest subnormal
    assert v[0x38] == 1.0 and v[0xB8] == -1.0                     # exponent field 7 = bias
    assert v[0x00] == 0.0 and v[0x80] == 0.0 and np.signbit(v[0x80])
    pos = v[0x00:0x7F]
    assert np.all(np.diff(pos) > 0)                               # monotone in the code
    assert np.array_equal(v[0x80:0xFF], -pos)                     # sign-magnitude
    # every value is an integer multiple of 2^-9 with at most 4 significant bits
    for x in pos[1:]:
        e = np.floor(np.log2(x))
        m = x / 2.0 ** (max(e, -6) - 3)
        assert m == np.round(m) and m < 16


def pin_e4m3_round_trip_and_monotone(lib):
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = oracle.e4m3_to_f64(codes, lib=lib).astype(np.float32)
    assert np.array_equal(oracle.f32_to_e4m3(vals, lib=lib), codes)       # every finite code is its own value's code
    x = np.linspace(-500, 500, 20001, dtype=np.float32)
    q = oracle.e4m3_to_f64(oracle.f32_to_e4m3(x, lib=lib), lib=lib)
    assert np.all(np.diff(q) >= 0)                                # rounding never reorders
    finite = np.abs(x) <= 448
    vals_pos = oracle.e4m3_to_f64(np.arange(0x00, 0x7F, dtype=np.uint8), lib=lib)
    for xi, qi in zip(x[finite][::97], q[finite][::97]):         # nearest representable value
        best = np.min(np.abs(np.concatenate([vals_pos, -vals_pos]) - xi))
        assert abs(qi - xi) == best


def pin_e4m3_ties_to_even_and_saturation(lib):
    vals = oracle.e4m3_to_f64(np.arange(0x00, 0x7F, dtype=np.uint8), lib=lib)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)       # exactly representable in binary32
    codes = oracle.f32_to_e4m3(mids, lib=lib)
    # a tie goes to the even code (even mantissa bit); just off the tie to the nearer one
    assert np.all(codes % 2 == 0)
    lo = oracle.f32_to_e4m3(np.nextafter(mids, np.float32(-np.inf)))
    hi = oracle.f32_to_e4m3(np.nextafter(mids, np.float32(np.inf)))
    assert np.array_equal(lo, np.arange(0, 0x7E, dtype=np.uint8))
    assert np.array_equal(hi, np.arange(1, 0x7F, dtype=np.uint8))
    big = np.array([464.0, 465.0, 1e9, np.inf, -464.0, -1e30, -np.inf], dtype=np.float32)
    assert oracle.f32_to_e4m3(big, lib=lib).tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0xFE]
    assert oracle.f32_to_e4m3(np.array([np.nan], dtype=np.float32), lib=lib)[0] in (0x7F, 0xFF)
    tiny = np.array([2.0 ** -10, -(2.0 ** -10), 2.0 ** -11], dtype=np.float32)
    assert oracle.f32_to_e4m3(tiny, lib=lib).tolist() == [0x00, 0x80, 0x00]


def pin_fp8_append_writes_codes_of_the_scaled_rows(lib):
    rng = np.random.default_rng(3)
    nb, hkv, bs, d = 6, 2, 16, 32
    kc = np.full((nb, hkv, bs, d), 0x55, dtype=np.uint8)
    vc = np.full((nb, hkv, bs, d), 0x55, dtype=np.uint8)
    k_new = rand_bf16(rng, (3, hkv, d))
    v_new = rand_bf16(rng, (3, hkv, d))
    slots = np.array([5 * bs + 3, -1, 0 * bs + 15], dtype=np.int32)
    k_scale, v_scale = 0.0375, 3.0
    oracle.cache_append_fp8(k_new, v_new, kc, vc, slots, k_scale, v_scale, lib=lib)
    f32 = lambda bits: (bits.astype(np.uint32) << 16).view(np.float32)  # noqa: E731
    want_k = np.full_like(kc, 0x55)
    want_v = np.full_like(vc, 0x55)
    for t, slot in enumerate(slots):
        if slot < 0:
            continue
        want_k[slot // bs, :, slot % bs, :] = oracle.f32_to_e4m3(f32(k_new[t]) * np.float32(oracle.inv_scale(k_scale)),
                                                                 lib=lib)
        want_v[slot // bs, :, slot % bs, :] = oracle.f32_to_e4m3(f32(v_new[t]) * np.float32(oracle.inv_scale(v_scale)),
                                                                 lib=lib)
    assert np.array_equal(kc, want_k) and np.array_equal(vc, want_v)


def _fp8_case(rng, lens, hkv, bs, d):
    codes_k = [rng.integers(0, 0x7F, (n, hkv, d)).astype(np.uint8) | (rng.integers(0, 2, (n, hkv, d)) * 0x80).astype(np.uint8)
               for n in lens]
    codes_v = [rng.integers(0, 0x7F, (n, hkv, d)).astype(np.uint8) | (rng.integers(0, 2, (n, hkv, d)) * 0x80).astype(np.uint8)
               for n in lens]
    nb = sum(-(-n // bs) for n in lens) + 2
    perm = rng.permutation(nb)
    kc8 = np.zeros((nb, hkv, bs, d), dtype=np.uint8)
    vc8 = np.zeros((nb, hkv, bs, d), dtype=np.uint8)
    bt = np.full((len(lens), max(-(-n // bs) for n in lens)), -1, dtype=np.int32)
    nxt = 0
    for s, n in enumerate(lens):
        for j in range(n):
            if j % bs == 0:
                bt[s, j // bs] = perm[nxt]
                nxt += 1
            kc8[bt[s, j // bs], :, j % bs, :] = codes_k[s][j]
            vc8[bt[s, j // bs], :, j % bs, :] = codes_v[s][j]
    return kc8, vc8, bt, nb


def pin_fp8_attention_equals_bf16_attention_on_exact_values(lib):
    # E4M3 values times a power-of-two scale are exact in bf16: the FP8 oracle
    # must then give bit for bit what the pinned bf16 oracle gives
    rng = np.random.default_rng(8)
    lens, qlens, hq, hkv, d, bs = [40, 17, 70], [1, 5, 1], 6, 2, 32, 16
    kc8, vc8, bt, nb = _fp8_case(rng, lens, hkv, bs, d)
    k_scale, v_scale = 2.0 ** -3, 2.0 ** 2
    to_bits = lambda x: (np.asarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)  # noqa: E731
    kc16 = to_bits(oracle.e4m3_to_f64(kc8, lib=lib) * k_scale)
    vc16 = to_bits(oracle.e4m3_to_f64(vc8, lib=lib) * v_scale)
    q = rand_bf16(rng, (sum(qlens), hq, d))
    qs = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    cl = np.array(lens, dtype=np.int32)
    a = oracle.paged_attention_fp8(q, kc8, vc8, bt, cl, qs, 0.2, k_scale, v_scale, lib=lib)
    b = oracle.paged_attention(q, kc16, vc16, bt, cl, qs, 0.2, lib=lib)
    assert np.array_equal(a, b)


def pin_fp8_scales_factor_out(lib):
    rng = np.random.default_rng(9)
    lens, hq, hkv, d, bs = [33, 90], 4, 1, 16, 32
    kc8, vc8, bt, nb = _fp8_case(rng, lens, hkv, bs, d)
    q = rand_bf16(rng, (2, hq, d))
    qs = np.array([0, 1, 2], dtype=np.int32)
    cl = np.array(lens, dtype=np.int32)
    base = oracle.paged_attention_fp8(q, kc8, vc8, bt, cl, qs, 0.25, 1.0, 1.0, lib=lib)
    # the V scale multiplies the output; the K scale multiplies the softmax scale
    np.testing.assert_allclose(oracle.paged_attention_fp8(q, kc8, vc8, bt, cl, qs, 0.25, 1.0, 3.0, lib=lib), 3.0 * base,
                               rtol=1e-13, atol=0)
    np.testing.assert_allclose(oracle.paged_attention_fp8(q, kc8, vc8, bt, cl, qs, 0.25, 0.5, 1.0, lib=lib),
                               oracle.paged_attention_fp8(q, kc8, vc8, bt, cl, qs, 0.125, 1.0, 1.0, lib=lib),
                               rtol=0, atol=1e-15)


ALL_FP8_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]


def test_e4m3_values_from_the_definition():
    pin_e4m3_values_from_the_definition(oracle.load())


def test_e4m3_round_trip_and_monotone():
    pin_e4m3_round_trip_and_monotone(oracle.load())


def test_e4m3_ties_to_even_and_saturation():
    pin_e4m3_ties_to_even_and_saturation(oracle.load())


def test_fp8_append_writes_codes_of_the_scaled_rows():
    pin_fp8_append_writes_codes_of_the_scaled_rows(oracle.load())


def test_fp8_attention_equals_bf16_attention_on_exact_values():
    pin_fp8_attention_equals_bf16_attention_on_exact_values(oracle.load())


def test_fp8_scales_factor_out():
    pin_fp8_scales_factor_out(oracle.load())


@pytest.mark.parametrize("mutation", range(9, 14))
def test_fp8_mutations_are_caught(mutation):
    # 9: decode bias 8, 10: encoding rounds toward zero, 11: no saturation,
    # 12: attention without the V scale, 13: append multiplies by the scale
    lib = oracle.load(mutation=mutation)
    failed = []
    for pin in ALL_FP8_PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"mutation {mutation} passed every FP8 pin"

