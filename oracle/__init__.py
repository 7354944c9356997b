"""fp64 CPU oracle for attention over a paged KV cache.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product package never imports it, and it imports nothing from
the product package: the two share no code.  Inputs reach both sides from the
seeded generators in ``paged_kv_cache_445_b200.workloads``, which hold no
attention arithmetic.

Two independent restatements live here:

* ``pa_oracle.c`` (loaded through ctypes) -- the paged definition in fp64:
  gather K/V through the block table, scores, max-subtracted softmax, PV.
* ``brute.py`` -- the contiguous numpy form of the same attention, used only to
  pin the paged oracle on tiny inputs.

Sources ("Inference optimization", AI Engineering from Scratch, Phase 10 / 12,
sections "KV cache", "Paged attention", "Build it -- Step 1" and "Step 2";
"vLLM serving internals", Phase 17 / 04, "PagedAttention as a virtual memory
system").  Every pinned function is listed in ``PINS`` below with the tests
that pin it; nothing here is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_lock = threading.Lock()
_lib = None

# function -> tests that pin it to the pages or to mathematics (see tests/test_oracle_pins.py)
PINS = {
    "paged_attention": [
        "test_golden_powers_of_two", "test_paged_equals_contiguous_brute",
        "test_block_permutation_invariance", "test_identical_keys_give_mean_of_v",
        "test_scale_zero_gives_mean_of_v", "test_single_token_returns_its_v_row",
        "test_dominant_key_selects_its_v_row", "test_gqa_equals_repeated_mha",
        "test_causal_chunk_from_zero_equals_textbook_sdpa", "test_chunk_split_invariance",
        "test_decode_row_equals_prefill_row", "test_shared_prefix_equals_private_copy",
        "test_empty_context_gives_zeros", "test_sampled_rows_equal_full_rows",
        "test_mutations_are_caught",
    ],
    "cache_append": ["test_append_is_a_byte_copy", "test_append_then_attend_reads_new_row"],
    "slot_mapping": ["test_slot_mapping_closed_form", "test_allocator_slots_match_oracle"],
    "e4m3_to_f64": ["test_e4m3_values_from_the_definition", "test_fp8_mutations_are_caught"],
    "f32_to_e4m3": ["test_e4m3_round_trip_and_monotone", "test_e4m3_ties_to_even_and_saturation",
                    "test_fp8_mutations_are_caught"],
    "cache_append_fp8": ["test_fp8_append_writes_codes_of_the_scaled_rows", "test_fp8_mutations_are_caught"],
    "paged_attention_fp8": ["test_fp8_attention_equals_bf16_attention_on_exact_values",
                            "test_fp8_scales_factor_out", "test_fp8_mutations_are_caught"],
}


def build(force: bool = False, mutation: int = 0) -> str:
    """Compile ``pa_oracle.c`` with gcc (-O2, OpenMP, no fast-math).

    ``mutation`` > 0 builds a deliberately broken variant used only by the
    test that checks the pins catch plausible mistakes.
    """
    os.makedirs(_BUILD, exist_ok=True)
    out = _LIB_PATH if mutation == 0 else os.path.join(_BUILD, f"liboracle_m{mutation}.so")
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", "-o", out + ".tmp", _SRC, "-lm"]
        if mutation:
            cmd.insert(1, f"-DORACLE_MUTATION={mutation}")
        subprocess.check_call(cmd)
        os.replace(out + ".tmp", out)
    return out


def _bind(lib):
    i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
    u16p = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
    f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
    ci = ctypes.c_int
    lib.oracle_slot_mapping.argtypes = [i32p, i32p, ci, i32p, i32p, ci, ci, ci]
    lib.oracle_slot_mapping.restype = ci
    lib.oracle_cache_append.argtypes = [u16p, u16p, u16p, u16p, i32p, ci, ci, ci, ci, ci]
    lib.oracle_cache_append.restype = ci
    lib.oracle_paged_attention.argtypes = [
        f64p, u16p, u16p, u16p, i32p, ci, i32p, i32p, ci, ci, ci, ci, ci, ci,
        ctypes.c_double, ctypes.c_void_p, ci]
    lib.oracle_paged_attention.restype = ci
    u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
    lib.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_to_f64.restype = ctypes.c_double
    lib.oracle_f32_to_e4m3.argtypes = [ctypes.c_float]
    lib.oracle_f32_to_e4m3.restype = ctypes.c_uint8
    lib.oracle_cache_append_fp8.argtypes = [u16p, u16p, u8p, u8p, i32p, ci, ci, ci, ci, ci, ctypes.c_float,
                                            ctypes.c_float]
    lib.oracle_cache_append_fp8.restype = ci
    lib.oracle_paged_attention_fp8.argtypes = [
        f64p, u16p, u8p, u8p, i32p, ci, i32p, i32p, ci, ci, ci, ci, ci, ci,
        ctypes.c_double, ctypes.c_double, ctypes.c_double, ctypes.c_void_p, ci]
    lib.oracle_paged_attention_fp8.restype = ci
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = ci
    lib.oracle_set_num_threads.argtypes = [ci]
    lib.oracle_set_num_threads.restype = None
    return lib


def load(mutation: int = 0):
    """Load (building if needed) the oracle library."""
    global _lib
    with _lock:
        if mutation:
            return _bind(ctypes.CDLL(build(mutation=mutation)))
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
        return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    """Threads the OpenMP runtime gives the oracle (OMP_NUM_THREADS or all cores)."""
    return int(load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Threads for the oracle's later calls from this thread (timing only: the
    result does not depend on it)."""
    load().oracle_set_num_threads(int(n))


def slot_mapping(block_tables, context_lens, query_start, block_size, num_blocks, lib=None):
    """int32 slot of every new token: table[s][pos // bs] * bs + pos % bs."""
    lib = lib or load()
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    qs = _c(query_start, np.int32)
    out = np.full(int(qs[-1]), -1, dtype=np.int32)
    rc = lib.oracle_slot_mapping(out, bt, bt.shape[1], cl, qs, len(cl), int(block_size), int(num_blocks))
    if rc != 0:
        raise ValueError(f"oracle_slot_mapping failed: {rc}")
    return out


def cache_append(k_new, v_new, k_cache, v_cache, slot_map, lib=None):
    """In-place byte copy of new K/V rows (bf16 bits, uint16) into their slots."""
    lib = lib or load()
    assert k_cache.dtype == np.uint16 and k_cache.flags.c_contiguous
    assert v_cache.dtype == np.uint16 and v_cache.flags.c_contiguous
    nb, hkv, bs, d = k_cache.shape
    kn = _c(k_new, np.uint16)
    vn = _c(v_new, np.uint16)
    sm = _c(slot_map, np.int32)
    rc = lib.oracle_cache_append(kn, vn, k_cache, v_cache, sm, len(sm), nb, hkv, d, bs)
    if rc != 0:
        raise ValueError(f"oracle_cache_append failed: {rc}")


def paged_attention(q, k_cache, v_cache, block_tables, context_lens, query_start, scale,
                    only=None, lib=None):
    """fp64 attention of every query row (or only the (token, head) pairs in
    ``only``) over the paged cache.  ``q`` is bf16 bits [T, Hq, d]."""
    lib = lib or load()
    q = _c(q, np.uint16)
    kc = _c(k_cache, np.uint16)
    vc = _c(v_cache, np.uint16)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    qs = _c(query_start, np.int32)
    t, hq, d = q.shape
    nb, hkv, bs, d2 = kc.shape
    assert d == d2 and int(qs[-1]) == t
    out = np.zeros((t, hq, d), dtype=np.float64)
    if only is not None:
        only_arr = _c(only, np.int32).reshape(-1, 2)
        ptr, n_only = only_arr.ctypes.data, len(only_arr)
    else:
        only_arr, ptr, n_only = None, None, 0
    rc = lib.oracle_paged_attention(out, q, kc, vc, bt, bt.shape[1], cl, qs, len(cl), hq, hkv, d,
                                    bs, nb, float(scale), ptr, n_only)
    if rc != 0:
        raise ValueError(f"oracle_paged_attention failed: {rc}")
    return out


def e4m3_to_f64(codes, lib=None) -> np.ndarray:
    """Values of E4M3 codes (OCP 8-bit float, "FN" variant)."""
    lib = lib or load()
    c = np.asarray(codes, dtype=np.uint8)
    return np.array([lib.oracle_e4m3_to_f64(int(x)) for x in c.ravel()], dtype=np.float64).reshape(c.shape)


def f32_to_e4m3(x, lib=None) -> np.ndarray:
    """E4M3 codes of binary32 values: round to nearest-even, saturate to +-448."""
    lib = lib or load()
    a = np.asarray(x, dtype=np.float32)
    return np.array([lib.oracle_f32_to_e4m3(float(v)) for v in a.ravel()], dtype=np.uint8).reshape(a.shape)


def inv_scale(scale: float) -> float:
    """The binary32 reciprocal the append multiplies by: fl32(1 / fl32(scale))."""
    return float(np.float32(1.0) / np.float32(scale))


def cache_append_fp8(k_new, v_new, k_cache, v_cache, slot_map, k_scale, v_scale, lib=None):
    """In-place E4M3 append: code = E4M3(bf16 value * fl32(1 / scale)), product in binary32."""
    lib = lib or load()
    assert k_cache.dtype == np.uint8 and k_cache.flags.c_contiguous
    assert v_cache.dtype == np.uint8 and v_cache.flags.c_contiguous
    nb, hkv, bs, d = k_cache.shape
    kn = _c(k_new, np.uint16)
    vn = _c(v_new, np.uint16)
    sm = _c(slot_map, np.int32)
    rc = lib.oracle_cache_append_fp8(kn, vn, k_cache, v_cache, sm, len(sm), nb, hkv, d, bs,
                                     inv_scale(k_scale), inv_scale(v_scale))
    if rc != 0:
        raise ValueError(f"oracle_cache_append_fp8 failed: {rc}")


def paged_attention_fp8(q, k_cache, v_cache, block_tables, context_lens, query_start, scale, k_scale, v_scale,
                        only=None, lib=None):
    """paged_attention over E4M3 caches (uint8 codes) with per-tensor scales."""
    lib = lib or load()
    q = _c(q, np.uint16)
    kc = _c(k_cache, np.uint8)
    vc = _c(v_cache, np.uint8)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    qs = _c(query_start, np.int32)
    t, hq, d = q.shape
    nb, hkv, bs, d2 = kc.shape
    assert d == d2 and int(qs[-1]) == t
    out = np.zeros((t, hq, d), dtype=np.float64)
    if only is not None:
        only_arr = _c(only, np.int32).reshape(-1, 2)
        ptr, n_only = only_arr.ctypes.data, len(only_arr)
    else:
        only_arr, ptr, n_only = None, None, 0
    rc = lib.oracle_paged_attention_fp8(out, q, kc, vc, bt, bt.shape[1], cl, qs, len(cl), hq, hkv, d, bs, nb,
                                        float(scale), float(k_scale), float(v_scale), ptr, n_only)
    if rc != 0:
        raise ValueError(f"oracle_paged_attention_fp8 failed: {rc}")
    return out


def decode_query_start(num_seqs: int) -> np.ndarray:
    """query_start for a pure decode batch: one query row per sequence."""
    return np.arange(num_seqs + 1, dtype=np.int32)
