"""The C-ABI library loads and exports every entry point of include/pa.h;
host-side argument checks answer without touching a GPU (CPU only)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from paged_kv_cache_445_b200.csrc import build as pabuild

HEADER = os.path.join(pabuild.ROOT, "include", "pa.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*PA_API\s+(?:const\s+)?[a-z_0-9]+\s*\*?\s*(pa_[a-z_0-9]+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    path = pabuild.build()
    lib = ctypes.CDLL(path)
    return lib


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("pa_cache_append", "pa_decode", "pa_prefill_chunk", "pa_workspace_bytes", "pa_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_only_the_boundary_is_exported():
    out = os.popen(f"nm -D --defined-only {pabuild.LIB}").read()
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert {n for n in exported if n.startswith("pa_")} == set(declared_functions())


def test_status_strings(lib):
    lib.pa_status_string.restype = ctypes.c_char_p
    for code in range(0, -8, -1):
        s = lib.pa_status_string(code).decode()
        assert s.startswith("PA_") or code == 0
    assert lib.pa_status_string(0).decode() == "PA_OK"
    assert b"unknown" in lib.pa_status_string(42)


def test_host_checks_answer_before_any_launch(lib):
    vp = ctypes.c_void_p
    lib.pa_decode.argtypes = [vp, vp, vp, vp, vp, ctypes.c_int, vp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                              ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float, vp, ctypes.c_size_t, vp, vp]
    fake = 4096
    # null output
    assert lib.pa_decode(None, fake, fake, fake, fake, 4, fake, 4, 8, 2, 128, 16, 10, 0.1, fake, 1 << 20, None,
                         None) == -1
    # Hq not a multiple of Hkv
    assert lib.pa_decode(fake, fake, fake, fake, fake, 4, fake, 4, 6, 4, 128, 16, 10, 0.1, fake, 1 << 20, None,
                         None) == -2
    # unsupported head_dim and block_size
    assert lib.pa_decode(fake, fake, fake, fake, fake, 4, fake, 4, 8, 2, 96, 16, 10, 0.1, fake, 1 << 20, None,
                         None) == -3
    assert lib.pa_decode(fake, fake, fake, fake, fake, 4, fake, 4, 8, 2, 128, 8, 10, 0.1, fake, 1 << 20, None,
                         None) == -3
    # group too wide for head_dim 256
    assert lib.pa_decode(fake, fake, fake, fake, fake, 4, fake, 4, 16, 1, 256, 16, 10, 0.1, fake, 1 << 20, None,
                         None) == -3
    lib.pa_cache_append.argtypes = [vp, vp, vp, vp, vp] + [ctypes.c_int] * 5 + [vp, vp]
    assert lib.pa_cache_append(fake, fake, fake, fake, fake, 0, 4, 2, 128, 16, None, None) == 0  # nothing to do
    assert lib.pa_cache_append(fake, fake, fake, fake, fake, 3, 4, 2, 100, 16, None, None) == -3
    assert lib.pa_cache_append(None, fake, fake, fake, fake, 3, 4, 2, 128, 16, None, None) == -1
    lib.pa_workspace_bytes.restype = ctypes.c_size_t
    lib.pa_workspace_bytes.argtypes = [ctypes.c_int] * 6
    assert lib.pa_workspace_bytes(4, 6, 4, 128, 8, 16) == 0  # bad group -> 0
    assert lib.pa_workspace_bytes(4, 8, 4, 128, 8, 24) == 0  # bad block size -> 0


def test_python_binding_imports_on_cpu():
    import paged_kv_cache_445_b200 as pa
    assert pa.pa_status_string(-4).startswith("PA_ERR_WORKSPACE")
    assert pa.status_bit(-5) == 32


def test_static_scratch_size_matches_the_header():
    from paged_kv_cache_445_b200 import _binding
    m = re.search(r"#define\s+PA_STATIC_SCRATCH_BYTES\s+\((\d+)u\s*\*\s*(\d+)u\s*\*\s*(\d+)u\)", open(HEADER).read())
    assert m, "PA_STATIC_SCRATCH_BYTES not found"
    assert int(m.group(1)) * int(m.group(2)) * int(m.group(3)) == _binding.STATIC_SCRATCH_BYTES


def test_every_entry_point_rejects_bad_arguments_before_touching_a_device():
    # each case returns from the host checks, before any CUDA call (this machine may have no GPU)
    from paged_kv_cache_445_b200 import _binding as b
    L, f, odd = b._lib, 4096, 4098  # f: a 16-byte aligned stand-in pointer; odd: a misaligned one

    def decode(out=f, q=f, ws=f, seqs=4, d=128):
        return L.pa_decode(out, q, f, f, f, 4, f, seqs, 8, 2, d, 16, 10, 0.1, ws, 1 << 20, None, None)
    assert decode(seqs=0) == b.PA_OK                       # empty batch: nothing to do
    assert decode(out=odd) == b.PA_ERR_SHAPE               # misaligned output
    assert decode(ws=None) == b.PA_ERR_NULL                # no workspace

    def fused(k_new, v_new):
        return L.pa_decode_append(f, f, k_new, v_new, f, f, f, 4, f, 4, 8, 2, 128, 16, 10, 0.1, f, 1 << 20, None,
                                  None)
    assert fused(None, f) == b.PA_ERR_NULL and fused(f, None) == b.PA_ERR_NULL
    assert fused(odd, f) == b.PA_ERR_SHAPE

    def fp8(k_scale=0.5, v_scale=0.25, d=128, k_new=None, v_new=None):
        return L.pa_decode_fp8(f, f, k_new, v_new, f, f, f, 4, f, 4, 8, 2, d, 16, 10, 0.1, k_scale, v_scale, f,
                               1 << 20, None, None)
    for ks, vs in ((0.0, 0.25), (0.5, -1.0), (float("inf"), 0.25), (0.5, float("nan"))):
        assert fp8(ks, vs) == b.PA_ERR_SHAPE, (ks, vs)
    assert fp8(d=64) == b.PA_ERR_UNSUPPORTED
    assert fp8(k_new=f) == b.PA_ERR_NULL

    def app8(n=3, d=128, ks=0.5):
        return L.pa_cache_append_fp8(f, f, f, f, f, n, 10, 2, d, 16, ks, 0.25, None, None)
    assert app8(ks=0.0) == b.PA_ERR_SHAPE and app8(d=100) == b.PA_ERR_UNSUPPORTED and app8(n=0) == b.PA_OK

    def chunk(qs=f, seqs=4, total=9):
        return L.pa_prefill_chunk(f, f, qs, f, f, f, 4, f, seqs, total, 8, 2, 128, 16, 10, 0.1, f, 1 << 20, None,
                                  None)
    assert chunk(qs=None) == b.PA_ERR_NULL and chunk(total=-1) == b.PA_ERR_SHAPE and chunk(seqs=0) == b.PA_OK

    assert L.pa_decode_cascade(f, f, f, None, f, f, f, 4, f, 4, 8, 2, 128, 16, 10, 0.1, f, f, 1, f, 1 << 20, None,
                               None) == b.PA_ERR_NULL
    assert L.pa_cascade_workspace_bytes(4, 6, 4, 128, 8, 16) == 0  # Hq not a multiple of Hkv
    assert L.pa_decode_static_scratch(f, f, f, f, f, 4, f, 4, 8, 2, 96, 16, 10, 0.1, None,
                                      None) == b.PA_ERR_UNSUPPORTED
    assert L.pa_decode_static_scratch(None, f, f, f, f, 4, f, 4, 8, 2, 128, 16, 10, 0.1, None, None) == b.PA_ERR_NULL
    # an empty batch gets pa_decode's answer, errors included
    for nb, hq, d in ((10, 8, 128), (0, 8, 128), (10, 6, 128), (10, 8, 96)):
        want = L.pa_decode(f, f, f, f, f, 4, f, 0, hq, 2, d, 16, nb, 0.1, f, 1 << 20, None, None)
        got = L.pa_decode_static_scratch(f, f, f, f, f, 4, f, 0, hq, 2, d, 16, nb, 0.1, None, None)
        assert got == want, (nb, hq, d, got, want)
    assert L.pa_decode_static_scratch(f, f, f, f, f, 4, f, 0, 8, 2, 128, 16, 0, 0.1, None, None) == b.PA_ERR_SHAPE


def test_oracle_and_product_share_no_code():
    # the oracle imports nothing of the product package, the product nothing of the oracle, and the
    # oracle's C file includes no header of the CUDA library
    import ast
    import glob
    root = pabuild.ROOT

    def imports(path):
        names = set()
        for node in ast.walk(ast.parse(open(path).read())):
            if isinstance(node, ast.Import):
                names |= {a.name.split(".")[0] for a in node.names}
            elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
                names.add(node.module.split(".")[0])
            elif isinstance(node, ast.ImportFrom) and node.level > 0:
                names.add(".")
        return names
    for path in glob.glob(os.path.join(root, "oracle", "*.py")):
        assert "paged_kv_cache_445_b200" not in imports(path), path
    for path in glob.glob(os.path.join(root, "paged_kv_cache_445_b200", "**", "*.py"), recursive=True):
        assert "oracle" not in imports(path), path
    c_src = open(os.path.join(root, "oracle", "pa_oracle.c")).read()
    included = re.findall(r'#include\s+[<"]([^>"]+)[>"]', c_src)
    assert included and all(not h.startswith("pa") for h in included), included
    for path in glob.glob(os.path.join(root, "paged_kv_cache_445_b200", "csrc", "*")):
        if path.endswith((".cu", ".cuh", ".h")):
            assert "pa_oracle" not in open(path).read(), path


def test_a_missing_library_fails_loudly(tmp_path):
    # the package without libpa.so: touching any entry point raises, there is no fallback
    import shutil
    import subprocess
    import sys
    pkg = os.path.join(pabuild.ROOT, "paged_kv_cache_445_b200")
    dst = tmp_path / "paged_kv_cache_445_b200"
    dst.mkdir()
    for name in os.listdir(pkg):
        if name.endswith(".py"):
            shutil.copy(os.path.join(pkg, name), dst / name)
    code = ("import paged_kv_cache_445_b200 as pa\n"
            "try:\n    pa.pa_decode\nexcept ImportError as e:\n    print('raised:', e)\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=tmp_path, capture_output=True, text=True, timeout=300,
                       env={**os.environ, "PYTHONPATH": str(tmp_path)})
    assert r.returncode == 0, r.stderr
    assert "raised:" in r.stdout and "no CPU fallback" in r.stdout


def test_plan_rejects_bad_arguments_before_touching_a_device():
    import ctypes as C
    from paged_kv_cache_445_b200 import _binding as b
    qs = (C.c_int32 * 3)(0, 5, 6)
    cl = (C.c_int32 * 2)(40, 7)
    plan = b.Plan()
    L = b._lib
    assert L.pa_plan_batch(None, cl, 2, 8, 2, 128, 16, 8, C.byref(plan)) == b.PA_ERR_NULL
    assert L.pa_plan_batch(qs, cl, 2, 8, 2, 128, 16, 8, None) == b.PA_ERR_NULL
    assert L.pa_plan_batch(qs, cl, 2, 6, 4, 128, 16, 8, C.byref(plan)) == b.PA_ERR_SHAPE       # Hq % Hkv
    assert L.pa_plan_batch(qs, cl, 2, 8, 2, 96, 16, 8, C.byref(plan)) == b.PA_ERR_UNSUPPORTED  # head_dim
    assert L.pa_plan_batch(qs, cl, 2, 8, 2, 128, 24, 8, C.byref(plan)) == b.PA_ERR_UNSUPPORTED  # block size
    bad = (C.c_int32 * 3)(1, 5, 6)  # query_start must start at 0
    assert L.pa_plan_batch(bad, cl, 2, 8, 2, 128, 16, 8, C.byref(plan)) == b.PA_ERR_SHAPE
    assert L.pa_prefill_chunk_planned(4096, 4096, None, 4096, 4096, 4096, 4, 4096, 2, 6, 8, 2, 128, 16, 10, 0.1,
                                      4096, 1 << 20, C.byref(plan), None, None) == b.PA_ERR_NULL


def test_calibrate_rejects_bad_arguments_before_touching_a_device():
    from paged_kv_cache_445_b200 import _binding as b
    L = b._lib
    assert L.pa_calibrate(None, 1 << 31, None, None) == b.PA_ERR_NULL
    assert L.pa_calibrate(4096 + 16, 1 << 31, None, None) == b.PA_ERR_SHAPE  # not 256-byte aligned


def test_fp8_varlen_rejects_bad_arguments_before_touching_a_device():
    from paged_kv_cache_445_b200 import _binding as b
    L, f = b._lib, 4096

    def call(qs=f, d=128, ks=0.5):
        return L.pa_prefill_chunk_fp8(f, f, qs, f, f, f, 4, f, 2, 6, 8, 2, d, 16, 10, 0.1, ks, 0.25, f, 1 << 20,
                                      None, None)
    assert call(qs=None) == b.PA_ERR_NULL
    assert call(d=64) == b.PA_ERR_UNSUPPORTED
    assert call(ks=0.0) == b.PA_ERR_SHAPE
