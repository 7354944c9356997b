"""ctypes binding of libpa.so: argument marshalling only.

Every function here checks the tensors' dtype, device, contiguity and shape,
passes raw device pointers, sizes and the current CUDA stream to the C entry
point of the same name (``include/pa.h``), and raises ``PAError`` on a
non-zero status.  All computation happens in the library's kernels; if the
library is missing this module fails to import -- there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

library_path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpa.so")
if not os.path.exists(library_path):
    raise ImportError(f"{library_path} is missing: build it with `python -m paged_kv_cache_445_b200.csrc.build` "
                      "(needs nvcc); there is no CPU fallback")
_lib = ctypes.CDLL(library_path)

_vp, _ci, _i32p = ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p
_lib.pa_cache_append.argtypes = [_vp, _vp, _vp, _vp, _i32p, _ci, _ci, _ci, _ci, _ci, _vp, _vp]
_lib.pa_cache_append.restype = _ci
_lib.pa_workspace_bytes.argtypes = [_ci, _ci, _ci, _ci, _ci, _ci]
_lib.pa_workspace_bytes.restype = ctypes.c_size_t
_lib.pa_decode.argtypes = [_vp, _vp, _vp, _vp, _i32p, _ci, _i32p, _ci, _ci, _ci, _ci, _ci, _ci, ctypes.c_float,
                           _vp, ctypes.c_size_t, _vp, _vp]
_lib.pa_decode.restype = _ci
_lib.pa_prefill_chunk.argtypes = [_vp, _vp, _i32p, _vp, _vp, _i32p, _ci, _i32p, _ci, _ci, _ci, _ci, _ci, _ci, _ci,
                                  ctypes.c_float, _vp, ctypes.c_size_t, _vp, _vp]
_lib.pa_prefill_chunk.restype = _ci
_lib.pa_decode_append.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i32p, _ci, _i32p, _ci, _ci, _ci, _ci, _ci, _ci,
                                  ctypes.c_float, _vp, ctypes.c_size_t, _vp, _vp]
_lib.pa_decode_append.restype = _ci
_lib.pa_cascade_workspace_bytes.argtypes = [_ci, _ci, _ci, _ci, _ci, _ci]
_lib.pa_cascade_workspace_bytes.restype = ctypes.c_size_t
_lib.pa_decode_cascade.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i32p, _ci, _i32p, _ci, _ci, _ci, _ci, _ci, _ci,
                                   ctypes.c_float, _i32p, _i32p, _ci, _vp, ctypes.c_size_t, _vp, _vp]
_lib.pa_decode_cascade.restype = _ci
_lib.pa_cache_append_fp8.argtypes = [_vp, _vp, _vp, _vp, _i32p, _ci, _ci, _ci, _ci, _ci, ctypes.c_float,
                                     ctypes.c_float, _vp, _vp]
_lib.pa_cache_append_fp8.restype = _ci
_lib.pa_decode_fp8.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i32p, _ci, _i32p, _ci, _ci, _ci, _ci, _ci, _ci,
                               ctypes.c_float, ctypes.c_float, ctypes.c_float, _vp, ctypes.c_size_t, _vp, _vp]
_lib.pa_decode_fp8.restype = _ci
_lib.pa_prefill_chunk_fp8.argtypes = [_vp, _vp, _i32p, _vp, _vp, _i32p, _ci, _i32p, _ci, _ci, _ci, _ci, _ci, _ci, _ci,
                                      ctypes.c_float, ctypes.c_float, ctypes.c_float, _vp, ctypes.c_size_t, _vp, _vp]
_lib.pa_prefill_chunk_fp8.restype = _ci
_lib.pa_decode_static_scratch.argtypes = [_vp, _vp, _vp, _vp, _i32p, _ci, _i32p, _ci, _ci, _ci, _ci, _ci, _ci,
                                          ctypes.c_float, _vp, _vp]
_lib.pa_decode_static_scratch.restype = _ci
_lib.pa_status_string.argtypes = [_ci]
_lib.pa_status_string.restype = ctypes.c_char_p
PLAN_WORDS = 16  # PA_PLAN_WORDS of include/pa.h


class Plan(ctypes.Structure):
    """pa_plan: the host plan of a varlen batch (opaque words)."""
    _fields_ = [("words", ctypes.c_int32 * PLAN_WORDS)]


_lib.pa_plan_batch.argtypes = [_vp, _vp, _ci, _ci, _ci, _ci, _ci, _ci, ctypes.POINTER(Plan)]
_lib.pa_plan_batch.restype = _ci
_lib.pa_prefill_chunk_planned.argtypes = [_vp, _vp, _i32p, _vp, _vp, _i32p, _ci, _i32p, _ci, _ci, _ci, _ci, _ci, _ci,
                                          _ci, ctypes.c_float, _vp, ctypes.c_size_t, ctypes.POINTER(Plan), _vp, _vp]
_lib.pa_prefill_chunk_planned.restype = _ci
_lib.pa_calibrate_bytes.argtypes = []
_lib.pa_calibrate_bytes.restype = ctypes.c_size_t
_lib.pa_calibrate.argtypes = [_vp, ctypes.c_size_t, _vp, _vp]
_lib.pa_calibrate.restype = _ci
_lib.pa_calibration.argtypes = [ctypes.POINTER(_ci), _vp]
_lib.pa_calibration.restype = _ci
_lib.pa_calibration_clear.argtypes = []
_lib.pa_calibration_clear.restype = None
_lib.pa_last_cuda_error.argtypes = []
_lib.pa_last_cuda_error.restype = _ci
_lib.pa_last_cuda_error_string.argtypes = []
_lib.pa_last_cuda_error_string.restype = ctypes.c_char_p

PA_OK = 0
PA_ERR_NULL, PA_ERR_SHAPE, PA_ERR_UNSUPPORTED, PA_ERR_WORKSPACE = -1, -2, -3, -4
PA_ERR_RANGE, PA_ERR_CUDA, PA_ERR_TIMEOUT = -5, -6, -7
STATIC_SCRATCH_BYTES = 64 * 1024 * 1024  # PA_STATIC_SCRATCH_BYTES of include/pa.h


def status_bit(code: int) -> int:
    """Bit a kernel ORs into the device status word for device error ``code``."""
    return 1 << (-code)


class PAError(RuntimeError):
    def __init__(self, code: int, detail: str | None = None):
        self.code = code
        msg = pa_status_string(code)
        super().__init__(f"{msg} ({detail})" if detail else msg)


def pa_status_string(code: int) -> str:
    return _lib.pa_status_string(int(code)).decode()


def pa_last_cuda_error() -> int:
    """cudaError_t (or CUresult) behind the last PA_ERR_CUDA on this thread; 0 if none."""
    return int(_lib.pa_last_cuda_error())


def pa_last_cuda_error_string() -> str:
    return _lib.pa_last_cuda_error_string().decode()


def _check(rc: int) -> None:
    if rc != PA_OK:
        raise PAError(rc, pa_last_cuda_error_string() if rc == PA_ERR_CUDA else None)


def _dev(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int | None = None) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got {tuple(t.shape)}")
    return t.data_ptr()


def _status_ptr(dev_status) -> int | None:
    if dev_status is None:
        return None
    return _dev(dev_status, "dev_status", torch.int32)


def _stream_ptr(stream) -> int | None:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream if hasattr(s, "cuda_stream") else int(s)


def pa_cache_append(k_new, v_new, k_cache, v_cache, slot_mapping, dev_status=None, stream=None) -> None:
    """Scatter k_new/v_new [T, Hkv, d] (bf16) into k_cache/v_cache
    [num_blocks, Hkv, block_size, d] at slot_mapping [T] (int32; < 0 = skip)."""
    kp = _dev(k_new, "k_new", torch.bfloat16, 3)
    vp = _dev(v_new, "v_new", torch.bfloat16, 3)
    kc = _dev(k_cache, "k_cache", torch.bfloat16, 4)
    vc = _dev(v_cache, "v_cache", torch.bfloat16, 4)
    sm = _dev(slot_mapping, "slot_mapping", torch.int32, 1)
    nb, hkv, bs, d = k_cache.shape
    if v_cache.shape != k_cache.shape or k_new.shape != v_new.shape:
        raise ValueError("k and v tensors must have the same shapes")
    if k_new.shape[1:] != (hkv, d) or slot_mapping.shape[0] != k_new.shape[0]:
        raise ValueError("k_new must be [T, Hkv, d] and slot_mapping [T]")
    _check(_lib.pa_cache_append(kp, vp, kc, vc, sm, k_new.shape[0], nb, hkv, d, bs, _status_ptr(dev_status),
                                _stream_ptr(stream)))


def pa_workspace_bytes(num_query_tokens: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                       max_blocks_per_seq: int, block_size: int) -> int:
    n = int(_lib.pa_workspace_bytes(num_query_tokens, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                                    block_size))
    if n == 0:
        raise PAError(PA_ERR_UNSUPPORTED)
    return n


def make_workspace(num_query_tokens: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                   max_blocks_per_seq: int, block_size: int, device=None) -> torch.Tensor:
    """A zero-filled workspace of pa_workspace_bytes() bytes (the zero fill is required once)."""
    n = pa_workspace_bytes(num_query_tokens, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, block_size)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def _attention_args(out, q, k_cache, v_cache, block_tables, context_lens, workspace):
    op = _dev(out, "out", torch.bfloat16, 3)
    qp = _dev(q, "q", torch.bfloat16, 3)
    kc = _dev(k_cache, "k_cache", torch.bfloat16, 4)
    vc = _dev(v_cache, "v_cache", torch.bfloat16, 4)
    bt = _dev(block_tables, "block_tables", torch.int32, 2)
    cl = _dev(context_lens, "context_lens", torch.int32, 1)
    ws = _dev(workspace, "workspace", torch.uint8, 1)
    if out.shape != q.shape:
        raise ValueError("out must have q's shape")
    if v_cache.shape != k_cache.shape or k_cache.shape[3] != q.shape[2]:
        raise ValueError("k_cache/v_cache must be [num_blocks, Hkv, block_size, d] with q's d")
    if block_tables.shape[0] != context_lens.shape[0]:
        raise ValueError("block_tables and context_lens must have one row per sequence")
    return op, qp, kc, vc, bt, cl, ws


def pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, workspace, dev_status=None,
              stream=None) -> None:
    """One decode row per sequence: q/out [B, Hq, d]; see include/pa.h."""
    op, qp, kc, vc, bt, cl, ws = _attention_args(out, q, k_cache, v_cache, block_tables, context_lens, workspace)
    nb, hkv, bs, d = k_cache.shape
    if q.shape[0] != context_lens.shape[0]:
        raise ValueError("pa_decode takes exactly one query row per sequence")
    _check(_lib.pa_decode(op, qp, kc, vc, bt, block_tables.shape[1], cl, context_lens.shape[0], q.shape[1], hkv, d,
                          bs, nb, float(scale), ws, workspace.numel(), _status_ptr(dev_status), _stream_ptr(stream)))


def pa_decode_append(out, q, k_new, v_new, k_cache, v_cache, block_tables, context_lens, scale, workspace,
                     dev_status=None, stream=None) -> None:
    """pa_cache_append of each sequence's newest row (k_new / v_new [B, Hkv, d],
    written at position context_lens[s] - 1 through the block table) and
    pa_decode, in one launch; see include/pa.h."""
    op, qp, kc, vc, bt, cl, ws = _attention_args(out, q, k_cache, v_cache, block_tables, context_lens, workspace)
    kn = _dev(k_new, "k_new", torch.bfloat16, 3)
    vn = _dev(v_new, "v_new", torch.bfloat16, 3)
    nb, hkv, bs, d = k_cache.shape
    if q.shape[0] != context_lens.shape[0]:
        raise ValueError("pa_decode_append takes exactly one query row per sequence")
    if k_new.shape != (context_lens.shape[0], hkv, d) or v_new.shape != k_new.shape:
        raise ValueError("k_new / v_new must be [num_seqs, Hkv, d]")
    _check(_lib.pa_decode_append(op, qp, kn, vn, kc, vc, bt, block_tables.shape[1], cl, context_lens.shape[0],
                                 q.shape[1], hkv, d, bs, nb, float(scale), ws, workspace.numel(),
                                 _status_ptr(dev_status), _stream_ptr(stream)))


def pa_cascade_workspace_bytes(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                               max_blocks_per_seq: int, block_size: int) -> int:
    n = int(_lib.pa_cascade_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                                            block_size))
    if n == 0:
        raise PAError(PA_ERR_UNSUPPORTED)
    return n


def make_cascade_workspace(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                           max_blocks_per_seq: int, block_size: int, device=None) -> torch.Tensor:
    """A zero-filled workspace of pa_cascade_workspace_bytes() bytes."""
    n = pa_cascade_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, block_size)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def pa_decode_cascade(out, q, k_cache, v_cache, block_tables, context_lens, scale, group_start, group_prefix,
                      workspace, k_new=None, v_new=None, dev_status=None, stream=None) -> None:
    """Decode attention for a batch with shared-prefix groups (sequences
    group_start[g] .. group_start[g+1]-1 share their first group_prefix[g]
    tokens); with k_new / v_new the step's append is fused in.  See include/pa.h."""
    op, qp, kc, vc, bt, cl, ws = _attention_args(out, q, k_cache, v_cache, block_tables, context_lens, workspace)
    gs = _dev(group_start, "group_start", torch.int32, 1)
    gp = _dev(group_prefix, "group_prefix", torch.int32, 1)
    if group_start.shape[0] != group_prefix.shape[0] + 1:
        raise ValueError("group_start must have one more entry than group_prefix")
    nb, hkv, bs, d = k_cache.shape
    if q.shape[0] != context_lens.shape[0]:
        raise ValueError("pa_decode_cascade takes exactly one query row per sequence")
    kn = vn = None
    if k_new is not None or v_new is not None:
        kn = _dev(k_new, "k_new", torch.bfloat16, 3)
        vn = _dev(v_new, "v_new", torch.bfloat16, 3)
        if k_new.shape != (context_lens.shape[0], hkv, d) or v_new.shape != k_new.shape:
            raise ValueError("k_new / v_new must be [num_seqs, Hkv, d]")
    _check(_lib.pa_decode_cascade(op, qp, kn, vn, kc, vc, bt, block_tables.shape[1], cl, context_lens.shape[0],
                                  q.shape[1], hkv, d, bs, nb, float(scale), gs, gp, group_prefix.shape[0], ws,
                                  workspace.numel(), _status_ptr(dev_status), _stream_ptr(stream)))


def pa_cache_append_fp8(k_new, v_new, k_cache, v_cache, slot_mapping, k_scale, v_scale, dev_status=None,
                        stream=None) -> None:
    """Append into an FP8 (E4M3 codes, uint8) cache with per-tensor scales; see include/pa.h."""
    kp = _dev(k_new, "k_new", torch.bfloat16, 3)
    vp = _dev(v_new, "v_new", torch.bfloat16, 3)
    kc = _dev(k_cache, "k_cache", torch.uint8, 4)
    vc = _dev(v_cache, "v_cache", torch.uint8, 4)
    sm = _dev(slot_mapping, "slot_mapping", torch.int32, 1)
    nb, hkv, bs, d = k_cache.shape
    if v_cache.shape != k_cache.shape or k_new.shape[1:] != (hkv, d) or v_new.shape != k_new.shape:
        raise ValueError("k_new/v_new [T, Hkv, d] and caches [num_blocks, Hkv, block_size, d] must agree")
    _check(_lib.pa_cache_append_fp8(kp, vp, kc, vc, sm, k_new.shape[0], nb, hkv, d, bs, float(k_scale),
                                    float(v_scale), _status_ptr(dev_status), _stream_ptr(stream)))


def pa_decode_fp8(out, q, k_cache, v_cache, block_tables, context_lens, scale, k_scale, v_scale, workspace,
                  k_new=None, v_new=None, dev_status=None, stream=None) -> None:
    """Decode over an FP8 cache; with k_new / v_new the step's append is fused in.  See include/pa.h."""
    op = _dev(out, "out", torch.bfloat16, 3)
    qp = _dev(q, "q", torch.bfloat16, 3)
    kc = _dev(k_cache, "k_cache", torch.uint8, 4)
    vc = _dev(v_cache, "v_cache", torch.uint8, 4)
    bt = _dev(block_tables, "block_tables", torch.int32, 2)
    cl = _dev(context_lens, "context_lens", torch.int32, 1)
    ws = _dev(workspace, "workspace", torch.uint8, 1)
    nb, hkv, bs, d = k_cache.shape
    if out.shape != q.shape or v_cache.shape != k_cache.shape or q.shape[2] != d:
        raise ValueError("out/q [B, Hq, d] and caches [num_blocks, Hkv, block_size, d] must agree")
    if q.shape[0] != context_lens.shape[0] or block_tables.shape[0] != context_lens.shape[0]:
        raise ValueError("one query row, one block-table row and one length per sequence")
    kn = vn = None
    if k_new is not None or v_new is not None:
        kn = _dev(k_new, "k_new", torch.bfloat16, 3)
        vn = _dev(v_new, "v_new", torch.bfloat16, 3)
        if k_new.shape != (context_lens.shape[0], hkv, d) or v_new.shape != k_new.shape:
            raise ValueError("k_new / v_new must be [num_seqs, Hkv, d]")
    _check(_lib.pa_decode_fp8(op, qp, kn, vn, kc, vc, bt, block_tables.shape[1], cl, context_lens.shape[0],
                              q.shape[1], hkv, d, bs, nb, float(scale), float(k_scale), float(v_scale), ws,
                              workspace.numel(), _status_ptr(dev_status), _stream_ptr(stream)))


def pa_prefill_chunk(out, q, query_start, k_cache, v_cache, block_tables, context_lens, scale, workspace,
                     dev_status=None, stream=None) -> None:
    """Varlen batch of prefill chunks, multi-token verification rows and
    decodes: q/out [Tq, Hq, d], query_start [B + 1]; see include/pa.h (which
    kernel takes which sequences)."""
    op, qp, kc, vc, bt, cl, ws = _attention_args(out, q, k_cache, v_cache, block_tables, context_lens, workspace)
    qs = _dev(query_start, "query_start", torch.int32, 1)
    if query_start.shape[0] != context_lens.shape[0] + 1:
        raise ValueError("query_start must have num_seqs + 1 entries")
    nb, hkv, bs, d = k_cache.shape
    _check(_lib.pa_prefill_chunk(op, qp, qs, kc, vc, bt, block_tables.shape[1], cl, context_lens.shape[0], q.shape[0],
                                 q.shape[1], hkv, d, bs, nb, float(scale), ws, workspace.numel(),
                                 _status_ptr(dev_status), _stream_ptr(stream)))


def _host_i32(a, name):
    import numpy as np
    if isinstance(a, torch.Tensor):
        if a.is_cuda:
            raise ValueError(f"{name} must be a host array (the plan is made on the host)")
        a = a.numpy()
    a = np.ascontiguousarray(a, dtype=np.int32)
    if a.ndim != 1:
        raise ValueError(f"{name} must be one-dimensional")
    return a


def pa_prefill_chunk_fp8(out, q, query_start, k_cache, v_cache, block_tables, context_lens, scale, k_scale, v_scale,
                         workspace, dev_status=None, stream=None) -> None:
    """pa_prefill_chunk over E4M3 caches (uint8 [num_blocks, Hkv, block_size, d])
    with per-tensor scales, as pa_decode_fp8."""
    op = _dev(out, "out", torch.bfloat16, 3)
    qp = _dev(q, "q", torch.bfloat16, 3)
    kc = _dev(k_cache, "k_cache", torch.uint8, 4)
    vc = _dev(v_cache, "v_cache", torch.uint8, 4)
    bt = _dev(block_tables, "block_tables", torch.int32, 2)
    cl = _dev(context_lens, "context_lens", torch.int32, 1)
    qs = _dev(query_start, "query_start", torch.int32, 1)
    ws = _dev(workspace, "workspace", torch.uint8, 1)
    if out.shape != q.shape or v_cache.shape != k_cache.shape or k_cache.shape[3] != q.shape[2]:
        raise ValueError("out/q [Tq, Hq, d] and caches [num_blocks, Hkv, block_size, d] must agree")
    if query_start.shape[0] != context_lens.shape[0] + 1 or block_tables.shape[0] != context_lens.shape[0]:
        raise ValueError("query_start must have num_seqs + 1 entries, one table row per sequence")
    nb, hkv, bs, d = k_cache.shape
    _check(_lib.pa_prefill_chunk_fp8(op, qp, qs, kc, vc, bt, block_tables.shape[1], cl, context_lens.shape[0],
                                     q.shape[0], q.shape[1], hkv, d, bs, nb, float(scale), float(k_scale),
                                     float(v_scale), ws, workspace.numel(), _status_ptr(dev_status),
                                     _stream_ptr(stream)))


def pa_plan_batch(query_start, context_lens, num_q_heads: int, num_kv_heads: int, head_dim: int, block_size: int,
                  max_blocks_per_seq: int) -> Plan:
    """Host plan of a varlen batch from HOST copies of query_start [B + 1] and
    context_lens [B]: which kernels have work, and how decode rows and
    prefill chunks share the SMs.  Make it with the device current that runs
    the call."""
    qs = _host_i32(query_start, "query_start")
    cl = _host_i32(context_lens, "context_lens")
    if qs.shape[0] != cl.shape[0] + 1:
        raise ValueError("query_start must have num_seqs + 1 entries")
    plan = Plan()
    _check(_lib.pa_plan_batch(qs.ctypes.data, cl.ctypes.data, cl.shape[0], num_q_heads, num_kv_heads, head_dim,
                              block_size, max_blocks_per_seq, ctypes.byref(plan)))
    return plan


def pa_prefill_chunk_planned(out, q, query_start, k_cache, v_cache, block_tables, context_lens, scale, workspace,
                             plan: Plan, dev_status=None, stream=None) -> None:
    """pa_prefill_chunk with a plan from pa_plan_batch (made for this batch)."""
    op, qp, kc, vc, bt, cl, ws = _attention_args(out, q, k_cache, v_cache, block_tables, context_lens, workspace)
    qs = _dev(query_start, "query_start", torch.int32, 1)
    if query_start.shape[0] != context_lens.shape[0] + 1:
        raise ValueError("query_start must have num_seqs + 1 entries")
    if not isinstance(plan, Plan):
        raise TypeError("plan must come from pa_plan_batch")
    nb, hkv, bs, d = k_cache.shape
    _check(_lib.pa_prefill_chunk_planned(op, qp, qs, kc, vc, bt, block_tables.shape[1], cl, context_lens.shape[0],
                                         q.shape[0], q.shape[1], hkv, d, bs, nb, float(scale), ws, workspace.numel(),
                                         ctypes.byref(plan), _status_ptr(dev_status), _stream_ptr(stream)))


def pa_calibrate(buffer: torch.Tensor | None = None, dev_status=None, stream=None) -> list[int]:
    """Time the decode kernel on every SM of the current device and keep per-SM
    weights for its split of the work; returns the weights.  ``buffer``: a
    CUDA tensor of at least pa_calibrate_bytes() bytes (overwritten); one is
    allocated for the call if None.  Waits for its own work."""
    need = int(_lib.pa_calibrate_bytes())
    if need == 0:
        raise PAError(PA_ERR_CUDA, "no CUDA device")
    if buffer is None:
        buffer = torch.empty(need, dtype=torch.uint8, device="cuda")
    if not buffer.is_cuda or not buffer.is_contiguous():
        raise ValueError("buffer must be a contiguous CUDA tensor")
    _check(_lib.pa_calibrate(buffer.data_ptr(), buffer.numel() * buffer.element_size(), _status_ptr(dev_status),
                             _stream_ptr(stream)))
    return pa_calibration()


def pa_calibration() -> list[int]:
    """The per-SM rates recorded for the current device ([] if none)."""
    n = _ci(0)
    rates = (ctypes.c_uint16 * 256)()
    rc = _lib.pa_calibration(ctypes.byref(n), rates)
    if rc == PA_ERR_RANGE:
        return []
    _check(rc)
    return list(rates[:n.value])


def pa_calibration_clear() -> None:
    """Forget every device's rates: decode splits its work equally again."""
    _lib.pa_calibration_clear()


def pa_decode_static_scratch(out, q, k_cache, v_cache, block_tables, context_lens, scale, dev_status=None,
                             stream=None) -> None:
    """pa_decode without a workspace argument, for callers that cannot allocate
    device memory when they launch: the library's own per-device scratch array
    (STATIC_SCRATCH_BYTES) is used instead.  Overlapping calls on one device
    race on that array; make the first call on a device before any stream
    capture.  See include/pa.h."""
    op = _dev(out, "out", torch.bfloat16, 3)
    qp = _dev(q, "q", torch.bfloat16, 3)
    kc = _dev(k_cache, "k_cache", torch.bfloat16, 4)
    vc = _dev(v_cache, "v_cache", torch.bfloat16, 4)
    bt = _dev(block_tables, "block_tables", torch.int32, 2)
    cl = _dev(context_lens, "context_lens", torch.int32, 1)
    if out.shape != q.shape:
        raise ValueError("out must have q's shape")
    if v_cache.shape != k_cache.shape or k_cache.shape[3] != q.shape[2]:
        raise ValueError("k_cache/v_cache must be [num_blocks, Hkv, block_size, d] with q's d")
    if block_tables.shape[0] != context_lens.shape[0] or q.shape[0] != context_lens.shape[0]:
        raise ValueError("one query row, one block-table row and one length per sequence")
    nb, hkv, bs, d = k_cache.shape
    rc = _lib.pa_decode_static_scratch(op, qp, kc, vc, bt, block_tables.shape[1], cl, context_lens.shape[0],
                                       q.shape[1], hkv, d, bs, nb, float(scale), _status_ptr(dev_status),
                                       _stream_ptr(stream))
    if rc == PA_ERR_WORKSPACE:
        raise PAError(rc, f"this batch needs more scratch than the {STATIC_SCRATCH_BYTES}-byte static array: "
                          "use pa_decode with a workspace")
    _check(rc)


def exported_symbols() -> list[str]:
    return ["pa_cache_append", "pa_workspace_bytes", "pa_decode", "pa_decode_append", "pa_cache_append_fp8",
            "pa_decode_fp8", "pa_cascade_workspace_bytes", "pa_decode_cascade", "pa_prefill_chunk",
            "pa_decode_static_scratch", "pa_status_string", "pa_last_cuda_error", "pa_last_cuda_error_string",
            "pa_plan_batch", "pa_prefill_chunk_planned", "pa_prefill_chunk_fp8", "pa_calibrate_bytes", "pa_calibrate", "pa_calibration",
            "pa_calibration_clear"]
