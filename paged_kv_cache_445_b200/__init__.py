"""Attention over a paged KV cache on B200 (sm_100a).

The compute path lives in ``libpa.so`` (``csrc/``), a C-ABI library whose
entry points are declared in ``include/pa.h``.  ``_binding`` is the thin
Python layer over it -- argument marshalling only -- and is imported lazily so
that the host-side pieces (``allocator``, ``workloads``, ``roofline``) load
without a GPU.  Touching any ``pa_*`` name loads the library; if it is missing
the import raises: there is no CPU fallback.
"""
from __future__ import annotations

__all__ = [
    "pa_cache_append", "pa_decode", "pa_decode_append", "pa_cache_append_fp8", "pa_decode_fp8",
    "pa_decode_cascade", "pa_cascade_workspace_bytes",
    "make_cascade_workspace", "pa_prefill_chunk", "pa_workspace_bytes", "pa_decode_static_scratch",
    "pa_status_string", "pa_last_cuda_error", "pa_last_cuda_error_string", "PAError", "library_path",
    "make_workspace", "status_bit", "pa_plan_batch", "pa_prefill_chunk_planned", "Plan",
    "pa_calibrate", "pa_calibration", "pa_calibration_clear", "pa_prefill_chunk_fp8",
]


def __getattr__(name):
    if name in __all__:
        from . import _binding
        return getattr(_binding, name)
    raise AttributeError(name)
