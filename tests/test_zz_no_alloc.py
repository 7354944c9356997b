"""pa_decode_static_scratch (decode with the library's own scratch array)
against pa_decode with a caller workspace, through the C ABI.

Collected last on purpose: it must pass both in a fresh process and after
every other test has used the library on this device.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from paged_kv_cache_445_b200 import workloads
from tests.gpu_helpers import DeviceStep, compare, i32, load_library

pytestmark = pytest.mark.gpu


def _static(ds: DeviceStep, out: torch.Tensor):
    import paged_kv_cache_445_b200 as pa
    pa.pa_decode_static_scratch(out, ds.q, ds.k_cache, ds.v_cache, ds.block_tables, ds.context_lens, ds.w.scale,
                                ds.status)


def test_static_scratch_matches_pa_decode_on_two_calls_in_a_row():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    load_library()
    # long contexts next to short ones: many (row, head) segments are split
    # between warps, so the scratch (barrier counters, segment records,
    # partial results) is really used
    batches = [
        workloads.custom([32000, 24999, 7, 300], [1, 1, 1, 1], 16, 2, 128, 16, seed=31, poison=True),
        workloads.custom([40, 1500, 9000], [1, 1, 1], 8, 1, 128, 16, seed=32, poison=True),
    ]
    for w in batches:  # a different shape between calls: what the last call left must not matter
        ds = DeviceStep(w)
        ds.append()
        ds.attend()  # pa_decode with its own zero-filled workspace
        torch.cuda.synchronize()
        want = ds.out.float().cpu().numpy().astype(np.float64)
        for call in range(2):
            got = torch.full_like(ds.out, 5.0)
            _static(ds, got)
            torch.cuda.synchronize()
            assert int(ds.status.item()) == 0, f"device status {int(ds.status.item())}"
            compare(got.float().cpu().numpy(), want, f"{w.name}, static-scratch call {call + 1}")


def test_static_scratch_rejects_a_batch_larger_than_the_array():
    import paged_kv_cache_445_b200 as pa
    num_seqs, hq, hkv, d, bs, max_blocks = 8000, 16, 2, 128, 16, 512
    assert pa.pa_workspace_bytes(num_seqs, hq, hkv, d, max_blocks, bs) > pa._binding.STATIC_SCRATCH_BYTES
    q = torch.zeros(num_seqs, hq, d, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(4, hkv, bs, d, dtype=torch.bfloat16, device="cuda")
    bt = i32(np.zeros((num_seqs, max_blocks), dtype=np.int32))
    cl = i32(np.ones(num_seqs, dtype=np.int32))
    out = torch.full_like(q, 3.0)
    with pytest.raises(pa.PAError) as e:
        pa.pa_decode_static_scratch(out, q, kc, kc, bt, cl, 0.1)
    assert e.value.code == pa._binding.PA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(out == 3.0)  # rejected before any launch
