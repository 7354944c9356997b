"""pa_decode_static_scratch: decode for callers that cannot allocate device
memory when they launch (a runtime replaying a recorded launch sequence, a
host with a fixed memory budget), using the library's own scratch array.

Checked through the C ABI against pa_decode with a caller workspace (the same
kernel and the same split of the work, so the output must be the same bits)
and against the fp64 oracle.  Collected last on purpose: it must pass both in
a fresh process and after every other test has used the library on this
device, and a failure here stops a run only after everything else has run.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from paged_kv_cache_445_b200 import workloads
from tests.gpu_helpers import DeviceStep, compare, i32, load_library, oracle_after_append

pytestmark = pytest.mark.gpu


def _static(ds: DeviceStep, out: torch.Tensor, block_tables=None):
    import paged_kv_cache_445_b200 as pa
    pa.pa_decode_static_scratch(out, ds.q, ds.k_cache, ds.v_cache,
                                ds.block_tables if block_tables is None else block_tables, ds.context_lens,
                                ds.w.scale, ds.status)


def _reference_bits(ds: DeviceStep) -> torch.Tensor:
    """pa_decode's output with a fresh zero-filled caller workspace."""
    ds.attend()
    torch.cuda.synchronize()
    assert int(ds.status.item()) == 0
    return ds.out.clone()


def _long_and_short():
    # long contexts next to short ones: many (row, head) segments are split
    # between warps, so the scratch (barrier counters, segment records,
    # partial results) is really used
    return [
        workloads.custom([32000, 24999, 7, 300], [1, 1, 1, 1], 16, 2, 128, 16, seed=31, poison=True),
        workloads.custom([40, 1500, 9000], [1, 1, 1], 8, 1, 128, 16, seed=32, poison=True),
    ]


def test_static_scratch_equals_pa_decode_bit_for_bit_on_two_calls_in_a_row():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    load_library()
    import oracle
    for k, w in enumerate(_long_and_short()):  # a different shape between calls: what the last call left must not matter
        ds = DeviceStep(w)
        ds.append()
        want = _reference_bits(ds)
        if k == 0:
            kc, vc = oracle_after_append(w)
            ref = oracle.paged_attention(w.q, kc, vc, w.block_tables, w.context_lens, w.query_start, w.scale)
        for call in range(2):
            got = torch.full_like(ds.out, 5.0)
            _static(ds, got)
            torch.cuda.synchronize()
            assert int(ds.status.item()) == 0, f"device status {int(ds.status.item())}"
            assert torch.equal(got.view(torch.int16), want.view(torch.int16)), \
                f"{w.name}, static-scratch call {call + 1}: not the bits of pa_decode"
            if k == 0:
                compare(got.float().cpu().numpy(), ref, f"{w.name}, static-scratch call {call + 1} vs the oracle")


def test_a_call_after_a_failed_call_needs_no_reset():
    import paged_kv_cache_445_b200 as pa
    load_library()
    w = _long_and_short()[0]
    ds = DeviceStep(w)
    ds.append()
    want = _reference_bits(ds)
    # a block ID outside the pool in sequence 0's table: the kernel skips the
    # tile, sets the RANGE bit and still runs to the end (nothing faults)
    bad = w.block_tables.copy()
    bad[0, 5] = w.num_blocks + 1000
    out = torch.full_like(ds.out, 5.0)
    _static(ds, out, block_tables=i32(bad))
    torch.cuda.synchronize()
    assert int(ds.status.item()) & pa.status_bit(pa._binding.PA_ERR_RANGE)
    # the next good call on the same shared array: correct with no reset of it
    ds.status.zero_()
    got = torch.full_like(ds.out, 5.0)
    _static(ds, got)
    torch.cuda.synchronize()
    assert int(ds.status.item()) == 0
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))


def test_static_scratch_rejects_a_batch_larger_than_the_array():
    import paged_kv_cache_445_b200 as pa
    load_library()
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
