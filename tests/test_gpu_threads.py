"""Two host threads call the library at once, each on its own CUDA stream
with its own workspace: every result matches the oracle.

The entry points keep only per-device launch set-up (shared-memory opt-in,
CTAs per SM) between calls, in atomics.  The calls run in a fresh process so
that the two threads' first calls also race on that set-up.
"""
from __future__ import annotations

import os
import subprocess
import sys
import textwrap

import pytest
import torch

from tests.gpu_helpers import load_library

pytestmark = pytest.mark.gpu

_SCRIPT = textwrap.dedent("""
    import sys, threading
    import numpy as np
    import torch
    sys.path.insert(0, {root!r})
    import oracle
    import paged_kv_cache_445_b200 as pa
    from paged_kv_cache_445_b200 import workloads
    from tests.gpu_helpers import DeviceStep, compare, oracle_after_append

    cases = [
        workloads.custom([3000, 17, 900, 5000], [1, 1, 1, 1], 16, 2, 128, 16, seed=41, poison=True),
        workloads.custom([700, 64, 2500], [1, 1, 1], 8, 1, 256, 32, seed=42, poison=True),
        workloads.custom([2000, 300], [40, 1], 32, 4, 128, 16, seed=43, poison=True),
        workloads.custom([64, 1000, 33], [1, 1, 1], 16, 1, 64, 16, seed=44, poison=True),
    ]
    refs = []
    for w in cases:
        kc, vc = oracle_after_append(w)
        refs.append(oracle.paged_attention(w.q, kc, vc, w.block_tables, w.context_lens, w.query_start, w.scale))
    steps = [DeviceStep(w) for w in cases]
    streams = [torch.cuda.Stream() for _ in range(2)]
    for k, ds in enumerate(steps):  # the appends first, on the default stream
        ds.append()
    torch.cuda.synchronize()
    start = threading.Barrier(2)
    errors = []

    def worker(t):
        try:
            mine = steps[t::2]
            with torch.cuda.stream(streams[t]):
                start.wait()
                for it in range(25):
                    for ds in mine:
                        ds.attend()
            streams[t].synchronize()
        except Exception as e:  # reported by the main thread
            errors.append(repr(e))

    threads = [threading.Thread(target=worker, args=(t,)) for t in range(2)]
    for th in threads:
        th.start()
    for th in threads:
        th.join()
    assert not errors, errors
    torch.cuda.synchronize()
    for ds, ref, w in zip(steps, refs, cases):
        assert int(ds.status.item()) == 0, (w.name, int(ds.status.item()))
        compare(ds.out.float().cpu().numpy(), ref, w.name)
    print("threads ok")
""")


def test_two_host_threads_on_two_streams_each_match_the_oracle():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    load_library()
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _SCRIPT.format(root=root)], cwd=root, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "threads ok" in r.stdout, (r.stdout[-2000:], r.stderr[-4000:])
