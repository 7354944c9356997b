"""The N>1 plumbing of bench.py on CPU: two gloo ranks, as torchrun would start them.

Each rank runs its own batch (weak scaling, no collective on the data path);
the only collectives are the barriers around the timed region and the MAX of
the step times / SUM of the bytes that make the whole-job number.
"""
from __future__ import annotations

import hashlib
import json
import os
import socket
import time

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
from paged_kv_cache_445_b200 import workloads


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    r, wsize, local = bench.dist_setup(world, backend="gloo")
    w = workloads.standard(1, seed=bench.rank_seed(1, r))
    kv_bytes = float(np.asarray(w.context_lens, dtype=np.int64).sum() * 2 * w.num_kv_heads * w.head_dim * 2)
    # a "step" whose length differs by rank: the slowest one must decide the time
    bench.barrier(wsize)
    t0 = time.perf_counter()
    time.sleep(0.05 * (r + 1))
    my_ms = (time.perf_counter() - t0) * 1e3
    bench.barrier(wsize)
    ms_max = bench.max_over_ranks(my_ms, wsize, device="cpu")
    total = bench.reduce_over_ranks(kv_bytes, wsize, "sum", device="cpu")
    digests = [None] * wsize
    dist.all_gather_object(digests, hashlib.sha256(w.q.tobytes()).hexdigest())
    with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
        json.dump({"rank": r, "world": wsize, "local": local, "my_ms": my_ms, "ms_max": ms_max,
                   "kv_bytes": kv_bytes, "total": total, "digests": digests,
                   "value": bench.compose_value(total, ms_max)}, f)
    dist.destroy_process_group()


def test_two_gloo_ranks_time_by_the_slowest_and_sum_the_bytes(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    slowest = max(r["my_ms"] for r in res)
    for r in res:
        assert r["world"] == world
        assert r["ms_max"] == pytest.approx(slowest)        # every rank sees the max
        assert r["total"] == pytest.approx(sum(x["kv_bytes"] for x in res))
        assert r["value"] == pytest.approx(r["total"] / (slowest * 1e-3) / 1e9)
    # weak scaling: each rank drew its own batch
    assert res[0]["digests"][0] != res[0]["digests"][1]
    assert res[0]["digests"] == res[1]["digests"]


def test_world_size_must_match_gpus(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "2")
    with pytest.raises(SystemExit):
        bench.dist_setup(1, backend="gloo")


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.main(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "1"])
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_one_line(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    bench.main(["--impl", "reference", "--steps", "2", "--warmup", "3", "--workload", "1",
                "--reference-seconds", "2"])
    lines = [l for l in capsys.readouterr().out.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_launch_count_per_step():
    decode = workloads.custom([40, 90], [1, 1], 16, 2, 128, 16, seed=1)
    mixed = workloads.custom([200, 30], [48, 1], 16, 2, 128, 16, seed=1)
    mixed_d64 = workloads.custom([200, 30], [48, 1], 16, 2, 64, 16, seed=1)
    assert bench.step_launches(decode) == 2
    # append, chunk kernel, the two multi-row kernels, rows kernel (pa_prefill_chunk launches
    # every kernel that may have work at head_dim 128, whatever the row counts are)
    assert bench.step_launches(mixed) == 5
    assert bench.step_launches(mixed_d64) == 2
    verify = workloads.custom([200, 30, 90], [4, 2, 8], 16, 2, 128, 16, seed=1)
    assert bench.verify_batch(verify) and not bench.verify_batch(mixed) and not bench.verify_batch(decode)


def test_l2_is_flushed_exactly_for_workloads_whose_kv_fits_in_it():
    from paged_kv_cache_445_b200 import roofline
    flushed = []
    for cfg in (1, 2, 3, 4, 5, 6):
        w = workloads.standard(cfg)
        unique = roofline.unique_kv_bytes(w.block_tables, w.context_lens, w.block_size, w.num_kv_heads, w.head_dim)
        if bench.l2_flush_needed(unique):
            flushed.append(cfg)
            assert bench.l2_note(True, 0, unique).startswith("flushed")
    # the tiny case and the shared-prefix batch (86 MB of distinct KV) fit in the 126 MB L2
    assert flushed == [1, 4]
    assert bench.FLUSH_BYTES > bench.L2_BYTES


def test_cpu_baseline_reports_all_cores_and_one_core():
    import oracle
    cores = oracle.num_threads()
    line = bench.oracle_baseline(workloads.standard(1), 0.2)
    assert line["kind"] == "oracle" and line["cores"] == cores and line["value"] > 0
    if cores > 1:
        assert line["single_core"]["cores"] == 1 and line["single_core"]["value"] > 0
    assert oracle.num_threads() == cores  # the thread count is restored
