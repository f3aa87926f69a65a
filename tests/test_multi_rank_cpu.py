"""The multi-GPU path of the benchmark, run as world-size-2 gloo ranks on CPU.

The path shards by sequence batch: every rank runs its own seeded batch of
the workload (weak scaling) with no data-path collective. The ranks meet only
to take the slowest rank's times (MAX) and the sum of the work (SUM); the
whole-job throughput is the summed FLOPs over the slowest rank's time. These
tests run that host logic on two real processes without a GPU.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, per_rank, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        w, r, lr = bench._dist()
        stats, totals = per_rank[rank]
        red_stats, red_totals = bench.reduce_over_ranks(stats, totals, w)
        results[rank] = {"dist": (w, r, lr), "stats": red_stats, "totals": red_totals,
                         "seed": bench.rank_seed(rank)}
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _run(world, per_rank):
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, per_rank, results))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        codes = [p.exitcode for p in procs]
        out = dict(results)
    assert codes == [0] * world, codes
    return out


@pytest.fixture(scope="module")
def two_ranks():
    per_rank = {
        0: ([4.00, 35.0, 3.95], [4.15e12, 85484.0]),
        1: ([4.40, 33.0, 4.31], [3.90e12, 80001.0]),
    }
    return per_rank, _run(2, per_rank)


def test_ranks_read_their_environment(two_ranks):
    _, res = two_ranks
    assert res[0]["dist"] == (2, 0, 0)
    assert res[1]["dist"] == (2, 1, 1)


def test_times_take_the_slowest_rank(two_ranks):
    per_rank, res = two_ranks
    want = [max(per_rank[0][0][i], per_rank[1][0][i]) for i in range(3)]
    for r in (0, 1):  # every rank holds the same reduced values
        assert res[r]["stats"] == pytest.approx(want)


def test_work_is_summed(two_ranks):
    per_rank, res = two_ranks
    want = [per_rank[0][1][i] + per_rank[1][1][i] for i in range(2)]
    for r in (0, 1):
        assert res[r]["totals"] == pytest.approx(want)


def test_whole_job_throughput(two_ranks):
    per_rank, res = two_ranks
    stats, totals = res[0]["stats"], res[0]["totals"]
    ms = stats[0]  # slowest rank's time per step
    v = bench.throughput_tflops(totals[0], ms)
    assert v == pytest.approx((4.15e12 + 3.90e12) / 4.40e-3 / 1e12)
    # weak scaling: the job is not faster than the slower rank working alone
    assert v <= sum(f / (t[0] * 1e-3) / 1e12 for t, f in
                    ((per_rank[r][0], per_rank[r][1][0]) for r in (0, 1))) + 1e-9


def test_each_rank_draws_its_own_batch(two_ranks):
    _, res = two_ranks
    assert res[0]["seed"] != res[1]["seed"]
    assert bench.rank_seed(0) == res[0]["seed"]


def test_single_rank_needs_no_process_group():
    stats, totals = bench.reduce_over_ranks([1.0, 2.0, 3.0], [5.0, 6.0], world=1)
    assert stats == [1.0, 2.0, 3.0] and totals == [5.0, 6.0]


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    called = []
    monkeypatch.setattr(bench, "_workload", lambda *a, **k: called.append(1))

    class A:
        pass
    assert bench.run_reference(A(), world=2, rank=1) is None
    assert called == []


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the CPU oracle on a bounded sample) prints
    one JSON line with the keys the driver reads."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "1", "--ref-total-s", "2"],
                       capture_output=True, text=True, timeout=600, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("{")][-1]
    d = json.loads(line)
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
