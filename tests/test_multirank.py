"""The N > 1 plumbing of bench.py on the host: world-size-2 gloo process groups.

The attention path shards with no exchange (each rank runs its own replica on its
own inputs), so the only cross-rank steps are the barrier around the timed region,
the max over ranks of the elapsed time, and rank 0 alone printing.  These tests run
that plumbing on CPU ranks; nothing here needs a GPU.
"""
import multiprocessing as mp
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, elapsed, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    try:
        w, r, _ = bench.dist_setup(world, backend="gloo")
        bench.barrier(w)
        ms = bench.max_over_ranks(elapsed[r], w)
        bench.barrier(w)
        q.put((r, w, ms, bench.aggregate_gbs(w, 1e9, 10, ms)))
    except Exception as e:  # reported to the parent, which fails the test
        q.put(("error", rank, repr(e)))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def _run_ranks(world, elapsed):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, elapsed, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert not [o for o in out if o[0] == "error"], out
    return sorted(out)


def test_max_over_ranks_and_barrier_gloo():
    """Every rank gets the slowest rank's time; the whole-job rate divides all
    ranks' bytes by it."""
    out = _run_ranks(2, [3.0, 5.0])
    assert [o[0] for o in out] == [0, 1]
    for r, w, ms, gbs in out:
        assert w == 2 and ms == 5.0
        assert gbs == pytest.approx(2 * 1e9 * 10 / 5e-3 / 1e9)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert bench.aggregate_gbs(1, 2e9, 4, 8.0) == pytest.approx(1000.0)


def test_reference_arm_on_a_nonzero_rank_exits_quietly():
    """Under torchrun only rank 0 runs and prints the reference line."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "1"], env=env, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_cpulist_parsing():
    """The e2e leg reads the GPU's NUMA-local CPUs from a sysfs CPU list."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.parse_cpulist("0-3,8,10-11\n") == {0, 1, 2, 3, 8, 10, 11}
    assert bench.parse_cpulist("5") == {5}
    assert bench.parse_cpulist("") == set()


def test_reference_arm_line_has_the_contract_keys():
    """`bench.py --impl reference` (the float64 oracle on host cores) prints one
    JSON line with the contract's keys, its own cpu_baseline and a zero-copy e2e."""
    import json
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(k, None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "1"], env=env, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 1 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert "workload" in d["config"]
