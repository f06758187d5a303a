"""bench.py's multi-rank host logic on world_size 2 with the gloo backend (CPU).

Each rank of a data-parallel run processes its own batch (no collective on the
data path); the only collective is the max over ranks of the timed region.
"""
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank], world, "cpu")
        out[rank] = got
        out[10 + rank] = bench.rank_seed(rank)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_seeds_gloo():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == [2.0, 10.0] and res[1] == [2.0, 10.0]
    assert res[10] != res[11]  # each rank draws a different batch


def _stub_rank(rank, world, out):
    """One rank of a two-rank job with a stubbed step: rank r 'took' 10 + 5 r ms for 4
    steps; the line comes from the max over ranks, as bench.py's own ranks build it."""
    sys.path.insert(0, ROOT)
    import bench
    ms, e2e_ms = bench.max_over_ranks([10.0 + 5.0 * rank, 40.0 - rank], world, "cpu")
    if rank == 0:
        out["line"] = bench.build_line(bench.WORKLOAD, world, 4, 3, ms, (e2e_ms, 2, 123), 4,
                                       None, None)
    out[f"env{rank}"] = (os.environ["RANK"], os.environ["WORLD_SIZE"], os.environ["MASTER_ADDR"])


def test_spawned_ranks_report_one_line_over_both_ranks():
    """bench.launch_ranks (used by --gpus N without an outer torchrun) forms a two-rank
    gloo group; the reported value counts both ranks' images over the slower rank's time."""
    sys.path.insert(0, ROOT)
    import bench
    with mp.Manager() as m:
        out = m.dict()
        bench.launch_ranks(2, _stub_rank, out, backend="gloo")
        res = dict(out)
    line = res["line"]
    c = bench.WORKLOAD
    assert line["n_gpus"] == 2 and line["steps"] == 4 and line["scaling"] == "weak"
    assert abs(line["ms_per_step"] - 15.0 / 4) < 1e-12  # the slower rank
    assert abs(line["value"] - c.flops() * 2 * 4 / 15e-3 / 1e12) < 1e-9 * line["value"]
    assert abs(line["e2e"]["ms_per_step"] - 40.0 / 2) < 1e-12
    assert res["env0"] == ("0", "2", "127.0.0.1") and res["env1"] == ("1", "2", "127.0.0.1")


def test_max_over_ranks_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 4.0], 1) == [3.0, 4.0]


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_line_shape():
    """Rank 0 of the reference arm prints one JSON line with the contract's keys."""
    import json
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "dtype", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert torch.tensor(line["value"]).isfinite()
