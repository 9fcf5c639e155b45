"""The bench's multi-rank plumbing on CPU: two gloo ranks, no GPU.

The path shards by sequence (every rank runs its own replica of the workload, no collective on the
data path), so what has to hold across ranks is the timing contract: every rank takes the same
reductions in the same order, the slowest rank's device time sets the job time, the job rate counts
the units of all ranks, and each replica draws its own inputs.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        mine = [12.5, 40.0][rank]       # per-rank device time of the timed region (ms)
        e2e = [30.0, 21.0][rank]
        total = bench.max_over_ranks(mine, world, "cpu")
        total_e2e = bench.max_over_ranks(e2e, world, "cpu")
        rate = bench.job_rate(64, world, 20, total)
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"total": total, "e2e": total_e2e, "rate": rate,
                       "seed": bench.replica_seed(0, rank)}, f)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_rank_timing_takes_the_slowest_rank(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    for r in res:
        assert r["total"] == 40.0 and r["e2e"] == 30.0  # both ranks see the max
        # 64 units per rank-step, 2 ranks, 20 steps over the slowest rank's 40 ms
        assert r["rate"] == pytest.approx(64 * 2 * 20 / 0.040)
    assert res[0]["seed"] != res[1]["seed"]  # each replica draws its own sequences


def test_job_rate_is_weak_scaling():
    # the same per-rank time with twice the ranks is twice the job rate
    assert bench.job_rate(32, 2, 10, 5.0) == pytest.approx(2 * bench.job_rate(32, 1, 10, 5.0))


def test_sweep_workload_names():
    c = bench.workload_config("sweep_dsa_4096")
    assert (c.L, c.sink, c.swa, c.K_sparse, c.M, c.layers) == (4096, 0, 0, 2048, 0, 1)
    c = bench.workload_config("sweep_lsa_262144")
    assert (c.L, c.sink, c.swa, c.K_sparse, c.M, c.layers) == (262144, 16, 1024, 1008, 1024, 2)
    with pytest.raises(SystemExit):
        bench.workload_config("sweep_xyz_4096")
    # the pooling ablation's setting (Table 11): 128K decode, M = 128 pages
    c = bench.workload_config("table11_minmax_8")
    assert (c.L, c.B, c.M, c.sub_block, c.page) == (131072, 32, 128, 8, 128)
    assert bench.workload_config("table11_mean_16").sub_block == 16
    with pytest.raises(SystemExit):
        bench.workload_config("table11_max_8")


def test_reference_arm_under_torchrun_two_ranks():
    """`bench.py --impl reference` launched as two ranks: rank 0 alone times the oracle and
    prints one JSON line; the other rank exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--workload", "sweep_dsa_4096", "--cpu-budget", "0.05"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    p = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["value"] > 0 and line["e2e"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"] == "sweep_b8_4096_dsa"


def test_training_workload_names_and_key_counts():
    """train_<L> parses to the Table 2 shape, and the |S_t| the backward's flop count uses equals
    the sizes of the oracle's region split (sink + window + min(K_sparse, dyn)) at every position,
    including the short rows at the start of the sequence."""
    import numpy as np

    import oracle
    cfg = bench.workload_config("train_8192")
    assert (cfg.B, cfg.T, cfg.L, cfg.H, cfg.K_sparse) == (1, 8192, 8192, 128, 1008)
    with pytest.raises(SystemExit):
        bench.workload_config("train_x")
    t = np.arange(0, 3000)
    got = bench.attended_keys(t, cfg.sink, cfg.swa, cfg.K_sparse)
    for ti in list(range(0, 40)) + [1038, 1039, 1040, 1041, 2047, 2048, 2063, 2064, 2999]:
        (s0, s1), (w0, w1), (d0, d1) = oracle.regions(ti, cfg.sink, cfg.swa)
        want = (s1 - s0) + (w1 - w0) + min(cfg.K_sparse, max(0, d1 - d0))
        assert got[ti] == want, ti
    assert got[2999] == 2048


def test_scorer_traffic_only_for_the_captured_source(monkeypatch):
    """The roofline's DRAM traffic is reported only for the scorer source its ncu capture was
    taken on; any other source gets null and the reason."""
    sha = bench.scorer_source_sha()
    assert len(sha) == 16
    monkeypatch.setitem(bench.SCORER_TRAFFIC, "w",
                        {"bytes": 1.0e9, "source_sha": sha, "how": "a capture"})
    assert bench.scorer_traffic("w") == (1.0e9, "a capture")
    monkeypatch.setitem(bench.SCORER_TRAFFIC, "w",
                        {"bytes": 1.0e9, "source_sha": "0" * 16, "how": "a capture"})
    b, why = bench.scorer_traffic("w")
    assert b is None and "changed" in why
    assert bench.scorer_traffic("no_such_workload") == (None, None)
