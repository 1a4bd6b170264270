"""The multi-rank path of the benchmark on CPU: two gloo ranks run the same
setup, barrier and max-over-ranks timing as the NCCL ranks on GPUs, and each
rank draws its own independent sequence (weak scaling, no data-path
collective)."""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    from gen import full_inputs, get_config

    w, r, _ = bench.dist_setup(world, backend="gloo")
    assert (w, r) == (world, rank)
    # the slowest rank sets the time
    t = bench.max_over_ranks(10.0 + rank, w)
    # independent inputs per rank: a small instance drawn with the rank's seed
    cfg = get_config("prefill").with_(seq=256, heads=4, kv_heads=1)
    q = full_inputs(cfg, device="cpu", seed=bench.rank_seed(cfg, r))["q"].float()
    sums = [torch.zeros(1, dtype=torch.float64) for _ in range(w)]
    dist.all_gather(sums, q.double().sum().reshape(1))
    bench.barrier(w)
    res = {"rank": r, "t": t, "sums": [float(x) for x in sums],
           "value": bench.job_throughput(cfg.seq, w, t)}
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump(res, f)
    bench.finish(w)


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    for r in res:
        assert r["t"] == 10.0 + (world - 1)  # max over ranks, on every rank
        assert r["value"] == pytest.approx(256 * world / (r["t"] * 1e-3))
    # both ranks saw the same gathered checksums, and the ranks' inputs differ
    assert res[0]["sums"] == res[1]["sums"]
    assert res[0]["sums"][0] != res[0]["sums"][1]


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr[-2000:]
    assert p.stdout.strip() == ""
