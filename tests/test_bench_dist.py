"""The multi-process side of bench.py on CPU (gloo, world size 2): the max-over-ranks step time,
the whole-job throughput of replicas, and the reference arm under torchrun, where rank 0 alone
runs the oracle and prints the JSON line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, values, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    assert bench.dist_env() == (world, rank, rank)
    bench.init_dist(rank)
    assert dist.get_backend() == "gloo"
    m = bench.max_over_ranks(values[rank], world, "cpu")
    out[rank] = (m, bench.throughput(world, m))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_replica_throughput():
    world, values = 2, [3.5, 7.25]  # ms per step seen by each rank
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), values, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        m, v = res[rank]
        assert m == max(values)            # every rank sees the slowest replica's time
        assert v == pytest.approx(world * 1e3 / max(values))


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(4.0, 1, "cpu") == 4.0
    assert bench.throughput(1, 4.0) == pytest.approx(250.0)


def test_reference_arm_under_torchrun_prints_once():
    env = dict(os.environ, OMP_NUM_THREADS="2", CUDA_VISIBLE_DEVICES="")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}", "bench.py",
           "--impl", "reference", "--workload", "tiny", "--gpus", "2", "--steps", "1",
           "--warmup", "3"]
    p = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout  # rank 0 alone prints
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
