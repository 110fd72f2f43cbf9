"""Host logic of the multi-GPU bench on CPU: N replicas, no collective on the data path,
the time taken as the max over ranks and the throughput summed over replicas.  Two
gloo ranks on 127.0.0.1."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import bench
    import synth
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(1.5 + rank, world)       # rank 1 is the slow one
        bench.barrier(world)
        x = synth.activation(64, 256, "student_t", seed=bench.replica_seed(1, rank), device="cpu",
                             outlier_frac=0.01, outlier_scale=50.0)
        torch.save({"ms": ms, "x": x, "tflops": bench.job_tflops(2e12, ms, world)},
                   os.path.join(out_dir, "rank%d.pt" % rank))
    finally:
        dist.destroy_process_group()


def test_two_gloo_replicas(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    r = [torch.load(os.path.join(tmp_path, "rank%d.pt" % i)) for i in range(world)]
    # every rank sees the slowest rank's time
    assert r[0]["ms"] == r[1]["ms"] == 2.5
    # whole-job throughput: both replicas' work over the slowest time
    assert r[0]["tflops"] == pytest.approx(2 * 2e12 / 2.5e-3 / 1e12)
    # each replica quantizes its own batch
    assert not torch.equal(r[0]["x"], r[1]["x"])


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr
    assert p.stdout.strip() == ""
