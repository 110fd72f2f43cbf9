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


def test_step_statistics():
    sys.path.insert(0, ROOT)
    import bench
    st = bench.step_stats([3.0, 1.0, 2.0, 10.0, 4.0, 5.0, 6.0, 7.0, 8.0, 9.0, 2.5])
    assert st["min"] == 1.0 and st["median"] == 5.0 and st["n"] == 11
    assert st["p90"] == 9.0          # the 10th of 11 sorted values
    assert st["mean"] == round(sum([3, 1, 2, 10, 4, 5, 6, 7, 8, 9, 2.5]) / 11, 4)


def test_block_roofline_burst_and_sustained():
    """A block's tensor floor: each linear's FLOPs at 4x (W4A4) or 2x (W4A8) the bf16
    figure, burst or sustained; an all-W4A4 block at 4 PFLOP/s bf16 takes its FLOPs / 16e15."""
    sys.path.insert(0, ROOT)
    import bench
    import synth
    M, ctx = 75600, 512
    peaks = {"bf16_tflops": 4000.0, "bf16_tflops_sustained": 3000.0}
    burst = bench.linears_roofline_ms(synth, M, ctx, 0x00, peaks)
    assert abs(burst - synth.block_flops(M, ctx) / 16e15 * 1e3) < 1e-9
    assert abs(bench.linears_roofline_ms(synth, M, ctx, 0x00, peaks, sustained=True) - burst * 4 / 3) < 1e-9
    # every linear in W4A8 halves the rate
    assert abs(bench.linears_roofline_ms(synth, M, ctx, 0xFF, peaks) - 2 * burst) < 1e-9
    # no sustained figure: the burst one stands in
    assert bench.linears_roofline_ms(synth, M, ctx, 0x00, {"bf16_tflops": 4000.0}, sustained=True) == burst


def test_reference_arm_prints_one_line_with_its_own_baseline():
    """Rank 0 of the reference arm: the CPU oracle on a bounded sample, one JSON line with the
    same metric, impl "reference", an e2e that is the line's own value and no device copies."""
    import json
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--workload", "small_w4a4", "--ref-step-seconds", "0.5"],
                       capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr
    line = json.loads(p.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["e2e"]["value"] == line["value"] and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
