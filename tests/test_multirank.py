"""The multi-GPU host path of bench.py on CPU: two gloo ranks.

bench.py runs one independent replica per GPU (the path has no exchange step)
and reports the whole-job throughput as the total work of all ranks over the
slowest rank's time.  Here two gloo ranks check the max-over-ranks reduction
and the aggregate that bench.py uses, without a GPU.
"""
import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, out_path):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        ms = [3.0, 5.0][rank]                       # rank 1 is the slower one
        t = bench.max_over_ranks(ms, dist, torch.device("cpu"))
        flops = [2.0e12, 2.0e12][rank]
        value, t_max = bench.aggregate([t, t], [flops, flops])
        dist.barrier()
        if rank == 0:
            with open(out_path, "w") as f:
                f.write(f"{t} {value} {t_max}\n")
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time(tmp_path):
    out = tmp_path / "result.txt"
    port = 29500 + (os.getpid() % 2000)
    mp.start_processes(_rank_main, args=(2, port, str(out)), nprocs=2, join=True, start_method="spawn")
    t, value, t_max = map(float, out.read_text().split())
    assert t == 5.0 and t_max == 5.0
    # 2 ranks x 2 TFLOP over 5 ms = 800 TFLOP/s
    assert value == pytest.approx(800.0)


def test_max_over_ranks_without_a_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1.25, None, torch.device("cpu")) == 1.25


def test_kernel_launch_count_per_step():
    sys.path.insert(0, ROOT)
    import bench
    from block_sparse_attention_fractal_b200 import synth
    assert bench.kernel_launches_per_step(synth.WORKLOADS["wan480p"]) == 8
    assert bench.kernel_launches_per_step(synth.WORKLOADS["hunyuan720p"]) == 7
    assert bench.kernel_launches_per_step(synth.WORKLOADS["density_sweep"]) == 6
