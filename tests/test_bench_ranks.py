"""The replica-only multi-GPU logic of bench.py on CPU: two gloo ranks (no GPU).

Every rank runs its own replica; the job's time is the maximum over ranks, every rank takes the
same collective steps, and the reference arm runs on rank 0 only.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

pytestmark = pytest.mark.cpu


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        bench.barrier(world)
        ms = bench.max_over_ranks(1.5 + rank, world, device="cpu")
        bench.barrier(world)
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(repr(ms))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_barrier_with_two_gloo_ranks(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    got = [float(open(tmp_path / f"r{r}.txt").read()) for r in range(2)]
    assert got == [2.5, 2.5]


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import argparse
    import bench
    from mixture_experts_decode_gemv_b200.synthetic import CONFIGS
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    args = argparse.Namespace(m=1, steps=1, warmup=0)
    bench.run_reference(args, CONFIGS["tiny"], 1)
    assert capsys.readouterr().out == ""


def test_both_arms_print_the_same_config():
    import bench
    from mixture_experts_decode_gemv_b200.synthetic import CONFIGS
    c = CONFIGS["llama4_scout"]
    assert bench.config_dict(c, 64, 1) == bench.config_dict(c, 64, 1)
    assert set(bench.config_dict(c, 64, 1)) == {"workload", "m", "weights", "l2_policy",
                                                 "parallelism"}


def test_single_rank_helpers_need_no_process_group():
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25
    bench.barrier(1)
