"""The replica path across ranks (CPU, gloo, world size 2): every rank sees the
slowest rank's timing, and the whole-job value counts one layer per rank."""
import os
import tempfile

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _rank(rank, world, init_file, out_dir):
    import bench
    dist.init_process_group("gloo", init_method=f"file://{init_file}", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(10.0 + 7.5 * rank)
        value = bench.whole_job_ms_per_layer(got, world)
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(f"{got} {value}")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_gloo():
    world = 2
    with tempfile.TemporaryDirectory() as d:
        init_file = os.path.join(d, "init")
        mp.start_processes(_rank, args=(world, init_file, d), nprocs=world, join=True, start_method="spawn")
        vals = [open(os.path.join(d, f"r{r}.txt")).read().split() for r in range(world)]
    for got, value in vals:
        assert float(got) == pytest.approx(17.5)
        assert float(value) == pytest.approx(17.5 / 2)


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.whole_job_ms_per_layer(8.0, 1) == 8.0
