"""The multi-rank paths across ranks (CPU, gloo, world size 2): every rank sees
the slowest rank's timing; replicas count one layer per rank; a head-sharded
layer splits the heads into balanced contiguous slices, every rank derives the
same zone shapes from the replicated features, and the per-rank results
reassemble into the single-process result."""
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


def test_head_shard_partition():
    from dynamic_block_sparse_shape_b200.shard import head_shard, parse_head_slice
    for heads in (1, 2, 3, 7, 24):
        for world in range(1, heads + 1):
            spans = [head_shard(heads, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == heads
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)
    assert head_shard(24, 8, 7) == (21, 24)
    assert parse_head_slice("0:3", 24) == (0, 3)
    for bad in ((24, 0, 0), (24, 2, 2), (2, 3, 0)):
        with pytest.raises(ValueError):
            head_shard(*bad)
    import bench
    assert bench.whole_job_ms_per_layer(8.0, 4, "heads") == 8.0
    assert bench.whole_job_ms_per_layer(8.0, 4, "replicas") == 2.0


def _tiny_layer(heads=4):
    """Features, Q/K/V on a 4x8x16 grid (two zones), oracle stages end to end."""
    import numpy as np
    rng = np.random.default_rng(12)
    grid, zone = (4, 8, 16), (4, 8, 8)
    N, d = 4 * 8 * 16, 8
    F = rng.normal(size=(N, 32))
    Q, K, V = (rng.normal(size=(N, heads, d)) for _ in range(3))
    return grid, zone, F, Q, K, V


def _layer_outputs(grid, zone, F, Q, K, V, h0, h1):
    import math
    from oracle import prism_oracle as O
    cand = [(4, 4, 4), (2, 4, 8), (4, 8, 2), (1, 8, 8)]
    idx, _, _ = O.zone_shapes(grid, zone, cand, F=F)
    blocks = O.block_tokens(grid, zone, cand, idx)
    q, k, v = Q[:, h0:h1], K[:, h0:h1], V[:, h0:h1]
    sc = 1 / math.sqrt(q.shape[2])
    sel = O.block_select(O.block_pool(q, blocks), O.block_pool(k, blocks), sc, 1, 0.3)
    out, _ = O.masked_attention_fwd(q, k, v, O.token_mask(sel["mask"], blocks, q.shape[0]), sc)
    return idx, out


def _shard_rank(rank, world, init_file, out_dir):
    import numpy as np
    import torch
    from dynamic_block_sparse_shape_b200.shard import head_shard
    dist.init_process_group("gloo", init_method=f"file://{init_file}", rank=rank, world_size=world)
    try:
        grid, zone, F, Q, K, V = _tiny_layer()
        h0, h1 = head_shard(Q.shape[1], world, rank)
        idx, out = _layer_outputs(grid, zone, F, Q, K, V, h0, h1)
        shapes = [torch.zeros(len(idx), dtype=torch.int64) for _ in range(world)]
        dist.all_gather(shapes, torch.as_tensor(idx, dtype=torch.int64))
        parts = [torch.zeros((out.shape[0], 2, out.shape[2]), dtype=torch.float64) for _ in range(world)]
        dist.all_gather(parts, torch.as_tensor(out))
        if rank == 0:
            np.save(os.path.join(out_dir, "shapes.npy"), torch.stack(shapes).numpy())
            np.save(os.path.join(out_dir, "out.npy"), torch.cat(parts, dim=1).numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_head_sharded_layer_reassembles_gloo():
    import numpy as np
    world = 2
    with tempfile.TemporaryDirectory() as d:
        init_file = os.path.join(d, "init")
        mp.start_processes(_shard_rank, args=(world, init_file, d), nprocs=world, join=True, start_method="spawn")
        shapes = np.load(os.path.join(d, "shapes.npy"))
        out = np.load(os.path.join(d, "out.npy"))
    grid, zone, F, Q, K, V = _tiny_layer()
    idx, full = _layer_outputs(grid, zone, F, Q, K, V, 0, Q.shape[1])
    assert (shapes == idx[None, :]).all()  # every rank derived the same partition
    assert np.allclose(out, full, atol=1e-12)
