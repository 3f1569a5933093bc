"""Multi-process host logic on the CPU: world size 2, gloo backend, ranks as
spawned processes (no GPU).

* the row-sharded NVFP4 exchange (fp4_post_weight_grid_b200.sharded): each
  rank computes its local max, the ranks all-reduce it (MAX), each rank sweeps
  its own rows -- run here with the oracle standing in for the CUDA kernels --
  and every rank's rows must equal those rows of the single-process
  quantization of the whole weight;
* the row split covers every row exactly once;
* the benchmark's time reduction returns the slowest rank's time on every rank,
  and the ranks draw different synthetic replicas.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port):
    import sys
    for p in (ROOT, os.path.join(ROOT, "tests")):
        if p not in sys.path:
            sys.path.insert(0, p)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))


def _sharded_worker(rank, world, port, out_dir):
    _init(rank, world, port)
    try:
        import oracle
        import synth
        from fp4_post_weight_grid_b200.sharded import row_shard_protocol, shard_rows
        rows, cols = 37, 256
        w = synth.q_proj(rows, cols, seed=17).float().numpy()
        start, stop = shard_rows(rows, world, rank)
        mine = np.ascontiguousarray(w[start:stop])

        def local_absmax():
            return torch.tensor([float(oracle.global_absmax(mine))], dtype=torch.float32)

        def all_reduce_max(t):
            dist.all_reduce(t, op=dist.ReduceOp.MAX)

        def sweep(amax):
            return oracle.nvfp4_quant(mine, S=oracle.global_scale(np.float32(amax.item())))

        res = row_shard_protocol(local_absmax, all_reduce_max, sweep)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), start=start, stop=stop, codes=res["codes"],
                 scales=res["scales"], loss=res["loss"], S=np.float32(res["S"]))
    finally:
        dist.destroy_process_group()


def _timing_worker(rank, world, port, out_dir):
    _init(rank, world, port)
    try:
        import bench
        got = bench.max_over_ranks(1.5 + rank, dist, torch.device("cpu"))
        np.savez(os.path.join(out_dir, f"t{rank}.npz"), got=got, seed=bench.rank_seed(rank))
    finally:
        dist.destroy_process_group()


def test_row_split_covers_every_row_once():
    from fp4_post_weight_grid_b200.sharded import shard_rows
    for rows in (0, 1, 7, 37, 4096):
        for world in (1, 2, 3, 8):
            seen = []
            for r in range(world):
                a, b = shard_rows(rows, world, r)
                assert 0 <= a <= b <= rows
                seen.extend(range(a, b))
            assert seen == list(range(rows))
    with pytest.raises(ValueError):
        shard_rows(4, 2, 2)


def test_row_sharded_nvfp4_equals_unsharded(tmp_path, orc):
    world = 2
    mp.start_processes(_sharded_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    import synth
    w = synth.q_proj(37, 256, seed=17).float().numpy()
    full = orc.nvfp4_quant(w, S=orc.global_scale(orc.global_absmax(w)))
    covered = 0
    for r in range(world):
        d = np.load(tmp_path / f"rank{r}.npz")
        a, b = int(d["start"]), int(d["stop"])
        covered += b - a
        assert np.float32(d["S"]) == np.float32(full["S"])          # global scale of the whole weight
        assert np.array_equal(d["codes"], full["codes"][a:b])
        assert np.array_equal(d["scales"], full["scales"][a:b])
        assert np.array_equal(d["loss"].view(np.uint32), full["loss"][a:b].view(np.uint32))
    assert covered == 37


def test_bench_time_is_the_slowest_rank(tmp_path):
    world = 2
    mp.start_processes(_timing_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    seeds = set()
    for r in range(world):
        d = np.load(tmp_path / f"t{r}.npz")
        assert float(d["got"]) == 2.5
        seeds.add(int(d["seed"]))
    assert len(seeds) == world
