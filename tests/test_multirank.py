"""Multi-rank host logic of bench.py on CPU with the gloo backend, world size
2: every rank draws its own keys (weak scaling, no collective on the data
path), and the job's time is the max over ranks, which every rank agrees on."""
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


def _worker(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from gen import synthetic as G
        # each rank's own (small) key slab, from its rank-specific seed
        seed = bench.rank_key_seed(1234, rank)
        keys = G.make_keys(seed, [300, 257], 300, 3, None, device="cpu")
        # a per-rank "elapsed time"; the job's time is the slowest rank's
        elapsed = [12.5, 17.25][rank]
        mx = bench.max_over_ranks(elapsed, world, "cpu")
        value = bench.job_throughput(557, world, 4, mx)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), keys0=keys[0].numpy(), mx=mx, value=value,
                 seed=seed)
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, start_method="spawn", join=True)
    r0 = np.load(tmp_path / "rank0.npz")
    r1 = np.load(tmp_path / "rank1.npz")
    assert float(r0["mx"]) == float(r1["mx"]) == 17.25
    # whole-job throughput: both ranks' decisions over the slowest rank's time
    assert float(r0["value"]) == float(r1["value"]) == pytest.approx(557 * 2 * 4 / 17.25e-3)
    assert int(r0["seed"]) != int(r1["seed"])
    assert r0["keys0"].shape == r1["keys0"].shape
    assert not np.array_equal(r0["keys0"], r1["keys0"])  # each rank scores its own batch


def test_single_rank_needs_no_process_group():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.job_throughput(100, 1, 2, 1000.0) == pytest.approx(200.0)
