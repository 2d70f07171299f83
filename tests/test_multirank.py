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


# ---------------------------------------------------------------- sharded top-K
# The chunks of each row are split over two gloo ranks; fm_select_topk_sharded
# runs its real exchange protocol (a histogram all-reduce per radix pass, then
# an all-gather of the tie counts).  The GPU phases cannot run here, so each
# rank drives a host stand-in with the same phase contract (the kernels'
# version is checked on the GPU in test_gpu_sharded_topk.py); the union of the
# ranks' masks must equal the oracle's top-K of the whole rows.
class _HostShard:
    PASSES = [(21, 11), (10, 11), (0, 10)]  # (shift, bits) of the three digits

    def __init__(self, ens_local, k, n_valid_local):
        self.ens = np.ascontiguousarray(ens_local, dtype=np.float32)
        self.B, self.N = self.ens.shape
        self.k = int(k)
        self.nv = np.asarray(n_valid_local)
        self.hist = torch.zeros(self.B, 2048, dtype=torch.int32)
        self.eq_local = torch.zeros(self.B, dtype=torch.int32)

    def _keys(self, b):
        u = self.ens[b, :self.nv[b]].view(np.uint32).astype(np.int64)
        return u | (1 << 31)  # scores >= 0: the bit pattern is monotone

    def begin(self):
        self.mode = ["select"] * self.B
        self.prefix = [0] * self.B
        self.rem = [self.k] * self.B
        self.need = [0] * self.B
        self.cnt = [0] * self.B
        self.hist.zero_()

    def hist_pass(self, p):
        shift, bits = self.PASSES[p]
        hi = shift + bits
        self.hist.zero_()
        for b in range(self.B):
            if self.mode[b] != "select":
                continue
            keys = self._keys(b)
            if hi < 32:
                keys = keys[(keys >> hi) == (self.prefix[b] >> hi)]
            digits = (keys >> shift) & ((1 << bits) - 1)
            self.hist[b, :1 << bits] = torch.from_numpy(np.bincount(digits, minlength=1 << bits).astype(np.int32))
        return self.hist

    def pick(self, p):
        shift, bits = self.PASSES[p]
        for b in range(self.B):
            if self.mode[b] != "select":
                continue
            h = self.hist[b, :1 << bits].numpy().astype(np.int64)
            if p == 0 and (h.sum() == 0 or self.rem[b] >= h.sum()):
                self.mode[b] = "empty" if h.sum() == 0 else "all"
                continue
            acc = 0
            for d in range((1 << bits) - 1, -1, -1):
                if acc + h[d] >= self.rem[b]:
                    self.prefix[b] |= d << shift
                    self.rem[b] -= acc
                    if p == 2:
                        self.need[b], self.cnt[b] = self.rem[b], int(h[d])
                    break
                acc += h[d]

    def ties(self):
        for b in range(self.B):
            split = self.mode[b] == "select" and self.need[b] != self.cnt[b]
            self.eq_local[b] = int((self._keys(b) == self.prefix[b]).sum()) if split else 0
        return self.eq_local

    def mask(self, eq_all, shard):
        keep = np.zeros((self.B, self.N), bool)
        for b in range(self.B):
            n = int(self.nv[b])
            if self.mode[b] == "all":
                keep[b, :n] = True
            elif self.mode[b] == "select":
                keys = self._keys(b)
                eq = keys == self.prefix[b]
                rank = int(eq_all[:shard, b].sum()) + np.cumsum(eq) - 1
                keep[b, :n] = (keys > self.prefix[b]) | (eq & (rank < self.need[b]))
        return keep


def _sharded_rows(seed):
    """Three rows of 700 chunks: spread scores, scores on a coarse grid (ties
    at the K-th value split across the ranks), and a short row; ragged."""
    rng = np.random.default_rng(seed)
    N = 700
    ens = np.zeros((4, N), np.float32)
    ens[0] = rng.random(N, dtype=np.float32)
    ens[1] = rng.integers(0, 6, N).astype(np.float32) / 8
    ens[2] = rng.random(N, dtype=np.float32)
    ens[3] = rng.integers(0, 3, N).astype(np.float32) / 4
    n_valid = np.array([700, 650, 120, 700], np.int32)
    return ens, n_valid


def _sharded_worker(rank, world, port, out_dir, split, k):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import importlib.util
        spec = importlib.util.spec_from_file_location("fm_binding", os.path.join(ROOT, "learned_kv_chunk_b200", "fm.py"))
        fm = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(fm)
        ens, n_valid = _sharded_rows(77)
        lo, hi = (0, split) if rank == 0 else (split, ens.shape[1])
        nv_local = np.clip(n_valid - lo, 0, hi - lo)
        shard = _HostShard(ens[:, lo:hi], k, nv_local)
        keep = fm.fm_select_topk_sharded(None, k, exchange=fm.TorchDistExchange(), shard=shard)
        np.save(os.path.join(out_dir, f"keep{rank}.npy"), keep)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("split,k", [(350, 300), (101, 300), (600, 64), (350, 5000)])
def test_sharded_topk_two_ranks_gloo(tmp_path, split, k):
    port = _free_port()
    mp.start_processes(_sharded_worker, args=(2, port, str(tmp_path), split, k), nprocs=2,
                       start_method="spawn", join=True)
    keep = np.concatenate([np.load(tmp_path / "keep0.npy"), np.load(tmp_path / "keep1.npy")], axis=1)
    import sys
    sys.path.insert(0, ROOT)
    from oracle import retriever as O
    ens, n_valid = _sharded_rows(77)
    want = O.select_topk(ens, n_valid, k)
    assert np.array_equal(keep, want)
    assert (keep.sum(1) == np.minimum(k, n_valid)).all()
