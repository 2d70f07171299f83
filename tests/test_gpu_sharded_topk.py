"""The sharded top-K kernels (fm_topk_shard_*) on one GPU: every row's chunks
are split into G consecutive slices, each slice driven as its own shard in
lockstep, with the two exchanges (sum of the histograms, gather of the tie
counts) done between the phases on the device by the test.  No kernel waits on
another shard's.  The union of the slices' masks must equal the top-K rule on
the whole rows, and fm_select_topk's mask on them."""
import numpy as np
import pytest
import torch

from tests import helpers as H

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from learned_kv_chunk_b200 import fm  # noqa: E402  (loads libfm.so; raises if missing)

DEV = torch.device("cuda", 0)


def sharded_mask(ens: torch.Tensor, n_valid: np.ndarray, k: int, cuts):
    """Runs the phases for the slices [cuts[g], cuts[g+1]) of every row."""
    shards = []
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        nv_local = torch.from_numpy(np.clip(n_valid - lo, 0, hi - lo).astype(np.int32)).to(DEV)
        shards.append(fm.TopKShard(ens[:, lo:hi].contiguous(), k, nv_local))
    for s in shards:
        s.begin()
    for p in range(3):
        total = torch.stack([s.hist_pass(p) for s in shards]).sum(0, dtype=torch.int32)
        for s in shards:
            s.hist.copy_(total)
            s.pick(p)
    eq_all = torch.stack([s.ties() for s in shards]).contiguous()
    keep = torch.cat([s.mask(eq_all, g) for g, s in enumerate(shards)], dim=1)
    torch.cuda.synchronize()
    return keep.cpu().numpy()


def _rows(kind: str, B: int, N: int, seed: int):
    g = torch.Generator().manual_seed(seed)
    if kind == "spread":
        return torch.rand(B, N, generator=g)
    if kind == "ties":  # few distinct values: the K-th value's ties span the slices
        return torch.randint(0, 24, (B, N), generator=g).float() / 24.0
    return torch.full((B, N), 0.5)  # all equal


@pytest.mark.parametrize("kind", ["spread", "ties", "equal"])
@pytest.mark.parametrize("G", [2, 3, 4])
def test_sharded_topk_matches_whole_row_rule(kind, G):
    B, N = 5, 3 * 8192 + 77  # several blocks per slice and a ragged tail
    ens = _rows(kind, B, N, 40 + G)
    nv = np.array([N, N - 5000, 100, 0, 9000], np.int32)  # row 2 lives in the first slice only
    rng = np.random.default_rng(G)
    cuts = [0] + sorted(rng.choice(np.arange(1, N), G - 1, replace=False).tolist()) + [N]
    ens_d = ens.to(DEV)
    for k in (1, 37, 4096, 9000, 30000):
        keep = sharded_mask(ens_d, nv, k, cuts)
        H.check_topk_against_rule(keep, ens.numpy(), nv, k)
        whole = fm.fm_select_topk(ens_d, k, torch.from_numpy(nv).to(DEV)).cpu().numpy()
        np.testing.assert_array_equal(keep, whole)


def test_sharded_topk_one_long_row_over_eight_shards():
    """One row of 262144 chunks, K = 2048 (the single-row workload), in eight
    equal slices; then in three slices, the middle one a single chunk."""
    N, k = 262144, 2048
    ens = _rows("spread", 1, N, 9)
    nv = np.array([N], np.int32)
    for cuts in ([i * N // 8 for i in range(9)], [0, 1000, 1001, N]):
        keep = sharded_mask(ens.to(DEV), nv, k, cuts)
        H.check_topk_against_rule(keep, ens.numpy(), nv, k)
