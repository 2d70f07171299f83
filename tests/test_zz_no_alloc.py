"""fm_select_topk_static -- the top-K keep mask for callers that cannot
allocate device memory (a serving process whose memory is all handed to its
KV-cache pool, a plugin inside another framework's allocator, a decode loop
that cannot afford cudaMalloc's device synchronisation).  It takes its
scratch from a fixed array inside the library instead of a caller workspace.

Checked through the C ABI against fm_select_topk (the workspace entry point)
on two calls in a row with different shapes, so the second call starts from
whatever the first left in the shared array.  Masks are integer results:
they must match exactly.  This file is named to be collected last."""
import numpy as np
import pytest
import torch

from tests import helpers as H

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from learned_kv_chunk_b200 import fm  # noqa: E402  (loads libfm.so; raises if missing)

DEV = torch.device("cuda", 0)


def _scores(seed: int, B: int, N: int, levels: int) -> torch.Tensor:
    """Sigmoid-range scores with many exact ties (values on a coarse grid)."""
    g = torch.Generator().manual_seed(seed)
    return (torch.randint(0, levels, (B, N), generator=g).float() / levels).to(DEV)


CALLS = [  # (seed, B, N, n_valid, k, grid levels)
    (501, 6, 70001, [70001, 69000, 4097, 1, 0, 12345], 2048, 1000),
    (502, 3, 20000, [20000, 19999, 7777], 300, 7),  # heavy ties: the K-th value is split
]


def test_static_topk_matches_workspace_topk_twice():
    torch.cuda.set_device(DEV)
    for seed, B, N, nv, k, levels in CALLS:
        ens = _scores(seed, B, N, levels)
        n_valid = torch.tensor(nv, dtype=torch.int32, device=DEV)
        ref = fm.fm_select_topk(ens, k, n_valid)
        out = torch.full((B, N), True, dtype=torch.bool, device=DEV)
        got = fm.fm_select_topk_static(ens, k, n_valid, out=out)
        torch.cuda.synchronize()
        assert got.data_ptr() == out.data_ptr()
        assert torch.equal(got, ref), int((got != ref).sum())
        H.check_topk_against_rule(got.cpu().numpy(), ens.cpu().numpy(), nv, k)


def test_static_topk_rejects_sizes_beyond_its_scratch():
    B, N = 300, 262144
    assert fm.fm_topk_workspace_bytes(B, N) > (4 << 20)
    ens = torch.zeros(B, N, dtype=torch.float32, device=DEV)
    out = torch.zeros(B, N, dtype=torch.bool, device=DEV)
    with pytest.raises(fm.FMError) as exc:
        fm.fm_select_topk_static(ens, 10, None, out=out)
    assert exc.value.status == fm.FM_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert not bool(out.any())  # nothing was launched
