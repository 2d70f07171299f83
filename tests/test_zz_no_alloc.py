"""fm_select_topk_static -- the top-K keep mask for callers that cannot
allocate device memory (a serving process whose memory is all handed to its
KV-cache pool, a plugin inside another framework's allocator, a decode loop
that cannot afford cudaMalloc's device synchronisation).  It takes its
scratch from a fixed array inside the library instead of a caller workspace.

Checked through the C ABI against fm_select_topk (the workspace entry point)
on calls in a row with different shapes, so each call starts from whatever
the one before it left in the shared array.  The first call takes the
histogram form (the array cannot also hold its candidate lists); the second
the candidate path, right after it, so it starts from the row states and
counts the earlier call left behind; the others alternate between the
histogram form and the one-kernel form for rows of up to 16384 chunks,
which uses no scratch.  Masks are integer results:
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
    (501, 40, 300000, [300000, 299999, 4097, 1, 0] + [300000 - 7 * i for i in range(35)], 2048, 1000),
    (502, 2, 300000, [300000, 123457], 1000, 1000),  # the candidate path, after a histogram-form call
    (503, 5, 16384, [16384, 16000, 300, 1, 0], 700, 9),  # one kernel, heavy ties
    (504, 3, 20000, [20000, 19999, 7777], 300, 7),  # heavy ties: the K-th value is split
    (505, 6, 4000, [4000, 3999, 77, 2, 1, 0], 100, 1000),
]
STATIC_BYTES = 4 << 20


def _form(B: int, N: int, k: int) -> str:
    """The form fm_select_topk_static takes (include/fm.h): rows of up to
    16384 chunks the one-kernel form, which needs no scratch; longer rows the
    candidate path when the fixed array also holds the candidate lists and
    2k + 1024 <= min(16384, max(256, ceil(N / 16))), else the histogram
    form."""
    if N <= 16384:
        return "one-kernel"
    cap = min(16384, max(256, (N + 15) // 16))
    if fm.fm_topk_workspace_bytes_fast(B, N) <= STATIC_BYTES and 2 * k + 1024 <= cap:
        return "candidate"
    return "histogram"


def test_static_topk_calls_cover_every_form():
    forms = [_form(B, N, k) for _, B, N, _, k, _ in CALLS]
    assert forms == ["histogram", "candidate", "one-kernel", "histogram", "one-kernel"], forms
    assert all(fm.fm_topk_workspace_bytes(B, N) <= STATIC_BYTES for _, B, N, _, _, _ in CALLS)


def test_static_topk_matches_workspace_topk_in_a_row():
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
