"""The CUDA path on the edge cases the pages leave open, against the oracle:
negative per-chunk scales (the scale is a plain fp32 in the README's
"compressed_k format", so nothing keeps it non-negative; the relu acts on
the scaled dot product) and NaN values (an e4m3 NaN code S.1111.111 or a NaN
scale makes the chunk's score NaN; the max and mean ensembles carry it; top-K
ranks NaN below every number, ties by chunk index; NaN > thr is false)."""
import numpy as np
import pytest
import torch

import oracle.retriever as O
from gen import synthetic as G
from tests import helpers as H

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from learned_kv_chunk_b200 import fm  # noqa: E402  (loads libfm.so; raises if missing)

DEV = torch.device("cuda", 0)
NAN_SCALE = np.array([np.nan], "<f4").view(np.uint8)


@pytest.fixture(scope="module")
def weights():
    return G.make_weights(4343, 3)


@pytest.fixture(scope="module", params=[2, 3], ids=["pieces2", "pieces3"])
def retr(request, weights):
    r = fm.Retriever(weights, device=0, max_batch=8, q_pieces=request.param)
    yield r
    r.close()


def _negate_scales(t: torch.Tensor, b: int, idx):
    """Flips the sign bit of the little-endian fp32 scale of the given chunks."""
    t[b, idx, 131] ^= 0x80


def test_negative_scales_match_oracle(retr, weights):
    # Scores are formed per warp of 32 chunk rows (rows 32w .. 32w+31 of a
    # 128-chunk tile); a warp with any negative scale takes the exact
    # relu(s * dot) branch.  Cover a whole warp, a mixed warp, a ragged last
    # tile, and a row whose every scale is negative.
    case = H.make_case(3, 1001, [1001, 1001, 700], seed=31, weights=weights)
    for l, t in enumerate(case.comp_k):
        _negate_scales(t, 0, list(range(128, 160)))             # tile 1, warp 0: all negative
        _negate_scales(t, 0, [300 + l, 305, 317, 319])           # tile 2, warp 1: mixed
        _negate_scales(t, 0, list(range(896 + 64, 1001, 3)))     # last, ragged tile
        _negate_scales(t, 1, list(range(0, 1001)))               # the whole row
    for t in case.comp_k:
        assert (t[:, :1001, 131] & 0x80).any()
    keys = [k.to(DEV) for k in case.comp_k]
    q, w = retr.fm_query_prep(case.hidden.to(DEV), case.positions.to(DEV))
    nv = case.n_valid.to(DEV)
    scores = retr.fm_score(keys, q, w, n_valid=nv, N=case.N)
    ens, keep_thr, _ = retr.fm_score_fused(keys, q, w, mode="mean", threshold=0.5, n_valid=nv, N=case.N)
    torch.cuda.synchronize()
    retr.fm_sync_status()
    s_o = H.oracle_scores(case)
    s_g = scores.cpu().numpy().astype(np.float64)
    assert np.abs(s_g - s_o).max() <= H.SCORE_TOL, np.abs(s_g - s_o).max()
    e_g = ens.cpu().numpy()
    assert np.abs(e_g - O.ensemble(s_o, "mean")).max() <= H.SCORE_TOL
    np.testing.assert_array_equal(keep_thr.cpu().numpy(), O.select_threshold(e_g, case.n_valid.numpy(), 0.5))
    # the negative scales matter: the same chunks with positive scales score differently
    flipped = H.make_case(3, 1001, [1001, 1001, 700], seed=31, weights=weights)
    assert np.abs(H.oracle_scores(flipped)[:, 1] - s_o[:, 1]).max() > 10 * H.SCORE_TOL


def test_nan_codes_and_scales(retr, weights):
    case = H.make_case(2, 900, [900, 640], seed=32, weights=weights)
    plant = {  # (layer, row, chunk) -> how the record is made NaN
        (0, 0, 10): "code+", (1, 0, 10): None, (1, 0, 777): "code-", (2, 0, 500): "scale",
        (0, 1, 128): "code+", (2, 1, 639): "scale", (1, 1, 200): "code-",
    }
    for (l, b, n), how in plant.items():
        rec = case.comp_k[l][b, n]
        if how == "code+":
            rec[37] = 0x7F
        elif how == "code-":
            rec[0] = 0xFF
        elif how == "scale":
            rec[128:132] = torch.from_numpy(NAN_SCALE.copy())
    keys = [k.to(DEV) for k in case.comp_k]
    q, w = retr.fm_query_prep(case.hidden.to(DEV), case.positions.to(DEV))
    nv = case.n_valid.to(DEV)
    scores = retr.fm_score(keys, q, w, n_valid=nv, N=case.N)
    torch.cuda.synchronize()
    retr.fm_sync_status()
    s_o = H.oracle_scores(case)
    s_g = scores.cpu().numpy().astype(np.float64)
    np.testing.assert_array_equal(np.isnan(s_g), np.isnan(s_o))
    assert int(np.isnan(s_o).sum()) == sum(1 for how in plant.values() if how)
    fin = ~np.isnan(s_o)
    assert np.abs(s_g[fin] - s_o[fin]).max() <= H.SCORE_TOL
    for mode in ("max", "mean"):
        ens, keep_thr, _ = retr.fm_score_fused(keys, q, w, mode=mode, threshold=0.4, n_valid=nv, N=case.N)
        keep = fm.fm_select_topk(ens, 600, nv)
        torch.cuda.synchronize()
        e_g = ens.cpu().numpy()
        e_o = O.ensemble(s_o, mode)
        np.testing.assert_array_equal(np.isnan(e_g), np.isnan(e_o))
        assert np.abs(e_g[~np.isnan(e_o)] - e_o[~np.isnan(e_o)]).max() <= H.SCORE_TOL
        np.testing.assert_array_equal(keep_thr.cpu().numpy(),
                                      O.select_threshold(e_g, case.n_valid.numpy(), 0.4))
        H.check_topk_against_rule(keep.cpu().numpy(), e_g, case.n_valid.numpy(), 600)
        assert not keep.cpu().numpy()[np.isnan(e_g)].any()  # 600 < the finite chunks of each row


@pytest.mark.parametrize("form", ["cluster", "candidate", "histogram"])
def test_topk_and_threshold_rank_nan_last(form):
    g = torch.Generator().manual_seed(33)
    B, N = 4, (16384 if form == "cluster" else 70000)  # rows past 16384 chunks take the other forms
    ens = torch.rand(B, N, generator=g)
    ens[0, torch.randperm(N, generator=g)[:5000]] = float("nan")      # scattered NaNs
    ens[1, :] = float("nan")
    ens[1, torch.randperm(N, generator=g)[:100]] = 0.25                # K cuts into the NaNs
    ens[2, ::7] = float("nan")
    ens[2, 1::7] = 0.0                                                 # zeros rank above NaN
    nv = torch.tensor([N, N, N - 3, 1234], dtype=torch.int32)
    if form == "cluster":
        ens[1, torch.randperm(N, generator=g)[:60]] = 0.25  # some numbers in the NaN row
    nbytes = fm.fm_topk_workspace_bytes(B, N) if form == "histogram" else fm.fm_topk_workspace_bytes_fast(B, N)
    ws = torch.zeros(nbytes, device=DEV, dtype=torch.uint8)
    for k in (64, 500, 1300):
        keep = fm.fm_select_topk(ens.to(DEV), k, nv.to(DEV), workspace=ws)
        torch.cuda.synchronize()
        H.check_topk_against_rule(keep.cpu().numpy(), ens.numpy(), nv.numpy(), k)
    keep_thr = fm.fm_select_threshold(ens.to(DEV), 0.1, nv.to(DEV))
    np.testing.assert_array_equal(keep_thr.cpu().numpy(), O.select_threshold(ens.numpy(), nv.numpy(), 0.1))
