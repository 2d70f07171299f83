"""The toy sparse decode on the GPU against the oracle: the sparse attention
over the kept chunks, through the index list and from a resident buffer of
the kept records (several 128-chunk segments, ragged tails, empty rows,
out-of-range indices), the state update, and the decode loop teacher-forced
step by step (each step's GPU output against the oracle's step from the GPU's
own input state and keep mask; retrievals at t % 64 == 0 against the top-K
rule on the GPU's own scores)."""
import numpy as np
import pytest
import torch

import oracle.decode as OD
import oracle.retriever as O
from gen import synthetic as G
from tests import helpers as H

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from learned_kv_chunk_b200 import fm  # noqa: E402  (loads libfm.so; raises if missing)

DEV = torch.device("cuda", 0)
ATTN_TOL = 2e-5  # relative to the row's output scale; fp32 accumulation over <= 4096 chunks


def _check_attention(o_gpu, o_ref):
    scale = np.abs(o_ref).max(axis=(1, 2), keepdims=True) + 1e-30
    err = np.abs(o_gpu - o_ref) / scale
    assert err.max() <= ATTN_TOL, err.max()


@pytest.mark.parametrize("resident", [False, True], ids=["index_list", "resident"])
@pytest.mark.parametrize("max_sel", [1, 128, 300, 1000])
def test_sparse_attention_matches_masked_oracle(max_sel, resident):
    B, N = 5, 3000
    keys = G.make_keys(61, [N, 2500, 900, N, 10], N, 1, None)[0]
    rng = np.random.default_rng(max_sel)
    dens = np.array([0.05, 0.5, 1.0, 0.0, 1.0])
    keep = rng.random((B, N)) < dens[:, None]
    keep[:, 2500:] &= np.array([True, False, True, True, False])[:, None]
    keep[4, 10:] = False
    q = torch.from_numpy(rng.standard_normal((B, 32, 128)).astype(np.float32))
    idx, count = fm.fm_compact_mask(torch.from_numpy(keep).to(DEV), max_sel)
    if resident:  # the kept records gathered in order; the attention reads them without the list
        res = fm.fm_gather_records(keys.to(DEV), idx, count)
        o = fm.fm_decode_attention(q.to(DEV), res, None, count).cpu().numpy()
    else:
        o = fm.fm_decode_attention(q.to(DEV), keys.to(DEV), idx, count).cpu().numpy()
    # the oracle attends over exactly the chunks the index list holds (the first max_sel kept)
    used = np.zeros_like(keep)
    idx_h, cnt_h = idx.cpu().numpy(), count.cpu().numpy()
    for b in range(B):
        used[b, idx_h[b, :min(cnt_h[b], max_sel)]] = True
    x = OD.memory_vectors(keys.numpy())
    _check_attention(o, OD.masked_attention(q.numpy(), x, used))
    assert (o[3] == 0).all()  # nothing kept


def test_sparse_attention_skips_out_of_range_indices():
    B, N = 2, 500
    keys = G.make_keys(62, [N, N], N, 1, None)[0]
    q = torch.randn(B, 32, 128, generator=torch.Generator().manual_seed(3))
    idx = torch.tensor([[5, 7, N + 3, -2], [499, 0, 1, 2]], dtype=torch.int32)
    count = torch.tensor([4, 4], dtype=torch.int32)
    o = fm.fm_decode_attention(q.to(DEV), keys.to(DEV), idx.to(DEV), count.to(DEV)).cpu().numpy()
    keep = np.zeros((B, N), bool)
    keep[0, [5, 7]] = True
    keep[1, [499, 0, 1, 2]] = True
    _check_attention(o, OD.masked_attention(q.numpy(), OD.memory_vectors(keys.numpy()), keep))


def test_toy_update_matches_oracle_in_place():
    rng = np.random.default_rng(4)
    h = rng.standard_normal((3, 4096)).astype(np.float32)
    o = rng.standard_normal((3, 4096)).astype(np.float32)
    hd = torch.from_numpy(h).to(DEV)
    fm.fm_toy_decoder_update(hd, torch.from_numpy(o).to(DEV), out=hd)
    np.testing.assert_allclose(hd.cpu().numpy(), OD.toy_update(h, o.reshape(3, 32, 128)), rtol=2e-6, atol=2e-6)


@pytest.mark.parametrize("select", ["topk", "threshold"])
def test_decode_loop_teacher_forced(select):
    weights = G.make_weights(63, 3)
    r = fm.Retriever(weights, device=0, max_batch=8, q_pieces=2)
    try:
        B, N = 3, 2000
        nv = [2000, 1500, 300]
        case = H.make_case(B, N, nv, seed=64, weights=weights)
        keys = [k.to(DEV) for k in case.comp_k]
        kw = dict(top_k=256) if select == "topk" else dict(top_k=None, threshold=0.5)
        dec = fm.ToySparseDecoder(r, keys, case.n_valid.to(DEV), case.hidden.to(DEV), case.positions, **kw)
        x = OD.memory_vectors(case.comp_k[0].numpy())
        nv_np = case.n_valid.numpy()
        keep_prev = None
        for t in range(130):
            h_in = dec.hidden.cpu().numpy().astype(np.float64)
            h_out = dec.step().cpu().numpy()
            keep = dec.keep.cpu().numpy().astype(bool)
            if t % 64 == 0:
                ens = dec.ens.cpu().numpy()
                want = (O.select_topk(ens, nv_np, 256) if select == "topk"
                        else O.select_threshold(ens, nv_np, 0.5))
                np.testing.assert_array_equal(keep, want)
            else:
                np.testing.assert_array_equal(keep, keep_prev)  # the mask holds between retrievals
            keep_prev = keep
            ref = OD.toy_step(h_in, x, keep)
            assert np.abs(h_out - ref).max() <= 1e-4, (t, np.abs(h_out - ref).max())
        assert dec.t == 130
    finally:
        r.close()
