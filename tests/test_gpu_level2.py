"""The per-step selection over a resident set as one CUDA graph (fm_level2_*),
against the oracle and against the same stages launched one by one.

Level 1 (the retrieval path, top-1024 of each row's chunks, then compaction
and gather) builds the resident set; the graph then runs for two later decode
steps (new hidden states and positions written in place): its ensembled
scores must be within the score tolerance of the oracle's scores of the
resident chunks, its selected chunk ids must be the top-k rule applied to its
own scores, mapped through the resident index list, and both must equal the
eager launch of the same stages bit for bit."""
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


def _resident_set(r, case, K1):
    keys = [t.to(DEV) for t in case.comp_k]
    nv = case.n_valid.to(DEV)
    _, keep, _ = r.retrieve(case.hidden.to(DEV), keys, case.positions.to(DEV), nv, mode="max", top_k=K1,
                            N=case.N)
    idx, count = fm.fm_compact_mask(keep, K1)
    res_keys = [fm.fm_gather_records(k, idx, count) for k in keys]
    torch.cuda.synchronize()
    return keys, idx, count, res_keys


def _eager(r, res_keys, idx, count, hidden, positions, k, R):
    q, w = r.fm_query_prep(hidden, positions)
    ens, _, _ = r.fm_score_fused(res_keys, q, w, mode="max", n_valid=count, N=R)
    keep = fm.fm_select_topk(ens, k, count)
    slots, scount = fm.fm_compact_mask(keep, k)
    ids = torch.full((idx.shape[0], k), -1, dtype=torch.int32, device=DEV)
    B = idx.shape[0]
    fm.fm_gather_records(idx.view(torch.uint8).view(B, R, 4), slots, scount, ids.view(torch.uint8).view(B, k, 4))
    torch.cuda.synchronize()
    return ens, ids, scount


@pytest.mark.parametrize("B", [12, 5])  # tensor-core and CUDA-core query prep inside the graph
def test_level2_graph_matches_oracle_and_eager(B):
    weights = G.make_weights(777, 3)
    r = fm.Retriever(weights, device=0, max_batch=64, q_pieces=2)
    try:
        N, K1, k = 6000, 1024, 128
        nv = [6000, 5000, 700, 100, 4097, 6000, 1024, 1025, 3000, 60, 2048, 5999][:B]
        case = H.make_case(B, N, nv, seed=31, weights=weights)
        keys, idx, count, res_keys = _resident_set(r, case, K1)
        assert count.cpu().tolist() == [min(K1, n) for n in nv]
        step = fm.Level2Step(r, res_keys, idx, count, k=k, mode="max")
        for s, seed in enumerate((91, 92)):
            hidden = G.make_hidden(seed, B)
            positions = case.positions + 4 * (s + 1)
            step.hidden.copy_(hidden.to(DEV))
            step.positions.copy_(positions.to(DEV))
            step.launch()
            torch.cuda.synchronize()
            r.fm_sync_status()  # no bounded wait ran out inside the graph
            ens = step.scores().cpu().numpy()
            ids = step.out_ids.cpu().numpy()
            cnt = count.cpu().numpy()
            idx_h = idx.cpu().numpy()
            # scores of the resident chunks against the oracle
            q_o, w_o = H.oracle_queries(case.layers_np, hidden, positions)
            for b in range(B):
                c = int(cnt[b])
                chunks = idx_h[b, :c]
                per = [O.score_chunks(case.comp_k[l][b].numpy()[chunks], q_o[b, l], w_o[b, l]) for l in range(3)]
                want = O.ensemble(np.stack(per), "max")
                assert np.abs(ens[b, :c] - want).max() <= H.SCORE_TOL
                assert (ens[b, c:] == 0).all()
            # selection: the top-k rule on the graph's own scores, mapped to chunk ids
            keep = O.select_topk(ens, cnt, k)
            for b in range(B):
                sel = idx_h[b, np.flatnonzero(keep[b])]
                want_ids = np.full(k, -1, np.int32)
                want_ids[:len(sel)] = sel
                np.testing.assert_array_equal(ids[b], want_ids)
            np.testing.assert_array_equal(step.out_count.cpu().numpy(), np.minimum(cnt, k))
            # the same stages launched one by one
            ens_e, ids_e, cnt_e = _eager(r, res_keys, idx, count, hidden.to(DEV), positions.to(DEV), k, K1)
            assert torch.equal(ens_e.cpu(), torch.from_numpy(ens))
            assert torch.equal(ids_e.cpu(), torch.from_numpy(ids))
        step.close()
    finally:
        r.close()


def test_level2_rejects_bad_descriptors():
    weights = G.make_weights(778, 3)
    r = fm.Retriever(weights, device=0, max_batch=8, q_pieces=2)
    try:
        keys = [torch.zeros(2, 64, 132, dtype=torch.uint8, device=DEV) for _ in range(3)]
        idx = torch.zeros(2, 64, dtype=torch.int32, device=DEV)
        cnt = torch.full((2,), 64, dtype=torch.int32, device=DEV)
        with pytest.raises(fm.FMError):
            fm.Level2Step(r, keys, idx, cnt, k=65)  # k > R
        big = torch.zeros(9, 64, dtype=torch.int32, device=DEV)
        with pytest.raises(fm.FMError):
            fm.Level2Step(r, [torch.zeros(9, 64, 132, dtype=torch.uint8, device=DEV)] * 3, big,
                          torch.zeros(9, dtype=torch.int32, device=DEV), k=8)  # B > max_batch
    finally:
        r.close()


def test_level2_ties_take_the_lowest_slots():
    """Identical resident records give identical scores: the top-k must keep
    the first k slots of each row (ties to the lower slot), and a row with
    fewer resident chunks than k keeps them all."""
    weights = G.make_weights(779, 3)
    r = fm.Retriever(weights, device=0, max_batch=8, q_pieces=2)
    try:
        B, R, k = 3, 1024, 100
        rec = G.make_keys(80, [1], 4, 3, None)  # one record per layer
        res_keys = [t[:, :1].expand(B, R, 132).contiguous().to(DEV) for t in rec]
        ids = (torch.arange(R, dtype=torch.int32) * 7 + 3).repeat(B, 1).contiguous().to(DEV)
        count = torch.tensor([R, 1000, 60], dtype=torch.int32, device=DEV)
        step = fm.Level2Step(r, res_keys, ids, count, k=k)
        step.hidden.copy_(G.make_hidden(81, B).to(DEV))
        step.positions.copy_(torch.full((B,), 4096, dtype=torch.int64, device=DEV))
        step.launch()
        torch.cuda.synchronize()
        out = step.out_ids.cpu().numpy()
        idh = ids.cpu().numpy()
        np.testing.assert_array_equal(out[0], idh[0, :k])
        np.testing.assert_array_equal(out[1], idh[1, :k])
        np.testing.assert_array_equal(out[2, :60], idh[2, :60])
        assert (out[2, 60:] == -1).all()
        np.testing.assert_array_equal(step.out_count.cpu().numpy(), [k, k, 60])
        step.close()
    finally:
        r.close()


def test_level2_at_bench_size():
    """The bench's Level-2 shape (64 rows x 4096 resident chunks, top-512):
    every CTA of the scoring pass takes many units and rows change inside its
    range.  Several graph launches without an error recorded, scores of a few
    rows against the oracle, the top-k rule on the graph's own scores."""
    B, R, k, N1 = 64, 4096, 512, 262144
    weights = G.make_weights(5000, 3)
    layers_np = H.np_layers(weights)
    r = fm.Retriever(weights, device=0, max_batch=B, q_pieces=2)
    try:
        g = torch.Generator().manual_seed(5001)
        ids = torch.stack([torch.randperm(N1, generator=g)[:R].sort().values for _ in range(B)]).to(torch.int32)
        res_keys = G.make_keys(5002, [R] * B, R, 3, None, device=DEV)
        count = torch.full((B,), R, dtype=torch.int32, device=DEV)
        step = fm.Level2Step(r, res_keys, ids.to(DEV), count, k=k, mode="max")
        hidden = G.make_hidden(5003, B)
        positions = torch.full((B,), 4 * N1, dtype=torch.int64)
        step.hidden.copy_(hidden.to(DEV))
        step.positions.copy_(positions.to(DEV))
        for _ in range(4):
            step.launch()
        torch.cuda.synchronize()
        r.fm_sync_status()
        ens = step.scores().cpu().numpy()
        q_o, w_o = H.oracle_queries(layers_np, hidden, positions)
        for b in (0, 33, 63):
            per = [O.score_chunks(res_keys[l][b].cpu().numpy(), q_o[b, l], w_o[b, l]) for l in range(3)]
            assert np.abs(ens[b] - O.ensemble(np.stack(per), "max")).max() <= H.SCORE_TOL
        keep = O.select_topk(ens, np.full(B, R), k)
        idh = ids.numpy()
        out = step.out_ids.cpu().numpy()
        for b in range(B):
            np.testing.assert_array_equal(out[b], idh[b, np.flatnonzero(keep[b])])
        step.close()
    finally:
        r.close()
