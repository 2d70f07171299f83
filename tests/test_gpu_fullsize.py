"""Full-size workloads in the launch configuration bench.py times: the fused
scoring pass (ensemble written, per-layer scores not written) followed by the
top-K select, checked on sampled chunks against the oracle, one whole row
element by element against the oracle's scores, and every row's mask
through the oracle's selection rule."""
import numpy as np
import pytest
import torch

import oracle.retriever as O
from gen import synthetic as G
from tests import helpers as H

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from learned_kv_chunk_b200 import fm  # noqa: E402

DEV = torch.device("cuda", 0)


def _run(wl, cta_pairs=0):
    case = H.workload_case(wl, key_device=DEV)
    r = fm.Retriever(case.weights, device=0, max_batch=max(64, wl.B), cta_pairs=cta_pairs)
    try:
        q, w = r.fm_query_prep(case.hidden.to(DEV), case.positions.to(DEV))
        nv = case.n_valid.to(DEV)
        ens, keep_thr, _ = r.fm_score_fused(case.comp_k, q, w, mode=wl.mode, threshold=wl.threshold,
                                            n_valid=nv, N=wl.N)
        keep = fm.fm_select_topk(ens, wl.top_k, nv)
        torch.cuda.synchronize()
        r.fm_sync_status()
        return case, r, q, w, ens, keep, keep_thr
    except Exception:
        r.close()
        raise


@pytest.mark.parametrize("wl,cta_pairs", [(w, 0) for w in G.WORKLOADS[1:]] + [(G.WORKLOADS[3], 1)],
                         ids=[w.name for w in G.WORKLOADS[1:]] + [G.WORKLOADS[3].name + "_cta_pairs"])
def test_full_size_workload(wl, cta_pairs):
    """cta_pairs: the scoring pass on CTA pairs, on the ragged rows whose odd
    tile counts leave the pair's second CTA without a tile at a row's end."""
    case, r, q, w, ens, keep, keep_thr = _run(wl, cta_pairs)
    try:
        nv = case.n_valid.numpy()
        e_gpu = ens.cpu().numpy()
        k_gpu = keep.cpu().numpy()
        # keep-mask: bit-exact against the oracle's rule on the GPU's own scores
        H.check_topk_against_rule(k_gpu, e_gpu, nv, wl.top_k)
        if wl.threshold is not None:
            np.testing.assert_array_equal(keep_thr.cpu().numpy(),
                                          O.select_threshold(e_gpu, nv, wl.threshold))
        # properties at any size
        assert np.all((e_gpu >= 0) & (e_gpu <= 1))
        for b in range(wl.B):
            assert np.all(e_gpu[b, int(nv[b]):] == 0) and not k_gpu[b, int(nv[b]):].any()
        # sampled chunks of a few rows against the oracle, per layer and ensembled
        rng = np.random.default_rng(wl.index)
        rows = sorted(set([0, wl.B - 1] + list(rng.integers(0, wl.B, 2))))
        _, _, scores = r.fm_score_fused(case.comp_k, q, w, mode=wl.mode, n_valid=case.n_valid.to(DEV),
                                        N=wl.N, want_layers=True)
        torch.cuda.synchronize()
        for b in rows:
            n = int(nv[b])
            idx = np.unique(np.concatenate([rng.integers(0, n, 2000), [0, n - 1],
                                            np.nonzero(k_gpu[b])[0][:200]]))
            host = [case.comp_k[l][b, idx].cpu().numpy() for l in range(3)]
            s_o = np.stack([O.score_chunks(host[l], case.q_o[b, l], case.w_o[b, l]) for l in range(3)])
            s_g = scores[:, b, idx].cpu().numpy()
            assert np.abs(s_g - s_o).max() <= H.SCORE_TOL, np.abs(s_g - s_o).max()
            e_o = O.ensemble(s_o, wl.mode)
            assert np.abs(e_gpu[b, idx] - e_o).max() <= H.SCORE_TOL
        # one whole row against the oracle's own top-K (tolerance band at the K-th score)
        b = rows[-1]
        n = int(nv[b])
        full = np.stack([O.score_chunks(case.comp_k[l][b, :n].cpu().numpy(), case.q_o[b, l],
                                        case.w_o[b, l]) for l in range(3)])
        # every chunk of the row, per layer and ensembled, element by element
        d_layers = np.abs(scores[:, b, :n].cpu().numpy().astype(np.float64) - full).max()
        assert d_layers <= H.SCORE_TOL, d_layers
        e_row = np.zeros((1, wl.N))
        e_row[0, :n] = O.ensemble(full, wl.mode)
        assert np.abs(e_gpu[b, :n] - e_row[0, :n]).max() <= H.SCORE_TOL
        H.check_topk_near_oracle(k_gpu[b:b + 1], e_row, nv[b:b + 1], wl.top_k)
    finally:
        r.close()


def test_full_size_shared_keys():
    """The 64-row workload with one key tensor for every layer (the README
    Usage signature taken literally, the shared-keys form of the pass): many
    units per CTA, so the per-unit key stages and scale slots wrap many
    times.  Sampled chunks against the oracle, the mask against the rule."""
    wl = G.WORKLOADS[4]
    inp = G.make_query_inputs(wl)
    layers_np = H.np_layers(inp.weights)
    q_o, w_o = H.oracle_queries(layers_np, inp.hidden, inp.positions)
    key = G.make_keys(wl.seed(G.SEED_KEYS), [int(x) for x in inp.n_valid], wl.N, 1,
                      H.plant_dirs(q_o)[:1], device=DEV)[0]
    r = fm.Retriever(inp.weights, device=0, max_batch=wl.B)
    try:
        q, w = r.fm_query_prep(inp.hidden.to(DEV), inp.positions.to(DEV))
        nv = inp.n_valid.to(DEV)
        ens, _, scores = r.fm_score_fused([key] * 3, q, w, mode=wl.mode, n_valid=nv, N=wl.N, want_layers=True)
        keep = fm.fm_select_topk(ens, wl.top_k, nv)
        torch.cuda.synchronize()
        r.fm_sync_status()
        e_gpu = ens.cpu().numpy()
        H.check_topk_against_rule(keep.cpu().numpy(), e_gpu, inp.n_valid.numpy(), wl.top_k)
        rng = np.random.default_rng(404)
        for b in (0, 17, 63):
            idx = np.unique(np.concatenate([rng.integers(0, wl.N, 1500), [0, wl.N - 1]]))
            host = key[b, idx].cpu().numpy()
            s_o = np.stack([O.score_chunks(host, q_o[b, l], w_o[b, l]) for l in range(3)])
            assert np.abs(scores[:, b, idx].cpu().numpy() - s_o).max() <= H.SCORE_TOL
            assert np.abs(e_gpu[b, idx] - O.ensemble(s_o, wl.mode)).max() <= H.SCORE_TOL
    finally:
        r.close()
