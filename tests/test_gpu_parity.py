"""Parity of the CUDA path (through the C ABI) with the CPU oracle on small
cases that span several 128-chunk tiles and ragged tails."""
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


@pytest.fixture(scope="module")
def weights():
    return G.make_weights(4242, 3)


@pytest.fixture(scope="module", params=[(3, 0), (2, 0), (2, 1)], ids=["pieces3", "pieces2", "pieces2_cta_pairs"])
def retr(request, weights):
    pieces, pairs = request.param
    r = fm.Retriever(weights, device=0, max_batch=64, q_pieces=pieces, cta_pairs=pairs)
    yield r
    r.close()


def _dev(ts):
    return [t.to(DEV) for t in ts]


def _run_query(r, case):
    q, w = r.fm_query_prep(case.hidden.to(DEV), case.positions.to(DEV))
    torch.cuda.synchronize()
    return q, w


def test_query_prep_matches_oracle(retr, weights):
    case = H.make_case(5, 256, [256] * 5, seed=11, weights=weights,
                       positions=[0, 1, 16384, 1 << 18, 1 << 20])
    q, w = _run_query(retr, case)
    q = q.cpu().numpy().astype(np.float64)
    w = w.cpu().numpy().astype(np.float64)
    nrm = np.linalg.norm(case.q_o, axis=-1, keepdims=True)
    err = np.linalg.norm(q - case.q_o, axis=-1, keepdims=True) / nrm
    assert err.max() < 2e-5, err.max()
    np.testing.assert_allclose(w, case.w_o, rtol=1e-4, atol=1e-6)
    retr.fm_sync_status()


def test_tile_dot_products_layout(retr, weights):
    """Raw tensor-core dots of one tile against exact fp64 dots of the e4m3
    codes with the query: checks the A/B operand layouts and the pieces."""
    case = H.make_case(2, 640, [640, 640], seed=12, weights=weights)
    keys = _dev(case.comp_k)
    q, w = _run_query(retr, case)
    P = retr.cfg.q_pieces
    qh = q.cpu().numpy().astype(np.float64)
    for (l, b, t) in [(0, 0, 0), (2, 1, 3), (1, 0, 4)]:
        out, e = retr.fm_debug_tile_dots(keys, q, w, l, b, t)
        torch.cuda.synchronize()
        out = out.cpu().numpy().astype(np.float64)
        e = e.cpu().numpy()
        codes = case.comp_k[l][b, t * 128:(t + 1) * 128, :128].numpy()
        kv = O.e4m3_decode(codes).astype(np.float64)             # [128, 128]
        exact = kv @ qh[b, l].T                                    # [128, 64]
        assert np.all(out[:, P * 64:] == 0.0)  # columns past the pieces are untouched
        # two pieces share one accumulator (the tensor core adds p0 + p1, p1
        # stored unscaled): columns 64.. stay untouched; three pieces keep one
        # block each, p_k scaled by 16^k
        rec = np.zeros((128, 64))
        for p in range(P):
            rec += out[:, p * 64:(p + 1) * 64] * 16.0 ** (-p)
        rec *= 2.0 ** (-e[None, :].astype(np.float64))
        # split error: 2^-4P relative per query element, plus the e4m3
        # subnormal floor of the last piece (2^-10 of the head's scale when it
        # is stored unscaled, 2^-18 with three scaled pieces); doubled for
        # fp32 accumulation
        floor = (2.0 ** -10 if P == 2 else 2.0 ** -18) * 2.0 ** (-e.astype(np.float64))
        bound = (np.abs(kv) @ np.abs(qh[b, l]).T * 2.0 ** (-4 * P)
                 + np.abs(kv).sum(1, keepdims=True) * floor[None, :]) * 2 + 1e-6
        assert np.all(np.abs(rec - exact) <= bound), np.abs(rec - exact).max()


@pytest.mark.parametrize("B", [24, 40, 64, 300])
def test_query_prep_tensor_core_path_matches_oracle(weights, B):
    """Past 8 rows both projections run on the tensor cores (three-pass TF32:
    hi*hi + hi*lo + lo*hi with hi = tf32(x)); the result must keep fp32-level
    accuracy.  300 rows take two 256-column tiles."""
    g = np.random.default_rng(100 + B)
    hidden = g.standard_normal((B, G.HIDDEN)).astype(np.float32)
    pos = g.integers(0, 1 << 20, size=B).astype(np.int64)
    r = fm.Retriever(weights, device=0, max_batch=max(64, B))
    try:
        q, w = r.fm_query_prep(torch.from_numpy(hidden).to(DEV), torch.from_numpy(pos).to(DEV))
        torch.cuda.synchronize()
        r.fm_sync_status()
        layers = H.np_layers(weights)
        for b in range(0, B, max(1, B // 7)):  # a spread of rows, through the oracle
            qo, wo = zip(*[O.query_prep(lw, hidden[b:b + 1].astype(np.float64), pos[b:b + 1]) for lw in layers])
            qo = np.stack([x[0] for x in qo])  # [L, H, D]
            wo = np.stack([x[0] for x in wo])  # [L, H]
            qg = q[b].cpu().numpy().astype(np.float64)
            err = np.linalg.norm(qg - qo, axis=-1) / np.linalg.norm(qo, axis=-1)
            assert err.max() < 2e-5, (b, err.max())
            np.testing.assert_allclose(w[b].cpu().numpy(), wo, rtol=1e-4, atol=1e-6)
    finally:
        r.close()


@pytest.mark.parametrize("shape", [
    dict(B=1, N=4096, nv=[4096]),
    dict(B=3, N=1001, nv=[1001, 517, 0]),
    dict(B=4, N=700, nv=[1, 127, 128, 700]),
])
def test_scores_match_oracle(retr, weights, shape):
    case = H.make_case(shape["B"], shape["N"], shape["nv"], seed=13, weights=weights)
    keys = _dev(case.comp_k)
    q, w = _run_query(retr, case)
    nv = case.n_valid.to(DEV)
    scores = retr.fm_score(keys, q, w, n_valid=nv, N=case.N)
    torch.cuda.synchronize()
    s_gpu = scores.cpu().numpy().astype(np.float64)
    s_o = H.oracle_scores(case)
    err = np.abs(s_gpu - s_o)
    assert err.max() <= H.SCORE_TOL, err.max()
    # exact zeros past each row's valid length
    for b in range(shape["B"]):
        assert np.all(s_gpu[:, b, int(case.n_valid[b]):] == 0.0)
    assert np.all((s_gpu >= 0) & (s_gpu <= 1))
    retr.fm_sync_status()


@pytest.mark.parametrize("mode,thr", [("max", None), ("mean", 0.5)])
def test_fused_pass_ensemble_and_masks(retr, weights, mode, thr):
    case = H.make_case(3, 2000, [2000, 1500, 333], seed=14, weights=weights)
    keys = _dev(case.comp_k)
    q, w = _run_query(retr, case)
    nv = case.n_valid.to(DEV)
    ens, keep_thr, scores = retr.fm_score_fused(keys, q, w, mode=mode, threshold=thr, n_valid=nv,
                                                N=case.N, want_layers=True)
    keep = fm.fm_select_topk(ens, 100, nv)
    torch.cuda.synchronize()
    s_o = H.oracle_scores(case)
    e_o = O.ensemble(s_o, mode)
    e_gpu = ens.cpu().numpy()
    assert np.abs(e_gpu - e_o).max() <= H.SCORE_TOL
    assert np.abs(scores.cpu().numpy() - s_o).max() <= H.SCORE_TOL
    # the fused ensemble equals the standalone ensemble of the same per-layer scores
    ens2 = fm.fm_ensemble(scores, mode)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(ens2.cpu().numpy(), e_gpu)
    H.check_topk_against_rule(keep.cpu().numpy(), e_gpu, case.n_valid.numpy(), 100)
    H.check_topk_near_oracle(keep.cpu().numpy(), e_o, case.n_valid.numpy(), 100)
    if thr is not None:
        expect = O.select_threshold(e_gpu, case.n_valid.numpy(), thr)
        np.testing.assert_array_equal(keep_thr.cpu().numpy(), expect)
    if mode == "max":
        assert np.all(e_gpu[None] >= scores.cpu().numpy())


def test_zero_scale_records_score_one_half(retr, weights):
    case = H.make_case(1, 300, [300], seed=15, weights=weights)
    for t in case.comp_k:
        t[0, 5:40, 128:132] = 0      # scale 0.0f -> k = 0 -> sigmoid(0)
    keys = _dev(case.comp_k)
    q, w = _run_query(retr, case)
    s = retr.fm_score(keys, q, w).cpu().numpy()
    assert np.all(s[:, 0, 5:40] == 0.5)


@pytest.mark.parametrize("ties", [False, True])
def test_topk_exact_rule(ties):
    g = torch.Generator().manual_seed(5)
    B, N = 6, 50000
    if ties:
        ens = torch.randint(0, 40, (B, N), generator=g).float() / 40.0
    else:
        ens = torch.rand(B, N, generator=g)
    nv = torch.tensor([N, 49999, 1, 0, 20000, 4096], dtype=torch.int32)
    for k in (1, 7, 4096, 30000, 60000):
        keep = fm.fm_select_topk(ens.to(DEV), k, nv.to(DEV))
        torch.cuda.synchronize()
        H.check_topk_against_rule(keep.cpu().numpy(), ens.numpy(), nv.numpy(), k)


def test_topk_all_equal_and_no_n_valid():
    ens = torch.full((2, 10000), 0.5)
    keep = fm.fm_select_topk(ens.to(DEV), 333).cpu().numpy()
    assert keep[0, :333].all() and not keep[0, 333:].any() and keep.sum() == 666


def test_threshold_and_ensemble_kernels():
    g = torch.Generator().manual_seed(6)
    s = (torch.randint(0, 9, (3, 4, 777), generator=g).float() / 8.0)
    nv = torch.tensor([777, 0, 5, 400], dtype=torch.int32)
    for mode in ("max", "mean"):
        e = fm.fm_ensemble(s.to(DEV), mode).cpu().numpy()
        np.testing.assert_allclose(e, O.ensemble(s.numpy(), mode), rtol=1e-6, atol=1e-7)
        keep = fm.fm_select_threshold(torch.from_numpy(e).to(DEV), 0.5, nv.to(DEV)).cpu().numpy()
        np.testing.assert_array_equal(keep, O.select_threshold(e, nv.numpy(), 0.5))


def test_argument_errors(retr, weights):
    case = H.make_case(2, 256, [256, 256], seed=16, weights=weights)
    keys = _dev(case.comp_k)
    q, w = _run_query(retr, case)
    lib = fm.lib()
    import ctypes
    arr = (ctypes.c_void_p * 3)(*[k.data_ptr() for k in keys])
    bad = (ctypes.c_void_p * 3)(*[k.data_ptr() + 4 for k in keys])
    out = torch.empty(3, 2, 256, device=DEV)
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    assert lib.fm_score(retr.handle, bad, 256 * 132, None, 2, 256, P(q), P(w), P(out), st) == fm.FM_ERR_ALIGNMENT
    assert lib.fm_score(retr.handle, arr, 255 * 132, None, 2, 256, P(q), P(w), P(out), st) != fm.FM_OK
    assert lib.fm_score(retr.handle, arr, 256 * 132, None, 65, 256, P(q), P(w), P(out), st) == fm.FM_ERR_INVALID_ARG
    assert lib.fm_score(retr.handle, arr, 256 * 132, None, 2, 0, P(q), P(w), P(out), st) == fm.FM_ERR_INVALID_ARG
    ens = torch.zeros(2, 256, device=DEV)
    keep = torch.zeros(2, 256, device=DEV, dtype=torch.uint8)
    ws = torch.zeros(fm.fm_topk_workspace_bytes(2, 256), device=DEV, dtype=torch.uint8)
    assert lib.fm_select_topk(P(ens), None, 2, 256, 0, P(keep), P(ws), ws.numel(), st) == fm.FM_ERR_INVALID_ARG
    assert lib.fm_select_topk(P(ens), None, 2, 256, 5, P(keep), P(ws), 16, st) == fm.FM_ERR_INVALID_ARG
    assert lib.fm_score_fused(retr.handle, arr, 256 * 132, None, 2, 256, P(q), P(w), 7, 0.0, None,
                              P(ens), None, st) == fm.FM_ERR_INVALID_ARG
    retr.fm_sync_status()


def test_shared_keys_across_layers(retr, weights):
    """One compressed_k scored by all three layers' queries (the README "Usage"
    signature taken literally): the layers' pointers alias one key tensor."""
    case = H.make_case(3, 1001, [1001, 517, 129], seed=21, weights=weights)
    shared = case.comp_k[0].to(DEV)
    case.comp_k = [case.comp_k[0]] * 3  # the oracle scores the same keys for every layer
    q, w = _run_query(retr, case)
    s = retr.fm_score([shared] * 3, q, w, n_valid=case.n_valid.to(DEV), N=case.N).cpu().numpy()
    want = H.oracle_scores(case)
    assert np.abs(s - want).max() <= H.SCORE_TOL
    ens, keep_thr, _ = retr.fm_score_fused([shared] * 3, q, w, mode="mean", threshold=0.5,
                                           n_valid=case.n_valid.to(DEV), N=case.N)
    ens = ens.cpu().numpy()
    assert np.abs(ens - O.ensemble(want, "mean")).max() <= H.SCORE_TOL
    np.testing.assert_array_equal(keep_thr.cpu().numpy(), O.select_threshold(ens, case.n_valid.numpy(), 0.5))
    retr.fm_sync_status()


def test_topk_candidate_path_and_its_fallbacks():
    """Rows of 300000 scores (past the one-kernel cluster form), K = 4096, a
    workspace large enough for the candidate path: ordinary scores (the path
    finishes the row), large scores placed only where the threshold sample
    looks (too few candidates: the row falls back to the histogram passes),
    all scores equal (too many candidates), and a K-th value tied across the
    cut (ties need chunk order): every mask must equal the selection rule."""
    B, N, K = 4, 300000, 4096
    g = torch.Generator().manual_seed(12)
    ens = torch.rand(B, N, generator=g) * 0.5
    sampled = (torch.arange(8192, dtype=torch.int64) * N) // 8192
    ens[1, sampled] = 0.9 + torch.rand(8192, generator=g) * 0.05  # only sampled positions are large
    ens[2] = 0.5
    ens[3] = torch.randint(0, 8, (N,), generator=g).float() / 8.0  # heavy ties at the K-th value
    nv = torch.tensor([N, N, N - 17, 200000], dtype=torch.int32)
    ws = torch.zeros(fm.fm_topk_workspace_bytes_fast(B, N), device=DEV, dtype=torch.uint8)
    keep = fm.fm_select_topk(ens.to(DEV), K, nv.to(DEV), workspace=ws)
    torch.cuda.synchronize()
    H.check_topk_against_rule(keep.cpu().numpy(), ens.numpy(), nv.numpy(), K)
    # the same rows through the histogram passes only (a workspace too small for the candidate path)
    ws_min = torch.zeros(fm.fm_topk_workspace_bytes(B, N), device=DEV, dtype=torch.uint8)
    keep_min = fm.fm_select_topk(ens.to(DEV), K, nv.to(DEV), workspace=ws_min)
    assert torch.equal(keep.cpu(), keep_min.cpu())


def test_retrieve_host_call_matches_the_device_calls(retr, weights):
    """fm_retrieve_host (host buffers in, host masks out, through the C ABI)
    gives the masks of the device calls it composes, bit for bit."""
    case = H.make_case(3, 2000, [2000, 1500, 333], seed=22, weights=weights)
    hk = [k.pin_memory() for k in case.comp_k]
    hh, hp, hn = case.hidden.pin_memory(), case.positions.pin_memory(), case.n_valid.pin_memory()
    bufs = {}
    for _ in range(2):  # the second call reuses the staging buffers
        kt, kh = retr.retrieve_from_host(hh, hp, hk, hn, "mean", 100, 0.5, case.N, bufs)
        ens, keep_topk, keep_thr = retr.retrieve(case.hidden.to(DEV), _dev(case.comp_k), case.positions.to(DEV),
                                                 case.n_valid.to(DEV), "mean", 100, 0.5, case.N)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(kt.numpy(), keep_topk.cpu().numpy().astype(np.uint8))
        np.testing.assert_array_equal(kh.numpy(), keep_thr.cpu().numpy().astype(np.uint8))
        H.check_topk_near_oracle(kt.numpy().astype(bool), O.ensemble(H.oracle_scores(case), "mean"),
                                 case.n_valid.numpy(), 100)


@pytest.mark.parametrize("N", [1, 100, 4096, 16383, 16384, 16385, 65536, 131073, 262144])
def test_topk_rule_across_row_lengths(N):
    """Rows up to 16384 chunks (the one-kernel form) and past it (the
    candidate path): ordinary scores, a K-th value tied across the cut, all
    scores equal, ragged and empty rows, K past the row's length."""
    g = torch.Generator().manual_seed(N)
    B = 5
    ens = torch.rand(B, N, generator=g)
    ens[1] = torch.randint(0, 5, (N,), generator=g).float() / 5.0   # heavy ties
    ens[2] = 0.25
    nv = torch.tensor([N, N, N, max(0, N - 37), 0], dtype=torch.int32)
    for k in sorted({1, 3, min(N, 512), max(1, N // 3), N + 5}):
        keep = fm.fm_select_topk(ens.to(DEV), k, nv.to(DEV))
        torch.cuda.synchronize()
        H.check_topk_against_rule(keep.cpu().numpy(), ens.numpy(), nv.numpy(), k)


@pytest.mark.parametrize("B", [2, 12])
def test_query_prep_rank_2048(B):
    """A Q_LORA_RANK of 2048 (the pages leave the rank open): the RMSNorm
    block spans more than 2048 elements, on the GEMV path (B <= 8) and the
    tensor-core path."""
    weights = G.make_weights(4646, 3, rank=2048)
    g = np.random.default_rng(47 + B)
    hidden = g.standard_normal((B, G.HIDDEN)).astype(np.float32)
    pos = g.integers(0, 1 << 20, size=B).astype(np.int64)
    r = fm.Retriever(weights, device=0, max_batch=16, q_lora_rank=2048)
    try:
        q, w = r.fm_query_prep(torch.from_numpy(hidden).to(DEV), torch.from_numpy(pos).to(DEV))
        torch.cuda.synchronize()
        r.fm_sync_status()
        qo, wo = H.oracle_queries(H.np_layers(weights), torch.from_numpy(hidden), torch.from_numpy(pos))
        err = np.linalg.norm(q.cpu().numpy() - qo, axis=-1) / np.linalg.norm(qo, axis=-1)
        assert err.max() < 2e-5, err.max()
        np.testing.assert_allclose(w.cpu().numpy(), wo, rtol=1e-4, atol=1e-6)
    finally:
        r.close()


@pytest.mark.parametrize("shared", [False, True], ids=["three_key_tensors", "shared_keys"])
def test_rows_of_one_tile_between_longer_rows(retr, weights, shared):
    """Rows of a single 128-chunk tile give pairs with one unit, so the second
    epilogue group idles while the first runs on: each group's scale ring
    must stay in step with its own tiles.  With shared keys every layer's
    pointer is the one tensor (one key tile per unit for all layers)."""
    nv = [1000, 100, 50, 128, 1, 129, 700, 3, 90, 400]
    case = H.make_case(len(nv), 1000, nv, seed=23, weights=weights)
    if shared:
        case.comp_k = [case.comp_k[0]] * 3
    keys = _dev(case.comp_k) if not shared else [case.comp_k[0].to(DEV)] * 3
    q, w = _run_query(retr, case)
    n_valid = case.n_valid.to(DEV)
    s = retr.fm_score(keys, q, w, n_valid=n_valid, N=case.N).cpu().numpy()
    ens, _, _ = retr.fm_score_fused(keys, q, w, mode="max", n_valid=n_valid, N=case.N)
    torch.cuda.synchronize()
    retr.fm_sync_status()
    want = H.oracle_scores(case)
    assert np.abs(s - want).max() <= H.SCORE_TOL
    assert np.abs(ens.cpu().numpy() - O.ensemble(want, "max")).max() <= H.SCORE_TOL
