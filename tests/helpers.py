"""Shared helpers of the tests: synthetic cases and their oracle values."""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence

import numpy as np
import torch

import oracle.retriever as O
from gen import synthetic as G

SCORE_TOL = 2e-3  # |GPU - oracle| bound on per-layer and ensembled sigmoid scores


def np_layers(weights: List[dict]) -> List[dict]:
    return [{k: v.numpy().astype(np.float64) for k, v in w.items()} for w in weights]


def oracle_queries(layers_np, hidden: torch.Tensor, positions: torch.Tensor):
    """oracle q [B, L, H, D] and fused_w [B, L, H] (fp64)."""
    h = hidden.numpy().astype(np.float64)
    pos = positions.numpy()
    qs, ws = zip(*[O.query_prep(l, h, pos) for l in layers_np])
    return np.stack(qs, axis=1), np.stack(ws, axis=1)


def plant_dirs(q: np.ndarray) -> torch.Tensor:
    """[L, B, 128] head-0 query directions used to plant relevant chunks."""
    return torch.from_numpy(np.ascontiguousarray(q[:, :, 0, :].transpose(1, 0, 2))).float()


@dataclasses.dataclass
class Case:
    weights: List[dict]
    layers_np: List[dict]
    hidden: torch.Tensor
    positions: torch.Tensor
    n_valid: torch.Tensor
    comp_k: List[torch.Tensor]      # [B, N_pad, 132] uint8 (device given at build)
    N: int
    q_o: np.ndarray                 # oracle q
    w_o: np.ndarray                 # oracle fused_w
    mode: str = "max"
    top_k: int = 512
    threshold: Optional[float] = None


def make_case(B: int, N: int, n_valid: Sequence[int], seed: int = 7, N_pad: Optional[int] = None,
              key_device="cpu", weights=None, n_layers: int = 3, mode="max", top_k=64,
              threshold=None, positions: Optional[Sequence[int]] = None) -> Case:
    weights = weights if weights is not None else G.make_weights(seed * 10 + 1, n_layers)
    layers_np = np_layers(weights)
    hidden = G.make_hidden(seed * 10 + 2, B)
    nv = torch.tensor(list(n_valid), dtype=torch.int32)
    pos = torch.tensor(list(positions), dtype=torch.int64) if positions is not None else G.positions_for(nv)
    q_o, w_o = oracle_queries(layers_np, hidden, pos)
    N_pad = N_pad if N_pad is not None else ((N + 3) // 4) * 4
    keys = G.make_keys(seed * 10 + 3, [int(x) for x in nv], N_pad, n_layers, plant_dirs(q_o),
                       device=key_device)
    return Case(weights, layers_np, hidden, pos, nv, keys, N, q_o, w_o, mode, top_k, threshold)


def workload_case(wl: G.Workload, key_device="cpu") -> Case:
    inp = G.make_query_inputs(wl)
    layers_np = np_layers(inp.weights)
    q_o, w_o = oracle_queries(layers_np, inp.hidden, inp.positions)
    keys = G.make_keys(wl.seed(G.SEED_KEYS), [int(x) for x in inp.n_valid], wl.N, G.N_LAYERS,
                       plant_dirs(q_o), device=key_device)
    return Case(inp.weights, layers_np, inp.hidden, inp.positions, inp.n_valid, keys, wl.N, q_o,
                w_o, wl.mode, wl.top_k, wl.threshold)


def oracle_scores(case: Case, q=None, w=None, rows=None) -> np.ndarray:
    """Oracle per-layer scores [L, B, N] for every valid chunk (small cases)."""
    q = case.q_o if q is None else q
    w = case.w_o if w is None else w
    L = len(case.comp_k)
    B = case.hidden.shape[0]
    out = np.zeros((L, B, case.N))
    for l in range(L):
        ck = case.comp_k[l].cpu().numpy()
        for b in range(B) if rows is None else rows:
            n = int(case.n_valid[b])
            out[l, b, :n] = O.score_chunks(ck[b, :n], q[b, l], w[b, l])
    return out


def oracle_sampled_scores(case: Case, b: int, idx: np.ndarray, comp_k_host: List[np.ndarray]):
    """Oracle per-layer scores [L, len(idx)] of chunks idx of row b."""
    return np.stack([O.score_chunks(comp_k_host[l][idx], case.q_o[b, l], case.w_o[b, l])
                     for l in range(len(comp_k_host))])


def check_topk_against_rule(keep_gpu: np.ndarray, ens_gpu: np.ndarray, n_valid, k: int):
    """Bit-exact: the oracle's selection rule applied to the GPU's own scores."""
    expect = O.select_topk(ens_gpu, np.asarray(n_valid), k)
    bad = np.argwhere(expect != keep_gpu)
    assert bad.size == 0, f"{len(bad)} mask entries differ, first {bad[:5].tolist()}"


def check_topk_near_oracle(keep_gpu: np.ndarray, ens_oracle: np.ndarray, n_valid, k: int,
                           tol: float = SCORE_TOL):
    """Against the oracle's own scores, masks may differ only on chunks whose
    oracle score lies within tol of the row's K-th oracle score."""
    expect = O.select_topk(ens_oracle, np.asarray(n_valid), k)
    for b in range(ens_oracle.shape[0]):
        n = int(n_valid[b])
        if n == 0 or k >= n:
            continue
        kth = np.sort(ens_oracle[b, :n])[::-1][k - 1]
        diff = np.nonzero(expect[b] != keep_gpu[b])[0]
        if diff.size:
            far = np.abs(ens_oracle[b, diff] - kth) > tol
            assert not far.any(), (b, diff[far][:5], ens_oracle[b, diff[far][:5]], kth)
