"""Seeded synthetic inputs for the FlashMemory DS-V4 retriever path.

This module serves both the CPU oracle (tests) and the CUDA library (tests,
bench).  It holds none of the retriever's arithmetic: only random draws, the
OCP E4M3 encoding of key values (done by torch's own fp8 cast), and the packing
of the 132-byte compressed-key record that the retriever README describes under
"compressed_k format" (128 e4m3 bytes followed by one little-endian fp32
scale).

Input recipe (shared by every workload):
  * weights: fp32 N(0, 0.02); q_norm weight = 1 + N(0, 0.02); one independent
    set per CSA layer (l10, l12, l20), row-major [out, in], no biases;
  * hidden: fp32 N(0, 1), shape [B, 4096];
  * keys: for each chunk draw v ~ N(0,1)^128; for 1 % of the chunks of a row
    (chosen uniformly without replacement, the same chunks in every layer) set
    v = 0.5 v + 2 u, u the unit direction supplied by the caller (the row's
    head-0 query of that layer); scale = amax|v| / 448 in fp32; the codes are
    v / scale cast to e4m3 with round-to-nearest-even;
  * ragged lengths (one workload): n_b ~ Uniform{lo..hi}, rows padded to N
    with zero bytes;
  * positions: 4 * n_b (the CSA compression stride is not stated on the pages;
    four tokens per chunk is the reading used here).

Random streams are keyed by (seed, layer, row) so that any slab can be drawn
on its own, on CPU or on a CUDA device.  Values drawn on different devices
differ (torch's CPU and CUDA generators are different algorithms); every
comparison draws once and copies.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence

import torch

HIDDEN = 4096
Q_LORA_RANK = 1024
N_HEADS = 64
HEAD_DIM = 128
N_LAYERS = 3
LAYER_NAMES = ("l10", "l12", "l20")
RECORD_BYTES = HEAD_DIM + 4
E4M3_MAX = 448.0
PLANT_FRACTION = 0.01

ROPE = dict(rope_dim=64, base=160000.0, factor=16.0, orig_max_pos=65536.0,
            beta_fast=32.0, beta_slow=1.0)
RMS_EPS = 1e-6


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes and selection settings."""
    index: int
    name: str
    B: int
    N: int                      # chunks per row per layer (padded length)
    n_lo: Optional[int] = None  # ragged rows: n_b ~ U{n_lo..n_hi}
    n_hi: Optional[int] = None
    mode: str = "max"           # cross-layer ensemble
    top_k: int = 512
    threshold: Optional[float] = None
    prep_in_step: bool = True   # query-side prep is part of every step

    def seed(self, part: int) -> int:
        return 1000 * self.index + part

    @property
    def ragged(self) -> bool:
        return self.n_lo is not None


WORKLOADS: List[Workload] = [
    Workload(0, "B1_N4096_max_top512", B=1, N=4096, mode="max", top_k=512),
    Workload(1, "B8_N65536_mean_top512_thr0.5", B=8, N=65536, mode="mean",
             top_k=512, threshold=0.5),
    Workload(2, "B1_N262144_max_top2048", B=1, N=262144, mode="max", top_k=2048),
    Workload(3, "B32_ragged32768-131072_max_top1536", B=32, N=131072,
             n_lo=32768, n_hi=131072, mode="max", top_k=1536),
    Workload(4, "B64_N262144_max_top4096", B=64, N=262144, mode="max", top_k=4096),
]

SEED_WEIGHTS, SEED_HIDDEN, SEED_KEYS, SEED_LENGTHS, SEED_PLANT = 0, 1, 2, 3, 4


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)
    return g


def make_weights(seed: int, n_layers: int = N_LAYERS, hidden: int = HIDDEN,
                 rank: int = Q_LORA_RANK, n_heads: int = N_HEADS,
                 head_dim: int = HEAD_DIM) -> List[dict]:
    """Per-layer fp32 weights on the CPU: wq_a [rank, hidden], q_norm [rank],
    wq_b [n_heads*head_dim, rank], weights_proj [n_heads, hidden]."""
    out = []
    for l in range(n_layers):
        g = _gen(seed * 1_000_003 + 17 * l)
        out.append(dict(
            wq_a=torch.randn(rank, hidden, generator=g) * 0.02,
            q_norm=1.0 + torch.randn(rank, generator=g) * 0.02,
            wq_b=torch.randn(n_heads * head_dim, rank, generator=g) * 0.02,
            weights_proj=torch.randn(n_heads, hidden, generator=g) * 0.02,
        ))
    return out


def make_hidden(seed: int, B: int, hidden: int = HIDDEN) -> torch.Tensor:
    return torch.randn(B, hidden, generator=_gen(seed))


def make_lengths(wl: Workload) -> torch.Tensor:
    """int32 [B] valid chunk counts per row."""
    if not wl.ragged:
        return torch.full((wl.B,), wl.N, dtype=torch.int32)
    g = _gen(wl.seed(SEED_LENGTHS))
    return torch.randint(wl.n_lo, wl.n_hi + 1, (wl.B,), generator=g,
                         dtype=torch.int64).to(torch.int32)


def positions_for(n_valid: torch.Tensor) -> torch.Tensor:
    """int64 [B] decode positions: four tokens per compressed chunk."""
    return n_valid.to(torch.int64) * 4


def plant_indices(seed: int, b: int, n_b: int) -> torch.Tensor:
    """The chunks of row b that carry the planted direction (all layers)."""
    n_plant = int(PLANT_FRACTION * n_b + 0.5)
    g = _gen(seed * 1_000_003 + 7 * b + 3)
    return torch.randperm(n_b, generator=g)[:n_plant]


def encode_records(v: torch.Tensor) -> torch.Tensor:
    """Pack fp32 key vectors [n, 128] into 132-byte records [n, 132] uint8:
    scale = amax|v| / 448 (fp32), codes = e4m3(v / scale) with RNE."""
    amax = v.abs().amax(dim=-1)
    scale = (amax / E4M3_MAX).to(torch.float32)
    safe = torch.where(scale > 0, scale, torch.ones_like(scale))
    x = v / safe[:, None]
    x = torch.where(scale[:, None] > 0, x, torch.zeros_like(x))
    codes = x.to(torch.float8_e4m3fn).view(torch.uint8)
    rec = torch.empty(v.shape[0], RECORD_BYTES, dtype=torch.uint8, device=v.device)
    rec[:, :HEAD_DIM] = codes
    rec[:, HEAD_DIM:] = scale.contiguous().view(torch.uint8).view(-1, 4)
    return rec


def make_key_slab(seed: int, layer: int, b: int, n_b: int,
                  plant_dir: Optional[torch.Tensor], device="cpu",
                  plant_idx: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Records [n_b, 132] uint8 for one (layer, row)."""
    g = _gen(seed * 1_000_003 + 65_537 * (layer + 1) + b, device)
    v = torch.randn(n_b, HEAD_DIM, generator=g, device=device)
    if plant_dir is not None and n_b > 0:
        if plant_idx is None:
            plant_idx = plant_indices(seed, b, n_b)
        u = plant_dir.to(device=device, dtype=torch.float32)
        nrm = u.norm()
        u = u / nrm if float(nrm) > 0 else u
        idx = plant_idx.to(device)
        v[idx] = 0.5 * v[idx] + 2.0 * u
    return encode_records(v)


def make_keys(seed: int, n_valid: Sequence[int], N: int, n_layers: int = N_LAYERS,
              plant_dirs: Optional[torch.Tensor] = None, device="cpu") -> List[torch.Tensor]:
    """Per-layer key tensors [B, N, 132] uint8 (rows zero-padded past n_b).

    plant_dirs: [n_layers, B, 128] directions (head-0 queries) or None."""
    n_valid = [int(x) for x in n_valid]
    B = len(n_valid)
    out = []
    pidx = [plant_indices(seed, b, n_valid[b]) for b in range(B)]
    for l in range(n_layers):
        t = torch.zeros(B, N, RECORD_BYTES, dtype=torch.uint8, device=device)
        for b in range(B):
            pd = None if plant_dirs is None else plant_dirs[l, b]
            t[b, :n_valid[b]] = make_key_slab(seed, l, b, n_valid[b], pd, device, pidx[b])
        out.append(t)
    return out


@dataclasses.dataclass
class Inputs:
    wl: Workload
    weights: List[dict]
    hidden: torch.Tensor      # [B, 4096] fp32 (CPU)
    n_valid: torch.Tensor     # [B] int32 (CPU)
    positions: torch.Tensor   # [B] int64 (CPU)


def make_query_inputs(wl: Workload, n_layers: int = N_LAYERS) -> Inputs:
    """Everything but the keys (the keys need the planting directions)."""
    n_valid = make_lengths(wl)
    return Inputs(wl=wl,
                  weights=make_weights(wl.seed(SEED_WEIGHTS), n_layers),
                  hidden=make_hidden(wl.seed(SEED_HIDDEN), wl.B),
                  n_valid=n_valid,
                  positions=positions_for(n_valid))
