"""Plain CPU oracle of the toy sparse decode loop (numpy, fp64).

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
cpu_baseline / reference leg of bench.py may import this module.  It shares
no code with the CUDA library and never imports it.

Source: the FlashMemory DS-V4 Retriever README, "Toy inference reference":
every decode step the toy decoder runs a sparse memory attention over the N
compressed chunks, the chunks the last retrieval did not keep having their
attention logits set to -inf; every 64 steps the retriever scores all chunks,
ensembles the layers and selects the keep mask (top-K or sigmoid > thresh).

The toy decoder is not defined by the pages.  Readings taken here:
  * the query is the step's hidden state [4096] taken as 32 heads of 128;
  * the memory is the chunks' dequantized compressed records (the only
    per-chunk data the toy has), used as keys and values;
  * logits are q_h . x_i / sqrt(128); masked chunks get -inf; a row with no
    kept chunk attends to nothing and gives 0;
  * the next hidden state is RMSNorm(hidden + o), eps 1e-6, no gain;
  * positions advance by one token per step; the retrieval runs at the steps
    t with t % 64 == 0, starting at t = 0.

Parity pins: tests/test_oracle_pins.py.
"""
from __future__ import annotations

import math

import numpy as np

from oracle import retriever as R

N_HEADS = 32
HEAD_DIM = 128


def memory_vectors(comp_k: np.ndarray) -> np.ndarray:
    """[..., 132] records -> [..., 128] fp64 vectors e4m3(code) * scale."""
    return R.dequant(comp_k).astype(np.float64)


def masked_attention(q: np.ndarray, x: np.ndarray, keep: np.ndarray) -> np.ndarray:
    """q [B, H, D], x [B, N, D], keep [B, N] -> o [B, H, D]: per row and head,
    softmax over the chunks of q.x / sqrt(D) with -inf where not kept, then the
    weighted sum of the chunk vectors; 0 for a row with no kept chunk."""
    q = np.asarray(q, np.float64)
    x = np.asarray(x, np.float64)
    B, H, D = q.shape
    out = np.zeros((B, H, D))
    for b in range(B):
        kept = np.flatnonzero(keep[b])
        if kept.size == 0:
            continue
        logits = np.full((H, x.shape[1]), -np.inf)
        logits[:, kept] = q[b] @ x[b, kept].T / math.sqrt(D)
        m = logits.max(axis=1, keepdims=True)
        e = np.exp(logits - m)  # exp(-inf) = 0 for the masked chunks
        p = e / e.sum(axis=1, keepdims=True)
        out[b] = p @ x[b]
    return out


def toy_update(hidden: np.ndarray, o: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """RMSNorm(hidden + o flattened head-major), no gain."""
    h = np.asarray(hidden, np.float64) + np.asarray(o, np.float64).reshape(hidden.shape)
    return R.rms_norm(h, np.ones(h.shape[-1]), eps)


def toy_step(hidden: np.ndarray, x: np.ndarray, keep: np.ndarray) -> np.ndarray:
    """One decode step of the toy decoder for the given keep mask."""
    B = hidden.shape[0]
    q = np.asarray(hidden, np.float64).reshape(B, N_HEADS, HEAD_DIM)
    return toy_update(hidden, masked_attention(q, x, keep))
