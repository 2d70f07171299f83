"""Plain CPU oracle of the recall step that follows selection (pure Python
loops over numpy arrays).

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
cpu_baseline / reference leg of bench.py may import this module.  It shares
no code with the CUDA library and never imports it.

Source: the FlashMemory DS-V4 Retriever model card, "How it works (in
brief)": every 64 decode steps the Memory Indexer selects the query-critical
chunks, and that resident set is recalled from the CPU-side bulk KV cache to
the GPU (only recalled chunks and the compressed indexer keys stay on the
GPU).  The card does not say how the set is represented; the reading here is
the plainest one: the kept chunk indices of each row in increasing order, and
each kept chunk's fixed-size record copied to consecutive slots of a resident
buffer in that order.

Parity pins: tests/test_oracle_pins.py (a hand-worked case, brute-force
definitions on tiny inputs, invariants).
"""
from __future__ import annotations

import numpy as np


def compact_mask(keep: np.ndarray, max_sel: int):
    """keep [B, N] (nonzero = kept) -> (idx [B, max_sel] int32, count [B] int32).
    idx[b] lists row b's kept chunk indices in increasing order, at most
    max_sel of them, then -1; count[b] is how many chunks row b keeps (it may
    exceed max_sel)."""
    keep = np.asarray(keep)
    B, N = keep.shape
    idx = np.full((B, max_sel), -1, np.int32)
    count = np.zeros(B, np.int32)
    for b in range(B):
        j = 0
        for n in range(N):
            if keep[b, n]:
                if j < max_sel:
                    idx[b, j] = n
                j += 1
        count[b] = j
    return idx, count


def gather_records(src: np.ndarray, idx: np.ndarray, count: np.ndarray, dst: np.ndarray) -> np.ndarray:
    """Copies record idx[b, j] of src[b] ([B, n_src, rec] bytes) into slot j of
    dst[b] for j < min(count[b], max_sel) and 0 <= idx[b, j] < n_src; other
    slots keep what dst held.  Returns a new array."""
    out = np.array(dst, copy=True)
    B, n_src, _ = src.shape
    max_sel = idx.shape[1]
    for b in range(B):
        for j in range(min(int(count[b]), max_sel)):
            n = int(idx[b, j])
            if 0 <= n < n_src:
                out[b, j, :] = src[b, n, :]
    return out
