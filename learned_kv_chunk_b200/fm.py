"""Thin Python binding of libfm (ctypes).  Argument marshalling only: every
step of the retriever path runs in the library's CUDA kernels.  torch is used
for device memory and the current stream.

The functions carry the C ABI's names (include/fm.h); `Retriever` bundles a
context with its weights for convenience.  If libfm.so is missing, importing
this module raises: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("FM_LIBRARY_PATH") or os.path.join(_PKG, "lib", "libfm.so")

FM_OK, FM_ERR_INVALID_ARG, FM_ERR_ALIGNMENT, FM_ERR_UNSUPPORTED = 0, 1, 2, 3
FM_ERR_CUDA, FM_ERR_OOM, FM_ERR_DEVICE = 4, 5, 6
FM_ENSEMBLE_MAX, FM_ENSEMBLE_MEAN = 0, 1
MODES = {"max": FM_ENSEMBLE_MAX, "mean": FM_ENSEMBLE_MEAN}
FM_TOPK_SHARD_BINS = 2048


class fm_config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("q_lora_rank", ctypes.c_int),
                ("n_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("n_layers", ctypes.c_int), ("rope_dim", ctypes.c_int),
                ("rope_base", ctypes.c_double), ("rope_factor", ctypes.c_double),
                ("rope_orig_max_pos", ctypes.c_double), ("rope_beta_fast", ctypes.c_double),
                ("rope_beta_slow", ctypes.c_double), ("rms_eps", ctypes.c_float),
                ("max_batch", ctypes.c_int), ("q_pieces", ctypes.c_int), ("cta_pairs", ctypes.c_int)]


class fm_layer_weights(ctypes.Structure):
    _fields_ = [("wq_a", ctypes.c_void_p), ("q_norm", ctypes.c_void_p),
                ("wq_b", ctypes.c_void_p), ("weights_proj", ctypes.c_void_p)]


class fm_level2_desc(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_void_p), ("positions", ctypes.c_void_p),
                ("resident_keys", ctypes.c_void_p * 4), ("resident_ids", ctypes.c_void_p),
                ("resident_count", ctypes.c_void_p), ("B", ctypes.c_int), ("R", ctypes.c_int),
                ("k", ctypes.c_int), ("mode", ctypes.c_int), ("out_ids", ctypes.c_void_p),
                ("out_count", ctypes.c_void_p)]


class fm_host_batch(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("N", ctypes.c_int), ("hidden", ctypes.c_void_p),
                ("positions", ctypes.c_void_p), ("comp_k", ctypes.c_void_p * 4),
                ("row_stride_bytes", ctypes.c_int64), ("n_valid", ctypes.c_void_p), ("mode", ctypes.c_int),
                ("top_k", ctypes.c_int), ("thr", ctypes.c_float), ("keep_topk", ctypes.c_void_p),
                ("keep_thr", ctypes.c_void_p)]


class fm_device_staging(ctypes.Structure):
    _fields_ = [("comp_k", ctypes.c_void_p * 4), ("hidden", ctypes.c_void_p), ("positions", ctypes.c_void_p),
                ("n_valid", ctypes.c_void_p), ("q", ctypes.c_void_p), ("fused_w", ctypes.c_void_p),
                ("ens", ctypes.c_void_p), ("keep_topk", ctypes.c_void_p), ("keep_thr", ctypes.c_void_p),
                ("topk_ws", ctypes.c_void_p), ("topk_ws_bytes", ctypes.c_size_t)]


class FMError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.fm_strerror(status).decode() if _lib is not None else str(status)
        extra = ""
        if status == FM_ERR_CUDA:
            extra = f" (cudaError {_lib.fm_last_cuda_error()})"
        super().__init__(f"{where}: {msg}{extra}")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libfm.so not built at {LIB_PATH}; run `python -m learned_kv_chunk_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, I64, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    sig = {
        "fm_config_default": (None, [ctypes.POINTER(fm_config)]),
        "fm_create": (I, [ctypes.POINTER(fm_config), ctypes.POINTER(fm_layer_weights), I,
                          ctypes.POINTER(P)]),
        "fm_destroy": (I, [P]),
        "fm_query_prep": (I, [P, P, P, I, P, P, P]),
        "fm_score": (I, [P, P, I64, P, I, I, P, P, P, P]),
        "fm_ensemble": (I, [P, I, I, I, I, P, P]),
        "fm_score_fused": (I, [P, P, I64, P, I, I, P, P, I, F, P, P, P, P]),
        "fm_topk_workspace_bytes": (S, [I, I]),
        "fm_topk_workspace_bytes_fast": (S, [I, I]),
        "fm_select_topk": (I, [P, P, I, I, I, P, P, S, P]),
        "fm_select_threshold": (I, [P, P, I, I, F, P, P]),
        "fm_retrieve_host": (I, [P, ctypes.POINTER(fm_host_batch), ctypes.POINTER(fm_device_staging), P]),
        "fm_select_topk_static": (I, [P, P, I, I, I, P, P]),
        "fm_compact_workspace_bytes": (S, [I, I]),
        "fm_compact_mask": (I, [P, I, I, I, P, P, P, S, P]),
        "fm_gather_records": (I, [P, I64, I, I64, P, P, I, I, P, I64, P]),
        "fm_level2_create": (I, [P, ctypes.POINTER(fm_level2_desc), P, ctypes.POINTER(P)]),
        "fm_level2_launch": (I, [P, P]),
        "fm_level2_copy_scores": (I, [P, P, P]),
        "fm_level2_destroy": (I, [P]),
        "fm_decode_attention_workspace_bytes": (S, [I, I]),
        "fm_decode_attention": (I, [P, P, I64, I, P, P, I, I, P, P, S, P]),
        "fm_toy_decoder_update": (I, [P, P, I, I, F, P, P]),
        "fm_topk_shard_begin": (I, [P, I, I, I, P, P, S, P]),
        "fm_topk_shard_hist": (I, [P, I, I, I, P, P, S, P]),
        "fm_topk_shard_pick": (I, [I, I, I, P, P, S, P]),
        "fm_topk_shard_ties": (I, [P, I, I, P, P, S, P]),
        "fm_topk_shard_mask": (I, [P, I, I, P, I, P, P, S, P]),
        "fm_sync_status": (I, [P, P]),
        "fm_strerror": (ctypes.c_char_p, [I]),
        "fm_last_cuda_error": (I, []),
        "fm_launch_count": (ctypes.c_uint64, []),
        "fm_debug_fail_alloc": (None, [I]),
        "fm_debug_live_allocations": (I64, []),
        "fm_debug_stall_next_score": (I, [P, ctypes.c_uint64]),
        "fm_debug_tile_dots": (I, [P, P, I64, I, I, P, P, I, I, I, P, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def lib():
    return _lib


def _check(status: int, where: str):
    if status != FM_OK:
        raise FMError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, dtype, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def fm_config_default() -> fm_config:
    c = fm_config()
    _lib.fm_config_default(ctypes.byref(c))
    return c


def fm_launch_count() -> int:
    return int(_lib.fm_launch_count())


def fm_topk_workspace_bytes(B: int, N: int) -> int:
    return int(_lib.fm_topk_workspace_bytes(B, N))


def fm_topk_workspace_bytes_fast(B: int, N: int) -> int:
    return int(_lib.fm_topk_workspace_bytes_fast(B, N))


def _comp_k_array(comp_k: Sequence[torch.Tensor]):
    for i, t in enumerate(comp_k):
        _need(t, torch.uint8, f"comp_k[{i}]")
    return (ctypes.c_void_p * len(comp_k))(*[t.data_ptr() for t in comp_k])


def _keys_shape(comp_k: Sequence[torch.Tensor], N: Optional[int]):
    B, N_pad, rec = comp_k[0].shape
    if rec != 132:
        raise ValueError("compressed keys must be [B, N, 132] uint8")
    for t in comp_k:
        if tuple(t.shape) != (B, N_pad, rec):
            raise ValueError("every layer's keys must have the same shape")
    N = N_pad if N is None else N
    return B, N, N_pad * 132


def fm_ensemble(scores: torch.Tensor, mode: str = "max", out: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
    _need(scores, torch.float32, "scores")
    L, B, N = scores.shape
    ens = out if out is not None else torch.empty(B, N, device=scores.device, dtype=torch.float32)
    _check(_lib.fm_ensemble(_ptr(scores), L, B, N, MODES[mode], _ptr(ens), _stream(stream)),
           "fm_ensemble")
    return ens


def fm_select_topk(ens: torch.Tensor, k: int, n_valid: Optional[torch.Tensor] = None,
                   out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    _need(ens, torch.float32, "ens")
    B, N = ens.shape
    if n_valid is not None:
        _need(n_valid, torch.int32, "n_valid")
    keep = out if out is not None else torch.empty(B, N, device=ens.device, dtype=torch.bool)
    nbytes = fm_topk_workspace_bytes_fast(B, N)
    ws = workspace if workspace is not None else torch.empty(nbytes, device=ens.device, dtype=torch.uint8)
    _check(_lib.fm_select_topk(_ptr(ens), _ptr(n_valid), B, N, int(k), _ptr(keep), _ptr(ws),
                               ws.numel(), _stream(stream)), "fm_select_topk")
    return keep


def fm_select_topk_static(ens: torch.Tensor, k: int, n_valid: Optional[torch.Tensor] = None,
                          out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """fm_select_topk without a workspace: the library's fixed scratch array
    is used, so the C call allocates nothing (for callers that cannot
    allocate device memory).  Pass `out` to allocate nothing here either."""
    _need(ens, torch.float32, "ens")
    B, N = ens.shape
    if n_valid is not None:
        _need(n_valid, torch.int32, "n_valid")
    keep = out if out is not None else torch.empty(B, N, device=ens.device, dtype=torch.bool)
    _check(_lib.fm_select_topk_static(_ptr(ens), _ptr(n_valid), B, N, int(k), _ptr(keep),
                                      _stream(stream)), "fm_select_topk_static")
    return keep


def fm_select_threshold(ens: torch.Tensor, thr: float, n_valid: Optional[torch.Tensor] = None,
                        out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _need(ens, torch.float32, "ens")
    B, N = ens.shape
    if n_valid is not None:
        _need(n_valid, torch.int32, "n_valid")
    keep = out if out is not None else torch.empty(B, N, device=ens.device, dtype=torch.bool)
    _check(_lib.fm_select_threshold(_ptr(ens), _ptr(n_valid), B, N, float(thr), _ptr(keep),
                                    _stream(stream)), "fm_select_threshold")
    return keep


def fm_compact_mask(keep: torch.Tensor, max_sel: int, idx: Optional[torch.Tensor] = None,
                    count: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                    stream=None):
    """Keep mask [B, N] (bool or uint8, device) -> (idx [B, max_sel] int32, kept
    chunk indices in increasing order then -1; count [B] int32)."""
    if keep.dtype not in (torch.bool, torch.uint8):
        raise ValueError("keep must be bool or uint8")
    if not keep.is_cuda or not keep.is_contiguous():
        raise ValueError("keep must be a contiguous CUDA tensor")
    B, N = keep.shape
    dev = keep.device
    idx = idx if idx is not None else torch.empty(B, max_sel, device=dev, dtype=torch.int32)
    count = count if count is not None else torch.empty(B, device=dev, dtype=torch.int32)
    _need(idx, torch.int32, "idx")
    _need(count, torch.int32, "count")
    nbytes = int(_lib.fm_compact_workspace_bytes(B, N))
    ws = workspace if workspace is not None else torch.empty(nbytes, device=dev, dtype=torch.uint8)
    _check(_lib.fm_compact_mask(_ptr(keep), B, N, int(max_sel), _ptr(idx), _ptr(count), _ptr(ws), ws.numel(),
                                _stream(stream)), "fm_compact_mask")
    return idx, count


def fm_gather_records(src: torch.Tensor, idx: torch.Tensor, count: torch.Tensor,
                      dst: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Resident buffer [B, max_sel, rec] (uint8, device): slot j of row b holds
    record idx[b, j] of src[b] for j < min(count[b], max_sel); other slots are
    left as they were (zeros in a new buffer).  src [B, n_src, rec] uint8 on
    the device or in pinned host memory."""
    if src.dtype != torch.uint8 or src.dim() != 3 or not src.is_contiguous():
        raise ValueError("src must be a contiguous uint8 tensor [B, n_src, rec]")
    if not src.is_cuda and not src.is_pinned():
        raise ValueError("src must be on the device or in pinned host memory")
    _need(idx, torch.int32, "idx")
    _need(count, torch.int32, "count")
    B, n_src, rec = src.shape
    max_sel = idx.shape[1]
    if dst is None:
        dst = torch.zeros(B, max_sel, rec, device=idx.device, dtype=torch.uint8)
    _need(dst, torch.uint8, "dst")
    _check(_lib.fm_gather_records(_ptr(src), n_src * rec, n_src, rec, _ptr(idx), _ptr(count), B, max_sel,
                                  _ptr(dst), dst.stride(0), _stream(stream)), "fm_gather_records")
    return dst


class Level2Step:
    """The per-step selection over a resident set, as one CUDA graph
    (fm_level2_*): query prep for the step's hidden states, scoring of the
    resident records of every layer with the ensemble, top-k, and the kept
    slots mapped to chunk ids.  The graph reads `hidden` and `positions` at
    every launch: write the next step's values into them in place
    (Level2Step.hidden.copy_(...)) and call launch().

    resident_keys: per layer [B, R, 132] uint8 (fm_gather_records' output);
    resident_ids [B, R] int32 and resident_count [B] int32 (fm_compact_mask's
    output for the resident set)."""

    def __init__(self, retriever: "Retriever", resident_keys: Sequence[torch.Tensor],
                 resident_ids: torch.Tensor, resident_count: torch.Tensor, k: int = 512, mode: str = "max",
                 stream=None):
        for i, t in enumerate(resident_keys):
            _need(t, torch.uint8, f"resident_keys[{i}]")
        _need(resident_ids, torch.int32, "resident_ids")
        _need(resident_count, torch.int32, "resident_count")
        B, R = resident_ids.shape
        dev = resident_ids.device
        cfg = retriever.cfg
        self.hidden = torch.zeros(B, cfg.hidden, device=dev, dtype=torch.float32)
        self.positions = torch.zeros(B, device=dev, dtype=torch.int64)
        self.out_ids = torch.empty(B, k, device=dev, dtype=torch.int32)
        self.out_count = torch.empty(B, device=dev, dtype=torch.int32)
        self._keep_alive = (retriever, list(resident_keys), resident_ids, resident_count)
        self.B, self.R, self.k = B, R, int(k)
        d = fm_level2_desc()
        d.hidden, d.positions = self.hidden.data_ptr(), self.positions.data_ptr()
        for l, t in enumerate(resident_keys):
            d.resident_keys[l] = t.data_ptr()
        d.resident_ids, d.resident_count = resident_ids.data_ptr(), resident_count.data_ptr()
        d.B, d.R, d.k, d.mode = B, R, int(k), MODES[mode]
        d.out_ids, d.out_count = self.out_ids.data_ptr(), self.out_count.data_ptr()
        h = ctypes.c_void_p()
        _check(_lib.fm_level2_create(retriever.handle, ctypes.byref(d), _stream(stream), ctypes.byref(h)),
               "fm_level2_create")
        self._h = h

    def launch(self, stream=None):
        _check(_lib.fm_level2_launch(self._h, _stream(stream)), "fm_level2_launch")

    def scores(self, stream=None) -> torch.Tensor:
        """The ensembled scores [B, R] of the last step (a copy)."""
        out = torch.empty(self.B, self.R, device=self.out_ids.device, dtype=torch.float32)
        _check(_lib.fm_level2_copy_scores(self._h, _ptr(out), _stream(stream)), "fm_level2_copy_scores")
        return out

    def close(self):
        if getattr(self, "_h", None):
            _lib.fm_level2_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def fm_decode_attention(q: torch.Tensor, mem: torch.Tensor, idx: Optional[torch.Tensor], count: torch.Tensor,
                        out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                        stream=None) -> torch.Tensor:
    """The toy decoder's sparse attention over the kept chunks: q [B, 32, 128]
    fp32 (the hidden state [B, 4096] viewed as 32 heads), mem [B, N, 132]
    uint8 chunk records, idx/count from fm_compact_mask; with idx None, mem
    is the resident buffer [B, max_sel, 132] of the kept records in order
    (fm_gather_records).  Returns o [B, 32, 128]."""
    _need(q, torch.float32, "q")
    _need(mem, torch.uint8, "mem")
    if idx is not None:
        _need(idx, torch.int32, "idx")
    _need(count, torch.int32, "count")
    B, n_mem, rec = mem.shape
    if rec != 132:
        raise ValueError("mem must be [B, N, 132] uint8")
    max_sel = idx.shape[1] if idx is not None else n_mem
    out = out if out is not None else torch.empty(B, 32, 128, device=q.device, dtype=torch.float32)
    nbytes = int(_lib.fm_decode_attention_workspace_bytes(B, max_sel))
    ws = workspace if workspace is not None else torch.empty(nbytes, device=q.device, dtype=torch.uint8)
    _check(_lib.fm_decode_attention(_ptr(q), _ptr(mem), n_mem * 132, n_mem, _ptr(idx), _ptr(count), B, max_sel,
                                    _ptr(out), _ptr(ws), ws.numel(), _stream(stream)), "fm_decode_attention")
    return out


def fm_toy_decoder_update(hidden: torch.Tensor, attn_out: torch.Tensor, eps: float = 1e-6,
                          out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """hidden' = RMSNorm(hidden + attn_out) (no gain); out may be hidden itself."""
    _need(hidden, torch.float32, "hidden")
    _need(attn_out, torch.float32, "attn_out")
    B, H = hidden.shape
    out = out if out is not None else torch.empty_like(hidden)
    _check(_lib.fm_toy_decoder_update(_ptr(hidden), _ptr(attn_out), B, H, float(eps), _ptr(out),
                                      _stream(stream)), "fm_toy_decoder_update")
    return out


class ToySparseDecoder:
    """The README's toy decode loop ("Toy inference reference") on synthetic
    inputs: every `interval` (64) steps the retriever scores all chunks of the
    three layers for the current hidden state and the keep mask (top-K, or
    sigmoid > threshold) is compacted into index lists; every step the toy
    decoder attends over the kept chunks of the memory layer and updates its
    hidden state (fm_decode_attention, fm_toy_decoder_update).  Positions
    advance by one token per step from `positions`."""

    def __init__(self, retriever: "Retriever", comp_k: Sequence[torch.Tensor], n_valid: torch.Tensor,
                 hidden: torch.Tensor, positions: torch.Tensor, top_k: Optional[int] = 512,
                 threshold: Optional[float] = None, mode: str = "max", interval: int = 64,
                 memory_layer: int = 0):
        if (top_k is None) == (threshold is None):
            raise ValueError("give exactly one of top_k and threshold")
        self.r, self.comp_k, self.n_valid = retriever, list(comp_k), n_valid
        self.B, self.N = comp_k[0].shape[0], comp_k[0].shape[1]
        dev = hidden.device
        self.hidden = hidden.clone()
        self.positions0 = positions.detach().to("cpu", torch.int64)
        self.top_k, self.threshold, self.mode, self.interval = top_k, threshold, mode, int(interval)
        self.mem = self.comp_k[memory_layer]
        self.max_sel = int(top_k) if top_k is not None else self.N
        self.idx = torch.empty(self.B, self.max_sel, device=dev, dtype=torch.int32)
        self.count = torch.empty(self.B, device=dev, dtype=torch.int32)
        # top-K: the kept records are gathered once per retrieval into a
        # resident buffer that every step's attention reads in order
        self.resident = (torch.empty(self.B, self.max_sel, 132, device=dev, dtype=torch.uint8)
                         if top_k is not None else None)
        self.attn = torch.empty(self.B, 32, 128, device=dev, dtype=torch.float32)
        self._cws = torch.empty(int(_lib.fm_compact_workspace_bytes(self.B, self.N)), device=dev,
                                dtype=torch.uint8)
        self._aws = torch.empty(int(_lib.fm_decode_attention_workspace_bytes(self.B, self.max_sel)), device=dev,
                                dtype=torch.uint8)
        self.t = 0
        self.keep = None
        self.ens = None

    def retrieve(self):
        pos = (self.positions0 + self.t).to(self.hidden.device)
        ens, keep_topk, keep_thr = self.r.retrieve(self.hidden, self.comp_k, pos, self.n_valid, self.mode,
                                                   self.top_k, self.threshold, self.N)
        self.ens = ens
        self.keep = keep_topk if self.top_k is not None else keep_thr
        fm_compact_mask(self.keep, self.max_sel, idx=self.idx, count=self.count, workspace=self._cws)
        if self.resident is not None:
            fm_gather_records(self.mem, self.idx, self.count, self.resident)

    def attend(self):
        """The sparse attention of the current hidden state over the kept chunks."""
        if self.resident is not None:
            return fm_decode_attention(self.hidden.view(self.B, 32, 128), self.resident, None, self.count,
                                       out=self.attn, workspace=self._aws)
        return fm_decode_attention(self.hidden.view(self.B, 32, 128), self.mem, self.idx, self.count,
                                   out=self.attn, workspace=self._aws)

    def step(self):
        """One decode step; returns the new hidden state [B, 4096]."""
        if self.t % self.interval == 0:
            self.retrieve()
        self.attend()
        fm_toy_decoder_update(self.hidden, self.attn.view(self.B, -1), out=self.hidden)
        self.t += 1
        return self.hidden


class TopKShard:
    """One shard's side of the sharded top-K (fm_topk_shard_*): this shard's
    slice `ens_local` [B, N] of rows whose chunks are split over the shards in
    shard order, with its buffers (workspace, the histogram the shards sum, the
    tie count they gather, the keep mask).  The phases are called in the order
    fm_select_topk_sharded uses; the exchanges between them are the caller's."""

    def __init__(self, ens_local: torch.Tensor, k: int, n_valid_local: Optional[torch.Tensor] = None,
                 stream=None):
        _need(ens_local, torch.float32, "ens_local")
        if n_valid_local is not None:
            _need(n_valid_local, torch.int32, "n_valid_local")
        self.ens, self.k, self.n_valid, self.stream = ens_local, int(k), n_valid_local, stream
        self.B, self.N = ens_local.shape
        dev = ens_local.device
        self.ws = torch.empty(fm_topk_workspace_bytes(self.B, self.N), device=dev, dtype=torch.uint8)
        self.hist = torch.empty(self.B, FM_TOPK_SHARD_BINS, device=dev, dtype=torch.int32)
        self.eq_local = torch.empty(self.B, device=dev, dtype=torch.int32)
        self.keep = torch.empty(self.B, self.N, device=dev, dtype=torch.bool)

    def _tail(self):
        return _ptr(self.ws), self.ws.numel(), _stream(self.stream)

    def begin(self):
        _check(_lib.fm_topk_shard_begin(_ptr(self.n_valid), self.B, self.N, self.k, _ptr(self.hist),
                                        *self._tail()), "fm_topk_shard_begin")

    def hist_pass(self, p: int) -> torch.Tensor:
        """This slice's histogram of pass p, to be summed over the shards in place."""
        _check(_lib.fm_topk_shard_hist(_ptr(self.ens), self.B, self.N, p, _ptr(self.hist), *self._tail()),
               "fm_topk_shard_hist")
        return self.hist

    def pick(self, p: int):
        _check(_lib.fm_topk_shard_pick(self.B, self.N, p, _ptr(self.hist), *self._tail()),
               "fm_topk_shard_pick")

    def ties(self) -> torch.Tensor:
        """This slice's count of keys equal to the K-th, per row, to be gathered."""
        _check(_lib.fm_topk_shard_ties(_ptr(self.ens), self.B, self.N, _ptr(self.eq_local), *self._tail()),
               "fm_topk_shard_ties")
        return self.eq_local

    def mask(self, eq_all: torch.Tensor, shard: int) -> torch.Tensor:
        _need(eq_all, torch.int32, "eq_all")
        _check(_lib.fm_topk_shard_mask(_ptr(self.ens), self.B, self.N, _ptr(eq_all), int(shard),
                                       _ptr(self.keep), *self._tail()), "fm_topk_shard_mask")
        return self.keep


class TorchDistExchange:
    """The two exchanges of the sharded top-K over a torch.distributed group
    (NCCL between GPUs): a sum of the histograms and a gather of the tie counts.
    The shard index is the rank in the group."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def all_reduce_sum_(self, t: torch.Tensor):
        self.dist.all_reduce(t, op=self.dist.ReduceOp.SUM, group=self.group)

    def all_gather(self, t: torch.Tensor) -> torch.Tensor:
        t = t.contiguous()
        out = torch.empty(self.world * t.numel(), device=t.device, dtype=t.dtype)
        self.dist.all_gather_into_tensor(out, t.reshape(-1), group=self.group)
        return out.view((self.world,) + tuple(t.shape))


def fm_select_topk_sharded(ens_local: torch.Tensor, k: int, n_valid_local: Optional[torch.Tensor] = None,
                           exchange=None, shard=None) -> torch.Tensor:
    """Top-K keep mask of rows split over the ranks of a group: rank g holds the
    g-th consecutive slice of every row (`ens_local` [B, N_g]).  Returns this
    rank's slice of the mask that fm_select_topk gives on the whole rows.  Per
    pass one all-reduce of B*2048 int32, then one all-gather of B int32;
    scores never leave their GPU.  `exchange` defaults to the default
    torch.distributed group; `shard` (an object with TopKShard's phases)
    defaults to this library's kernels."""
    ex = exchange if exchange is not None else TorchDistExchange()
    sh = shard if shard is not None else TopKShard(ens_local, k, n_valid_local)
    sh.begin()
    for p in range(3):
        ex.all_reduce_sum_(sh.hist_pass(p))
        sh.pick(p)
    eq_all = ex.all_gather(sh.ties())
    return sh.mask(eq_all, ex.rank)


class Retriever:
    """A libfm context: the three CSA layers' weights on one device.

    weights: list (one per layer) of dicts with fp32 tensors wq_a [R, HID],
    q_norm [R], wq_b [H*D, R], weights_proj [H, HID] (CPU or CUDA)."""

    def __init__(self, weights: List[dict], device: int = 0, max_batch: int = 64,
                 q_pieces: int = 2, **overrides):
        cfg = fm_config_default()
        cfg.n_layers = len(weights)
        cfg.max_batch = max_batch
        cfg.q_pieces = q_pieces
        for k, v in overrides.items():
            setattr(cfg, k, v)
        self.cfg = cfg
        self.device = device
        keep = []
        arr = (fm_layer_weights * len(weights))()
        for i, w in enumerate(weights):
            ts = {k: w[k].detach().to(torch.float32).contiguous() for k in
                  ("wq_a", "q_norm", "wq_b", "weights_proj")}
            keep.append(ts)
            arr[i] = fm_layer_weights(*[ts[k].data_ptr() for k in ("wq_a", "q_norm", "wq_b", "weights_proj")])
        h = ctypes.c_void_p()
        _check(_lib.fm_create(ctypes.byref(cfg), arr, device, ctypes.byref(h)), "fm_create")
        self._h = h
        self.L = cfg.n_layers

    def close(self):
        if getattr(self, "_h", None):
            _lib.fm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def handle(self):
        return self._h

    def fm_query_prep(self, hidden: torch.Tensor, positions: torch.Tensor, q=None, fused_w=None,
                      stream=None):
        _need(hidden, torch.float32, "hidden")
        _need(positions, torch.int64, "positions")
        B = hidden.shape[0]
        dev = hidden.device
        q = q if q is not None else torch.empty(B, self.L, 64, 128, device=dev, dtype=torch.float32)
        fused_w = fused_w if fused_w is not None else torch.empty(B, self.L, 64, device=dev, dtype=torch.float32)
        _check(_lib.fm_query_prep(self._h, _ptr(hidden), _ptr(positions), B, _ptr(q), _ptr(fused_w),
                                  _stream(stream)), "fm_query_prep")
        return q, fused_w

    def fm_score(self, comp_k: Sequence[torch.Tensor], q: torch.Tensor, fused_w: torch.Tensor,
                 n_valid: Optional[torch.Tensor] = None, N: Optional[int] = None, out=None,
                 stream=None) -> torch.Tensor:
        B, N, stride = _keys_shape(comp_k, N)
        arr = _comp_k_array(comp_k)
        _need(q, torch.float32, "q")
        _need(fused_w, torch.float32, "fused_w")
        if n_valid is not None:
            _need(n_valid, torch.int32, "n_valid")
        scores = out if out is not None else torch.empty(self.L, B, N, device=q.device, dtype=torch.float32)
        _check(_lib.fm_score(self._h, arr, stride, _ptr(n_valid), B, N, _ptr(q), _ptr(fused_w),
                             _ptr(scores), _stream(stream)), "fm_score")
        return scores

    def fm_score_fused(self, comp_k: Sequence[torch.Tensor], q: torch.Tensor, fused_w: torch.Tensor,
                       mode: str = "max", threshold: Optional[float] = None,
                       n_valid: Optional[torch.Tensor] = None, N: Optional[int] = None,
                       want_layers: bool = False, ens=None, keep_thr=None, scores=None, stream=None):
        B, N, stride = _keys_shape(comp_k, N)
        arr = _comp_k_array(comp_k)
        _need(q, torch.float32, "q")
        _need(fused_w, torch.float32, "fused_w")
        if n_valid is not None:
            _need(n_valid, torch.int32, "n_valid")
        dev = q.device
        ens = ens if ens is not None else torch.empty(B, N, device=dev, dtype=torch.float32)
        if threshold is not None and keep_thr is None:
            keep_thr = torch.empty(B, N, device=dev, dtype=torch.bool)
        if want_layers and scores is None:
            scores = torch.empty(self.L, B, N, device=dev, dtype=torch.float32)
        thr = 0.0 if threshold is None else float(threshold)
        _check(_lib.fm_score_fused(self._h, arr, stride, _ptr(n_valid), B, N, _ptr(q), _ptr(fused_w),
                                   MODES[mode], thr, _ptr(scores), _ptr(ens),
                                   _ptr(keep_thr if threshold is not None else None),
                                   _stream(stream)), "fm_score_fused")
        return ens, keep_thr, scores

    def fm_sync_status(self, stream=None):
        _check(_lib.fm_sync_status(self._h, _stream(stream)), "fm_sync_status")

    def fm_debug_tile_dots(self, comp_k, q, fused_w, layer: int, b: int, t: int, N=None):
        B, N, stride = _keys_shape(comp_k, N)
        arr = _comp_k_array(comp_k)
        out = torch.zeros((128, 192), device=q.device, dtype=torch.float32)
        e = torch.zeros(64, device=q.device, dtype=torch.int32)
        _check(_lib.fm_debug_tile_dots(self._h, arr, stride, B, N, _ptr(q), _ptr(fused_w), layer, b, t,
                                       _ptr(out), _ptr(e), _stream()), "fm_debug_tile_dots")
        return out, e

    def retrieve_from_host(self, hidden, positions, comp_k, n_valid=None, mode="max", top_k=None,
                           threshold=None, N=None, device_buffers: Optional[dict] = None, sync=True):
        """The whole path for inputs in (pinned) host memory through the C call
        fm_retrieve_host: host inputs copied to device staging buffers, query
        prep, scoring, top-K, masks copied back.  Returns (keep_topk, keep_thr)
        as host uint8 tensors (either may be None).  `device_buffers` (a dict)
        keeps the staging buffers and the host masks between calls."""
        dev = torch.device("cuda", self.device)
        buf = device_buffers if device_buffers is not None else {}
        B, N_pad, rec = comp_k[0].shape
        N = N_pad if N is None else N
        for t in list(comp_k) + [hidden, positions] + ([n_valid] if n_valid is not None else []):
            if t.is_cuda or not t.is_contiguous():
                raise ValueError("fm_retrieve_host takes contiguous host tensors")

        def dbuf(name, shape, dtype):
            d = buf.get(name)
            if d is None or tuple(d.shape) != tuple(shape) or d.dtype != dtype:
                d = buf[name] = torch.empty(shape, dtype=dtype, device=dev)
            return d

        def hbuf(name, shape):
            h = buf.get(name)
            if h is None or tuple(h.shape) != tuple(shape):
                h = buf[name] = torch.empty(shape, dtype=torch.uint8, pin_memory=True)
            return h

        st = fm_device_staging()
        for l, t in enumerate(comp_k):
            st.comp_k[l] = dbuf(f"keys{l}", t.shape, torch.uint8).data_ptr()
        st.hidden = dbuf("hidden", hidden.shape, torch.float32).data_ptr()
        st.positions = dbuf("positions", positions.shape, torch.int64).data_ptr()
        st.n_valid = dbuf("n_valid", (B,), torch.int32).data_ptr()
        st.q = dbuf("q", (B, self.L, 64, 128), torch.float32).data_ptr()
        st.fused_w = dbuf("fused_w", (B, self.L, 64), torch.float32).data_ptr()
        st.ens = dbuf("ens", (B, N), torch.float32).data_ptr()
        st.keep_topk = dbuf("keep_topk", (B, N), torch.uint8).data_ptr()
        st.keep_thr = dbuf("keep_thr", (B, N), torch.uint8).data_ptr()
        ws = dbuf("topk_ws", (fm_topk_workspace_bytes_fast(B, N),), torch.uint8)
        st.topk_ws, st.topk_ws_bytes = ws.data_ptr(), ws.numel()
        hb = fm_host_batch()
        hb.B, hb.N = B, N
        hb.hidden, hb.positions = hidden.data_ptr(), positions.data_ptr()
        for l, t in enumerate(comp_k):
            hb.comp_k[l] = t.data_ptr()
        hb.row_stride_bytes = N_pad * rec
        hb.n_valid = n_valid.data_ptr() if n_valid is not None else None
        hb.mode = MODES[mode]
        hb.top_k = int(top_k) if top_k is not None else 0
        hb.thr = 0.0 if threshold is None else float(threshold)
        out_topk = hbuf("out_topk", (B, N)) if top_k is not None else None
        out_thr = hbuf("out_thr", (B, N)) if threshold is not None else None
        hb.keep_topk = out_topk.data_ptr() if out_topk is not None else None
        hb.keep_thr = out_thr.data_ptr() if out_thr is not None else None
        _check(_lib.fm_retrieve_host(self._h, ctypes.byref(hb), ctypes.byref(st), _stream()), "fm_retrieve_host")
        if sync:
            self.fm_sync_status()
        return out_topk, out_thr

    # the pages' calls, composed (README "Usage")
    def retrieve(self, hidden, comp_k, positions, n_valid=None, mode="max", top_k=None,
                 threshold=None, N=None):
        q, w = self.fm_query_prep(hidden, positions)
        ens, keep_thr, _ = self.fm_score_fused(comp_k, q, w, mode=mode, threshold=threshold,
                                               n_valid=n_valid, N=N)
        keep_topk = fm_select_topk(ens, top_k, n_valid) if top_k is not None else None
        return ens, keep_topk, keep_thr
