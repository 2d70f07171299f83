"""Plant plausible mistakes in the CPU oracle (on the CPU, one at a time) and
check that the pins in test_oracle_pins.py catch every one of them."""
import numpy as np
import pytest

import oracle.retriever as O
from tests import test_oracle_pins as P


def _e4m3_bias8(codes):
    c = np.asarray(codes).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -7, (1.0 + m / 8.0) * np.exp2(e - 8.0))
    return (sign * mag).astype(np.float32)


def _split_big_endian(comp_k, head_dim=128):
    comp_k = np.asarray(comp_k, np.uint8)
    s = np.ascontiguousarray(comp_k[..., head_dim:head_dim + 4]).view(">f4")[..., 0]
    return comp_k[..., :head_dim], s.astype(np.float32)


def _rms_no_eps(x, g, eps=1e-6):
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.mean(x * x, -1, keepdims=True)) * g


def _rms_sum(x, g, eps=1e-6):
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.sum(x * x, -1, keepdims=True) + eps) * g


def _yarn_reversed(rope_dim=64, base=160000.0, factor=16.0, orig_max_pos=65536.0,
                   beta_fast=32.0, beta_slow=1.0):
    j = np.arange(rope_dim // 2, dtype=np.float64)
    inv = base ** (-2.0 * j / rope_dim)
    ramp = np.clip((j - 15) / 10, 0, 1)
    return inv * ramp + inv / factor * (1 - ramp)


def _rotary_sign(q, theta, rope_dim=64):
    return O.__dict__["_orig_apply_rotary"](q, -np.asarray(theta), rope_dim)


def _rotary_interleaved(q, theta, rope_dim=64):
    q = np.array(q, np.float64, copy=True)
    c = np.cos(theta)[..., None, :]
    s = np.sin(theta)[..., None, :]
    x1 = q[..., 64::2].copy()
    x2 = q[..., 65::2].copy()
    q[..., 64::2] = x1 * c - x2 * s
    q[..., 65::2] = x2 * c + x1 * s
    return q


def _rotary_first_half(q, theta, rope_dim=64):
    q = np.array(q, np.float64, copy=True)
    c = np.cos(theta)[..., None, :]
    s = np.sin(theta)[..., None, :]
    x1 = q[..., 0:32].copy()
    x2 = q[..., 32:64].copy()
    q[..., 0:32] = x1 * c - x2 * s
    q[..., 32:64] = x2 * c + x1 * s
    return q


def _wht_unnormalised(q):
    return np.asarray(q, np.float64) @ O.hadamard_matrix(q.shape[-1]).T


def _score_relu_after_weight(comp_k, q, w):
    k = O.dequant(comp_k, q.shape[-1]).astype(np.float64)
    return O.sigmoid(np.maximum((k @ q.T) * w, 0).sum(-1))


def _score_no_scale(comp_k, q, w):
    codes, _ = O.split_records(comp_k, q.shape[-1])
    k = O.e4m3_decode(codes).astype(np.float64)
    return O.sigmoid(np.maximum(k @ q.T, 0) @ w)


def _score_transposed_q(comp_k, q, w):
    k = O.dequant(comp_k, q.shape[-1]).astype(np.float64)
    qt = q.T[: q.shape[0]] if q.shape[0] <= q.shape[1] else q
    return O.sigmoid(np.maximum(k[:, : qt.shape[1]] @ qt.T, 0) @ w)


def _score_scale_after_relu(comp_k, q, w):
    codes, scale = O.split_records(comp_k, q.shape[-1])
    k8 = O.e4m3_decode(codes).astype(np.float64)
    return O.sigmoid((np.maximum(k8 @ q.T, 0) * scale[:, None]) @ w)


def _score_relu_drops_nan(comp_k, q, w):
    k = O.dequant(comp_k, q.shape[-1]).astype(np.float64)
    return O.sigmoid(np.fmax(k @ q.T, 0) @ w)


def _ensemble_max_drops_nan(scores, mode="max"):
    s = np.asarray(scores, np.float64)
    return np.fmax.reduce(s, axis=0) if mode == "max" else O.__dict__["_orig_ensemble"](s, mode)


def _topk_nan_high(ens, n_valid, k):
    ens = np.asarray(ens, np.float64)
    keep = np.zeros(ens.shape, bool)
    for b in range(ens.shape[0]):
        n = int(n_valid[b])
        key = np.where(np.isnan(ens[b, :n]), np.inf, ens[b, :n])
        order = np.lexsort((np.arange(n), -key))
        keep[b, order[:min(k, n)]] = True
    return keep


def _threshold_nan_kept(ens, n_valid, thr):
    ens = np.asarray(ens)
    valid = np.arange(ens.shape[1])[None, :] < np.asarray(n_valid).reshape(-1, 1)
    return valid & ~(ens <= thr)


def _ensemble_sum(scores, mode="max"):
    s = np.asarray(scores, np.float64)
    return s.max(0) if mode == "max" else s.sum(0)


def _topk_ties_high(ens, n_valid, k):
    ens = np.asarray(ens)
    keep = np.zeros(ens.shape, bool)
    for b in range(ens.shape[0]):
        n = int(n_valid[b])
        order = np.lexsort((-np.arange(n), -ens[b, :n].astype(np.float64)))
        keep[b, order[:min(k, n)]] = True
    return keep


def _threshold_ge(ens, n_valid, thr):
    ens = np.asarray(ens)
    valid = np.arange(ens.shape[1])[None, :] < np.asarray(n_valid).reshape(-1, 1)
    return valid & (ens >= thr)


def _fused_w_wrong_scale(layer, hidden, positions, n_heads=64, head_dim=128, rms_eps=1e-6, rope=None):
    q, w = O.__dict__["_orig_query_prep"](layer, hidden, positions, n_heads, head_dim, rms_eps, rope)
    return q, w * (head_dim ** -0.5)


MUTATIONS = [
    ("e4m3_decode", _e4m3_bias8),
    ("split_records", _split_big_endian),
    ("linear", lambda W, x: np.asarray(x, np.float64) @ np.asarray(W, np.float64)),
    ("rms_norm", _rms_no_eps),
    ("rms_norm", _rms_sum),
    ("yarn_inv_freq", _yarn_reversed),
    ("apply_rotary", _rotary_sign),
    ("apply_rotary", _rotary_interleaved),
    ("apply_rotary", _rotary_first_half),
    ("hadamard_transform", _wht_unnormalised),
    ("hadamard_transform", lambda q: np.asarray(q, np.float64)),
    ("score_chunks", _score_relu_after_weight),
    ("score_chunks", _score_no_scale),
    ("score_chunks", _score_transposed_q),
    ("score_chunks", _score_scale_after_relu),
    ("score_chunks", _score_relu_drops_nan),
    ("ensemble", _ensemble_sum),
    ("ensemble", _ensemble_max_drops_nan),
    ("select_topk", _topk_ties_high),
    ("select_topk", _topk_nan_high),
    ("select_threshold", _threshold_ge),
    ("select_threshold", _threshold_nan_kept),
    ("query_prep", _fused_w_wrong_scale),
]

PINS = [getattr(P, n) for n in dir(P) if n.startswith("test_")]


@pytest.mark.parametrize("name,fn", MUTATIONS, ids=[f"{n}:{f.__name__}" for n, f in MUTATIONS])
def test_pins_catch_planted_mistake(monkeypatch, name, fn):
    monkeypatch.setitem(O.__dict__, "_orig_" + name, getattr(O, name))
    monkeypatch.setattr(O, name, fn)
    caught = []
    for pin in PINS:
        try:
            pin()
        except Exception:  # noqa: BLE001 - any failure counts as detection
            caught.append(pin.__name__)
    assert caught, f"no pin caught the mutation {name}:{fn.__name__}"


# ------------------------------------------------------------------ recall
import oracle.recall as OR  # noqa: E402


def _compact_count_capped(keep, max_sel):
    idx, count = OR.__dict__["_orig_compact_mask"](keep, max_sel)
    return idx, np.minimum(count, max_sel).astype(np.int32)


def _compact_fill_zero(keep, max_sel):
    idx, count = OR.__dict__["_orig_compact_mask"](keep, max_sel)
    return np.where(idx < 0, 0, idx).astype(np.int32), count


def _compact_descending(keep, max_sel):
    keep = np.asarray(keep)
    return OR.__dict__["_orig_compact_mask"](keep[:, ::-1], max_sel)


def _compact_one_based(keep, max_sel):
    idx, count = OR.__dict__["_orig_compact_mask"](keep, max_sel)
    return np.where(idx >= 0, idx + 1, -1).astype(np.int32), count


def _gather_ignores_idx(src, idx, count, dst):
    out = np.array(dst, copy=True)
    for b in range(src.shape[0]):
        m = min(int(count[b]), idx.shape[1], src.shape[1])
        out[b, :m] = src[b, :m]
    return out


def _gather_row_zero(src, idx, count, dst):
    return OR.__dict__["_orig_gather_records"](np.broadcast_to(src[:1], src.shape), idx, count, dst)


RECALL_MUTATIONS = [
    ("compact_mask", _compact_count_capped),
    ("compact_mask", _compact_fill_zero),
    ("compact_mask", _compact_descending),
    ("compact_mask", _compact_one_based),
    ("gather_records", _gather_ignores_idx),
    ("gather_records", _gather_row_zero),
]


@pytest.mark.parametrize("name,fn", RECALL_MUTATIONS, ids=[f"{n}:{f.__name__}" for n, f in RECALL_MUTATIONS])
def test_recall_pins_catch_planted_mistake(monkeypatch, name, fn):
    monkeypatch.setitem(OR.__dict__, "_orig_" + name, getattr(OR, name))
    monkeypatch.setattr(OR, name, fn)
    caught = []
    for pin in PINS:
        try:
            pin()
        except Exception:  # noqa: BLE001 - any failure counts as detection
            caught.append(pin.__name__)
    assert caught, f"no pin caught the mutation {name}:{fn.__name__}"


# -------------------------------------------------------------- toy decode
import math  # noqa: E402

import oracle.decode as OD  # noqa: E402


def _attn_generic(q, x, keep, scale=True, mask_value=-np.inf, normalise=True, over_heads=False):
    q = np.asarray(q, np.float64)
    x = np.asarray(x, np.float64)
    B, H, D = q.shape
    out = np.zeros((B, H, D))
    for b in range(B):
        if not keep[b].any():
            continue
        lg = q[b] @ x[b].T / (math.sqrt(D) if scale else 1.0)
        lg = np.where(keep[b][None, :], lg, mask_value)
        ax = 0 if over_heads else 1
        e = np.exp(lg - lg.max(axis=ax, keepdims=True))
        p = e / e.sum(axis=ax, keepdims=True) if normalise else e
        out[b] = p @ x[b]
    return out


def _update_no_residual(hidden, o, eps=1e-6):
    return OD.__dict__["_orig_toy_update"](np.zeros_like(hidden), o, eps)


def _step_dim_major(hidden, x, keep):
    B = hidden.shape[0]
    q = np.asarray(hidden, np.float64).reshape(B, 128, 32).transpose(0, 2, 1)
    return OD.toy_update(hidden, OD.masked_attention(q, x, keep))


DECODE_MUTATIONS = [
    ("masked_attention", lambda q, x, k: _attn_generic(q, x, k, scale=False)),
    ("masked_attention", lambda q, x, k: _attn_generic(q, x, k, mask_value=0.0)),
    ("masked_attention", lambda q, x, k: _attn_generic(q, x, k, normalise=False)),
    ("masked_attention", lambda q, x, k: _attn_generic(q, x, k, over_heads=True)),
    ("toy_update", _update_no_residual),
    ("toy_step", _step_dim_major),
]


@pytest.mark.parametrize("name,fn", DECODE_MUTATIONS, ids=[f"{n}:{i}" for i, (n, _) in enumerate(DECODE_MUTATIONS)])
def test_decode_pins_catch_planted_mistake(monkeypatch, name, fn):
    monkeypatch.setitem(OD.__dict__, "_orig_" + name, getattr(OD, name))
    monkeypatch.setattr(OD, name, fn)
    caught = []
    for pin in PINS:
        try:
            pin()
        except Exception:  # noqa: BLE001 - any failure counts as detection
            caught.append(pin.__name__)
    assert caught, f"no pin caught the mutation {name}"
