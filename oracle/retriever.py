"""Plain CPU oracle of the FlashMemory DS-V4 retriever path (numpy, fp64).

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
cpu_baseline / reference leg of bench.py may import this module.  It shares
no code, header, table or constant with the CUDA library and never imports it.

Source: the FlashMemory DS-V4 Retriever README (libertywing/FlashMemory-
Deepseek-V4, translated copy on bittide.aicompass.dev), sections
"compressed_k format", "Architecture" and "Joint checkpoint + ensemble", and
the decode-loop figure of its "Toy inference reference" section.  Every
function below restates one arrow of the Architecture figure in the order the
figure gives it.  Arithmetic is fp64 except where the README fixes fp32 (the
key dequantisation `fp8_values.view(float8_e4m3).float() * scale`).

Readings of points the pages leave open:
  * linear maps are bias-free, weights stored [out, in];
  * RMSNorm is x * (mean(x^2) + eps)^-1/2 * g;
  * RoPE acts on the last 64 dims in half-split pairs (64+j, 96+j); YaRN
    scales the inverse frequencies with the ramp between the beta_fast and
    beta_slow correction dims, and no magnitude factor is applied to q;
  * the Hadamard transform is the Sylvester (natural) order, scaled by
    128^-1/2, applied to q only;
  * e4m3 is the OCP "fn" variant (bias 7, no infinities, S.1111.111 = NaN);
  * the per-chunk scale multiplies the codes before the head dot products, so
    the relu sees the scaled dot product whatever the scale's sign;
  * a NaN code or scale makes the chunk's score NaN (relu, sigmoid and the
    ensembles carry NaN, as torch's do); top-K ranks NaN below every number,
    ties by chunk index, and NaN > thr is false;
  * top-K ties go to the lower chunk index, K >= n keeps every valid chunk;
    the threshold test is strict (score > thr);
  * chunks past a row's valid length score 0 and are never kept.

Parity pins for every function live in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import math

import numpy as np

# ----------------------------------------------------------------------------
# compressed_k record: 128 e4m3 bytes + one little-endian fp32 scale
# (README "compressed_k format"; restated on the news.ditty.ir summary page)
# ----------------------------------------------------------------------------


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """OCP E4M3 ("fn") byte -> float32 value (exact).

    sign = bit 7, exponent = bits 6..3 (bias 7), mantissa = bits 2..0;
    exponent 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; no infinities.
    """
    c = np.asarray(codes).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & ((c & 0x7) == 7), np.nan, mag)
    return (sign * mag).astype(np.float32)


def split_records(comp_k: np.ndarray, head_dim: int = 128):
    """[..., head_dim+4] uint8 -> (codes [..., head_dim] uint8, scale [...] float32)."""
    comp_k = np.asarray(comp_k, dtype=np.uint8)
    assert comp_k.shape[-1] == head_dim + 4
    codes = comp_k[..., :head_dim]
    scale = np.ascontiguousarray(comp_k[..., head_dim:head_dim + 4]).view("<f4")[..., 0]
    return codes, scale.astype(np.float32)


def dequant(comp_k: np.ndarray, head_dim: int = 128) -> np.ndarray:
    """k = e4m3(bytes[:D]).float() * f32(bytes[D:D+4]), in fp32 as the README writes it."""
    codes, scale = split_records(comp_k, head_dim)
    return (e4m3_decode(codes) * scale[..., None]).astype(np.float32)


# ----------------------------------------------------------------------------
# query side (README "Architecture", upper two chains)
# ----------------------------------------------------------------------------


def linear(W: np.ndarray, x: np.ndarray) -> np.ndarray:
    """y = W x for W [out, in] and x [..., in] (no bias)."""
    return np.asarray(x, np.float64) @ np.asarray(W, np.float64).T


def rms_norm(x: np.ndarray, g: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * g over the last axis."""
    x = np.asarray(x, np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(g, np.float64)


def yarn_correction_range(rope_dim, base, orig_max_pos, beta_fast, beta_slow):
    """Integer band [low, high] of rotary pair indices between YaRN's two
    correction dims: dim(r) = rope_dim * ln(orig / (2 pi r)) / (2 ln base)."""
    def dim_of(n_rot):
        return rope_dim * math.log(orig_max_pos / (n_rot * 2.0 * math.pi)) / (2.0 * math.log(base))
    low = max(math.floor(dim_of(beta_fast)), 0)
    high = min(math.ceil(dim_of(beta_slow)), rope_dim - 1)
    return low, high


def yarn_inv_freq(rope_dim=64, base=160000.0, factor=16.0, orig_max_pos=65536.0,
                  beta_fast=32.0, beta_slow=1.0) -> np.ndarray:
    """fp64 [rope_dim/2] rotary frequencies f_j with YaRN interpolation:
    f_j = inv_j (1 - ramp_j) + (inv_j / factor) ramp_j, inv_j = base^(-2j/rope_dim),
    ramp_j = clamp((j - low) / (high - low), 0, 1)."""
    half = rope_dim // 2
    j = np.arange(half, dtype=np.float64)
    inv = base ** (-2.0 * j / rope_dim)
    low, high = yarn_correction_range(rope_dim, base, orig_max_pos, beta_fast, beta_slow)
    span = (high - low) if high != low else 0.001
    ramp = np.clip((j - low) / span, 0.0, 1.0)
    return inv * (1.0 - ramp) + (inv / factor) * ramp


def rope_angles(positions: np.ndarray, freqs: np.ndarray) -> np.ndarray:
    """theta[b, j] = pos_b * f_j (fp64)."""
    return np.asarray(positions, np.float64)[..., None] * np.asarray(freqs, np.float64)


def apply_rotary(q: np.ndarray, theta: np.ndarray, rope_dim: int = 64) -> np.ndarray:
    """Rotate the last rope_dim dims of q [..., H, D] by theta [..., rope_dim/2]
    (broadcast over heads), half-split pairs (D-rope_dim+j, D-rope_dim/2+j):
    x1' = x1 cos - x2 sin, x2' = x2 cos + x1 sin.  Dims before them are kept."""
    q = np.array(q, np.float64, copy=True)
    D = q.shape[-1]
    half = rope_dim // 2
    lo = D - rope_dim
    c = np.cos(theta)[..., None, :]
    s = np.sin(theta)[..., None, :]
    x1 = q[..., lo:lo + half].copy()
    x2 = q[..., lo + half:D].copy()
    q[..., lo:lo + half] = x1 * c - x2 * s
    q[..., lo + half:D] = x2 * c + x1 * s
    return q


def hadamard_matrix(n: int) -> np.ndarray:
    """Sylvester-order Hadamard matrix H[i, j] = (-1)^popcount(i & j)."""
    i = np.arange(n)
    bits = np.bitwise_and(i[:, None], i[None, :])
    pc = np.zeros_like(bits)
    while np.any(bits):
        pc += bits & 1
        bits >>= 1
    return np.where(pc % 2 == 0, 1.0, -1.0)


def hadamard_transform(q: np.ndarray) -> np.ndarray:
    """Normalised Walsh-Hadamard transform of the last axis: H q / sqrt(D)."""
    D = q.shape[-1]
    return np.asarray(q, np.float64) @ hadamard_matrix(D).T / math.sqrt(D)


def query_prep(layer: dict, hidden: np.ndarray, positions: np.ndarray,
               n_heads: int = 64, head_dim: int = 128, rms_eps: float = 1e-6,
               rope: dict | None = None):
    """One CSA layer's indexer query and head weights.

    hidden [B, hid] -> wq_a -> RMSNorm(q_norm) -> wq_b -> [B, H, D]
    -> YaRN RoPE on the last 64 dims -> Hadamard  = q [B, H, D];
    hidden -> weights_proj -> * D^-1/2 H^-1/2     = fused_w [B, H].
    """
    rope = dict(rope or dict(rope_dim=64, base=160000.0, factor=16.0,
                             orig_max_pos=65536.0, beta_fast=32.0, beta_slow=1.0))
    B = hidden.shape[0]
    a = linear(layer["wq_a"], hidden)
    r = rms_norm(a, layer["q_norm"], rms_eps)
    qf = linear(layer["wq_b"], r).reshape(B, n_heads, head_dim)
    theta = rope_angles(positions, yarn_inv_freq(**rope))
    qr = apply_rotary(qf, theta, rope["rope_dim"])
    q = hadamard_transform(qr)
    fused_w = linear(layer["weights_proj"], hidden) * (head_dim ** -0.5 * n_heads ** -0.5)
    return q, fused_w


# ----------------------------------------------------------------------------
# key side and score (README "Architecture", last chain and score line)
# ----------------------------------------------------------------------------


def sigmoid(x):
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-np.asarray(x, np.float64)))


def score_chunks(comp_k: np.ndarray, q: np.ndarray, fused_w: np.ndarray) -> np.ndarray:
    """score[n] = sigmoid(sum_h relu(k_n . q_h) * fused_w_h) for one row.

    comp_k [n, D+4] uint8, q [H, D], fused_w [H] -> [n] fp64 in [0, 1]."""
    k = dequant(comp_k, q.shape[-1]).astype(np.float64)
    dots = k @ np.asarray(q, np.float64).T            # [n, H]
    logit = np.maximum(dots, 0.0) @ np.asarray(fused_w, np.float64)
    return sigmoid(logit)


def score_layer(comp_k: np.ndarray, n_valid: np.ndarray, q: np.ndarray,
                fused_w: np.ndarray) -> np.ndarray:
    """One layer, all rows: comp_k [B, N, D+4], q [B, H, D], fused_w [B, H]
    -> [B, N] fp64; chunks past n_valid[b] score 0."""
    B, N = comp_k.shape[:2]
    out = np.zeros((B, N), np.float64)
    for b in range(B):
        n = int(n_valid[b])
        out[b, :n] = score_chunks(comp_k[b, :n], q[b], fused_w[b])
    return out


# ----------------------------------------------------------------------------
# ensemble and selection (README "Joint checkpoint + ensemble", "Usage",
# and the retrieval step of the toy decode loop)
# ----------------------------------------------------------------------------


def ensemble(scores: np.ndarray, mode: str = "max") -> np.ndarray:
    """Per-chunk union (max, the default) or mean over the layer axis 0."""
    s = np.asarray(scores, np.float64)
    if mode == "max":
        return s.max(axis=0)
    if mode == "mean":
        acc = s[0].copy()
        for l in range(1, s.shape[0]):
            acc = acc + s[l]
        return acc / s.shape[0]
    raise ValueError(mode)


def select_topk(ens: np.ndarray, n_valid: np.ndarray, k: int) -> np.ndarray:
    """bool keep [B, N]: the min(k, n_b) highest scores of each row among its
    valid chunks, equal scores ordered by lower chunk index first."""
    ens = np.asarray(ens)
    B, N = ens.shape
    keep = np.zeros((B, N), bool)
    for b in range(B):
        n = int(n_valid[b])
        idx = np.arange(n)
        order = np.lexsort((idx, -ens[b, :n].astype(np.float64)))
        keep[b, order[:min(k, n)]] = True
    return keep


def select_threshold(ens: np.ndarray, n_valid: np.ndarray, thr: float) -> np.ndarray:
    """bool keep [B, N]: valid chunks whose score is strictly above thr."""
    ens = np.asarray(ens)
    B, N = ens.shape
    valid = np.arange(N)[None, :] < np.asarray(n_valid).reshape(B, 1)
    return valid & (ens > thr)


def retrieve(layers, hidden, positions, comp_k_layers, n_valid, mode="max",
             top_k=None, threshold=None):
    """Whole path: per-layer scores [L, B, N], ensemble [B, N], keep masks."""
    per_layer = []
    qs, ws = [], []
    for layer, ck in zip(layers, comp_k_layers):
        q, w = query_prep(layer, hidden, positions)
        qs.append(q)
        ws.append(w)
        per_layer.append(score_layer(ck, n_valid, q, w))
    scores = np.stack(per_layer)
    ens = ensemble(scores, mode)
    out = dict(q=np.stack(qs, axis=1), fused_w=np.stack(ws, axis=1),
               scores=scores, ens=ens)
    if top_k is not None:
        out["keep_topk"] = select_topk(ens, n_valid, top_k)
    if threshold is not None:
        out["keep_thr"] = select_threshold(ens, n_valid, threshold)
    return out
