"""Pins of the CPU oracle against facts that do not come from the oracle itself:
the OCP E4M3 encoding table, library routines (torch's fp8 cast, scipy's
Sylvester Hadamard matrix, numpy's stable argsort), closed forms, invariants
and brute force on tiny inputs.  CPU only."""
import math
import os
import struct

import numpy as np
import pytest
import torch

import oracle.retriever as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------- e4m3


def test_e4m3_ocp_points():
    rows = []
    with open(os.path.join(GOLDEN, "e4m3_ocp_points.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                c, v = line.split()
                rows.append((int(c, 16), float(v)))
    codes = np.array([c for c, _ in rows], np.uint8)
    got = O.e4m3_decode(codes)
    for (c, v), g in zip(rows, got):
        if math.isnan(v):
            assert math.isnan(g), hex(c)
        else:
            assert g == v and math.copysign(1, g) == math.copysign(1, v), (hex(c), g, v)


def test_e4m3_exhaustive_vs_torch_cast():
    codes = np.arange(256, dtype=np.uint8)
    ours = O.e4m3_decode(codes)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).float().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    # round trip through torch's encoder for every finite code
    back = torch.from_numpy(ours[~nan].copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    fin = codes[~nan]
    # -0 and +0 both decode to zero; the encoder keeps the sign
    assert np.array_equal(back, fin)


# ------------------------------------------------------------ record parsing


def _record(codes, scale):
    return np.frombuffer(bytes(codes) + struct.pack("<f", scale), np.uint8).copy()


def test_record_scale_is_little_endian_fp32_after_the_codes():
    rng = np.random.default_rng(0)
    codes = rng.integers(0, 0x7E, 128).astype(np.uint8)
    rec = _record(codes, 0.0123)
    c, s = O.split_records(rec[None])
    assert np.array_equal(c[0], codes)
    assert s[0] == np.float32(struct.unpack("<f", struct.pack("<f", 0.0123))[0])
    k = O.dequant(rec[None])[0]
    assert np.array_equal(k, (O.e4m3_decode(codes) * np.float32(0.0123)).astype(np.float32))


def test_zero_scale_gives_zero_key():
    rec = _record(np.full(128, 0x7E, np.uint8), 0.0)
    assert np.all(O.dequant(rec[None]) == 0)


def test_dequant_known_bytes():
    codes = np.zeros(128, np.uint8)
    codes[0], codes[1], codes[127] = 0x38, 0xC0, 0x01  # 1.0, -2.0, 2^-9
    k = O.dequant(_record(codes, 4.0)[None])[0]
    assert k[0] == 4.0 and k[1] == -8.0 and k[127] == 4.0 * 2.0 ** -9
    assert np.all(k[2:127] == 0)


# ---------------------------------------------------------------- linear maps


def test_linear_orientation_with_selection_matrix():
    # W [out=3, in=5] picks inputs 4, 0, 2: a transposed W cannot pass.
    W = np.zeros((3, 5))
    W[0, 4] = W[1, 0] = W[2, 2] = 1.0
    x = np.array([[10., 11., 12., 13., 14.], [1., 2., 3., 4., 5.]])
    assert np.array_equal(O.linear(W, x), [[14., 10., 12.], [5., 1., 3.]])


def test_linear_is_linear():
    rng = np.random.default_rng(1)
    W, x, y = rng.normal(size=(7, 9)), rng.normal(size=9), rng.normal(size=9)
    np.testing.assert_allclose(O.linear(W, 2 * x - 3 * y),
                               2 * O.linear(W, x) - 3 * O.linear(W, y), atol=1e-12)


# -------------------------------------------------------------------- RMSNorm


def test_rmsnorm_constant_input_closed_form():
    c, eps = 0.003, 1e-6
    g = np.linspace(0.5, 1.5, 16)
    out = O.rms_norm(np.full(16, c), g, eps)
    np.testing.assert_allclose(out, g * c / math.sqrt(c * c + eps), rtol=1e-14)


def test_rmsnorm_unit_rms_and_gain():
    rng = np.random.default_rng(2)
    x = rng.normal(size=(3, 1024)) * 5
    out = O.rms_norm(x, np.ones(1024))
    ms = np.mean(x * x, -1)
    np.testing.assert_allclose(np.sqrt(np.mean(out * out, -1)), np.sqrt(ms / (ms + 1e-6)), rtol=1e-12)
    g = rng.normal(size=1024)
    np.testing.assert_allclose(O.rms_norm(x, g), out * g, rtol=1e-12)


# ----------------------------------------------------------------- YaRN RoPE


def test_yarn_band_edges():
    # dim(32) = 64 ln(65536/(64 pi)) / (2 ln 160000) = 15.45..,
    # dim(1)  = 64 ln(65536/(2 pi))  / (2 ln 160000) = 24.71..
    low, high = O.yarn_correction_range(64, 160000.0, 65536.0, 32.0, 1.0)
    assert (low, high) == (15, 25)


def test_yarn_frequencies_closed_form():
    f = O.yarn_inv_freq()
    assert f.shape == (32,)
    for j in range(32):
        inv = 160000.0 ** (-j / 32.0)
        if j <= 15:
            assert f[j] == pytest.approx(inv, rel=1e-15)
        elif j >= 25:
            assert f[j] == pytest.approx(inv / 16.0, rel=1e-15)
    # middle of the band: ramp = (20 - 15) / 10 = 1/2
    inv20 = 160000.0 ** (-20 / 32.0)
    assert f[20] == pytest.approx(0.5 * inv20 + 0.5 * inv20 / 16.0, rel=1e-15)
    assert f[0] == 1.0


def test_rotary_pairing_and_sign():
    # a quarter turn sends e_{64+j} to e_{96+j} and e_{96+j} to -e_{64+j}
    for j in (0, 7, 31):
        q = np.zeros((1, 1, 128))
        q[0, 0, 64 + j] = 1.0
        theta = np.zeros((1, 32))
        theta[0, j] = math.pi / 2
        out = O.apply_rotary(q, theta)[0, 0]
        expect = np.zeros(128)
        expect[96 + j] = 1.0
        np.testing.assert_allclose(out, expect, atol=1e-15)
        q2 = np.zeros((1, 1, 128))
        q2[0, 0, 96 + j] = 1.0
        out2 = O.apply_rotary(q2, theta)[0, 0]
        expect2 = np.zeros(128)
        expect2[64 + j] = -1.0
        np.testing.assert_allclose(out2, expect2, atol=1e-15)


def test_rope_angle_is_position_times_frequency():
    f = O.yarn_inv_freq()
    pos = np.array([1 << 20, 12345])
    th = O.rope_angles(pos, f)
    assert th.shape == (2, 32)
    q = np.zeros((2, 1, 128))
    q[:, 0, 64 + 3] = 1.0
    out = O.apply_rotary(q, th)
    for b in range(2):
        a = float(pos[b]) * (160000.0 ** (-3 / 32.0))
        assert out[b, 0, 64 + 3] == pytest.approx(math.cos(a), abs=1e-12)
        assert out[b, 0, 96 + 3] == pytest.approx(math.sin(a), abs=1e-12)


def test_rope_identity_norm_untouched_and_composition():
    rng = np.random.default_rng(3)
    q = rng.normal(size=(2, 64, 128))
    f = O.yarn_inv_freq()
    zero = O.apply_rotary(q, O.rope_angles(np.zeros(2), f))
    np.testing.assert_array_equal(zero, q)
    pos = np.array([16384, 1 << 20])
    r = O.apply_rotary(q, O.rope_angles(pos, f))
    np.testing.assert_array_equal(r[..., :64], q[..., :64])
    np.testing.assert_allclose(np.linalg.norm(r, axis=-1), np.linalg.norm(q, axis=-1), rtol=1e-12)
    two = O.apply_rotary(O.apply_rotary(q, O.rope_angles(np.array([100, 7]), f)),
                         O.rope_angles(np.array([23, 1000]), f))
    one = O.apply_rotary(q, O.rope_angles(np.array([123, 1007]), f))
    np.testing.assert_allclose(two, one, atol=1e-11)


# ------------------------------------------------------------------ Hadamard


def test_hadamard_matches_scipy_sylvester():
    import scipy.linalg
    np.testing.assert_array_equal(O.hadamard_matrix(128), scipy.linalg.hadamard(128))


def test_hadamard_kron_construction():
    H2 = np.array([[1., 1.], [1., -1.]])
    H = np.ones((1, 1))
    for _ in range(7):
        H = np.kron(H, H2)
    np.testing.assert_array_equal(O.hadamard_matrix(128), H)


def test_wht_orthonormal_involution():
    H = O.hadamard_matrix(128)
    np.testing.assert_array_equal(H @ H, 128 * np.eye(128))
    rng = np.random.default_rng(4)
    x = rng.normal(size=(5, 128))
    y = O.hadamard_transform(x)
    np.testing.assert_allclose(O.hadamard_transform(y), x, atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    e0 = np.zeros(128)
    e0[0] = 1
    np.testing.assert_allclose(O.hadamard_transform(e0), np.full(128, 128 ** -0.5), rtol=1e-15)
    e1 = np.zeros(128)
    e1[1] = 1
    np.testing.assert_allclose(O.hadamard_transform(e1) * math.sqrt(128),
                               np.tile([1., -1.], 64), rtol=1e-15)


# ------------------------------------------------------- query prep, composed


def _tiny_layer(rng, hid=48, rank=32, H=3, D=128):
    return dict(wq_a=rng.normal(size=(rank, hid)) * 0.1,
                q_norm=1 + rng.normal(size=rank) * 0.1,
                wq_b=rng.normal(size=(H * D, rank)) * 0.1,
                weights_proj=rng.normal(size=(H, hid)) * 0.1)


def test_query_prep_order_of_steps():
    rng = np.random.default_rng(5)
    layer = _tiny_layer(rng)
    h = rng.normal(size=(2, 48))
    pos = np.array([0, 4096])
    q, w = O.query_prep(layer, h, pos, n_heads=3, head_dim=128)
    # undo the (involutive) Hadamard: the heads before rotation
    pre = O.hadamard_transform(q)
    a = h @ layer["wq_a"].T
    r = a / np.sqrt(np.mean(a * a, -1, keepdims=True) + 1e-6) * layer["q_norm"]
    qf = (r @ layer["wq_b"].T).reshape(2, 3, 128)
    # row 0 has position 0: no rotation at all
    np.testing.assert_allclose(pre[0], qf[0], atol=1e-12)
    # row 1: rotation leaves dims 0..63 and the rotated half's norm alone
    np.testing.assert_allclose(pre[1, :, :64], qf[1, :, :64], atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(pre[1, :, 64:], axis=-1),
                               np.linalg.norm(qf[1, :, 64:], axis=-1), rtol=1e-12)
    assert not np.allclose(pre[1, :, 64:], qf[1, :, 64:])
    # the head-weight branch: constant HEAD_DIM^-1/2 * N_HEADS^-1/2
    np.testing.assert_allclose(w, (h @ layer["weights_proj"].T) / math.sqrt(128 * 3), rtol=1e-13)


def test_head_weight_scale_constant():
    layer = dict(wq_a=np.eye(4), q_norm=np.ones(4), wq_b=np.zeros((64 * 128, 4)),
                 weights_proj=np.ones((64, 4)))
    _, w = O.query_prep(layer, np.array([[1., 0., 0., 0.]]), np.array([0]))
    np.testing.assert_allclose(w, np.full((1, 64), 0.011048543456039806), rtol=1e-15)


# --------------------------------------------------------------------- score


def _records_from_keys(k):
    """Exactly representable keys: k = codes * scale with scale 1."""
    codes = torch.from_numpy(np.asarray(k, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return np.stack([_record(c, 1.0) for c in codes])


def test_score_hand_example():
    # two heads, D = 128; q_h = e_h so dot_h = k[h]
    q = np.zeros((2, 128))
    q[0, 0] = q[1, 1] = 1.0
    k = np.zeros((3, 128))
    k[0, :2] = [1.0, -2.0]    # relu -> (1, 0):  logit = 0.5
    k[1, :2] = [-1.0, 2.0]    # relu -> (0, 2):  logit = 2 * (-0.25) = -0.5
    k[2, :2] = [3.0, 4.0]     # logit = 1.5 - 1.0 = 0.5
    w = np.array([0.5, -0.25])
    s = O.score_chunks(_records_from_keys(k), q, w)
    np.testing.assert_allclose(s, [0.6224593312018546, 0.3775406687981454, 0.6224593312018546],
                               rtol=1e-15)


def test_score_scale_applies_inside_relu():
    q = np.zeros((1, 128))
    q[0, 0] = 1.0
    codes = np.zeros(128, np.uint8)
    codes[0] = 0x38  # 1.0
    rec = np.stack([_record(codes, 0.5), _record(codes, 0.0)])
    s = O.score_chunks(rec, q, np.array([2.0]))
    np.testing.assert_allclose(s, [1 / (1 + math.exp(-1.0)), 0.5], rtol=1e-15)


def test_score_negative_scale_applies_inside_relu():
    # README "compressed_k format": the scale is a plain fp32, so it may be
    # negative; the key is codes * scale and the relu acts on k . q_h.  With
    # s = -0.5 and codes (1, -2) the key is (-0.5, 1): head dots (-0.5, 1),
    # relu (0, 1), logit 3 * 1 = 3.  Scaling after the relu would give
    # s * relu((1, -2)) = (-0.5, 0) and logit -1.
    q = np.zeros((2, 128))
    q[0, 0] = q[1, 1] = 1.0
    codes = np.zeros(128, np.uint8)
    codes[0], codes[1] = 0x38, 0xC0  # 1.0, -2.0
    rec = np.stack([_record(codes, -0.5), _record(codes, 0.5)])
    s = O.score_chunks(rec, q, np.array([2.0, 3.0]))
    # s = +0.5: key (0.5, -1), relu (0.5, 0), logit 1
    np.testing.assert_allclose(s, [1 / (1 + math.exp(-3.0)), 1 / (1 + math.exp(-1.0))], rtol=1e-15)


def test_nan_codes_and_scales_give_nan_scores():
    # OCP E4M3 "fn": S.1111.111 is NaN.  A NaN element makes every head dot
    # NaN, and relu and sigmoid carry it (as the README's torch ops do), so the
    # chunk's score is NaN; a NaN scale does the same.  Other chunks are
    # untouched.
    q = np.ones((3, 128))
    w = np.array([0.5, -0.25, 1.0])
    base = np.full(128, 0x30, np.uint8)  # 0.5
    bad_pos, bad_neg = base.copy(), base.copy()
    bad_pos[17], bad_neg[100] = 0x7F, 0xFF
    rec = np.stack([_record(base, 0.01), _record(bad_pos, 0.01), _record(bad_neg, 0.01),
                    _record(base, float("nan"))])
    s = O.score_chunks(rec, q, w)
    assert np.isfinite(s[0]) and np.all(np.isnan(s[1:]))
    k = 0.5 * float(np.float32(0.01))  # the scale is stored as fp32
    np.testing.assert_allclose(s[0], 1 / (1 + math.exp(-(0.5 - 0.25 + 1.0) * 128 * k)), rtol=1e-12)


def test_ensemble_carries_nan():
    s = np.array([[0.2, 0.3], [np.nan, 0.9], [0.7, 0.1]])
    for mode in ("max", "mean"):
        e = O.ensemble(s, mode)
        assert np.isnan(e[0]) and np.isfinite(e[1])


def test_topk_and_threshold_rank_nan_below_every_number():
    nan = float("nan")
    ens = np.array([[0.2, nan, 0.1, 0.0, nan, 0.7]])
    n = np.array([6])
    assert O.select_topk(ens, n, 3)[0].tolist() == [True, False, True, False, False, True]
    assert O.select_topk(ens, n, 4)[0].tolist() == [True, False, True, True, False, True]
    # NaNs come last, in index order; K >= n keeps every valid chunk
    assert O.select_topk(ens, n, 5)[0].tolist() == [True, True, True, True, False, True]
    assert O.select_topk(ens, n, 6)[0].all()
    assert O.select_threshold(ens, n, 0.05)[0].tolist() == [True, False, True, False, False, True]
    assert not O.select_threshold(ens, n, -1.0)[0, [1, 4]].any()


def test_score_degenerate_cases_and_range():
    rng = np.random.default_rng(6)
    q = rng.normal(size=(64, 128))
    w = rng.normal(size=64)
    # zero scale -> k = 0 -> sigma(0) = 1/2 exactly
    zero = np.stack([_record(rng.integers(0, 0x7E, 128).astype(np.uint8), 0.0) for _ in range(3)])
    assert np.all(O.score_chunks(zero, q, w) == 0.5)
    # a key anti-aligned with every head -> every relu is 0
    qpos = np.abs(q)
    neg = _records_from_keys(-np.ones((1, 128)))
    assert O.score_chunks(neg, qpos, w)[0] == 0.5
    recs = np.stack([_record(rng.integers(0, 0x7E, 128).astype(np.uint8), float(s))
                     for s in rng.uniform(0, 1, 64)])
    s = O.score_chunks(recs, q * 10, w * 10)
    assert np.all((s >= 0) & (s <= 1))


def test_score_brute_force_tiny():
    rng = np.random.default_rng(7)
    H, N = 4, 8
    q = rng.normal(size=(H, 128))
    w = rng.normal(size=H)
    recs = np.stack([_record(rng.integers(0, 0x7E, 128).astype(np.uint8),
                             float(rng.uniform(0.001, 0.01))) for _ in range(N)])
    got = O.score_chunks(recs, q, w)
    for n in range(N):
        scale = struct.unpack("<f", bytes(recs[n, 128:132]))[0]
        kv = [float(torch.tensor([int(b)], dtype=torch.uint8).view(torch.float8_e4m3fn).float()) * scale
              for b in recs[n, :128]]
        logit = 0.0
        for h in range(H):
            d = sum(kv[i] * q[h, i] for i in range(128))
            logit += max(d, 0.0) * w[h]
        assert got[n] == pytest.approx(1.0 / (1.0 + math.exp(-logit)), rel=1e-6, abs=1e-7)


def test_score_layer_pads_with_zero():
    rng = np.random.default_rng(8)
    ck = np.zeros((2, 6, 132), np.uint8)
    for b in range(2):
        for n in range(6):
            ck[b, n] = _record(rng.integers(0, 0x7E, 128).astype(np.uint8), 0.01)
    s = O.score_layer(ck, np.array([6, 2]), rng.normal(size=(2, 64, 128)), rng.normal(size=(2, 64)))
    assert np.all(s[1, 2:] == 0) and np.all(s[1, :2] > 0) and np.all(s[0] > 0)


# ------------------------------------------------------------------ ensemble


def test_ensemble_values():
    s = np.array([[[0.1, 0.9]], [[0.4, 0.2]], [[0.7, 0.3]]])
    np.testing.assert_allclose(O.ensemble(s, "max"), [[0.7, 0.9]])
    np.testing.assert_allclose(O.ensemble(s, "mean"), [[0.4, 1.4 / 3]], rtol=1e-15)


def test_ensemble_max_ge_mean_and_identical_layers():
    rng = np.random.default_rng(9)
    s = rng.uniform(size=(3, 4, 50))
    assert np.all(O.ensemble(s, "max") >= O.ensemble(s, "mean") - 1e-15)
    same = np.stack([s[0]] * 3)
    np.testing.assert_allclose(O.ensemble(same, "mean"), s[0], rtol=1e-15)
    np.testing.assert_array_equal(O.ensemble(same, "max"), s[0])


# ----------------------------------------------------------------- selection


def test_topk_matches_stable_argsort():
    rng = np.random.default_rng(10)
    ens = rng.integers(0, 20, size=(3, 200)).astype(np.float32) / 20  # many ties
    nv = np.array([200, 150, 7])
    keep = O.select_topk(ens, nv, 30)
    for b in range(3):
        n = nv[b]
        order = np.argsort(-ens[b, :n].astype(np.float64), kind="stable")
        expect = np.zeros(200, bool)
        expect[order[:min(30, n)]] = True
        np.testing.assert_array_equal(keep[b], expect)
        assert keep[b].sum() == min(30, n)


def test_topk_brute_force_and_ties():
    ens = np.array([[0.5, 0.7, 0.7, 0.2, 0.7, 0.9]])
    keep = O.select_topk(ens, np.array([6]), 3)
    # 0.9 first, then the two lowest-index 0.7s
    np.testing.assert_array_equal(keep[0], [False, True, True, False, False, True])
    keep = O.select_topk(ens, np.array([6]), 10)
    assert keep.all()
    keep = O.select_topk(ens, np.array([3]), 10)
    np.testing.assert_array_equal(keep[0], [True, True, True, False, False, False])
    dup = np.full((1, 40), 0.25)
    np.testing.assert_array_equal(O.select_topk(dup, np.array([40]), 9)[0], np.arange(40) < 9)


def test_topk_keeps_everything_above_kth():
    rng = np.random.default_rng(11)
    ens = rng.uniform(size=(2, 1000))
    keep = O.select_topk(ens, np.array([1000, 1000]), 100)
    for b in range(2):
        kth = np.sort(ens[b])[::-1][99]
        assert np.all(keep[b][ens[b] > kth]) and not np.any(keep[b][ens[b] < kth])


def test_threshold_is_strict_and_respects_length():
    ens = np.array([[0.5, 0.50000006, 0.4, 0.9, 0.9]], np.float32)
    keep = O.select_threshold(ens, np.array([4]), 0.5)
    np.testing.assert_array_equal(keep[0], [False, True, False, True, False])


# ------------------------------------------------------------------ recall
import oracle.recall as OR  # noqa: E402


def test_compact_hand_example():
    keep = np.array([[0, 1, 1, 0, 1, 0], [0, 0, 0, 0, 0, 0], [1, 1, 1, 1, 1, 1]], np.uint8)
    idx, count = OR.compact_mask(keep, 4)
    assert idx.tolist() == [[1, 2, 4, -1], [-1, -1, -1, -1], [0, 1, 2, 3]]
    assert count.tolist() == [3, 0, 6]  # row 2 keeps more than it can list


def test_compact_matches_flatnonzero_and_invariants():
    rng = np.random.default_rng(3)
    keep = rng.random((5, 300)) < np.array([0.0, 0.02, 0.5, 0.97, 1.0])[:, None]
    idx, count = OR.compact_mask(keep, 64)
    for b in range(5):
        nz = np.flatnonzero(keep[b])  # library routine
        assert count[b] == keep[b].sum() == len(nz)
        m = min(len(nz), 64)
        assert np.array_equal(idx[b, :m], nz[:m])
        assert (idx[b, m:] == -1).all()
        assert (np.diff(idx[b, :m]) > 0).all() and keep[b, idx[b, :m]].all()


def test_gather_hand_example_and_untouched_slots():
    src = np.arange(2 * 5 * 3, dtype=np.uint8).reshape(2, 5, 3)
    idx = np.array([[4, 0, -1], [2, 9, 1]], np.int32)  # 9 is out of range: skipped
    count = np.array([2, 3], np.int32)
    dst = np.full((2, 3, 3), 255, np.uint8)
    out = OR.gather_records(src, idx, count, dst)
    assert out[0, 0].tolist() == [12, 13, 14] and out[0, 1].tolist() == [0, 1, 2]
    assert (out[0, 2] == 255).all()  # past count
    assert out[1, 0].tolist() == [21, 22, 23] and (out[1, 1] == 255).all()
    assert out[1, 2].tolist() == [18, 19, 20]
    assert (dst == 255).all()  # the input is not modified


def test_gather_matches_fancy_indexing():
    rng = np.random.default_rng(4)
    src = rng.integers(0, 256, (3, 50, 132), dtype=np.uint8)
    keep = rng.random((3, 50)) < 0.3
    idx, count = OR.compact_mask(keep, 20)
    out = OR.gather_records(src, idx, count, np.zeros((3, 20, 132), np.uint8))
    for b in range(3):
        m = min(int(count[b]), 20)
        assert np.array_equal(out[b, :m], src[b][np.flatnonzero(keep[b])[:m]])  # library routine
        assert not out[b, m:].any()


# -------------------------------------------------------------- toy decode
import oracle.decode as OD  # noqa: E402


def _vecs(seed, B, N, D=128):
    return np.random.default_rng(seed).standard_normal((B, N, D))


def test_attention_single_kept_chunk_returns_it():
    x = _vecs(1, 2, 7)
    q = np.random.default_rng(2).standard_normal((2, 32, 128))
    keep = np.zeros((2, 7), bool)
    keep[0, 3] = True
    keep[1, 6] = True
    o = OD.masked_attention(q, x, keep)
    np.testing.assert_allclose(o[0], np.broadcast_to(x[0, 3], (32, 128)), rtol=1e-14)
    np.testing.assert_allclose(o[1], np.broadcast_to(x[1, 6], (32, 128)), rtol=1e-14)


def test_attention_two_chunks_closed_form():
    # q = 2 e_0 and x_1 = 3 e_0, x_2 = -e_0 + e_5: logits 6/sqrt(128) and -2/sqrt(128)
    q = np.zeros((1, 32, 128))
    q[0, :, 0] = 2.0
    x = np.zeros((1, 3, 128))
    x[0, 1, 0] = 3.0
    x[0, 2, 0] = -1.0
    x[0, 2, 5] = 1.0
    x[0, 0, :] = 1e6  # a masked chunk: must not matter
    keep = np.array([[False, True, True]])
    p1 = 1.0 / (1.0 + math.exp(-(6.0 + 2.0) / math.sqrt(128)))
    want = p1 * x[0, 1] + (1 - p1) * x[0, 2]
    o = OD.masked_attention(q, x, keep)
    np.testing.assert_allclose(o[0, 7], want, rtol=1e-13, atol=1e-15)


def test_attention_masked_chunks_do_not_matter_and_empty_row_is_zero():
    rng = np.random.default_rng(5)
    x = _vecs(6, 2, 40)
    q = rng.standard_normal((2, 32, 128))
    keep = rng.random((2, 40)) < 0.4
    keep[1] = False
    o = OD.masked_attention(q, x, keep)
    x2 = x.copy()
    x2[~keep] = rng.standard_normal(((~keep).sum(), 128)) * 1e3
    np.testing.assert_allclose(OD.masked_attention(q, x2, keep), o, rtol=1e-12, atol=1e-12)
    assert (o[1] == 0).all()
    # softmax weights of the kept chunks: the output is a convex combination
    sub = x[0, keep[0]]
    assert (o[0] <= sub.max(axis=0) + 1e-12).all() and (o[0] >= sub.min(axis=0) - 1e-12).all()


def test_attention_heads_are_independent_and_equal_vectors_give_the_vector():
    x = np.tile(_vecs(7, 1, 1), (1, 9, 1))
    q = np.random.default_rng(8).standard_normal((1, 32, 128))
    o = OD.masked_attention(q, x, np.ones((1, 9), bool))
    np.testing.assert_allclose(o[0], np.broadcast_to(x[0, 0], (32, 128)), rtol=1e-13)
    # a query aligned with chunk j for head 5 only: head 5 weights chunk j most
    x = _vecs(9, 1, 6) / 10
    q = np.zeros((1, 32, 128))
    q[0, 5] = 40.0 * x[0, 2] / np.linalg.norm(x[0, 2])
    o = OD.masked_attention(q, x, np.ones((1, 6), bool))
    assert np.argmin(np.linalg.norm(x[0] - o[0, 5], axis=1)) == 2
    np.testing.assert_allclose(o[0, 4], x[0].mean(axis=0), rtol=1e-12)  # head 4: zero query, uniform weights


def test_toy_step_is_rmsnorm_of_residual():
    rng = np.random.default_rng(10)
    h = rng.standard_normal((2, 4096))
    x = _vecs(11, 2, 30)
    keep = rng.random((2, 30)) < 0.5
    out = OD.toy_step(h, x, keep)
    o = OD.masked_attention(h.reshape(2, 32, 128), x, keep).reshape(2, 4096)
    v = h + o
    np.testing.assert_allclose(np.sqrt(np.mean(out * out, axis=1)), np.sqrt(np.mean(v * v, axis=1) /
                               (np.mean(v * v, axis=1) + 1e-6)), rtol=1e-12)
    cos = (out * v).sum(1) / np.linalg.norm(out, axis=1) / np.linalg.norm(v, axis=1)
    np.testing.assert_allclose(cos, 1.0, rtol=1e-12)
    # head h of the query is hidden[h*128:(h+1)*128]: one kept chunk makes o = x for every head
    keep1 = np.zeros((2, 30), bool)
    keep1[:, 4] = True
    out1 = OD.toy_step(h, x, keep1)
    want = h + np.tile(x[:, 4], (1, 32))
    np.testing.assert_allclose(out1, want / np.sqrt(np.mean(want * want, 1, keepdims=True) + 1e-6), rtol=1e-12)
