"""Pins of the decoder oracle against closed forms, textbook values,
independent library routines and invariants (no GPU).

Each case is built so that a plausible slip in ``oracle/decoder.py`` -- a
swapped sin/cos lane, a missing attention scale, a transposed weight, a
dropped residual or LayerNorm, a wrong head split -- changes the result.
"""
import math
import os

import numpy as np
import pytest
from scipy.stats import norm

from oracle import decoder as D

GOLD = os.path.join(os.path.dirname(__file__), "golden")
S8, C8, R2 = math.sin(math.pi / 8), math.cos(math.pi / 8), math.sqrt(2) / 2


def _zero_weights(C, F, H=None):
    z = lambda *s: np.zeros(s, np.float64)
    return dict(Wq=z(C, 64), bq=z(C), Wk=z(C, C), bk=z(C), Wv=z(C, C), bv=z(C),
                Wo=z(C, C), bo=z(C), W1=z(F, C), b1=z(F), W2=z(C, F), b2=z(C),
                ln_kv_g=np.ones(C), ln_kv_b=z(C), ln1_g=np.ones(C), ln1_b=z(C),
                ln2_g=np.ones(C), ln2_b=z(C), w_head=z(C), b_head=z(1))


def test_fourier_embedding_matches_hand_worked_values():
    want = np.zeros(64)
    sym = {"r2": R2, "s8": S8, "c8": C8}
    for line in open(os.path.join(GOLD, "fourier_pe_closed_form.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        lane, val = line.split()
        neg = val.startswith("-")
        v = sym.get(val.lstrip("-"))
        v = float(val.lstrip("-")) if v is None else v
        want[int(lane)] = -v if neg else v
    got = D.fourier_embed(np.array([[0.25, 0.5, -0.125]]))[0]
    np.testing.assert_allclose(got, want, atol=1e-12)
    assert np.all(got[51:] == 0)


def test_grid_points_cell_centred_and_nested():
    R = 4
    p = D.grid_points(R)
    assert p.shape == (64, 3)
    np.testing.assert_allclose(p[0], [-0.75, -0.75, -0.75])
    np.testing.assert_allclose(p[1], [-0.75, -0.75, -0.25])     # z fastest
    np.testing.assert_allclose(p[R * R], [-0.25, -0.75, -0.75])  # x slowest
    # the 8 children of a voxel at 2R average to the parent centre
    kids = D.grid_points(2 * R, np.array([((2 * 1 + a) * 8 + (2 * 2 + b)) * 8 + (2 * 3 + c)
                                          for a in (0, 1) for b in (0, 1) for c in (0, 1)]))
    np.testing.assert_allclose(kids.mean(axis=0), D.grid_points(R, np.array([(1 * 4 + 2) * 4 + 3]))[0])


def test_layer_norm_closed_form():
    x = np.array([[1.0, 2.0, 3.0, 4.0]])
    want = (x - 2.5) / math.sqrt(1.25 + 1e-5)
    np.testing.assert_allclose(D.layer_norm(x, np.ones(4), np.zeros(4)), want, rtol=1e-14)
    g, b = np.array([2.0, 1.0, 0.5, -1.0]), np.array([0.1, 0.0, -0.2, 0.3])
    np.testing.assert_allclose(D.layer_norm(x, g, b), want * g + b, rtol=1e-14)


def test_gelu_textbook_values_and_normal_cdf():
    # GELU(x) = x * Phi(x); Phi(1) = 0.841344746068543 (standard normal table)
    np.testing.assert_allclose(D.gelu(np.array([0.0, 1.0, -1.0])),
                               [0.0, 0.8413447460685429, -0.15865525393145707], atol=1e-15)
    x = np.linspace(-6, 6, 97)
    np.testing.assert_allclose(D.gelu(x), x * norm.cdf(x), rtol=1e-12, atol=1e-15)


def test_attention_two_tokens_closed_form():
    # one head; s = q.k / 8 ; p0 = sigmoid(s0 - s1)
    t = 3.0
    q = np.zeros((1, 64)); q[0, 0] = t
    K = np.zeros((1, 2, 64)); K[0, 0, 0] = 1.0; K[0, 1, 0] = -1.0
    V = np.zeros((1, 2, 64)); V[0, 0, 5] = 1.0; V[0, 1, 7] = 1.0
    p0 = 1.0 / (1.0 + math.exp(-2 * t / 8))
    a = D.attention(q, K, V)[0]
    assert a[5] == pytest.approx(p0, abs=1e-14)
    assert a[7] == pytest.approx(1 - p0, abs=1e-14)


def test_attention_heads_use_their_own_slices():
    # head 0 prefers token 0, head 1 prefers token 1 (same logit magnitude)
    q = np.zeros((1, 128)); q[0, 0] = 8.0; q[0, 64] = 8.0
    K = np.zeros((2, 2, 64))
    K[0, 0, 0] = 1.0; K[0, 1, 0] = 0.0
    K[1, 0, 0] = 0.0; K[1, 1, 0] = 1.0
    V = np.zeros((2, 2, 64))
    V[0, 0, 1] = 1.0; V[0, 1, 2] = 1.0
    V[1, 0, 3] = 1.0; V[1, 1, 4] = 1.0
    hi = math.e / (math.e + 1.0)
    a = D.attention(q, K, V)[0]
    np.testing.assert_allclose(a[[1, 2]], [hi, 1 - hi], atol=1e-14)
    np.testing.assert_allclose(a[[64 + 3, 64 + 4]], [1 - hi, hi], atol=1e-14)


def test_attention_closed_forms_identical_rows_and_single_token():
    rng = np.random.default_rng(1)
    q = rng.standard_normal((5, 128))
    K = rng.standard_normal((2, 7, 64))
    v = rng.standard_normal((2, 1, 64))
    V = np.repeat(v, 7, axis=1)
    # identical V rows -> output is that row whatever the weights
    a = D.attention(q, K, V)
    np.testing.assert_allclose(a, np.tile(v.reshape(1, 128), (5, 1)), atol=1e-13)
    # identical K rows -> uniform weights -> mean of V
    Kc = np.repeat(rng.standard_normal((2, 1, 64)), 7, axis=1)
    V2 = rng.standard_normal((2, 7, 64))
    a2 = D.attention(q, Kc, V2)
    np.testing.assert_allclose(a2, np.tile(V2.mean(axis=1).reshape(1, 128), (5, 1)), atol=1e-13)
    # a single token
    a3 = D.attention(q, K[:, :1], V2[:, :1])
    np.testing.assert_allclose(a3, np.tile(V2[:, 0].reshape(1, 128), (5, 1)), atol=1e-14)


def test_attention_subset_ignores_unselected_tokens():
    q = np.zeros((1, 64)); q[0, 0] = 2.0
    K = np.zeros((1, 4, 64)); K[0, 1, 0] = 1.0; K[0, 3, 0] = -1.0
    V = np.full((1, 4, 64), 1e6)
    V[0, 1] = 0.0; V[0, 3] = 0.0; V[0, 1, 9] = 1.0; V[0, 3, 9] = -1.0
    a = D.attention(q, K, V, sel=np.array([1, 3]))[0]
    # tanh form of p0 - p1 with logits +-2/8
    assert a[9] == pytest.approx(math.tanh(2.0 / 8.0), abs=1e-14)
    assert np.abs(a).max() < 2


def test_decoder_head_after_layernorm_closed_form():
    # C=64: q = PE (identity on the 51 lanes), no attention/MLP contribution,
    # dec = w_head . LN2(q).  At the origin PE = 24 ones (cos 0) and zeros.
    C = 64
    w = _zero_weights(C, 64)
    w["Wq"][:51, :51] = np.eye(51)
    mean, var = 24 / 64, 24 / 64 * (1 - 24 / 64)
    K = np.zeros((1, 3, 64)); V = np.zeros((1, 3, 64))
    p = np.zeros((1, 3))
    for lane, val in ((0, 0.0), (27, 1.0)):
        w["w_head"][:] = 0; w["w_head"][lane] = 1.0
        got = D.decode_points(p, K, V, w, query_ln=True)[0]
        assert got == pytest.approx((val - mean) / math.sqrt(var + 1e-5), abs=1e-13)
    # without query-side LayerNorm the head reads q directly: dec = x
    w["w_head"][:] = 0; w["w_head"][0] = 1.0; w["b_head"][0] = 0.25
    pts = np.array([[0.3, -0.2, 0.9], [-0.7, 0.1, 0.0]])
    np.testing.assert_allclose(D.decode_points(pts, K, V, w, query_ln=False), pts[:, 0] + 0.25, atol=1e-14)


def test_decoder_mlp_residual_closed_form():
    # x2 = q + W2 GELU(W1 q + b1) + b2 with W1 = W2 = I: dec_c = q_c + GELU(q_c + b1_c) + b2_c
    C = 64
    w = _zero_weights(C, 64)
    w["Wq"][:51, :51] = np.eye(51)
    w["W1"][:] = np.eye(64); w["W2"][:] = np.eye(64)
    w["b1"][0] = 0.1; w["b2"][0] = -0.05
    w["w_head"][0] = 1.0
    K = np.zeros((1, 2, 64)); V = np.zeros((1, 2, 64))
    x = np.array([-0.8, -0.1, 0.3, 0.95])
    pts = np.stack([x, np.zeros(4), np.zeros(4)], axis=1)
    want = x + (x + 0.1) * norm.cdf(x + 0.1) - 0.05
    np.testing.assert_allclose(D.decode_points(pts, K, V, w, query_ln=False), want, atol=1e-13)


def test_decoder_kv_path_and_output_projection_closed_form():
    # Two tokens z0 = (+1,-1,...), z1 = -z0 -> LN_kv(z) = +-z0/s, s = sqrt(1+1e-5).
    # Wk = Wv = I, q = bq = t z0 (Wq = 0) -> logits +-8t/s, so a = tanh(8t/s) z0/s.
    # Wo = permutation P (x1 = q + P a): lane 0 reads a[1] = -tanh(8t/s)/s.
    C = 64
    z0 = np.array([1.0 if i % 2 == 0 else -1.0 for i in range(C)])
    z = np.stack([z0, -z0])
    s = math.sqrt(1.0 + 1e-5)
    for t in (0.05, 0.3):
        w = _zero_weights(C, 64)
        w["Wk"][:] = np.eye(C); w["Wv"][:] = np.eye(C)
        w["bq"][:] = t * z0
        P = np.roll(np.eye(C), 1, axis=1)    # (P a)_c = a_{c+1}
        w["Wo"][:] = P
        w["w_head"][0] = 1.0
        K, V = D.precompute_kv(z, w)
        got = D.decode_points(np.zeros((1, 3)), K, V, w, query_ln=False)[0]
        want = t * z0[0] + math.tanh(8 * t / s) * z0[1] / s
        assert got == pytest.approx(want, abs=1e-13)


def test_value_bias_makes_output_query_independent():
    # Wv = 0 -> every V row equals bv -> a = bv for every query and subset
    rng = np.random.default_rng(3)
    C = 128
    w = _zero_weights(C, 32)
    w["Wq"] = rng.standard_normal((C, 64)) * 0.3
    w["Wk"] = rng.standard_normal((C, C)) * 0.3
    w["bv"] = rng.standard_normal(C)
    w["Wo"] = np.eye(C)
    z = rng.standard_normal((9, C))
    K, V = D.precompute_kv(z, w)
    pts = rng.uniform(-1, 1, (6, 3))
    pe = D.fourier_embed(pts)
    q = pe @ w["Wq"].T
    w["w_head"][3] = 1.0
    want = q[:, 3] + w["bv"][3]
    np.testing.assert_allclose(D.decode_points(pts, K, V, w, query_ln=False), want, atol=1e-12)
    np.testing.assert_allclose(D.decode_points(pts, K, V, w, query_ln=False, sel=np.array([2, 5])),
                               want, atol=1e-12)


def test_token_permutation_invariance():
    import workloads as W
    spec = W.DecoderSpec(C=128, H=2, F=256, N=40, query_ln=True, dtype="f32")
    d = W.make_decoder(spec, seed=7, key=99, stress=True)
    z, w = d["z"][0], d["weights"]
    pts = W.make_points(16, seed=7, key=99)[0]
    K, V = D.precompute_kv(z, w)
    perm = np.random.default_rng(0).permutation(spec.N)
    K2, V2 = D.precompute_kv(z[perm], w)
    np.testing.assert_allclose(D.decode_points(pts, K, V, w), D.decode_points(pts, K2, V2, w),
                               atol=1e-12)


def test_sphere_sdf_closed_forms():
    sp = np.array([[0.0, 0.0, 0.0, 0.5], [0.6, 0.0, 0.0, 0.1]])
    p = np.array([[0.0, 0.0, 0.0], [0.0, 0.9, 0.0], [0.6, 0.0, 0.0], [0.3, 0.0, 0.0]])
    want = [-0.5, 0.4, -0.1, -0.2]
    np.testing.assert_allclose(D.sphere_sdf(p, sp), want, atol=1e-15)
    dec = np.array([0.0, 100.0, -100.0, 0.5])
    np.testing.assert_allclose(D.field(p, dec, sp, 0.01), np.array(want) + 0.01 * np.tanh(dec),
                               atol=1e-15)
    assert np.all(D.field(p, dec, None, 0.01) == dec)


def test_decoder_query_layernorm_before_mlp_closed_form():
    # query_ln = True, attention silent (V = 0, Wo = 0): x1 = q = PE(p) on lanes 0..50.
    # W1 = W2 = I: x2 = x1 + GELU(LN1(x1)), dec = LN2(x2)[0].  At p = (0.5, 0, 0) the
    # embedding is worked out by hand: lane 0 = 0.5, sin(pi/2) = 1 at lane 3, sin(2^k pi/2)
    # = 0 for k >= 1, cos(pi/2) = 0 at lane 27, cos(pi) = -1 at lane 28, cos(2^k pi/2) = 1
    # at lanes 29..34 (k >= 2), and y = z = 0 give sin = 0, cos = 1 at lanes 35..50.
    C = 64
    w = _zero_weights(C, 64)
    w["Wq"][:51, :51] = np.eye(51)
    w["W1"][:] = np.eye(64); w["W2"][:] = np.eye(64)
    w["w_head"][0] = 1.0
    x1 = np.zeros(64)
    x1[0] = 0.5
    x1[3] = 1.0
    x1[28] = -1.0
    x1[29:35] = 1.0
    x1[35:51] = 1.0
    np.testing.assert_allclose(D.fourier_embed(np.array([[0.5, 0.0, 0.0]]))[0], x1, atol=1e-14)

    def ln(v):   # biased variance, eps 1e-5, unit gain, zero shift
        m = v.mean()
        return (v - m) / math.sqrt(((v - m) ** 2).mean() + 1e-5)

    def gelu(v):
        return v * norm.cdf(v)

    want = ln(x1 + gelu(ln(x1)))[0]
    K = np.zeros((1, 2, 64)); V = np.zeros((1, 2, 64))
    got = D.decode_points(np.array([[0.5, 0.0, 0.0]]), K, V, w, query_ln=True)[0]
    assert got == pytest.approx(want, abs=1e-12)
    # the case separates the plausible slips: LN1 dropped, or the residual taken after LN1
    # (x2 = LN1(x1) + MLP, post-norm style)
    for slip in (ln(x1 + gelu(x1)), ln(ln(x1) + gelu(ln(x1)))):
        assert abs(slip[0] - want) > 1e-2


def test_tsdf_head_reads_the_same_final_features():
    # the tSDF head is a second linear head on LN2(x2): at the origin (C = 64, q = PE on
    # 51 lanes, 24 ones at the cos lanes) a unit weight on lane 27 reads (1 - 3/8) / sigma
    C = 64
    w = _zero_weights(C, 64)
    w["Wq"][:51, :51] = np.eye(51)
    w["w_head"][0] = 1.0
    w["w_tsdf"] = np.zeros(C); w["w_tsdf"][27] = 1.0
    w["b_tsdf"] = np.array([0.125])
    K = np.zeros((1, 3, 64)); V = np.zeros((1, 3, 64))
    mean, var = 24 / 64, 24 / 64 * (1 - 24 / 64)
    dec, t = D.decode_points(np.zeros((1, 3)), K, V, w, query_ln=True, return_tsdf=True)
    assert dec[0] == pytest.approx((0 - mean) / math.sqrt(var + 1e-5), abs=1e-13)
    assert t[0] == pytest.approx((1 - mean) / math.sqrt(var + 1e-5) + 0.125, abs=1e-13)


def test_tsdf_field_truncates_the_distance():
    sp = np.array([[0.0, 0.0, 0.0, 0.5]])
    p = np.array([[0.0, 0.0, 0.52], [0.0, 0.45, 0.0], [0.9, 0.0, 0.0], [0.0, 0.0, 0.0]])
    got = D.tsdf_field(p, np.zeros(4), sp, 0.01, trunc=0.1)
    np.testing.assert_allclose(got, [0.2, -0.5, 1.0, -1.0], atol=1e-14)
    t = np.array([0.0, 0.0, 0.0, 0.0]) + 3.0
    np.testing.assert_allclose(D.tsdf_field(p, t, sp, 0.01, trunc=0.1),
                               np.clip((np.array([0.02, -0.05, 0.4, -0.5]) + 0.01 * np.tanh(3.0)) / 0.1, -1, 1),
                               atol=1e-14)
    assert np.array_equal(D.tsdf_field(p, t, None, 0.01, 0.1), t)
