"""Pins of the vecset-encoder oracle: invariance to the order of the cloud's
points, equivariance in the latent tokens, and closed forms of the block."""
import math

import numpy as np
import pytest

from oracle import decoder as D
from oracle import encoder as E


def _block(C, F, rng, scale=0.3):
    w = {k: rng.standard_normal(s) * scale for k, s in
         (("Wq", (C, 64)), ("Wk", (C, C)), ("Wv", (C, C)), ("Wo", (C, C)), ("W1", (F, C)), ("W2", (C, F)))}
    for k, n in (("bq", C), ("bk", C), ("bv", C), ("bo", C), ("b1", F), ("b2", C), ("ln_kv_b", C),
                 ("ln1_b", C), ("ln2_b", C)):
        w[k] = rng.standard_normal(n) * 0.1
    for k in ("ln_kv_g", "ln1_g", "ln2_g"):
        w[k] = 1.0 + rng.standard_normal(C) * 0.1
    w["w_head"] = np.zeros(C)
    w["b_head"] = np.zeros(1)
    return w


def test_vecset_is_invariant_to_the_order_of_the_points():
    rng = np.random.default_rng(0)
    C, F = 128, 256
    w = _block(C, F, rng)
    w_in, b_in = rng.standard_normal((C, 64)) * 0.3, rng.standard_normal(C) * 0.1
    pts = rng.uniform(-1, 1, (50, 3))
    q = pts[:7]
    z = E.encode(pts, q, w_in, b_in, w)
    perm = rng.permutation(50)
    np.testing.assert_allclose(E.encode(pts[perm], q, w_in, b_in, w), z, atol=1e-12)
    qp = rng.permutation(7)   # tokens follow their query points
    np.testing.assert_allclose(E.encode(pts, q[qp], w_in, b_in, w), z[qp], atol=1e-12)


def test_identical_points_give_the_value_row():
    # every point at the same place: identical keys and values, so the attention output is
    # that value row whatever the query; x1 = q + Wo v + bo and x2 follows by hand
    rng = np.random.default_rng(1)
    C, F = 64, 64
    w = _block(C, F, rng)
    w_in, b_in = rng.standard_normal((C, 64)) * 0.3, rng.standard_normal(C) * 0.1
    p0 = np.array([[0.2, -0.4, 0.7]])
    pts = np.repeat(p0, 9, axis=0)
    q = rng.uniform(-1, 1, (3, 3))
    z = E.encode(pts, q, w_in, b_in, w)
    u = D.fourier_embed(p0) @ w_in.T + b_in
    mu, var = u.mean(), u.var()
    v = ((u - mu) / math.sqrt(var + 1e-5) * w["ln_kv_g"] + w["ln_kv_b"]) @ w["Wv"].T + w["bv"]
    qq = D.fourier_embed(q) @ w["Wq"].T + w["bq"]
    x1 = qq + v @ w["Wo"].T + w["bo"]
    m1 = x1.mean(axis=1, keepdims=True)
    h = (x1 - m1) / np.sqrt(x1.var(axis=1, keepdims=True) + 1e-5) * w["ln1_g"] + w["ln1_b"]
    g = h @ w["W1"].T + w["b1"]
    from scipy.stats import norm
    x2 = x1 + (g * norm.cdf(g)) @ w["W2"].T + w["b2"]
    np.testing.assert_allclose(z, x2, atol=1e-12)


def test_point_features_orientation_by_a_permutation():
    # W_in moves embedding lane i to output lane (i + 5) mod 64: u[(i + 5) % 64] = pe[i].  At
    # p = (0.25, 0.5, -0.125): lane 0 holds x = 0.25 (-> u[5]), lane 3 sin(pi/4) (-> u[8]),
    # lane 27 cos(pi/4) (-> u[32]), lane 4 sin(pi/2) = 1 (-> u[9]); b_in adds 1 to u[5]
    w_in = np.roll(np.eye(64), 5, axis=0)
    b_in = np.zeros(64); b_in[5] = 1.0
    u = E.point_features(np.array([[0.25, 0.5, -0.125]]), w_in, b_in)[0]
    r2 = math.sqrt(2) / 2
    assert u[5] == pytest.approx(1.25, abs=1e-14)
    assert u[8] == pytest.approx(r2, abs=1e-14) and u[32] == pytest.approx(r2, abs=1e-14)
    assert u[9] == pytest.approx(1.0, abs=1e-14)
