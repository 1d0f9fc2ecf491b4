"""Pins of the local (MSVS-style) decoder oracle: the neighbour rule (order,
float32 distances, ties), AVS-Conv closed forms, translation invariance, and a
hand-worked multi-scale fusion."""
import numpy as np
import pytest

from oracle import decoder as D
from oracle import local as L


def test_knn_order_and_ties_by_hand():
    # anchors on the x axis at -1, 1, 0.5, -0.5, 2 (indices 0..4): from x = 0 the nearest are
    # 2 and 3 (distance 0.5, tie -> index 2 first), then 0 and 1 (tie -> 0 first), then 4
    a = np.array([[-1, 0, 0], [1, 0, 0], [0.5, 0, 0], [-0.5, 0, 0], [2, 0, 0]], np.float32)
    assert L.knn(np.zeros((1, 3)), a, 5)[0].tolist() == [2, 3, 0, 1, 4]
    assert L.knn(np.array([[1.9, 0, 0]]), a, 2)[0].tolist() == [4, 1]


def test_knn_distances_are_float32_in_a_fixed_order():
    # A = (a, 0, 0) and B = (0, b, c): in float64 B is nearer to the origin by 2.5e-9, in
    # float32 (x, y, then z) both squared distances are the same number, so the tie rule puts
    # the smaller index first
    a, b, c = 0.31638941168785095, 0.3066110610961914, 0.07805071771144867
    x = np.zeros((1, 3), np.float32)
    A, B = [a, 0, 0], [0, b, c]
    assert a * a - (b * b + c * c) > 2e-9                       # float64: B nearer
    assert L.knn(x, np.array([A, B], np.float32), 2)[0].tolist() == [0, 1]
    assert L.knn(x, np.array([B, A], np.float32), 2)[0].tolist() == [0, 1]


def _scale(C, rng, hidden=4):
    return {"W1": rng.standard_normal((hidden, 3)), "b1": rng.standard_normal(hidden),
            "W2": rng.standard_normal((C, hidden)), "b2": rng.standard_normal(C)}


def test_avs_conv_closed_forms():
    rng = np.random.default_rng(0)
    a = rng.uniform(-1, 1, (40, 3)).astype(np.float32)
    F = rng.standard_normal((40, 6))
    x = rng.uniform(-1, 1, (5, 3))
    K = 4
    nb = L.knn(x, a, K)
    w = _scale(6, rng)
    w["W2"][:] = 0.0
    w["b2"][:] = 0.0                    # no dynamic weight: the mean-pooling residual alone
    np.testing.assert_allclose(L.avs_conv(x, a, F, w, K), F[nb].mean(axis=1), atol=1e-14)
    w["b2"][:] = 2.5                    # constant weight c: (1 + c) times the mean
    np.testing.assert_allclose(L.avs_conv(x, a, F, w, K), 3.5 * F[nb].mean(axis=1), atol=1e-13)


def test_avs_conv_is_translation_invariant():
    # dyadic coordinates keep every float32 difference exact under a dyadic shift
    rng = np.random.default_rng(1)
    a = (rng.integers(-60, 60, (50, 3)) / 64.0).astype(np.float32)
    x = (rng.integers(-60, 60, (6, 3)) / 64.0 + 1 / 128).astype(np.float32)
    F = rng.standard_normal((50, 5))
    w = _scale(5, rng)
    s = np.array([0.25, -0.5, 0.125], np.float32)
    np.testing.assert_allclose(L.avs_conv(x + s, a + s, F, w, 3), L.avs_conv(x, a, F, w, 3), atol=1e-12)


def test_multi_scale_fusion_by_hand():
    # two scales, K = 1, no dynamic weight (f = F of the nearest anchor), Wf = I, wo = e_1:
    # sdf = GELU(F0[nearest] concatenated with F1[nearest])[1] + b_o
    a0 = np.array([[0.5, 0, 0], [-0.5, 0, 0]], np.float32)
    a1 = np.array([[0, 0.3, 0], [0, -0.9, 0], [0, 0.2, 0]], np.float32)
    F0 = np.array([[1.0, -2.0], [3.0, 4.0]])
    F1 = np.array([[0.5], [0.25], [-1.5]])
    rng = np.random.default_rng(2)
    ws = []
    for C in (2, 1):
        w = _scale(C, rng)
        w["W2"][:] = 0.0
        w["b2"][:] = 0.0
        ws.append(w)
    fuse = {"Wf": np.eye(3), "bf": np.zeros(3), "wo": np.array([0.0, 1.0, 0.0]), "bo": np.array([0.125])}
    x = np.array([[0.4, 0.1, 0.0], [-0.4, 0.19, 0.0]])
    got = L.decode_local(x, [a0, a1], [F0, F1], ws, fuse, K=1)
    want = D.gelu(np.array([-2.0, 4.0])) + 0.125      # nearest scale-0 anchors: 0 then 1
    np.testing.assert_allclose(got, want, atol=1e-14)
    fuse["wo"] = np.array([0.0, 0.0, 1.0])            # nearest scale-1 anchors: 2 (y 0.2) twice
    np.testing.assert_allclose(L.decode_local(x, [a0, a1], [F0, F1], ws, fuse, K=1),
                               D.gelu(np.array([-1.5, -1.5])) + 0.125, atol=1e-14)
