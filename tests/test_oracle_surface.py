"""Pins of the surface-extraction oracle (marching cubes traced from corner
signs): every one of the 256 sign patterns, closed forms (a plane, a sphere)
and invariants that any correct extraction has (a closed surface is
watertight, consistently oriented and of Euler characteristic 2)."""
import math
from collections import Counter

import numpy as np
import pytest

from oracle import decoder as OD
from oracle import surface as S


def _crossed_edges(config):
    inside = [(config >> c) & 1 for c in range(8)]
    out = set()
    for e in range(12):
        c0, c1 = S._edge_corners(e)
        if inside[c0] != inside[c1]:
            out.add(e)
    return out


def test_every_sign_pattern_gives_loops_over_its_crossed_edges():
    most = 0
    for config in range(256):
        loops = S.cube_loops(config)
        edges = [e for l in loops for e in l]
        assert sorted(edges) == sorted(_crossed_edges(config)), config
        assert all(len(l) >= 3 for l in loops)
        tris = S.cube_triangles(config)
        assert len(tris) == sum(len(l) - 2 for l in loops)
        most = max(most, len(tris))
    assert S.cube_loops(0) == [] and S.cube_loops(255) == []
    # one inside corner: a triangle around it; its normal points away from the corner
    (t,) = S.cube_triangles(1)
    p = [S._edge_mid(e) for e in t]
    n = np.cross(p[1] - p[0], p[2] - p[0])
    assert np.dot(n, p[0] - np.zeros(3)) > 0
    assert most <= 12


def _edges_of(tris):
    c = Counter()
    for a, b, d in tris:
        for u, v in ((a, b), (b, d), (d, a)):
            c[(u, v)] += 1
    return c


def test_plane_closed_form():
    # f = x - c with c between sample layers i0 and i0 + 1: one quad per cube of layer i0
    R, i0 = 10, 4
    x = -1.0 + (2 * np.arange(R) + 1) / R
    c = (x[i0] + x[i0 + 1]) / 2 + 0.013
    f = np.broadcast_to((x - c)[:, None, None], (R, R, R)).copy()
    m = S.marching_cubes(f)
    assert m["triangles"].shape[0] == 2 * (R - 1) ** 2
    assert m["vertices"].shape[0] == R * R
    np.testing.assert_allclose(m["vertices"][:, 0], c, atol=1e-14)
    v = m["vertices"][m["triangles"]]
    n = np.cross(v[:, 1] - v[:, 0], v[:, 2] - v[:, 0])
    assert np.all(n[:, 0] > 0) and np.allclose(n[:, 1:], 0)   # towards f > 0


def test_sphere_is_closed_oriented_and_measures_right():
    R, r = 40, 0.55
    p = OD.grid_points(R)
    f = (np.linalg.norm(p - np.array([0.03, -0.02, 0.05]), axis=1) - r).reshape(R, R, R)
    m = S.marching_cubes(f)
    V, T = m["vertices"].shape[0], m["triangles"].shape[0]
    e = _edges_of(m["triangles"].tolist())
    # watertight and consistently oriented: every directed edge once, its reverse once
    assert all(n == 1 for n in e.values())
    assert all((v, u) in e for (u, v) in e)
    E = len(e) // 2
    assert V - E + T == 2
    vol = S.mesh_volume(m["vertices"], m["triangles"])
    area = S.mesh_area(m["vertices"], m["triangles"])
    assert vol == pytest.approx(4 / 3 * math.pi * r ** 3, rel=0.01)
    assert area == pytest.approx(4 * math.pi * r ** 2, rel=0.02)
    assert np.abs(np.linalg.norm(m["vertices"] - [0.03, -0.02, 0.05], axis=1) - r).max() < 2e-3


def test_random_field_is_watertight_inside_the_grid():
    # noise makes every face pattern appear; away from the grid's outer faces each
    # directed edge appears once and its reverse once (neighbouring cubes agree)
    rng = np.random.default_rng(0)
    R = 9
    f = rng.standard_normal((R, R, R))
    f[rng.random((R, R, R)) < 0.05] = 0.0
    m = S.marching_cubes(f)
    e = _edges_of(m["triangles"].tolist())
    assert all(n == 1 for n in e.values())
    vox = m["vertices"]
    lo, hi = -1 + 1 / R, 1 - 1 / R
    for (u, v) in e:
        if (v, u) in e:
            continue
        # an unmatched edge lies on the outer boundary of the sampled region
        pu, pv = vox[u], vox[v]
        on = [np.isclose(pu[a], b) and np.isclose(pv[a], b) for a in range(3) for b in (lo, hi)]
        assert any(on), (pu, pv)
    assert m["cube_tris"].sum() == m["triangles"].shape[0]
    assert m["cube_verts"].sum() == m["vertices"].shape[0]
