"""Pins of the hierarchical-decoding oracle: brute force on tiny grids,
closed forms of the marking/dilation, and the Lipschitz guarantee of an exact
sphere SDF (no GPU)."""
import itertools

import numpy as np
import pytest

from oracle import decoder as D
from oracle import hierarchy as HV


def _brute_mark(f, thr):
    R = f.shape[0]
    out = np.zeros(f.shape, bool)
    for i, j, k in itertools.product(range(R), repeat=3):
        s = f[i, j, k] < 0
        hit = abs(f[i, j, k]) < thr
        for di, dj, dk in itertools.product((-1, 0, 1), repeat=3):
            a, b, c = i + di, j + dj, k + dk
            if 0 <= a < R and 0 <= b < R and 0 <= c < R and (f[a, b, c] < 0) != s:
                hit = True
        out[i, j, k] = hit
    return out


def _brute_dilate(m):
    R = m.shape[0]
    out = np.zeros(m.shape, bool)
    for i, j, k in itertools.product(range(R), repeat=3):
        out[i, j, k] = any(m[a, b, c] for a in range(max(0, i - 1), min(R, i + 2))
                           for b in range(max(0, j - 1), min(R, j + 2))
                           for c in range(max(0, k - 1), min(R, k + 2)))
    return out


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_mark_and_dilate_match_brute_force(seed):
    rng = np.random.default_rng(seed)
    R = 7
    f = rng.standard_normal((R, R, R)).astype(np.float32) * 0.6 + 0.2
    f[rng.random(f.shape) < 0.05] = 0.0          # exact zeros count as outside
    thr = HV.near_threshold(R)
    m = HV.mark(f, thr)
    np.testing.assert_array_equal(m, _brute_mark(f, thr))
    np.testing.assert_array_equal(HV.dilate(m), _brute_dilate(m))


def test_single_inside_voxel_closed_form():
    R = 9
    f = np.ones((R, R, R), np.float32)
    f[4, 4, 4] = -1.0
    m = HV.mark(f, np.float32(0.5))
    want = np.zeros_like(m); want[3:6, 3:6, 3:6] = True
    np.testing.assert_array_equal(m, want)
    want2 = np.zeros_like(m); want2[2:7, 2:7, 2:7] = True
    np.testing.assert_array_equal(HV.dilate(m), want2)
    # at a corner the cube is clipped
    f2 = np.ones((R, R, R), np.float32); f2[0, 0, 0] = -1.0
    m2 = HV.mark(f2, np.float32(0.5))
    assert m2.sum() == 8 and m2[:2, :2, :2].all()


def test_near_surface_band_uses_float32_threshold():
    R = 96
    thr = HV.near_threshold(R)
    assert thr == np.float32(4.0 / 96)
    f = np.full((R, R, R), 1.0, np.float32)
    f[10, 10, 10] = np.nextafter(thr, np.float32(0))    # just below: marked
    f[20, 20, 20] = thr                                  # equal: not marked
    m = HV.mark(f, thr)
    assert m[10, 10, 10] and not m[20, 20, 20] and m.sum() == 1


def test_compaction_children_and_fill():
    rng = np.random.default_rng(5)
    R = 6
    act = rng.random((R, R, R)) < 0.2
    par = HV.compact(act)
    assert par.size == act.sum() and np.all(np.diff(par) > 0)
    assert np.all(act.ravel()[par])
    kids = HV.children(par, R)
    assert kids.size == 8 * par.size and np.all(np.diff(kids) > 0)
    np.testing.assert_array_equal(np.unique(HV.parent_of(kids, 2 * R)), par)
    # every fine voxel whose parent is active is a child, and no other
    allf = np.arange((2 * R) ** 3)
    np.testing.assert_array_equal(np.sort(allf[act.ravel()[HV.parent_of(allf, 2 * R)]]), kids)
    fc = rng.standard_normal((R, R, R))
    vals = rng.standard_normal(kids.size)
    ff = HV.fill(fc, kids, vals).ravel()
    np.testing.assert_array_equal(ff[kids], vals)
    rest = np.setdiff1d(allf, kids)
    np.testing.assert_array_equal(ff[rest], fc.ravel()[HV.parent_of(rest, 2 * R)])


def test_hierarchical_exact_sdf_lipschitz_guarantee():
    """With the exact sphere SDF (1-Lipschitz), every decoded voxel equals the
    dense value and every inherited voxel keeps the dense sign: a parent with
    |f| >= 2h cannot change sign within the distance sqrt(3) h / 2 of its
    children, and a sign change next to it would have marked it."""
    rng = np.random.default_rng(11)
    sp = np.concatenate([rng.uniform(-0.6, 0.6, (6, 3)), rng.uniform(0.05, 0.3, (6, 1))], axis=1)
    r0, L = 8, 4

    def dec_level(level, R, idx):
        return D.sphere_sdf(D.grid_points(R, idx), sp)

    res = HV.hierarchical(dec_level, r0, L)
    Rf = r0 << (L - 1)
    dense = D.sphere_sdf(D.grid_points(Rf), sp).reshape(Rf, Rf, Rf)
    g = res["grid"]
    last = res["levels"][-1]
    np.testing.assert_array_equal(g.ravel()[last["children"]], dense.ravel()[last["children"]])
    np.testing.assert_array_equal(g < 0, dense < 0)
    # fewer queries than dense decoding
    n_q = r0 ** 3 + sum(lv["children"].size for lv in res["levels"][1:])
    assert n_q < 0.6 * Rf ** 3


def test_tsdf_rule_equals_a_distance_band_for_an_exact_field():
    # dec_scale = 0: tsdf = clip(sdf / trunc), so |tsdf| < 0.95 marks exactly the voxels with
    # |sdf| < 0.95 trunc (grid chosen so that no voxel sits on the band edge)
    from oracle import decoder as D
    R, trunc = 24, 0.2
    sp = np.array([[0.1, -0.05, 0.02, 0.437]])
    p = D.grid_points(R)
    f = D.sphere_sdf(p, sp).reshape(R, R, R)
    t = D.tsdf_field(p, np.zeros(p.shape[0]), sp, 0.0, trunc).reshape(R, R, R)
    assert np.abs(np.abs(f) - 0.95 * trunc).min() > 1e-4
    near = np.abs(t.astype(np.float32)) < np.float32(0.95)
    assert np.array_equal(HV.mark(f, 0.0, near=near), HV.mark(f, 0.95 * trunc))
    assert near.sum() > (np.abs(f) < HV.near_threshold(R)).sum()     # a wider band than 2 h


def test_hierarchical_carries_the_tsdf_grid():
    # decode_level returning (field, tsdf): the tsdf grid is inherited like the field and its
    # band decides the refinement; with a zero tsdf everywhere every voxel is near: all refined
    from oracle import decoder as D
    sp = np.array([[0.0, 0.0, 0.0, 0.5]])

    def dl(level, R, idx):
        p = D.grid_points(R, idx)
        return D.sphere_sdf(p, sp), np.zeros(idx.size)

    out = HV.hierarchical(dl, 4, 3, tsdf_threshold=0.95)
    assert out["levels"][0]["active"].all() and out["levels"][1]["active"].all()
    assert out["levels"][2]["tsdf"].shape == (16, 16, 16) and not out["levels"][2]["tsdf"].any()
