"""Oracle: hierarchical (coarse-to-fine) volume decoding, step by step.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

FlashVDM summary, section 4.1 item 1 ("Hierarchical Volume Decoding"):
decode the whole volume at a low resolution; find the voxels that meet the
surface, i.e. whose neighbours have a different SDF sign; subdivide them and
query only the new sub-voxels; repeat up to the target resolution.  Two
corner-case fixes: also select voxels whose truncated SDF is below a
threshold (thin structures), and dilate the selected set once.  The
techwalker article (section 5) adds that voxels wholly inside or outside are
skipped and labelled directly.

Readings taken here:

* neighbourhood = the 3x3x3 cube around a voxel, clipped at the grid border
  (border voxels simply have fewer neighbours);
* inside means ``f < 0``; ``f == 0`` counts as outside;
* the synthetic field has no tSDF channel, so the near-surface rule is
  ``|f| < 2 h`` with ``h = 2 / R`` the current level's voxel width; the
  threshold is the float32 value ``float32(4 / R)`` and the comparison is made
  in the grid's own precision;
* the marking is recomputed on every level's dense grid (decoded or inherited
  values) -- "repeat this process";
* one dilation = one pass of the same 3x3x3 cube;
* a fine voxel whose parent is not selected inherits the parent's value (and
  hence its sign), recursively.
"""
from __future__ import annotations

from typing import Callable, Dict, List, Optional

import numpy as np

_OFFSETS = [(di, dj, dk) for di in (-1, 0, 1) for dj in (-1, 0, 1) for dk in (-1, 0, 1)]


def near_threshold(R: int) -> np.float32:
    """``2 h`` for voxel width ``h = 2/R``, as a float32 value."""
    return np.float32(4.0 / R)


def _shift_views(a: np.ndarray, pad_value):
    """Yield, for each of the 27 cube offsets, the array of neighbour values
    (``pad_value`` where the neighbour falls outside the grid)."""
    R = a.shape[0]
    p = np.full((R + 2, R + 2, R + 2), pad_value, dtype=a.dtype)
    p[1:-1, 1:-1, 1:-1] = a
    for di, dj, dk in _OFFSETS:
        yield p[1 + di:1 + di + R, 1 + dj:1 + dj + R, 1 + dk:1 + dk + R]


def mark(f: np.ndarray, thr, near: Optional[np.ndarray] = None) -> np.ndarray:
    """Boundary mark of a dense level grid ``f[R,R,R]``.

    ``mark(v) = (exists in-grid u in cube(v): (f_u < 0) != (f_v < 0)) or near(v)``
    with ``near(v) = |f_v| < thr``, or the given ``near`` mask (the tSDF rule:
    ``|tsdf_v| < threshold``, section 4.1 item 1 "key details" 1; 0.95 on the
    techwalker article, section 5).
    """
    f = np.asarray(f)
    inside = f < 0
    # out-of-grid neighbours take v's own sign so they never count as a change
    change = np.zeros(f.shape, dtype=bool)
    R = f.shape[0]
    p = np.zeros((R + 2, R + 2, R + 2), dtype=np.int8)
    p[...] = -1
    p[1:-1, 1:-1, 1:-1] = inside.astype(np.int8)
    for di, dj, dk in _OFFSETS:
        nb = p[1 + di:1 + di + R, 1 + dj:1 + dj + R, 1 + dk:1 + dk + R]
        change |= (nb >= 0) & (nb != inside)
    return change | ((np.abs(f) < thr) if near is None else np.asarray(near, bool))


def dilate(m: np.ndarray) -> np.ndarray:
    """One 3x3x3 dilation, clipped at the border."""
    out = np.zeros(m.shape, dtype=bool)
    for nb in _shift_views(np.asarray(m, bool), False):
        out |= nb
    return out


def compact(active: np.ndarray) -> np.ndarray:
    """Linear indices of the active voxels in ascending order (int64)."""
    return np.flatnonzero(np.asarray(active).ravel()).astype(np.int64)


def children(parents: np.ndarray, R: int) -> np.ndarray:
    """Linear indices, at resolution 2R, of the 8 children of each parent
    (ascending order overall)."""
    parents = np.asarray(parents, np.int64)
    i, rem = np.divmod(parents, R * R)
    j, k = np.divmod(rem, R)
    R2 = 2 * R
    out = []
    for di in (0, 1):
        for dj in (0, 1):
            for dk in (0, 1):
                out.append(((2 * i + di) * R2 + (2 * j + dj)) * R2 + (2 * k + dk))
    return np.sort(np.concatenate(out)) if out else np.zeros(0, np.int64)


def parent_of(idx: np.ndarray, R2: int) -> np.ndarray:
    """Parent linear index (resolution R2/2) of fine voxels at resolution R2."""
    idx = np.asarray(idx, np.int64)
    i, rem = np.divmod(idx, R2 * R2)
    j, k = np.divmod(rem, R2)
    R = R2 // 2
    return ((i >> 1) * R + (j >> 1)) * R + (k >> 1)


def fill(f_coarse: np.ndarray, child_idx: np.ndarray, child_val: np.ndarray) -> np.ndarray:
    """Dense fine grid: decoded values where the parent is active, else the
    parent's value."""
    R = f_coarse.shape[0]
    R2 = 2 * R
    fine = np.repeat(np.repeat(np.repeat(f_coarse, 2, axis=0), 2, axis=1), 2, axis=2).copy()
    flat = fine.reshape(-1)
    flat[np.asarray(child_idx, np.int64)] = child_val
    return flat.reshape(R2, R2, R2)


def hierarchical(decode_level: Callable[[int, int, np.ndarray], np.ndarray],
                 r0: int, n_levels: int, dilation: int = 1,
                 dtype=np.float64, coarse: Optional[np.ndarray] = None,
                 tsdf_threshold: Optional[float] = None) -> Dict:
    """Coarse-to-fine decoding.

    ``decode_level(level, R, idx)`` returns field values at the voxels
    ``idx`` (linear, resolution R) of level ``level`` (0 = coarse); with
    ``tsdf_threshold`` it returns ``(field, tsdf)`` and the near-surface rule
    is ``|tsdf| < tsdf_threshold`` (compared in float32), the tSDF grid being
    decoded and inherited like the field.
    ``coarse`` optionally supplies the level-0 grid instead of decoding it.
    Returns the final dense grid and, per level, the masks, active parents,
    decoded children and their values.
    """
    R = r0
    use_t = tsdf_threshold is not None
    tg = None
    if coarse is None:
        r = decode_level(0, R, np.arange(R ** 3, dtype=np.int64))
        if use_t:
            r, t0 = r
            tg = np.asarray(t0, dtype).reshape(R, R, R)
        f = np.asarray(r).astype(dtype).reshape(R, R, R)
    else:
        f = np.asarray(coarse, dtype).reshape(R, R, R)
    levels: List[Dict] = [{"R": R, "grid": f, "tsdf": tg}]
    for lv in range(1, n_levels):
        near = None
        if use_t:
            near = np.abs(tg.astype(np.float32)) < np.float32(tsdf_threshold)
        m = mark(f, near_threshold(R), near=near)
        act = m
        for _ in range(dilation):
            act = dilate(act)
        parents = compact(act)
        kids = children(parents, R)
        r = decode_level(lv, 2 * R, kids)
        if use_t:
            r, tv = r
            tg = fill(tg, kids, np.asarray(tv).astype(dtype))
        vals = np.asarray(r).astype(dtype)
        f = fill(f, kids, vals)
        levels[-1].update(mark=m, active=act, parents=parents)
        R *= 2
        levels.append({"R": R, "grid": f, "children": kids, "values": vals, "tsdf": tg})
    return {"grid": f, "levels": levels}
