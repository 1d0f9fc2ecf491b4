"""Oracle: surface extraction (marching cubes) from a decoded SDF volume.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

The pipeline's last stage turns the decoded volume into a mesh (techwalker
article, section 1: image encoding -> diffusion sampling -> VAE decoding ->
surface extraction).  The pages name no extraction method; the plainest
reading is marching cubes on the grid of decoded samples: every cube of 2^3
neighbouring samples whose corners have both signs holds a piece of the zero
level set, and the piece is a set of closed polygons whose vertices sit on the
cube's edges where the field crosses zero (linear interpolation).

Nothing here is a memorised case table: each cube's polygons are traced from
its 8 corner signs with the rules below, written out once in plain Python.

Conventions (shared with the CUDA path by specification, not by code):

* samples: the voxel centres of an R^3 grid, ``x_i = -1 + (2 i + 1) / R``;
  cube (i, j, k) has its minimum corner at sample (i, j, k), i, j, k < R - 1;
* corner c = 4 ci + 2 cj + ck sits at (i + ci, j + cj, k + ck); inside means
  f < 0 (f == 0 is outside);
* edge e = 4 a + 2 u + v runs along axis a (0: i, 1: j, 2: k) between the two
  corners whose other two coordinates, in increasing axis order, are (u, v);
* a face holds the 4 edges along its two axes; with two sign changes around
  it, one segment joins its two crossed edges; with four (diagonal corners
  alike), two segments each cut off one inside corner ("inside corners are
  never joined across a face"), which both cubes sharing the face agree on;
* each segment A -> B is oriented so that an inside corner P of its side
  satisfies ((B - A) x (P - A)) . n < 0 with n the face's outward normal
  (edge midpoints stand for A and B); the segments then chain into closed
  loops, each listed from its smallest edge id in segment direction, loops in
  order of their smallest edge id; a loop l0 .. l(m-1) becomes a fan from its
  apex l_s, the first l_s in loop order none of whose fan diagonals
  (l_s, l_(s+q)), 2 <= q <= m - 2, joins two edges of one cube face (such a
  diagonal would lie in the face, where the neighbouring cube draws it too);
  the fan is (l_s, l_(s+1), l_(s+2)), (l_s, l_(s+2), l_(s+3)), ... (indices
  mod m); every loop of the 256 patterns has such an apex; triangle normals
  point to the outside (f > 0) region;
* vertices: the crossed edge from sample p0 to p1 = p0 + 1 along axis a sits
  at p0 + t (p1 - p0), t = f0 / (f0 - f1); it belongs to sample p0;
* order: samples (vertex owners) and cubes (by minimum corner) are both
  ordered by 8^3 block in linear block order, then linear order inside the
  block; a sample's vertices in axis order; triangles cube by cube in loop
  and fan order.
"""
from __future__ import annotations

from typing import Dict, List, Tuple

import numpy as np

_CORNER = [((c >> 2) & 1, (c >> 1) & 1, c & 1) for c in range(8)]


def _edge_corners(e: int) -> Tuple[int, int]:
    """The two corners of edge e (axis bit 0 first)."""
    a, u, v = e // 4, (e >> 1) & 1, e & 1
    others = [x for x in range(3) if x != a]
    lo = [0, 0, 0]
    lo[others[0]], lo[others[1]] = u, v
    hi = list(lo)
    hi[a] = 1
    idx = lambda p: 4 * p[0] + 2 * p[1] + p[2]
    return idx(lo), idx(hi)


def _edge_mid(e: int) -> np.ndarray:
    c0, c1 = _edge_corners(e)
    return (np.array(_CORNER[c0], float) + np.array(_CORNER[c1], float)) / 2.0


def _face_cycle(a: int, s: int) -> List[int]:
    """Corners of face (axis a, side s) in cyclic order around the square."""
    others = [x for x in range(3) if x != a]
    cyc = []
    for u, v in ((0, 0), (1, 0), (1, 1), (0, 1)):
        p = [0, 0, 0]
        p[a], p[others[0]], p[others[1]] = s, u, v
        cyc.append(4 * p[0] + 2 * p[1] + p[2])
    return cyc


def _edge_of(c0: int, c1: int) -> int:
    p, q = _CORNER[c0], _CORNER[c1]
    a = [x for x in range(3) if p[x] != q[x]][0]
    others = [x for x in range(3) if x != a]
    return 4 * a + 2 * p[others[0]] + p[others[1]]


def cube_loops(config: int) -> List[List[int]]:
    """Oriented loops (lists of edge ids) of a cube whose inside corners are the
    set bits of ``config`` (bit c = corner c inside)."""
    inside = [(config >> c) & 1 == 1 for c in range(8)]
    nxt: Dict[int, int] = {}
    for a in range(3):
        for s in range(2):
            n = np.zeros(3)
            n[a] = 1.0 if s else -1.0
            cyc = _face_cycle(a, s)
            crossed = [_edge_of(cyc[q], cyc[(q + 1) % 4]) for q in range(4)
                       if inside[cyc[q]] != inside[cyc[(q + 1) % 4]]]
            if not crossed:
                continue
            if len(crossed) == 2:
                segs = [(crossed[0], crossed[1], [c for c in cyc if inside[c]][0])]
            else:
                # diagonal corners alike: cut off each inside corner separately
                segs = []
                for q in range(4):
                    if inside[cyc[q]]:
                        segs.append((_edge_of(cyc[q - 1], cyc[q]), _edge_of(cyc[q], cyc[(q + 1) % 4]), cyc[q]))
            for ea, eb, pin in segs:
                A, B, P = _edge_mid(ea), _edge_mid(eb), np.array(_CORNER[pin], float)
                if np.dot(np.cross(B - A, P - A), n) > 0:
                    ea, eb = eb, ea
                assert ea not in nxt, "two segments leave one edge"
                nxt[ea] = eb
    loops = []
    seen = set()
    for start in sorted(nxt):
        if start in seen:
            continue
        loop = [start]
        seen.add(start)
        e = nxt[start]
        while e != start:
            loop.append(e)
            seen.add(e)
            e = nxt[e]
        loops.append(loop)
    return loops


def _faces(e: int) -> set:
    """The two cube faces (axis, side) that hold edge e."""
    c0, c1 = _edge_corners(e)
    p, q = _CORNER[c0], _CORNER[c1]
    return {(a, p[a]) for a in range(3) if p[a] == q[a]}


def cube_triangles(config: int) -> List[Tuple[int, int, int]]:
    """Fan triangulation of the cube's loops (edge-id triples), each fan from the
    first apex in loop order whose diagonals lie in no face."""
    tris = []
    for loop in cube_loops(config):
        m = len(loop)
        for s in range(m):
            r = loop[s:] + loop[:s]
            if all(not (_faces(r[0]) & _faces(r[q])) for q in range(2, m - 1)):
                break
        else:
            raise AssertionError(f"loop {loop} has no apex")
        for q in range(1, m - 1):
            tris.append((r[0], r[q], r[q + 1]))
    return tris


def _block_order(R: int, n: int) -> np.ndarray:
    """Linear indices (i, j, k) -> i R^2 + j R + k of the points of [0, n)^3 in
    block order: 8^3 blocks in linear block order, linear order inside a block
    (n = R for samples, R - 1 for cubes' minimum corners)."""
    i, j, k = np.meshgrid(np.arange(n), np.arange(n), np.arange(n), indexing="ij")
    i, j, k = i.ravel(), j.ravel(), k.ravel()
    nb = (R + 7) // 8
    blk = ((i >> 3) * nb + (j >> 3)) * nb + (k >> 3)
    loc = ((i & 7) * 8 + (j & 7)) * 8 + (k & 7)
    order = np.lexsort((loc, blk))
    return (i[order] * R + j[order]) * R + k[order]


def marching_cubes(f: np.ndarray) -> Dict[str, np.ndarray]:
    """Mesh of the zero level set of a dense grid ``f[R,R,R]`` (every cube).

    Returns ``vertices [V,3]`` (float64 xyz), ``triangles [T,3]`` (vertex
    indices), ``cube_ids`` / ``cube_tris``: each cube with a crossing (linear
    index of its minimum corner) and its triangle count, and ``cube_verts``:
    the vertex count of each sample that owns vertices, all in output order."""
    f = np.asarray(f)
    R = f.shape[0]
    flat = f.ravel()
    inside = flat < 0
    h = 2.0 / R
    order = _block_order(R, R - 1)
    # corners' linear offsets
    offs = np.array([(ci * R + cj) * R + ck for ci, cj, ck in _CORNER])
    cfg = np.zeros(order.size, np.int64)
    for c in range(8):
        cfg |= inside[order + offs[c]].astype(np.int64) << c
    crossing = (cfg != 0) & (cfg != 255)
    # a cube's own vertices: its edges 0 (axis i), 4 (axis j), 8 (axis k) when crossed
    own_axis_off = [R * R, R, 1]
    vid: Dict[Tuple[int, int], int] = {}
    verts: List[np.ndarray] = []
    for smp in _block_order(R, R):
        i, rem = divmod(int(smp), R * R)
        j, k = divmod(rem, R)
        for a in range(3):
            if (i, j, k)[a] == R - 1:
                continue
            q = smp + own_axis_off[a]
            if inside[smp] != inside[q]:
                f0, f1 = float(flat[smp]), float(flat[q])
                t = f0 / (f0 - f1)
                p = np.array([-1.0 + (2 * i + 1) / R, -1.0 + (2 * j + 1) / R, -1.0 + (2 * k + 1) / R])
                p[a] += t * h
                vid[(int(smp), a)] = len(verts)
                verts.append(p)
    tris = []
    cube_ids, cube_tris, cube_verts = [], [], []
    for cube, c in zip(order[crossing], cfg[crossing]):
        i, rem = divmod(int(cube), R * R)
        j, k = divmod(rem, R)
        ts = cube_triangles(int(c))
        for tri in ts:
            idx = []
            for e in tri:
                c0, _ = _edge_corners(e)
                ci, cj, ck = _CORNER[c0]
                owner = ((i + ci) * R + (j + cj)) * R + (k + ck)
                idx.append(vid[(owner, e // 4)])
            tris.append(idx)
        cube_ids.append(int(cube))
        cube_tris.append(len(ts))
    for smp in _block_order(R, R):
        nv = sum(1 for a in range(3) if (int(smp), a) in vid)
        if nv:
            cube_verts.append(nv)
    return {"vertices": np.array(verts, np.float64).reshape(-1, 3),
            "triangles": np.array(tris, np.int64).reshape(-1, 3),
            "cube_ids": np.array(cube_ids, np.int64), "cube_tris": np.array(cube_tris, np.int64),
            "cube_verts": np.array(cube_verts, np.int64)}


def mesh_volume(vertices: np.ndarray, triangles: np.ndarray) -> float:
    """Signed volume enclosed by a closed, outward-oriented triangle mesh
    (divergence theorem: sum of v0 . (v1 x v2) / 6)."""
    v = np.asarray(vertices, np.float64)[np.asarray(triangles)]
    return float(np.einsum("ij,ij->i", v[:, 0], np.cross(v[:, 1], v[:, 2])).sum() / 6.0)


def mesh_area(vertices: np.ndarray, triangles: np.ndarray) -> float:
    v = np.asarray(vertices, np.float64)[np.asarray(triangles)]
    return float(np.linalg.norm(np.cross(v[:, 1] - v[:, 0], v[:, 2] - v[:, 0]), axis=1).sum() / 2.0)
