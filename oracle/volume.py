"""Oracle: whole-volume decoding of one shape (dense grid or coarse-to-fine).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Wires ``decoder``, ``hierarchy`` and ``adaptive`` together for one shape of a
workload: the VAE decode stage of the pipeline (techwalker article, section 1:
image encoding -> diffusion sampling -> VAE decoding -> surface extraction).
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np

from . import adaptive as A
from . import decoder as D
from . import hierarchy as HV


def shape_kv(z: np.ndarray, w: Dict[str, np.ndarray]):
    """K, V ``[H,N,64]`` of one shape's vecset ``z[N,C]``."""
    return D.precompute_kv(z, w)


def dense_grid(K, V, w, R: int, query_ln: bool, spheres=None, dec_scale: float = 0.0,
               idx: Optional[np.ndarray] = None) -> np.ndarray:
    """Field (or raw decoder output without spheres) at grid voxels ``idx``
    (all R^3 voxels by default), float64."""
    p = D.grid_points(R, idx)
    dec = D.decode_points(p, K, V, w, query_ln)
    return D.field(p, dec, spheres, dec_scale)


def hierarchical_volume(K, V, w, r0: int, n_levels: int, query_ln: bool, spheres=None,
                        dec_scale: float = 0.0, adaptive: bool = False, seed: int = 0,
                        tile: int = 8, n_probe: int = 64, top_k: int = 1024,
                        coarse: Optional[np.ndarray] = None, keep_tiles: bool = False,
                        tsdf_trunc: Optional[float] = None, tsdf_threshold: float = 0.95) -> Dict:
    """Hierarchical decoding of one shape, optionally with adaptive KV on the
    fine levels.  Returns ``hierarchy.hierarchical``'s dict plus, per fine
    level, the raw decoder outputs (``dec``) and adaptive tile records.  With
    ``tsdf_trunc`` the decoder's tSDF head drives the near-surface rule
    (``|tsdf| < tsdf_threshold``) instead of ``|f| < 2h``."""
    extras = {}
    want_t = tsdf_trunc is not None

    def decode_level(level: int, R: int, idx: np.ndarray):
        p = D.grid_points(R, idx)
        if level == 0 or not adaptive:
            r = D.decode_points(p, K, V, w, query_ln, return_tsdf=want_t)
            dec = r[0] if want_t else r
            extras[level] = {"dec": dec}
            f = D.field(p, dec, spheres, dec_scale)
            return (f, D.tsdf_field(p, r[1], spheres, dec_scale, tsdf_trunc)) if want_t else f
        out = A.adaptive_level(level, R, idx, K, V, w, query_ln, spheres, dec_scale, seed,
                               tile=tile, n_probe=n_probe, k=top_k, keep_tiles=keep_tiles,
                               tsdf_trunc=tsdf_trunc)
        extras[level] = out
        return (out["values"], out["tsdf"]) if want_t else out["values"]

    res = HV.hierarchical(decode_level, r0, n_levels, coarse=coarse,
                          tsdf_threshold=tsdf_threshold if want_t else None)
    for lv, e in extras.items():
        res["levels"][lv].update({k: v for k, v in e.items() if k not in ("values", "tsdf")})
    return res


def compare_volumes(a: np.ndarray, b: np.ndarray) -> Dict:
    """Counts behind the volume IoU of two fields on the same grid (aipaper.cc
    summary, section 5 "Evaluation Metrics": V-IoU of the inside sets; Table 3
    reports it per acceleration).  Inside means ``f < 0``.  ``max_abs_diff`` is
    computed in the fields' own precision."""
    a = np.asarray(a).ravel()
    b = np.asarray(b).ravel()
    ia, ib = a < 0, b < 0
    both = int((ia & ib).sum())
    union = int(ia.sum()) + int(ib.sum()) - both
    return {"inside_a": int(ia.sum()), "inside_b": int(ib.sum()), "inside_both": both,
            "same_sign": int((ia == ib).sum()),
            "v_iou": both / union if union else 1.0,
            "max_abs_diff": float(np.abs(a - b).max()) if a.size else 0.0}
