"""Oracle: adaptive KV selection on the fine levels of hierarchical decoding.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

FlashVDM summary, section 4.1 item 2 ("Adaptive KV Selection"): split the
volume into small sub-volumes; in each, randomly sample a small part of the
queries; score all vecset tokens with the attention of those samples; keep the
Top-K tokens (key/value pairs) for the sub-volume; every other query of the
sub-volume attends to those K tokens only.  Queries of different sub-volumes
are packed to run in parallel ("packing" note).  The techwalker article
(section 5) describes the same procedure as "trial queries in a small region".

Readings taken here (the pages give no sizes, sampler, score or tie rule):

* sub-volumes are aligned 8^3 tiles of the fine level's grid; only the level's
  active (subdivided) fine voxels are queries;
* "randomly sample" is made reproducible by ranking the tile's queries by
  ``splitmix64(splitmix64(seed ^ (level << 32)) ^ linear_index)`` (ties by the
  smaller index) and taking the first ``n_probe`` (64); a tile with at most
  ``n_probe`` queries decodes all of them densely and selects nothing;
* a token's score is its softmax probability summed over heads and probes;
* Top-K keeps the ``k`` largest scores, ties to the smaller token index; the
  kept set is used in ascending token order; one subset is shared by all heads;
* probes keep their full-attention result; the other queries attend over the
  kept subset, softmax renormalised over it;
* the coarse level is decoded densely; adaptive selection runs on fine levels.

SplitMix64 is the generator of Steele, Lea and Flood, "Fast splittable
pseudorandom number generators" (OOPSLA 2014), in its common 64-bit finaliser
form: add the golden-ratio increment, then two xor-shift-multiply rounds and a
final xor-shift.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np

from . import decoder as D

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def splitmix64(x) -> np.ndarray:
    """SplitMix64 output for state ``x`` (uint64 array, arithmetic mod 2^64)."""
    z = np.asarray(x, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = z + _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def probe_key(seed: int, level: int, idx: np.ndarray) -> np.ndarray:
    """Per-query random rank key of fine level ``level``."""
    salt = splitmix64(np.uint64(seed) ^ (np.uint64(level) << np.uint64(32)))
    return splitmix64(np.asarray(idx, np.uint64) ^ salt)


def tile_of(idx: np.ndarray, R: int, tile: int) -> np.ndarray:
    """Linear id of the aligned ``tile^3`` sub-volume holding each fine voxel."""
    idx = np.asarray(idx, np.int64)
    i, rem = np.divmod(idx, R * R)
    j, k = np.divmod(rem, R)
    nt = R // tile
    return ((i // tile) * nt + (j // tile)) * nt + (k // tile)


def choose_probes(idx: np.ndarray, n_probe: int, seed: int, level: int) -> np.ndarray:
    """Boolean mask over ``idx`` (one tile's queries): the ``n_probe`` queries
    with the smallest (key, index)."""
    idx = np.asarray(idx, np.int64)
    if idx.size <= n_probe:
        return np.ones(idx.size, dtype=bool)
    key = probe_key(seed, level, idx)
    order = np.lexsort((idx, key))   # primary key, then index
    m = np.zeros(idx.size, dtype=bool)
    m[order[:n_probe]] = True
    return m


def token_scores(q: np.ndarray, K: np.ndarray) -> np.ndarray:
    """Softmax probabilities summed over heads and the given queries: ``[N]``."""
    return D.attention_probs(q, K).sum(axis=(0, 1))


def top_k(score: np.ndarray, k: int) -> np.ndarray:
    """Indices of the ``k`` largest scores (ties to the smaller index), in
    ascending index order."""
    score = np.asarray(score, np.float64)
    n = score.size
    if k >= n:
        return np.arange(n, dtype=np.int64)
    order = np.lexsort((np.arange(n), -score))
    return np.sort(order[:k]).astype(np.int64)


def query_vectors(p: np.ndarray, w: Dict[str, np.ndarray]) -> np.ndarray:
    return D.linear(D.fourier_embed(p), w["Wq"], w["bq"])


def adaptive_level(level: int, R: int, kids: np.ndarray, K: np.ndarray, V: np.ndarray,
                   w: Dict[str, np.ndarray], query_ln: bool, spheres: Optional[np.ndarray],
                   dec_scale: float, seed: int, tile: int = 8, n_probe: int = 64,
                   k: int = 1024, sel_override: Optional[Dict[int, np.ndarray]] = None,
                   keep_tiles: bool = False, tsdf_trunc: Optional[float] = None) -> Dict:
    """Field values of fine level ``level`` at the active voxels ``kids``.

    ``sel_override`` maps tile id -> token subset and replaces the oracle's
    own selection for that tile (used to compare a decode given the same
    selection).  Returns ``values`` (aligned with ``kids``), ``dec`` (raw
    decoder outputs) and, with ``keep_tiles``, per-tile probes/scores/subsets.
    With ``tsdf_trunc`` the tSDF head is decoded too (same attention) and
    ``tsdf`` holds ``decoder.tsdf_field`` at ``kids``.
    """
    if R % tile:
        raise ValueError("fine resolution must be a multiple of the tile edge")
    kids = np.asarray(kids, np.int64)
    vals = np.empty(kids.size, np.float64)
    decs = np.empty(kids.size, np.float64)
    tsdf = np.empty(kids.size, np.float64) if tsdf_trunc is not None else None
    want_t = tsdf is not None
    tiles = {}
    tid = tile_of(kids, R, tile)
    order = np.lexsort((kids, tid))
    bounds = np.flatnonzero(np.diff(tid[order])) + 1
    for grp in np.split(order, bounds):
        if grp.size == 0:
            continue
        t = int(tid[grp[0]])
        idx = kids[grp]                       # ascending within the tile
        pts = D.grid_points(R, idx)
        probe = choose_probes(idx, n_probe, seed, level)
        dec = np.empty(idx.size, np.float64)
        traw = np.empty(idx.size, np.float64)
        r = D.decode_points(pts[probe], K, V, w, query_ln, return_tsdf=want_t)
        if want_t:
            dec[probe], traw[probe] = r
        else:
            dec[probe] = r
        info = {"idx": idx, "probe": probe}
        if (~probe).any():
            score = token_scores(query_vectors(pts[probe], w), K)
            sel = top_k(score, k)
            if sel_override is not None and t in sel_override:
                sel = np.asarray(sel_override[t], np.int64)
            r = D.decode_points(pts[~probe], K, V, w, query_ln, sel=sel, return_tsdf=want_t)
            if want_t:
                dec[~probe], traw[~probe] = r
            else:
                dec[~probe] = r
            info.update(score=score, sel=sel)
        decs[grp] = dec
        vals[grp] = D.field(pts, dec, spheres, dec_scale)
        if want_t:
            tsdf[grp] = D.tsdf_field(pts, traw, spheres, dec_scale, tsdf_trunc)
        if keep_tiles:
            tiles[t] = info
    out = {"values": vals, "dec": decs}
    if want_t:
        out["tsdf"] = tsdf
    if keep_tiles:
        out["tiles"] = tiles
    return out
