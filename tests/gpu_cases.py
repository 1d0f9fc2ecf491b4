"""Shared set-up for the GPU parity tests: build a decoder on the device and
in the oracle from the same seeded arrays, and compare hierarchical outputs
level by level.  Imported by the gpu-marked tests only."""
from __future__ import annotations

import numpy as np

import workloads as W
from oracle import adaptive as OA
from oracle import decoder as OD
from oracle import hierarchy as OH

TOL = {"f32": 1e-4, "bf16": 2e-2}


class Case:
    """One shape's decoder: device tensors, oracle K/V, spheres."""

    def __init__(self, spec: W.DecoderSpec, key: int, B: int = 1, stress: bool = False,
                 n_spheres: int = 0, sphere_key: int = 0, seed: int = 0):
        import torch
        import neural_sdf_volume_b200 as vdm
        self.spec = spec
        d = W.make_decoder(spec, seed=seed, key=key, B=B, stress=stress)
        self.w = d["weights"]
        self.z = d["z"]
        self.dec = vdm.Decoder.from_numpy(self.w, spec.C, spec.H, spec.F, spec.query_ln, spec.dtype)
        self.K, self.V = vdm.vdm_precompute_kv(self.dec, torch.from_numpy(self.z).cuda())
        self._okv = {}
        self.spheres_np = (W.make_spheres(n_spheres, seed, sphere_key, B) if n_spheres else None)
        self.spheres = (torch.from_numpy(self.spheres_np).cuda() if n_spheres else None)

    def okv(self, b: int = 0):
        if b not in self._okv:
            self._okv[b] = OD.precompute_kv(self.z[b], self.w)
        return self._okv[b]

    def oracle_dec(self, p: np.ndarray, b: int = 0, sel=None) -> np.ndarray:
        K, V = self.okv(b)
        return OD.decode_points(p, K, V, self.w, self.spec.query_ln, sel=sel)

    def sp(self, b: int = 0):
        return None if self.spheres_np is None else self.spheres_np[b]


def unpack_words(words: np.ndarray, R: int) -> np.ndarray:
    """Blocked refine mask (one uint64 per 4^3 block) -> bool [R,R,R]."""
    nb = R // 4
    w = words.astype(np.uint64).reshape(nb, nb, nb)
    bits = ((w[..., None] >> np.arange(64, dtype=np.uint64)) & np.uint64(1)).astype(bool)
    bits = bits.reshape(nb, nb, nb, 4, 4, 4)           # (bi, bj, bk, di, dj, dk)
    return bits.transpose(0, 3, 1, 4, 2, 5).reshape(R, R, R)


def debug_buffers(B: int, r0: int, L: int, adaptive: bool, k: int, max_tiles: int):
    import torch
    dbg = {"grid": [], "active": [], "dec": [], "tile_ids": [], "sel": [], "max_tiles": max_tiles}
    for l in range(L):
        R = r0 << l
        dbg["grid"].append(torch.empty((B, R ** 3), device="cuda", dtype=torch.float32))
        dbg["dec"].append(torch.full((B, R ** 3), float("nan"), device="cuda", dtype=torch.float32))
        dbg["active"].append(torch.zeros((B, (R // 4) ** 3), device="cuda", dtype=torch.int64)
                             if l < L - 1 else None)
        if adaptive and l > 0:
            dbg["tile_ids"].append(torch.full((B, max_tiles), -1, device="cuda", dtype=torch.int32))
            dbg["sel"].append(torch.full((B, max_tiles, k), -1, device="cuda", dtype=torch.int32))
        else:
            dbg["tile_ids"].append(None)
            dbg["sel"].append(None)
    return dbg


def check_levels(case: Case, b: int, r0: int, L: int, dbg, dec_scale: float, adaptive: bool,
                 n_probe: int, seed: int, sample: int = 0, rng=None, report=None):
    """Level-by-level parity of one shape's hierarchical decode.

    * refine masks bit-exact vs the oracle's mark+dilate of the GPU's own grid;
    * inherited voxels equal their parent's value exactly;
    * decoded voxels: raw decoder output within tolerance of the oracle at the
      same points (adaptive non-probes attend over the GPU's selection), and the
      stored field equals sphere SDF + scale tanh(dec) of the GPU's own dec.
    ``sample`` > 0 compares a random subset of the decoded voxels only.
    """
    tol = TOL[case.spec.dtype]
    rng = rng or np.random.default_rng(0)
    report = report if report is not None else {}
    grids = [dbg["grid"][l][b].cpu().numpy() for l in range(L)]
    decs = [dbg["dec"][l][b].cpu().numpy() for l in range(L)]
    worst = 0.0
    for l in range(L):
        R = r0 << l
        g = grids[l].reshape(R, R, R)
        if l < L - 1:
            words = dbg["active"][l][b].cpu().numpy().view(np.uint64)
            act_gpu = unpack_words(words, R)
            act_ref = OH.dilate(OH.mark(g, OH.near_threshold(R)))
            assert np.array_equal(act_gpu, act_ref), f"level {l}: refine mask differs " \
                f"({int((act_gpu != act_ref).sum())} voxels)"
        if l == 0:
            decoded = np.arange(R ** 3)
        else:
            Rp = R // 2
            act_p = unpack_words(dbg["active"][l - 1][b].cpu().numpy().view(np.uint64), Rp)
            decoded = OH.children(OH.compact(act_p), Rp)
            inherited = np.setdiff1d(np.arange(R ** 3), decoded)
            par = OH.parent_of(inherited, R)
            assert np.array_equal(g.ravel()[inherited], grids[l - 1].ravel()[par]), \
                f"level {l}: inherited voxels differ from their parents"
        report[f"decoded_{l}"] = int(decoded.size)
        dv = decs[l][decoded]
        assert np.isfinite(dv).all(), f"level {l}: some decoded voxels were not written"
        # stored field is consistent with the GPU's own raw decoder output
        pts_all = OD.grid_points(R, decoded)
        fld = OD.field(pts_all, dv.astype(np.float64), case.sp(b), dec_scale)
        assert np.abs(g.ravel()[decoded] - fld).max() < 1e-5
        idx = decoded if not sample or decoded.size <= sample else \
            np.sort(rng.choice(decoded, sample, replace=False))
        if l > 0 and adaptive:
            want = _oracle_adaptive_dec(case, b, R, decoded, idx, dbg, l, n_probe, seed)
        else:
            want = case.oracle_dec(OD.grid_points(R, idx), b)
        got = decs[l][idx].astype(np.float64)
        err = float(np.abs(got - want).max()) if idx.size else 0.0
        worst = max(worst, err)
        report[f"err_{l}"] = err
        assert err <= tol, f"level {l}: max abs dec error {err} > {tol}"
    report["worst"] = worst
    return report


def _oracle_adaptive_dec(case, b, R, decoded, idx, dbg, l, n_probe, seed):
    """Oracle raw decoder output at voxels ``idx`` of adaptive level ``l``:
    probes / small sub-volumes with full attention, the others over the GPU's
    Top-K subset of their sub-volume."""
    tiles = OA.tile_of(decoded, R, 8)
    tid_gpu = dbg["tile_ids"][l][b].cpu().numpy()
    sel_gpu = dbg["sel"][l][b].cpu().numpy()
    row = {int(t): n for n, t in enumerate(tid_gpu) if t >= 0}
    want = np.empty(idx.size)
    idx_tiles = OA.tile_of(idx, R, 8)
    pos = {int(v): n for n, v in enumerate(idx)}
    checked = [0]
    for t in np.unique(idx_tiles):
        members = np.sort(decoded[tiles == t])
        probe = OA.choose_probes(members, n_probe, seed, l)
        mine = idx[idx_tiles == t]
        is_probe = probe[np.searchsorted(members, mine)]
        dense_pts = mine[is_probe]
        if dense_pts.size:
            v = case.oracle_dec(OD.grid_points(R, dense_pts), b)
            for p_, x in zip(dense_pts, v):
                want[pos[int(p_)]] = x
        sparse_pts = mine[~is_probe]
        if sparse_pts.size:
            assert int(t) in row, f"tile {t} has no GPU selection"
            sel = sel_gpu[row[int(t)]]
            assert (sel >= 0).all() and np.all(np.diff(sel) > 0)
            if checked[0] < 16:   # the selection itself: the oracle's Top-K from the same probes
                K, _ = case.okv(b)
                q = OA.query_vectors(OD.grid_points(R, members[probe]), case.w)
                top = OA.top_k(OA.token_scores(q, K), sel.size)
                overlap = len(np.intersect1d(sel, top)) / sel.size
                assert overlap >= 0.9, f"tile {t}: Top-K overlap {overlap}"
                checked[0] += 1
            v = case.oracle_dec(OD.grid_points(R, sparse_pts), b, sel=sel)
            for p_, x in zip(sparse_pts, v):
                want[pos[int(p_)]] = x
    return want
