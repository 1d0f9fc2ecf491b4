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

    def oracle_dec(self, p: np.ndarray, b: int = 0, sel=None, want_attn: bool = False):
        K, V = self.okv(b)
        return OD.decode_points(p, K, V, self.w, self.spec.query_ln, sel=sel, return_attn=want_attn)

    def sp(self, b: int = 0):
        return None if self.spheres_np is None else self.spheres_np[b]


def unpack_words(words: np.ndarray, R: int) -> np.ndarray:
    """Blocked refine mask (one uint64 per 4^3 block) -> bool [R,R,R]."""
    nb = R // 4
    w = words.astype(np.uint64).reshape(nb, nb, nb)
    bits = ((w[..., None] >> np.arange(64, dtype=np.uint64)) & np.uint64(1)).astype(bool)
    bits = bits.reshape(nb, nb, nb, 4, 4, 4)           # (bi, bj, bk, di, dj, dk)
    return bits.transpose(0, 3, 1, 4, 2, 5).reshape(R, R, R)


def debug_buffers(B: int, r0: int, L: int, adaptive: bool, k: int, max_tiles: int,
                  n_probe: int = 0, N: int = 0, C: int = 0, attn_stride: int = 0):
    """Device buffers for ``vdm_hier_debug``; unwritten entries keep a sentinel
    (NaN, -1 or -2) so that a missing write shows."""
    import torch
    dbg = {"grid": [], "active": [], "dec": [], "tile_ids": [], "sel": [], "probes": [], "scores": [],
           "attn": [], "max_tiles": max_tiles, "attn_stride": attn_stride}
    for l in range(L):
        R = r0 << l
        dbg["grid"].append(torch.empty((B, R ** 3), device="cuda", dtype=torch.float32))
        dbg["dec"].append(torch.full((B, R ** 3), float("nan"), device="cuda", dtype=torch.float32))
        dbg["active"].append(torch.zeros((B, (R // 4) ** 3), device="cuda", dtype=torch.int64)
                             if l < L - 1 else None)
        if adaptive and l > 0:
            dbg["tile_ids"].append(torch.full((B, max_tiles), -1, device="cuda", dtype=torch.int32))
            dbg["sel"].append(torch.full((B, max_tiles, k), -1, device="cuda", dtype=torch.int32))
            dbg["probes"].append(torch.full((B, max_tiles, n_probe), -2, device="cuda", dtype=torch.int32)
                                 if n_probe else None)
            dbg["scores"].append(torch.full((B, max_tiles, N), float("nan"), device="cuda",
                                            dtype=torch.float32) if N else None)
        else:
            for key in ("tile_ids", "sel", "probes", "scores"):
                dbg[key].append(None)
        if attn_stride:
            rows = -(-R ** 3 // attn_stride)
            dbg["attn"].append(torch.full((B, rows, C), float("nan"), device="cuda", dtype=torch.float32))
        else:
            dbg["attn"].append(None)
    return dbg


def check_levels(case: Case, b: int, r0: int, L: int, dbg, dec_scale: float, adaptive: bool,
                 n_probe: int, seed: int, sample: int = 0, rng=None, report=None,
                 score_tiles: int = 16, attn_rows: int = 256):
    """Level-by-level parity of one shape's hierarchical decode.

    * refine masks bit-exact vs the oracle's mark+dilate of the GPU's own grid;
    * inherited voxels equal their parent's value exactly;
    * decoded voxels: raw decoder output within tolerance of the oracle at the
      same points (adaptive non-probes attend over the GPU's selection), and the
      stored field equals sphere SDF + scale tanh(dec) of the GPU's own dec;
    * adaptive levels (when the debug buffers hold them): the sub-volume list,
      every sub-volume's probe set and rank order exactly the oracle's
      (``choose_probes``), every selection exactly the oracle's Top-K rule on
      the GPU's own scores, and the scores of ``score_tiles`` sub-volumes within
      2e-2 * max of the oracle's ``token_scores``;
    * attention output (when exported): up to ``attn_rows`` sampled voxels per
      level within 2e-2 * max|a| of the oracle's.
    ``sample`` > 0 compares a random subset of the decoded voxels only.
    """
    tol = TOL[case.spec.dtype]
    rng = rng or np.random.default_rng(0)
    report = report if report is not None else {}
    grids = [dbg["grid"][l][b].cpu().numpy() for l in range(L)]
    decs = [dbg["dec"][l][b].cpu().numpy() for l in range(L)]
    stride = int(dbg.get("attn_stride", 0) or 0)
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
        ad = None
        if l > 0 and adaptive:
            ad = AdaptiveLevel(case, b, R, decoded, dbg, l, n_probe, seed)
            if dbg.get("probes") and dbg["probes"][l] is not None:
                report[f"probe_tiles_{l}"] = ad.check_probes()
            if dbg.get("scores") and dbg["scores"][l] is not None:
                report[f"topk_tiles_{l}"], report[f"score_err_{l}"] = ad.check_selection(score_tiles, rng)
            want = ad.oracle(idx)[0]
        else:
            want = case.oracle_dec(OD.grid_points(R, idx), b)
        got = decs[l][idx].astype(np.float64)
        err = float(np.abs(got - want).max()) if idx.size else 0.0
        worst = max(worst, err)
        report[f"err_{l}"] = err
        assert err <= tol, f"level {l}: max abs dec error {err} > {tol}"
        if stride and dbg["attn"][l] is not None:
            cand = decoded[decoded % stride == 0]
            if cand.size > attn_rows:
                cand = np.sort(rng.choice(cand, attn_rows, replace=False))
            if cand.size:
                a_gpu = dbg["attn"][l][b].cpu().numpy()[cand // stride].astype(np.float64)
                assert np.isfinite(a_gpu).all(), f"level {l}: attention rows not written"
                if ad is not None:
                    a_ref = ad.oracle(cand, want_attn=True)[1]
                else:
                    a_ref = case.oracle_dec(OD.grid_points(R, cand), b, want_attn=True)[1]
                aerr = float(np.abs(a_gpu - a_ref).max())
                scale = float(np.abs(a_ref).max())
                report[f"attn_err_{l}"] = aerr / scale
                assert aerr <= 2e-2 * scale, f"level {l}: attention error {aerr} > 2e-2 * {scale}"
    report["worst"] = worst
    return report


class AdaptiveLevel:
    """Oracle view of one adaptive level, built from the GPU's decoded set and
    debug exports: sub-volumes, probes (``choose_probes``), scores, Top-K."""

    def __init__(self, case, b, R, decoded, dbg, l, n_probe, seed):
        self.case, self.b, self.R, self.l = case, b, R, l
        self.n_probe, self.seed = n_probe, seed
        self.dbg = dbg
        self.tiles = OA.tile_of(decoded, R, 8)
        self.decoded = decoded
        self.tid_gpu = dbg["tile_ids"][l][b].cpu().numpy()
        self.sel_gpu = dbg["sel"][l][b].cpu().numpy()
        self.row = {int(t): n for n, t in enumerate(self.tid_gpu) if t >= 0}
        order = np.argsort(self.tiles, kind="stable")
        self._members = {}
        ts = self.tiles[order]
        bounds = np.flatnonzero(np.diff(ts)) + 1
        for grp in np.split(order, bounds):
            if grp.size:
                self._members[int(self.tiles[grp[0]])] = np.sort(decoded[grp])
        self._probe = {}

    def members(self, t):
        return self._members[int(t)]

    def probe_mask(self, t):
        if t not in self._probe:
            self._probe[t] = OA.choose_probes(self.members(t), self.n_probe, self.seed, self.l)
        return self._probe[t]

    def check_probes(self):
        """The sub-volume list and every probe set (in rank order) exactly the oracle's."""
        uniq = np.array(sorted(self._members))
        mt = self.tid_gpu.size
        assert np.array_equal(self.tid_gpu[:min(mt, uniq.size)], uniq[:mt]), \
            f"level {self.l}: sub-volume list differs"
        pr = self.dbg["probes"][self.l][self.b].cpu().numpy()
        n = min(mt, uniq.size)
        for i in range(n):
            t = int(uniq[i])
            mem = self.members(t)
            nd = min(mem.size, self.n_probe)
            got = pr[i, :nd]
            assert np.all(pr[i, nd:] == -1), f"level {self.l} sub-volume {t}: probe padding"
            if mem.size <= self.n_probe:
                assert np.array_equal(np.sort(got), mem), f"level {self.l} sub-volume {t}: dense set"
            else:
                key = OA.probe_key(self.seed, self.l, mem)
                want = mem[np.lexsort((mem, key))[:self.n_probe]]
                assert np.array_equal(got, want), f"level {self.l} sub-volume {t}: probes differ"
        return n

    def check_selection(self, score_tiles, rng):
        """Every selection = Top-K rule on the GPU's scores; sampled scores vs oracle."""
        sc = self.dbg["scores"][self.l][self.b].cpu().numpy()
        K, _ = self.case.okv(self.b)
        H = K.shape[0]
        sel_rows = [i for i, t in enumerate(self.tid_gpu) if t >= 0 and
                    self.members(int(t)).size > self.n_probe]
        k = self.sel_gpu.shape[1]
        for i in sel_rows:
            s = sc[i].astype(np.float64)
            assert np.isfinite(s).all(), f"level {self.l} row {i}: scores not written"
            assert np.array_equal(self.sel_gpu[i], OA.top_k(s, k)), \
                f"level {self.l} sub-volume {self.tid_gpu[i]}: selection is not the Top-K of its scores"
            assert abs(s.sum() - self.n_probe * H) <= 2e-3 * self.n_probe * H
        pick = sel_rows if len(sel_rows) <= score_tiles else \
            sorted(rng.choice(sel_rows, score_tiles, replace=False))
        worst = 0.0
        for i in pick:
            t = int(self.tid_gpu[i])
            mem = self.members(t)
            q = OA.query_vectors(OD.grid_points(self.R, mem[self.probe_mask(t)]), self.case.w)
            want = OA.token_scores(q, K)
            err = float(np.abs(sc[i] - want).max())
            worst = max(worst, err / max(1.0, want.max()))
            assert err <= 2e-2 * max(1.0, want.max()), \
                f"level {self.l} sub-volume {t}: score error {err}"
        return len(sel_rows), worst

    def oracle(self, idx, want_attn=False):
        """Oracle raw decoder output (and attention output) at voxels ``idx``:
        probes / small sub-volumes with full attention, the others over the
        GPU's Top-K subset of their sub-volume."""
        C = self.case.spec.C
        want = np.empty(idx.size)
        attn = np.empty((idx.size, C)) if want_attn else None
        idx_tiles = OA.tile_of(idx, self.R, 8)
        for t in np.unique(idx_tiles):
            mem = self.members(t)
            probe = self.probe_mask(int(t))
            here = np.flatnonzero(idx_tiles == t)
            mine = idx[here]
            is_probe = probe[np.searchsorted(mem, mine)]
            for sub, sel in ((here[is_probe], None), (here[~is_probe], "gpu")):
                if sub.size == 0:
                    continue
                if sel == "gpu":
                    assert int(t) in self.row, f"tile {t} has no GPU selection"
                    sel = self.sel_gpu[self.row[int(t)]]
                    assert (sel >= 0).all() and np.all(np.diff(sel) > 0)
                r = self.case.oracle_dec(OD.grid_points(self.R, idx[sub]), self.b, sel=sel,
                                         want_attn=want_attn)
                if want_attn:
                    want[sub], attn[sub] = r
                else:
                    want[sub] = r
        return want, attn
