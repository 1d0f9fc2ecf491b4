"""GPU parity of hierarchical volume decoding and adaptive KV selection.

Small cases run the whole oracle procedure and compare every level; the full
workloads (96->192->384 dense and adaptive, 4 x 128->256->512 slim adaptive)
are checked level by level on sampled decoded voxels plus bit-exact refine
masks and exact inheritance."""
import numpy as np
import pytest

import workloads as W
from oracle import adaptive as OA
from oracle import decoder as OD
from oracle import volume as OV

from gpu_cases import TOL, Case, check_levels, debug_buffers

pytestmark = pytest.mark.gpu


def _run(case, B, r0, L, adaptive, n_probe=64, top_k=1024, seed=0, dec_scale=0.01, max_tiles=0,
         attn_stride=0, exports=True):
    import neural_sdf_volume_b200 as vdm
    p = vdm.hier_params(r0, L, adaptive, 8, n_probe, top_k, seed)
    k = min(top_k, case.spec.N)
    mt = max_tiles or (r0 << (L - 1)) // 8
    mt = mt ** 3 if not max_tiles else max_tiles
    dbg = debug_buffers(B, r0, L, adaptive, k, mt, n_probe=n_probe if exports else 0,
                        N=case.spec.N if exports else 0, C=case.spec.C, attn_stride=attn_stride)
    grid, stats = vdm.vdm_decode_hierarchical(case.dec, case.K, case.V, p, case.spheres, dec_scale,
                                              debug=dbg)
    return grid, stats, dbg


def _analytic_sign_agreement(grid, spheres, Rf, margin=0.011, chunk=1 << 20):
    """Share of the voxels with |sphere SDF| > margin whose final value has the
    sphere SDF's sign: there field = sphere SDF + 0.01 tanh(dec) cannot change
    sign, whatever the decoder says.  Returns (agreeing, counted)."""
    g = grid.reshape(-1)
    agree = counted = 0
    for s0 in range(0, Rf ** 3, chunk):
        idx = np.arange(s0, min(s0 + chunk, Rf ** 3))
        sd = OD.sphere_sdf(OD.grid_points(Rf, idx), spheres)
        m = np.abs(sd) > margin
        agree += int(((g[idx][m] < 0) == (sd[m] < 0)).sum())
        counted += int(m.sum())
    return agree, counted


@pytest.mark.parametrize("stress", [False, True])
@pytest.mark.parametrize("adaptive,n_probe", [(False, 16), (True, 16), (True, 32), (True, 64)])
def test_small_hierarchical_matches_full_oracle(adaptive, n_probe, stress):
    """12 -> 24 -> 48 with the full-width bf16 decoder (N=256, C=512): every
    level checked (probe sets and Top-K exact, attention output at sampled
    voxels), then the final sign compared with the oracle's own run.  16 probes
    per sub-volume score on CUDA cores, 32 and 64 on the tensor cores.  The
    stress weights give attention logits of order 5 and a value bias, so a
    wrong gathered row or a wrong softmax shows in the output."""
    spec = W.DecoderSpec(C=512, H=8, F=2048, N=256, query_ln=True, dtype="bf16")
    case = Case(spec, key=2, n_spheres=5, sphere_key=3, stress=stress)
    grid, stats, dbg = _run(case, 1, 12, 3, adaptive, n_probe=n_probe, top_k=64, attn_stride=7)
    rep = check_levels(case, 0, 12, 3, dbg, 0.01, adaptive, n_probe, 0, score_tiles=64,
                       attn_rows=400)
    if adaptive:   # the exact checks ran on some sub-volumes
        assert rep["probe_tiles_1"] > 0 and rep["probe_tiles_2"] > 0
        assert rep["topk_tiles_1"] + rep["topk_tiles_2"] > 0
    assert stats[0]["decoded"][0] == 12 ** 3
    assert stats[0]["decoded"][1] == rep["decoded_1"] and stats[0]["decoded"][2] == rep["decoded_2"]
    K, V = case.okv()
    ref = OV.hierarchical_volume(K, V, case.w, 12, 3, True, case.sp(), 0.01, adaptive=adaptive,
                                 seed=0, n_probe=n_probe, top_k=64)
    g = grid[0].cpu().numpy()
    agree = float(((g < 0) == (ref["grid"] < 0)).mean())
    assert agree >= 0.9999, agree


def test_fp32_hierarchical_exact_sdf_closed_form():
    """dec_scale = 0: the field is the exact sphere SDF, so every decoded voxel
    equals the analytic value and the hierarchical sign equals the dense sign
    everywhere (1-Lipschitz argument)."""
    import torch
    spec = W.DecoderSpec(C=64, H=1, F=256, N=64, query_ln=True, dtype="f32")
    case = Case(spec, key=1, n_spheres=6, sphere_key=7)
    grid, stats, dbg = _run(case, 1, 8, 4, False, dec_scale=0.0)
    Rf = 64
    dense = OD.sphere_sdf(OD.grid_points(Rf), case.sp()).reshape(Rf, Rf, Rf)
    g = grid[0].cpu().numpy()
    assert np.array_equal(g < 0, dense < 0)
    d3 = dbg["dec"][3][0].cpu().numpy()
    dec_vox = np.flatnonzero(np.isfinite(d3))
    assert np.abs(g.ravel()[dec_vox] - dense.ravel()[dec_vox]).max() < 2e-6
    assert stats[0]["decoded"][3] < 0.6 * Rf ** 3


def test_adaptive_k_equal_n_is_dense_decode():
    """top_k = N: the adaptive path must give the dense path's values."""
    spec = W.DecoderSpec(C=256, H=4, F=512, N=96, query_ln=False, dtype="bf16")
    case = Case(spec, key=4, n_spheres=4, sphere_key=4)
    g1, s1, d1 = _run(case, 1, 8, 3, False)
    g2, s2, d2 = _run(case, 1, 8, 3, True, n_probe=8, top_k=96)
    a = d1["dec"][2][0].cpu().numpy()
    b = d2["dec"][2][0].cpu().numpy()
    m = np.isfinite(a)
    assert np.array_equal(m, np.isfinite(b))
    assert np.abs(a[m] - b[m]).max() <= 2e-3


@pytest.mark.parametrize("cid", [3, 4])
def test_full_size_96_to_384(cid):
    """Full workloads 3 and 4: masks bit-exact, sampled decoded voxels and
    attention rows within tolerance, (4) every sub-volume's probes and Top-K
    exact and 32 sub-volumes' scores within tolerance per level, and the final
    sign equal to the analytic sign on >= 99.99 % of the voxels whose sign the
    decoder term cannot change."""
    cfg = W.CONFIGS[cid]
    case = Case(cfg.dec, key=cfg.seed_key, n_spheres=cfg.n_spheres, sphere_key=cfg.sphere_key)
    grid, stats, dbg = _run(case, 1, cfg.r0, cfg.n_levels, cfg.adaptive, cfg.n_probe, cfg.top_k,
                            dec_scale=cfg.dec_scale, max_tiles=16384, attn_stride=4099)
    rep = check_levels(case, 0, cfg.r0, cfg.n_levels, dbg, cfg.dec_scale, cfg.adaptive,
                       cfg.n_probe, 0, sample=256, score_tiles=32, attn_rows=64)
    n_dec = sum(stats[0]["decoded"][:3])
    saved = 1.0 - n_dec / 384 ** 3
    agree, counted = _analytic_sign_agreement(grid[0].cpu().numpy(), case.sp(), 384)
    print(f"config {cid}: decoded per level {stats[0]['decoded'][:3]}, queries saved {saved:.3f}, "
          f"sign agreement {agree}/{counted}, {rep}")
    assert saved > 0.8
    assert agree >= 0.9999 * counted


def test_full_size_batched_slim_adaptive():
    cfg = W.CONFIGS[5]
    case = Case(cfg.dec, key=cfg.seed_key, B=cfg.B, n_spheres=cfg.n_spheres, sphere_key=cfg.sphere_key)
    grid, stats, dbg = _run(case, cfg.B, cfg.r0, cfg.n_levels, True, cfg.n_probe, cfg.top_k,
                            dec_scale=cfg.dec_scale, max_tiles=40000, attn_stride=8191)
    for b in (0, 3):
        assert stats[b]["tiles"][2] <= 40000
        check_levels(case, b, cfg.r0, cfg.n_levels, dbg, cfg.dec_scale, True, cfg.n_probe, 0,
                     sample=128, rng=np.random.default_rng(b), score_tiles=16, attn_rows=64)
        agree, counted = _analytic_sign_agreement(grid[b].cpu().numpy(), case.sp(b), 512)
        assert agree >= 0.9999 * counted, (b, agree, counted)


def test_select_kv_scores_and_topk_given_the_same_scores():
    """vdm_select_kv with a sub-volume of 130 probes (more than the tensor-core
    route's 128 rows, so the CUDA-core route): scores within tolerance of the
    oracle's; the selection is exactly the oracle's Top-K rule applied to the
    GPU's own scores."""
    import torch
    import neural_sdf_volume_b200 as vdm
    spec = W.DecoderSpec(C=512, H=8, F=2048, N=700, query_ln=True, dtype="bf16")
    case = Case(spec, key=2, stress=True)
    counts = [0, 1, 64, 65, 130]
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    pts = W.make_points(int(off[-1]), seed=3, key=3)[0]
    k = 100
    sel, score, pdec = vdm.vdm_select_kv(case.dec, case.K, case.V, torch.from_numpy(pts).cuda(),
                                         torch.from_numpy(off).cuda(), k, want_scores=True, want_probe_dec=True)
    sel = sel.cpu().numpy()
    score = score.cpu().numpy().astype(np.float64)
    # the probes' decoded values (full attention)
    assert np.abs(pdec.cpu().numpy() - case.oracle_dec(pts)).max() <= TOL["bf16"]
    K, V = case.okv()
    for t in range(len(counts)):
        assert np.array_equal(sel[t], OA.top_k(score[t], k)), f"tile {t}"
        if counts[t] == 0:
            assert np.array_equal(sel[t], np.arange(k))
            continue
        q = OA.query_vectors(pts[off[t]:off[t + 1]], case.w)
        want = OA.token_scores(q, K)
        # scores sum to probes x heads; bf16 K and weights give ~1% relative error
        assert abs(score[t].sum() - counts[t] * 8) < 1e-3 * counts[t] * 8
        assert np.abs(score[t] - want).max() <= 2e-2 * max(1.0, want.max())
        overlap = len(np.intersect1d(sel[t], OA.top_k(want, k))) / k
        assert overlap >= 0.9, overlap


def test_select_kv_tensor_core_route_scores_and_topk():
    """vdm_select_kv with at most 128 probes per sub-volume (the tensor-core
    route, ragged counts including 0 and a full 128): scores within tolerance
    of the oracle's, the selection exactly the Top-K rule on the GPU's scores."""
    import torch
    import neural_sdf_volume_b200 as vdm
    spec = W.DecoderSpec(C=512, H=8, F=2048, N=700, query_ln=True, dtype="bf16")
    case = Case(spec, key=2, stress=True)
    counts = [0, 1, 31, 64, 100, 128, 0, 17]
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    pts = W.make_points(int(off[-1]), seed=5, key=3)[0]
    k = 100
    sel, score, pdec = vdm.vdm_select_kv(case.dec, case.K, case.V, torch.from_numpy(pts).cuda(),
                                         torch.from_numpy(off).cuda(), k, want_scores=True, want_probe_dec=True)
    sel = sel.cpu().numpy()
    score = score.cpu().numpy().astype(np.float64)
    assert np.abs(pdec.cpu().numpy() - case.oracle_dec(pts)).max() <= TOL["bf16"]
    K, V = case.okv()
    for t in range(len(counts)):
        assert np.array_equal(sel[t], OA.top_k(score[t], k)), f"tile {t}"
        if counts[t] == 0:
            assert np.array_equal(sel[t], np.arange(k))
            assert not score[t].any()
            continue
        want = OA.token_scores(OA.query_vectors(pts[off[t]:off[t + 1]], case.w), K)
        assert abs(score[t].sum() - counts[t] * 8) < 1e-3 * counts[t] * 8
        assert np.abs(score[t] - want).max() <= 2e-2 * max(1.0, want.max())


def test_select_kv_reproduces_the_hierarchical_selection():
    """The public selection call run on a hierarchical level's own probes (as
    points, in rank order) gives that level's scores and kept tokens bit for
    bit: both run the same tensor-core kernels."""
    import torch
    import neural_sdf_volume_b200 as vdm
    spec = W.DecoderSpec(C=512, H=8, F=2048, N=256, query_ln=True, dtype="bf16")
    case = Case(spec, key=2, n_spheres=5, sphere_key=3, stress=True)
    n_probe, k = 64, 64
    grid, stats, dbg = _run(case, 1, 12, 3, True, n_probe=n_probe, top_k=k)
    checked = 0
    for l in (1, 2):
        R = 12 << l
        sel_h = dbg["sel"][l][0].cpu().numpy()
        # sub-volume i holds 8 children per refined parent of its 4^3 parent block (one mask word);
        # those with more queries than probes were scored
        tiles = dbg["tile_ids"][l][0].cpu().numpy()
        tiles = tiles[tiles >= 0]
        words = dbg["active"][l - 1][0].cpu().numpy().view(np.uint64)[tiles]
        n_q = 8 * np.array([bin(int(w)).count("1") for w in words])
        rows = np.flatnonzero(n_q > n_probe)
        if rows.size == 0:
            continue
        vox = dbg["probes"][l][0].cpu().numpy()[rows].astype(np.int64)
        assert (vox >= 0).all()
        ijk = np.stack([vox // (R * R), (vox // R) % R, vox % R], axis=-1).reshape(-1, 3)
        xyz = (np.float32(-1.0) + (2 * ijk + 1).astype(np.float32) / np.float32(R)).astype(np.float32)
        off = (np.arange(rows.size + 1) * n_probe).astype(np.int32)
        sel, score = vdm.vdm_select_kv(case.dec, case.K, case.V, torch.from_numpy(xyz).cuda(),
                                       torch.from_numpy(off).cuda(), k, want_scores=True)
        assert np.array_equal(sel.cpu().numpy(), sel_h[rows]), l
        assert np.array_equal(score.cpu().numpy(), dbg["scores"][l][0].cpu().numpy()[rows]), l
        checked += rows.size
    assert checked > 0
