"""GPU parity of K/V projection and dense decoding against the CPU oracle.

Tolerances: max abs error of the raw decoder output <= 1e-4 for float32
decoders and <= 2e-2 for bf16 decoders."""
import numpy as np
import pytest

import workloads as W
from oracle import decoder as OD

from gpu_cases import TOL, Case

pytestmark = pytest.mark.gpu


def test_kv_projection_matches_oracle():
    import torch
    for dt, tol in (("f32", 1e-5), ("bf16", None)):
        spec = W.DecoderSpec(C=128, H=2, F=128, N=77, query_ln=True, dtype=dt)
        c = Case(spec, key=11, stress=True)
        K, V = c.okv()
        Kg = c.K[0].float().cpu().numpy()
        Vg = c.V[0].float().cpu().numpy()
        if tol is None:   # bf16 storage: one rounding of a value of magnitude <= ~4
            np.testing.assert_allclose(Kg, K, rtol=2 ** -8, atol=1e-3)
            np.testing.assert_allclose(Vg, V, rtol=2 ** -8, atol=1e-3)
        else:
            np.testing.assert_allclose(Kg, K, atol=tol)
            np.testing.assert_allclose(Vg, V, atol=tol)


def test_tiny_fp32_config_full_grid():
    """32^3 grid, N=256, C=64, float32: every voxel within 1e-4 of the oracle."""
    import neural_sdf_volume_b200 as vdm
    cfg = W.CONFIGS[1]
    c = Case(cfg.dec, key=cfg.seed_key)
    out = vdm.vdm_decode_dense(c.dec, c.K, c.V, grid_R=32)[0].cpu().numpy()
    want = c.oracle_dec(OD.grid_points(32))
    err = np.abs(out - want).max()
    assert err <= 1e-4, err


@pytest.mark.parametrize("dtype,C,H,F,N", [("f32", 64, 1, 256, 256), ("f32", 256, 4, 512, 300),
                                           ("bf16", 512, 8, 2048, 200), ("bf16", 256, 4, 512, 129)])
@pytest.mark.parametrize("stress", [False, True])
def test_points_mode_ragged(dtype, C, H, F, N, stress):
    """Random points, M not a multiple of the query tile, N not a multiple of
    the token block; the stress weights give attention logits of order 5."""
    import torch
    import neural_sdf_volume_b200 as vdm
    spec = W.DecoderSpec(C=C, H=H, F=F, N=N, query_ln=C != 256, dtype=dtype)
    c = Case(spec, key=20 + C, stress=stress)
    M = 333
    pts = W.make_points(M, seed=1, key=C)
    out = vdm.vdm_decode_dense(c.dec, c.K, c.V, xyz=torch.from_numpy(pts).cuda())[0].cpu().numpy()
    want = c.oracle_dec(pts[0])
    err = np.abs(out - want).max()
    assert err <= TOL[dtype], err


def test_batched_shapes_and_analytic_term():
    import torch
    import neural_sdf_volume_b200 as vdm
    spec = W.DecoderSpec(C=256, H=4, F=512, N=96, query_ln=False, dtype="bf16")
    c = Case(spec, key=5, B=3, n_spheres=5, sphere_key=5)
    R = 10
    out = vdm.vdm_decode_dense(c.dec, c.K, c.V, grid_R=R, spheres=c.spheres, dec_scale=0.01).cpu().numpy()
    raw = vdm.vdm_decode_dense(c.dec, c.K, c.V, grid_R=R).cpu().numpy()
    p = OD.grid_points(R)
    for b in range(3):
        want = c.oracle_dec(p, b)
        assert np.abs(raw[b] - want).max() <= 2e-2
        fld = OD.field(p, raw[b].astype(np.float64), c.sp(b), 0.01)
        assert np.abs(out[b] - fld).max() < 1e-6


def test_empty_and_single_query():
    import torch
    import neural_sdf_volume_b200 as vdm
    spec = W.DecoderSpec(C=64, H=1, F=64, N=1, query_ln=True, dtype="f32")
    c = Case(spec, key=9, stress=True)
    out = vdm.vdm_decode_dense(c.dec, c.K, c.V, xyz=torch.zeros((1, 0, 3), device="cuda"))
    assert out.shape == (1, 0)
    pts = np.array([[[0.1, -0.2, 0.3]]], np.float32)
    got = vdm.vdm_decode_dense(c.dec, c.K, c.V, xyz=torch.from_numpy(pts).cuda())[0].cpu().numpy()
    assert abs(got[0] - c.oracle_dec(pts[0])[0]) <= 1e-4


def test_dense_decode_is_deterministic():
    import neural_sdf_volume_b200 as vdm
    spec = W.DecoderSpec(C=512, H=8, F=2048, N=150, query_ln=True, dtype="bf16")
    c = Case(spec, key=2)
    a = vdm.vdm_decode_dense(c.dec, c.K, c.V, grid_R=9).cpu().numpy()
    b = vdm.vdm_decode_dense(c.dec, c.K, c.V, grid_R=9).cpu().numpy()
    assert np.array_equal(a, b)


def test_full_size_dense_bf16_sampled():
    """The dense bf16 workload at full size (N=3072, C=512, 8 heads, 128^3
    points); 1024 voxels drawn at random are compared with the oracle."""
    import neural_sdf_volume_b200 as vdm
    cfg = W.CONFIGS[2]
    c = Case(cfg.dec, key=cfg.seed_key)
    out = vdm.vdm_decode_dense(c.dec, c.K, c.V, grid_R=128)[0].cpu().numpy()
    assert np.isfinite(out).all()
    idx = np.sort(np.random.default_rng(0).choice(128 ** 3, 1024, replace=False))
    want = c.oracle_dec(OD.grid_points(128, idx))
    err = np.abs(out[idx] - want).max()
    assert err <= 2e-2, err
