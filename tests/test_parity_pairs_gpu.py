"""GPU parity of tensor-core decoding on CTA pairs (vdm_set_cta_pairs(1)):
each 256-row MMA spans the two CTAs of a cluster, each CTA holding half of
every weight / key / value tile.  Same tolerances as the single-CTA path, and
the two paths agree to within float32 summation-order differences."""
import numpy as np
import pytest

import workloads as W
from oracle import volume as OV

from gpu_cases import TOL, Case, check_levels, debug_buffers

pytestmark = pytest.mark.gpu


def _pairs(on: bool):
    import neural_sdf_volume_b200 as vdm
    vdm.vdm_set_cta_pairs(on)


@pytest.mark.parametrize("C,H,F,N", [(512, 8, 2048, 200), (256, 4, 512, 129), (128, 2, 256, 300)])
@pytest.mark.parametrize("stress", [False, True])
def test_pairs_points_mode_ragged(C, H, F, N, stress):
    """M = 333 random points: three 128-query units, so the second CTA pair has
    one empty half; N not a multiple of the 128-token block."""
    import torch
    import neural_sdf_volume_b200 as vdm
    spec = W.DecoderSpec(C=C, H=H, F=F, N=N, query_ln=C != 256, dtype="bf16")
    c = Case(spec, key=40 + C, stress=stress)
    pts = torch.from_numpy(W.make_points(333, seed=2, key=C)).cuda()
    try:
        _pairs(True)
        got = vdm.vdm_decode_dense(c.dec, c.K, c.V, xyz=pts)[0].cpu().numpy()
    finally:
        _pairs(False)
    single = vdm.vdm_decode_dense(c.dec, c.K, c.V, xyz=pts)[0].cpu().numpy()
    want = c.oracle_dec(pts[0].cpu().numpy())
    assert np.abs(got - want).max() <= TOL["bf16"]
    assert np.abs(got - single).max() <= 1e-4


def test_pairs_grid_mode_full_width():
    """A 24^3 grid with the full-width decoder (N=3072): 108 units, 54 pairs."""
    import neural_sdf_volume_b200 as vdm
    spec = W.DecoderSpec(C=512, H=8, F=2048, N=3072, query_ln=True, dtype="bf16")
    c = Case(spec, key=2)
    try:
        _pairs(True)
        got = vdm.vdm_decode_dense(c.dec, c.K, c.V, grid_R=24)[0].cpu().numpy().reshape(-1)
    finally:
        _pairs(False)
    rng = np.random.default_rng(5)
    idx = rng.choice(24 ** 3, 300, replace=False)
    from oracle import decoder as OD
    want = c.oracle_dec(OD.grid_points(24, idx))
    assert np.abs(got[idx] - want).max() <= TOL["bf16"]


@pytest.mark.parametrize("stress", [False, True])
def test_pairs_small_hierarchical_adaptive_levels(stress):
    """12 -> 24 -> 48 with adaptive KV on CTA pairs: the sparse pass pairs two
    query slots of one sub-volume (gathered keys split by token, values by head
    dimension); every level is checked against the oracle, probes and Top-K
    exactly, attention output at sampled voxels."""
    import neural_sdf_volume_b200 as vdm
    spec = W.DecoderSpec(C=512, H=8, F=2048, N=256, query_ln=True, dtype="bf16")
    case = Case(spec, key=2, n_spheres=5, sphere_key=3, stress=stress)
    p = vdm.hier_params(12, 3, True, 8, 32, 64, 0)
    dbg = debug_buffers(1, 12, 3, True, 64, 6 ** 3, n_probe=32, N=256, C=512, attn_stride=7)
    try:
        _pairs(True)
        grid, stats = vdm.vdm_decode_hierarchical(case.dec, case.K, case.V, p, case.spheres, 0.01, debug=dbg)
    finally:
        _pairs(False)
    rep = check_levels(case, 0, 12, 3, dbg, 0.01, True, 32, 0, score_tiles=64, attn_rows=400)
    assert stats[0]["decoded"][1] == rep["decoded_1"] and stats[0]["decoded"][2] == rep["decoded_2"]
    K, V = case.okv()
    ref = OV.hierarchical_volume(K, V, case.w, 12, 3, True, case.sp(), 0.01, adaptive=True,
                                 seed=0, n_probe=32, top_k=64)
    agree = float(((grid[0].cpu().numpy() < 0) == (ref["grid"] < 0)).mean())
    assert agree >= 0.9999, agree
