"""GPU parity of the local (MSVS-style) decoder query (vdm_decode_local): the
neighbour sets bit-exact against the oracle's rule (index work), and the SDF
within the fp32 tolerance of the oracle's AVS-Conv and multi-scale fusion."""
import numpy as np
import pytest

import workloads as W
from oracle import local as OL

pytestmark = pytest.mark.gpu


def _points(n, rng):
    # uniform points, points right next to anchors, and points outside the unit cube
    return rng.uniform(-1.0, 1.0, (n, 3)).astype(np.float32)


@pytest.mark.parametrize("K,n_anchors,channels", [(8, (512, 2048), (64, 32)), (3, (40, 300), (16, 8)),
                                                  (16, (2048,), (32,))])
def test_local_decoder_matches_oracle(K, n_anchors, channels):
    import torch
    import neural_sdf_volume_b200 as vdm
    sp = W.make_spheres(6, seed=0, key=51)[0]
    d = W.make_local_decoder(sp, n_anchors=n_anchors, channels=channels, seed=0, key=52)
    ld = vdm.LocalDecoder.from_numpy(d, K)
    rng = np.random.default_rng(K)
    near = d["anchors"][0][rng.choice(n_anchors[0], 64)] + rng.normal(0, 1e-3, (64, 3)).astype(np.float32)
    outside = rng.uniform(-1.6, 1.6, (64, 3)).astype(np.float32)
    x = np.concatenate([_points(700, rng), near.astype(np.float32), outside])
    out, knn = vdm.vdm_decode_local(ld, torch.from_numpy(x).cuda(), want_knn=True)
    out = out.cpu().numpy()
    knn = knn.cpu().numpy()
    for s, a in enumerate(d["anchors"]):
        assert np.array_equal(knn[:, s, :], OL.knn(x, a, K)), f"scale {s}: neighbour sets differ"
    want = OL.decode_local(x, d["anchors"], d["feats"], d["scales"], d["fuse"], K)
    assert np.abs(out - want).max() <= 1e-4 * max(1.0, np.abs(want).max())


def test_local_decoder_empty_and_errors():
    import torch
    import neural_sdf_volume_b200 as vdm
    sp = W.make_spheres(2, seed=0, key=53)[0]
    d = W.make_local_decoder(sp, n_anchors=(64,), channels=(8,), seed=0, key=53)
    ld = vdm.LocalDecoder.from_numpy(d, 4)
    assert vdm.vdm_decode_local(ld, torch.zeros((0, 3), device="cuda")).shape == (0,)
    ld.cs.K = 65
    with pytest.raises(vdm.VdmError) as ei:
        vdm.vdm_decode_local(ld, torch.zeros((4, 3), device="cuda"))
    assert ei.value.status == 2


def test_local_decoder_several_chunks():
    """More queries than one chunk of the neighbour buffer (262,144), with and
    without the neighbour export: sampled rows against the oracle, and the
    two calls' SDF values identical."""
    import torch
    import neural_sdf_volume_b200 as vdm
    sp = W.make_spheres(6, seed=0, key=54)[0]
    d = W.make_local_decoder(sp, n_anchors=(1024, 4096), channels=(32, 16), seed=0, key=55)
    K = 8
    ld = vdm.LocalDecoder.from_numpy(d, K)
    rng = np.random.default_rng(7)
    x = rng.uniform(-1.0, 1.0, (300_000, 3)).astype(np.float32)
    xt = torch.from_numpy(x).cuda()
    out, knn = vdm.vdm_decode_local(ld, xt, want_knn=True)
    out2 = vdm.vdm_decode_local(ld, xt)
    out, out2, knn = out.cpu().numpy(), out2.cpu().numpy(), knn.cpu().numpy()
    assert np.array_equal(out, out2)
    rows = np.concatenate([rng.choice(x.shape[0], 600, replace=False), [0, 262_143, 262_144, x.shape[0] - 1]])
    for s, a in enumerate(d["anchors"]):
        assert np.array_equal(knn[rows, s, :], OL.knn(x[rows], a, K)), f"scale {s}"
    want = OL.decode_local(x[rows], d["anchors"], d["feats"], d["scales"], d["fuse"], K)
    assert np.abs(out[rows] - want).max() <= 1e-4 * max(1.0, np.abs(want).max())
