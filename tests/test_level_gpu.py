"""GPU parity of one level step without the decoder (vdm_refine_level):
refine mask bit-exact against the oracle's marking and dilation, the refined
voxel list and counts exact (index work), and the inherited fine grid equal to
its parents' values bit for bit."""
import numpy as np
import pytest

import workloads as W
from oracle import decoder as OD
from oracle import hierarchy as OH

from gpu_cases import unpack_words

pytestmark = pytest.mark.gpu


def _fields():
    R = 64
    sp = W.make_spheres(7, seed=0, key=12)[0]
    yield "spheres", OD.sphere_sdf(OD.grid_points(R), sp).reshape(R, R, R).astype(np.float32)
    rng = np.random.default_rng(4)
    f = rng.standard_normal((40, 40, 40)).astype(np.float32)
    f[rng.random(f.shape) < 0.7] = 0.5       # sparse sign changes, some near-threshold values
    f[rng.random(f.shape) < 0.02] = 0.0
    yield "noise", f
    yield "outside", np.full((16, 16, 16), 2.0, np.float32)
    g = np.full((8, 8, 8), 2.0, np.float32)
    g[0, 0, 0] = -1.0                         # a corner voxel: clipping at the border
    yield "corner", g


@pytest.mark.parametrize("name,f", list(_fields()))
def test_refine_level_matches_oracle(name, f):
    import torch
    import neural_sdf_volume_b200 as vdm
    R = f.shape[0]
    tf = torch.from_numpy(f).cuda()
    fine = torch.full((2 * R,) * 3, float("nan"), device="cuda")
    parents = torch.full((R ** 3,), -1, device="cuda", dtype=torch.int32)
    mask, counts = vdm.vdm_refine_level(tf, fine=fine, parents=parents)
    act = OH.dilate(OH.mark(f, OH.near_threshold(R)))
    got = unpack_words(mask.cpu().numpy().view(np.uint64), R)
    assert np.array_equal(got, act), name
    n = int(act.sum())
    c = counts.cpu().numpy()
    assert c[0] == n
    nb = R // 4
    blocks = act.reshape(nb, 4, nb, 4, nb, 4).any(axis=(1, 3, 5))
    assert c[1] == int(blocks.sum())
    pl = parents.cpu().numpy()[:n].astype(np.int64)
    assert np.array_equal(np.sort(pl), OH.compact(act))
    # grouped by 4^3 block in block order, ascending bit order inside a block
    i, rem = np.divmod(pl, R * R)
    j, k = np.divmod(rem, R)
    word = ((i // 4) * nb + j // 4) * nb + k // 4
    bit = ((i % 4) * 4 + j % 4) * 4 + k % 4
    assert np.array_equal(np.lexsort((bit, word)), np.arange(n))
    want = np.repeat(np.repeat(np.repeat(f, 2, 0), 2, 1), 2, 2)
    assert np.array_equal(fine.cpu().numpy(), want)
