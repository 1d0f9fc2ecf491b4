"""GPU parity of vdm_compare_volumes (V-IoU counts, sign agreement, largest
difference) against the oracle's plain definition: integer counts bit-exact."""
import numpy as np
import pytest

from oracle import volume as OV

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,offset", [(1_000_003, 0), (1_000_003, 1), (7, 0), (0, 0), (384 ** 3, 0)])
def test_compare_volumes_matches_oracle(n, offset):
    import torch
    import neural_sdf_volume_b200 as vdm
    rng = np.random.default_rng(n + offset)
    a = rng.standard_normal(n + offset).astype(np.float32)
    b = (a + rng.standard_normal(n + offset).astype(np.float32) * 0.3).astype(np.float32)
    if n > 10:   # exact zeros of both signs count as outside
        a[offset:offset + 5] = 0.0
        b[offset + 3:offset + 8] = -0.0
    ta = torch.from_numpy(a).cuda()[offset:]
    tb = torch.from_numpy(b).cuda()[offset:]
    got = vdm.vdm_compare_volumes(ta, tb)
    want = OV.compare_volumes(a[offset:], b[offset:])
    for k in ("inside_a", "inside_b", "inside_both", "same_sign"):
        assert got[k] == want[k], k
    assert got["max_abs_diff"] == want["max_abs_diff"]
    assert got["v_iou"] == want["v_iou"]
