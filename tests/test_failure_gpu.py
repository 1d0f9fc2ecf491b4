"""Failure detection without a GPU fault: a withheld completion signal makes
the tensor-core decoder's bounded waits expire; the call that made the launch
reports VDM_ERR_TIMEOUT and the CUDA context stays usable (later calls decode
bit-identically)."""
import numpy as np
import pytest

import workloads as W

from gpu_cases import Case

pytestmark = pytest.mark.gpu

SHORT_WAIT = 20_000_000          # cycles, ~10 ms per wait


def _case():
    spec = W.DecoderSpec(C=256, H=4, F=512, N=128, query_ln=False, dtype="bf16")
    return Case(spec, key=8, n_spheres=3, sphere_key=8)


def _expect_timeout(fn):
    import neural_sdf_volume_b200 as vdm
    with pytest.raises(vdm.VdmError) as ei:
        fn()
    assert ei.value.status == 5, str(ei.value)
    assert "bounded wait" in str(ei.value)


@pytest.mark.parametrize("launch", [1, 2])
def test_withheld_signal_times_out_and_context_survives(launch):
    """Two levels, two decode launches: the withheld signal in the first (the
    coarse pass, reported after the level's marking) or in the second (the
    last level, reported by the final check before the call returns)."""
    import torch
    import neural_sdf_volume_b200 as vdm
    case = _case()
    params = vdm.hier_params(8, 2, False)
    ref, _ = vdm.vdm_decode_hierarchical(case.dec, case.K, case.V, params, case.spheres, 0.01)
    ref = ref.cpu().numpy()
    vdm.vdm_debug_inject(launch, SHORT_WAIT)
    try:
        _expect_timeout(lambda: vdm.vdm_decode_hierarchical(case.dec, case.K, case.V, params,
                                                             case.spheres, 0.01))
    finally:
        vdm.vdm_debug_inject(0, 0)
    torch.cuda.synchronize()
    again, _ = vdm.vdm_decode_hierarchical(case.dec, case.K, case.V, params, case.spheres, 0.01)
    assert np.array_equal(again.cpu().numpy(), ref)


def test_dense_decode_reports_its_own_timeout():
    """The dense call returns the timeout of its own launch, and the next,
    unrelated call is not blamed for it."""
    import torch
    import neural_sdf_volume_b200 as vdm
    case = _case()
    ref = vdm.vdm_decode_dense(case.dec, case.K, case.V, grid_R=12).cpu().numpy()
    vdm.vdm_debug_inject(1, SHORT_WAIT)
    try:
        _expect_timeout(lambda: vdm.vdm_decode_dense(case.dec, case.K, case.V, grid_R=12))
    finally:
        vdm.vdm_debug_inject(0, 0)
    torch.cuda.synchronize()
    again = vdm.vdm_decode_dense(case.dec, case.K, case.V, grid_R=12).cpu().numpy()
    assert np.array_equal(again, ref)
