"""Failure detection without a GPU fault: a withheld completion signal makes
the tensor-core decoder's bounded waits expire; the call reports
VDM_ERR_TIMEOUT and the CUDA context stays usable."""
import numpy as np
import pytest

import workloads as W

from gpu_cases import Case

pytestmark = pytest.mark.gpu


def test_withheld_signal_times_out_and_context_survives():
    import torch
    import neural_sdf_volume_b200 as vdm
    spec = W.DecoderSpec(C=256, H=4, F=512, N=128, query_ln=False, dtype="bf16")
    case = Case(spec, key=8, n_spheres=3, sphere_key=8)
    params = vdm.hier_params(8, 2, False)
    ref, _ = vdm.vdm_decode_hierarchical(case.dec, case.K, case.V, params, case.spheres, 0.01)
    ref = ref.cpu().numpy()
    vdm.vdm_debug_inject(1, 20_000_000)          # ~10 ms per wait
    try:
        with pytest.raises(vdm.VdmError) as ei:
            vdm.vdm_decode_hierarchical(case.dec, case.K, case.V, params, case.spheres, 0.01)
        assert ei.value.status == 5, str(ei.value)
        assert "bounded wait" in str(ei.value)
    finally:
        vdm.vdm_debug_inject(0, 0)
    torch.cuda.synchronize()
    again, _ = vdm.vdm_decode_hierarchical(case.dec, case.K, case.V, params, case.spheres, 0.01)
    assert np.array_equal(again.cpu().numpy(), ref)
