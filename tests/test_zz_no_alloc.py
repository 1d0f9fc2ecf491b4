"""The no-allocation entry point gives the same volume as the workspace one.

vdm_decode_hierarchical_noalloc exists for callers that may not allocate
device memory themselves (applications that own the whole device memory
budget, latency-critical code that avoids cudaMalloc/cudaFree because they can
synchronise the device).  It runs the hierarchical decoder on a scratch array
built into the library.  This file is collected last so that a run that stops
at its first failure has already run every other test; it also passes on its
own in a fresh process."""
import ctypes as C

import numpy as np
import pytest

import workloads as W

from gpu_cases import Case

pytestmark = pytest.mark.gpu


def _call_noalloc(vdm, case, params, out, B):
    cd = case.dec.cstruct()
    an = vdm.CAnalytic()
    an.spheres = case.spheres.data_ptr()
    an.n_spheres = int(case.spheres.shape[1])
    an.dec_scale = 0.01
    stats = (vdm.CHierStats * B)()
    import torch
    st = vdm._lib.vdm_decode_hierarchical_noalloc(
        C.byref(cd), case.K.data_ptr(), case.V.data_ptr(), B, case.spec.N, C.byref(params),
        C.byref(an), out.data_ptr(), stats, None, torch.cuda.current_stream().cuda_stream)
    return st, stats


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    import torch
    import neural_sdf_volume_b200 as vdm
    spec = W.DecoderSpec(C=256, H=4, F=512, N=512, query_ln=False, dtype="bf16")
    B = 2
    case = Case(spec, key=5, B=B, n_spheres=6, sphere_key=5)
    params = vdm.hier_params(16, 3, adaptive=True, n_probe=32, top_k=128, seed=3)
    ref, ref_stats = vdm.vdm_decode_hierarchical(case.dec, case.K, case.V, params, case.spheres, 0.01)
    ref = ref.cpu().numpy()
    for call in range(2):
        out = torch.full((B, 64, 64, 64), float("nan"), device="cuda")
        st, stats = _call_noalloc(vdm, case, params, out, B)
        assert st == 0, vdm._lib.vdm_last_error()
        got = out.cpu().numpy()
        assert np.isfinite(got).all(), f"call {call}: voxels left unwritten"
        # same kernels on the same inputs: the library's results are bit-identical run to run
        assert np.array_equal(got, ref), f"call {call}: max abs difference {np.abs(got - ref).max()}"
        for b in range(B):
            assert list(stats[b].decoded) == ref_stats[b]["decoded"]


def test_noalloc_rejects_problems_larger_than_its_scratch():
    import torch
    import neural_sdf_volume_b200 as vdm
    spec = W.DecoderSpec(C=256, H=4, F=512, N=64, query_ln=False, dtype="bf16")
    case = Case(spec, key=6, n_spheres=2, sphere_key=6)
    params = vdm.hier_params(64, 3, adaptive=True, n_probe=64, top_k=64)   # needs > 32 MiB
    out = torch.empty((1, 256, 256, 256), device="cuda")
    st, _ = _call_noalloc(vdm, case, params, out, 1)
    assert st == 2 and b"scratch" in vdm._lib.vdm_last_error()
