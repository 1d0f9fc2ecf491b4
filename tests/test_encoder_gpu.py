"""GPU parity of vecset encoding (vdm_encode) against the oracle's encoder:
point features, keys and values of the cloud, and each latent token's block
output; then the round trip (encode, then decode the vecset) against the
oracle's round trip."""
import numpy as np
import pytest

import workloads as W
from oracle import decoder as OD
from oracle import encoder as OE

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("spec,M,N", [
    (W.DecoderSpec(C=512, H=8, F=2048, N=1, query_ln=True, dtype="bf16"), 1000, 200),
    (W.DecoderSpec(C=256, H=4, F=512, N=1, query_ln=False, dtype="bf16"), 777, 131),
    (W.DecoderSpec(C=64, H=1, F=256, N=1, query_ln=True, dtype="f32"), 300, 50)])
@pytest.mark.parametrize("stress", [False, True])
def test_encode_matches_oracle(spec, M, N, stress):
    import torch
    import neural_sdf_volume_b200 as vdm
    blk = W.make_decoder(spec, seed=0, key=41, stress=stress)["weights"]
    proj = W.make_encoder_input_proj(spec.C, seed=0, key=41, dtype=spec.dtype)
    sp = W.make_spheres(6, seed=0, key=42)[0]
    cloud = W.make_point_cloud(sp, M, N, seed=0, key=43)
    dev = vdm.Decoder.from_numpy(blk, spec.C, spec.H, spec.F, spec.query_ln, spec.dtype)
    tdt = torch.float32 if spec.dtype == "f32" else torch.bfloat16
    W_in = torch.from_numpy(proj["W_in"]).cuda().to(tdt)
    b_in = torch.from_numpy(proj["b_in"]).cuda()
    z = vdm.vdm_encode(dev, W_in, b_in, torch.from_numpy(cloud["points"][None]).cuda(),
                       torch.from_numpy(cloud["queries"][None]).cuda())[0].cpu().numpy()
    want = OE.encode(cloud["points"], cloud["queries"], proj["W_in"], proj["b_in"], blk, spec.query_ln)
    tol = 1e-4 if spec.dtype == "f32" else 2e-2
    assert np.abs(z - want).max() <= tol * max(1.0, np.abs(want).max())


def test_encode_then_decode_round_trip():
    """Encode a sphere-union cloud into 512 tokens of width 512 and decode them
    with the full decoder: the decoder output at grid points matches the
    oracle's encode + decode within the bf16 tolerance."""
    import torch
    import neural_sdf_volume_b200 as vdm
    spec = W.DecoderSpec(C=512, H=8, F=2048, N=512, query_ln=True, dtype="bf16")
    enc = W.make_decoder(spec, seed=0, key=44)["weights"]
    dec_w = W.make_decoder(spec, seed=0, key=45)["weights"]
    proj = W.make_encoder_input_proj(spec.C, seed=0, key=44)
    sp = W.make_spheres(8, seed=0, key=46)[0]
    cloud = W.make_point_cloud(sp, 4096, 512, seed=0, key=47)
    e = vdm.Decoder.from_numpy(enc, spec.C, spec.H, spec.F, True, "bf16")
    d = vdm.Decoder.from_numpy(dec_w, spec.C, spec.H, spec.F, True, "bf16")
    z = vdm.vdm_encode(e, torch.from_numpy(proj["W_in"]).cuda().bfloat16(), torch.from_numpy(proj["b_in"]).cuda(),
                       torch.from_numpy(cloud["points"][None]).cuda(), torch.from_numpy(cloud["queries"][None]).cuda())
    K, V = vdm.vdm_precompute_kv(d, z)
    out = vdm.vdm_decode_dense(d, K, V, grid_R=10)[0].cpu().numpy()
    z_o = OE.encode(cloud["points"], cloud["queries"], proj["W_in"], proj["b_in"], enc, True)
    Ko, Vo = OD.precompute_kv(z_o, dec_w)
    want = OD.decode_points(OD.grid_points(10), Ko, Vo, dec_w, True)
    assert np.abs(out - want).max() <= 2e-2
