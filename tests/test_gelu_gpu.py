"""The decoder's GELU (x Phi(x), erf by Abramowitz & Stegun formula 7.1.26) through
the test hook `vdm_debug_gelu`:

- the pair form that feeds the MLP's second matrix equals the scalar form rounded
  to bf16 (round to nearest even), bit for bit;
- the scalar form is within 1e-6 max(1, |x|) of x Phi(x) in float64 (the
  formula's |erf error| <= 1.5e-7 plus the hardware reciprocal and exponential)."""
import numpy as np
import pytest
from scipy.special import erf

pytestmark = pytest.mark.gpu


def _bf16_rne(v: np.ndarray) -> np.ndarray:
    b = v.astype(np.float32).view(np.uint32).astype(np.uint64)
    r = ((b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32)


def test_gelu_pair_form_and_error_bound():
    import torch

    import neural_sdf_volume_b200 as vdm

    rng = np.random.default_rng(5)
    x = np.concatenate([np.linspace(-10.0, 10.0, 1 << 20 | 1), rng.normal(0.0, 2.0, 1 << 16),
                        [0.0, -0.0, 1e-30, -1e-30, 40.0, -40.0, 0.5]]).astype(np.float32)
    pair, scalar = vdm.vdm_debug_gelu(torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    pair = pair.cpu().numpy()
    scalar = scalar.cpu().numpy()
    assert np.array_equal(pair.view(np.uint32), _bf16_rne(scalar).view(np.uint32))
    xd = x.astype(np.float64)
    exact = 0.5 * xd * (1.0 + erf(xd / np.sqrt(2.0)))
    err = np.abs(scalar.astype(np.float64) - exact)
    assert (err <= 1e-6 * np.maximum(1.0, np.abs(xd))).all(), (err.max(), x[np.argmax(err)])
