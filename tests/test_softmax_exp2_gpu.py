"""The tensor-core decoder computes a quarter of its softmax exponentials as
2^x = 2^round(x) * p(x - round(x)) with a fitted cubic p (instead of the
special-function unit).  Checked here against 2^x in float64 (numpy), over the
range the softmax uses (x = S - m <= 8 by the stale-maximum rule, and far below
0), through the library's test hook `vdm_debug_exp2`.

Bound: relative error <= 1e-4 for -125 <= x <= 9 (the fit's own bound is
7.5e-5 in float32 Horner form); below -125 the result is in [0, 2^-124] (near
-126 the scaled result leaves the normal range, where it is not accurate)."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _exp2_gpu(x: np.ndarray) -> np.ndarray:
    import torch

    import neural_sdf_volume_b200 as vdm

    y = vdm.vdm_debug_exp2(torch.from_numpy(x.astype(np.float32)).cuda())
    torch.cuda.synchronize()
    return y.cpu().numpy()


def test_polynomial_exp2_relative_error_bound():
    rng = np.random.default_rng(7)
    x = np.concatenate([
        np.linspace(-125.0, 9.0, 1 << 20 | 1),                 # dense sweep, odd count (last pair half used)
        rng.uniform(-30.0, 8.0, 1 << 18),                      # the softmax's usual range
        np.arange(-125, 10, dtype=np.float64),                 # integers: f = 0
        np.arange(-125, 9, dtype=np.float64) + 0.5,            # round-half cases
    ]).astype(np.float32)
    y = _exp2_gpu(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert np.isfinite(y).all()
    assert rel.max() <= 1e-4, (rel.max(), x[np.argmax(rel)])
    # the polynomial is not the identity: its error is of the fitted size, not of float32 rounding
    assert rel.max() > 1e-6


def test_polynomial_exp2_below_the_normal_range_and_minus_infinity():
    x = np.concatenate([np.linspace(-126.0, -125.0, 4097),
                        [-126.5, -127.0, -140.0, -1000.0, -np.inf, -3.4e38]]).astype(np.float32)
    y = _exp2_gpu(x).astype(np.float64)
    assert (y >= 0.0).all() and (y <= 2.0 ** -124).all(), y


def test_polynomial_exp2_empty_and_single():
    import torch

    import neural_sdf_volume_b200 as vdm

    assert vdm.vdm_debug_exp2(torch.empty(0, device="cuda")).numel() == 0
    y = _exp2_gpu(np.array([3.0], np.float32))
    assert abs(y[0] / 8.0 - 1.0) <= 1e-4
