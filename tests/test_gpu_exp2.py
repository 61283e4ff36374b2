"""The FMA-pipe exponential used for part of the softmax's 2^x, against exp2 in fp64.

Its error bound is the polynomial's fitted bound (1.0e-4 relative, float32 Horner)
plus float32 rounding of the range reduction; the softmax rounds P to bf16 (2^-9)
right after, so 2e-4 relative is the bar."""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


def _run(x):
    import mask_skipping_flashattention_b200 as bfa
    y = bfa.selftest_exp2(torch.as_tensor(x, dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


def test_exp2_poly_relative_error_over_softmax_range():
    # the softmax passes s*c - m <= 8; everything down to the underflow point
    x = np.concatenate([np.linspace(-126.0, 8.0, 400001), np.arange(-126, 9, dtype=np.float64) + 0.5])
    x32 = x.astype(np.float32)
    y = _run(x32)
    ref = np.exp2(x32.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 2e-4, rel.max()


def test_exp2_poly_integers_exact_and_masked_zero():
    n = np.arange(-126, 9, dtype=np.float32)
    assert np.array_equal(_run(n), np.exp2(n.astype(np.float64)))
    y = _run(np.array([-np.inf, -1e30, -200.0, -127.0], dtype=np.float32))
    assert np.array_equal(y, np.zeros(4))


def test_exp2_poly_monotone_up_to_its_error_on_fine_grid():
    # monotone inside each reduction interval; at the switch points n + 1/2 the two
    # polynomial ends may differ by up to the fitted error
    x = np.linspace(-20.0, 8.0, 200001).astype(np.float32)
    y = _run(x)
    assert np.all(np.diff(y) >= -2e-4 * y[1:])
