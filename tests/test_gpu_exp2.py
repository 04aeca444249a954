"""The polynomial 2^x that the attention kernel evaluates on the FMA pipe for
a share of its softmax exponentials, held to its stated error bound (relative
<= 1e-4 on [-125, 8]) against an exact 2^x of the same fp32 inputs."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _poly_exp2(x: torch.Tensor) -> torch.Tensor:
    from joint_video_audio_b200 import _binding as B
    y = torch.empty_like(x)
    B.h3blk_selftest_exp2(x.data_ptr(), y.data_ptr(), x.numel(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return y


def test_exp2_polynomial_within_its_error_bound():
    grid = np.linspace(-125.0, 8.0, 1 << 22, dtype=np.float32)
    k = np.arange(-125, 9, dtype=np.float32)
    # integers, the rounding boundaries between them (n + 1/2 and its fp32
    # neighbours), and points just inside each unit interval
    edges = np.concatenate([k, k + 0.5, np.nextafter(k + 0.5, np.float32(-np.inf)),
                            np.nextafter(k + 0.5, np.float32(np.inf)), k + 1e-3, k - 1e-3])
    x = np.concatenate([grid, edges[(edges >= -125) & (edges <= 8)]]).astype(np.float32)
    y = _poly_exp2(torch.from_numpy(x).cuda()).cpu().numpy().astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert np.all(np.isfinite(y))
    assert rel.max() <= 1e-4, f"max relative error {rel.max():.3e} at x = {x[np.argmax(rel)]}"
    # integers are exact to within the fit's error at f = 0
    ki = np.isin(x, k)
    assert np.abs(y[ki] / ref[ki] - 1).max() <= 1e-4


def test_exp2_polynomial_clamps_below_minus_125():
    x = torch.tensor([-125.0, -126.0, -200.0, -1e30], device="cuda")
    y = _poly_exp2(x).cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(y, 2.0 ** -125, rtol=1e-4)


def test_exp2_polynomial_odd_length():
    x = torch.linspace(-3, 3, 7, device="cuda")
    y = _poly_exp2(x).cpu().double()
    np.testing.assert_allclose(y.numpy(), np.exp2(x.cpu().double().numpy()), rtol=1e-4)
