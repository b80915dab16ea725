"""The attention softmax's exponential on the device (stca_selftest_ex2),
against 2^x in float64: the FMA-pipe form (range reduction to [-1/2, 1/2], a
degree-3 minimax polynomial for relative error) within its stated 1.5e-4
relative error over [-126, 8], alone and in the packed two-at-a-time form the
kernels use; the MUFU ex2.approx within 2^-21; and the clamp below -126."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _run(x, method, gpu):
    import torch
    import target_attention_jagged_b200 as S
    xd = torch.from_numpy(x.astype(np.float32)).to(gpu)
    yd = torch.empty_like(xd)
    S.stca_selftest_ex2(xd, yd, method)
    torch.cuda.synchronize()
    return yd.cpu().numpy().astype(np.float64)


def _inputs():
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-126.0, 8.0, 2_000_001),
                        rng.uniform(-126.0, 8.0, 1_000_000),
                        np.arange(-126, 9, dtype=np.float64),            # integers
                        np.arange(-126, 8, dtype=np.float64) + 0.5,      # reduction boundaries
                        [-0.0, 1e-30, -1e-30]]).astype(np.float32)
    return x


@pytest.mark.parametrize("method", [1, 2])
def test_fma_form_within_bound(gpu, method):
    x = _inputs()
    y = _run(x, method, gpu)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert np.all(np.isfinite(y))
    assert rel.max() <= 1.5e-4, f"max relative error {rel.max():.3e} at x = {x[np.argmax(rel)]}"


def test_fma_form_clamps_below_range(gpu):
    x = np.array([-126.5, -200.0, -1e4, -np.inf], dtype=np.float32)
    for method in (1, 2):
        y = _run(x, method, gpu)
        assert np.allclose(y, 2.0 ** -126, rtol=2e-4), y


def test_mufu_form(gpu):
    x = _inputs()
    y = _run(x, 0, gpu)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() <= 2.0 ** -21, f"max relative error {rel.max():.3e}"
