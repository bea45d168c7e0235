"""The exponential the forward kernel evaluates on the FMA pipe for a share of its
probabilities (exp2_poly_x2), through attn_selftest_exp2, against exp2 in fp64.

Over x in [-125, 64] the relative error must stay below 2^-18 (the fitted polynomial's
2^-18.5 plus fp32 Horner rounding); at the integer and half-integer boundaries of the
range reduction too; below -125 the value is clamped to about 2^-125."""
import numpy as np
import pytest

from long_context_attention_fwd_b200 import capi

torch = pytest.importorskip("torch")


def _run(x: np.ndarray) -> np.ndarray:
    xt = torch.from_numpy(x.astype(np.float32)).cuda()
    y = torch.full_like(xt, float("nan"))
    st = capi.attn_selftest_exp2(xt.data_ptr(), y.data_ptr(), xt.numel(),
                                 torch.cuda.current_stream().cuda_stream)
    capi.check(st, "attn_selftest_exp2")
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


@pytest.mark.gpu
def test_relative_error_over_the_range():
    rng = np.random.default_rng(7)
    grid = np.linspace(-125.0, 64.0, 1 << 21)
    ints = np.arange(-125, 65, dtype=np.float64)
    edges = np.concatenate([ints, ints + 0.5, ints - 0.5, np.nextafter(ints + 0.5, 0),
                            np.nextafter(ints - 0.5, 0)])
    x = np.concatenate([grid, edges[(edges >= -125) & (edges <= 64)],
                        rng.uniform(-1, 1, 1 << 18), [0.0, -0.0]]).astype(np.float32)
    if x.size % 2:
        x = np.append(x, np.float32(1.0))
    y = _run(x)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert np.isfinite(y).all()
    assert rel.max() <= 2.0 ** -18, float(np.log2(rel.max()))


@pytest.mark.gpu
def test_clamped_below():
    x = np.array([-125.5, -126.0, -200.0, -1e30, -np.inf, -125.0], dtype=np.float32)
    y = _run(x)
    assert (y[:5] > 0).all() and (y[:5] <= 2.0 ** -124).all()
    assert abs(y[5] / 2.0 ** -125 - 1.0) <= 2.0 ** -18
