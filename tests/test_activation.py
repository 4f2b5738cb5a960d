"""The generalized attention's activations (GELU, SiLU and their derivatives)
through ba_selftest_activation, the device functions the GDPA kernels call,
against fp64 values computed on the host from the definitions.

Stated bound (include/ba.h): GELU's Phi comes from erf by Abramowitz &
Stegun's formula 7.1.26, whose absolute error is at most 1.5e-7, so Phi is
off by at most 7.5e-8 before float32 rounding; 2^x and reciprocals from the
special-function unit add relative errors near 2^-22. The test allows
1e-6 max(1, |x|) on the value and on the derivative, which covers those and
the float32 arithmetic around them with room to spare; a wrong coefficient,
a missing density term or a sign error in the tail is far outside it.
"""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_kunlun_b200 as ba

pytestmark = pytest.mark.gpu

_erf = np.frompyfunc(math.erf, 1, 1)


def exact(act, x):
    x = x.astype(np.float64)
    if act == ba.BA_ACT_GELU:
        cdf = 0.5 * (1.0 + _erf(x / math.sqrt(2.0)).astype(np.float64))
        pdf = np.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)
        return x * cdf, cdf + x * pdf
    with np.errstate(over="ignore"):
        sg = 1.0 / (1.0 + np.exp(-x))
    return x * sg, sg * (1.0 + x * (1.0 - sg))


def gpu(act, x):
    xd = torch.from_numpy(x.astype(np.float32)).cuda()
    y, dy = torch.empty_like(xd), torch.empty_like(xd)
    assert ba.ba_selftest_activation(act, xd, y, dy) == ba.BA_OK
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64), dy.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("act", [ba.BA_ACT_GELU, ba.BA_ACT_SILU], ids=["gelu", "silu"])
def test_activation_and_derivative_within_the_stated_bound(act):
    x = np.concatenate([np.linspace(-12.0, 12.0, 1 << 20), np.linspace(-0.01, 0.01, 4097),
                        [-80.0, -30.0, -9.0, 9.0, 30.0, 80.0]]).astype(np.float32)
    y, dy = gpu(act, x)
    assert not np.isnan(dy).any(), "the kernels' value / derivative forms disagree"
    ry, rdy = exact(act, x)
    tol = 1e-6 * np.maximum(1.0, np.abs(x.astype(np.float64)))
    for name, got, ref in (("value", y, ry), ("derivative", dy, rdy)):
        err = np.abs(got - ref)
        i = int(np.argmax(err / tol))
        assert np.all(err <= tol), f"{name}: error {err[i]:.3e} at x = {x[i]} (bound {tol[i]:.1e})"


@pytest.mark.parametrize("act", [ba.BA_ACT_GELU, ba.BA_ACT_SILU], ids=["gelu", "silu"])
def test_activation_limits(act):
    x = np.array([-1e30, -1e4, 0.0, 1e4, 1e30], dtype=np.float32)
    y, dy = gpu(act, x)
    np.testing.assert_array_equal(y, [0.0, 0.0, 0.0, 1e4, np.float32(1e30)])
    np.testing.assert_allclose(dy, [0.0, 0.0, 0.5, 1.0, 1.0], rtol=0, atol=1e-7)


def test_activation_selftest_rejects_bad_arguments():
    x = torch.zeros(4, device="cuda")
    assert ba.ba_selftest_activation(7, x, x.clone(), x.clone()) == ba.BA_ERR_INVALID_ARG
