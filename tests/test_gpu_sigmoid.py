"""Accuracy of the kernels' in-register sigma, measured through the C ABI
against the exact logistic function (fp64 oracle).

EXP mode: relative error of sigma and sigma' below 1e-3 over [-80, 80] where
the value is a normal fp32 number (the degree-4 reciprocal polynomial leaves
< 3.4e-4 in sigma and twice that in sigma' = u g^2; ex2.approx adds ~1e-7).
TANH mode: the hardware tanh.approx form; its error is measured and reported
(absolute error, which is what bounds it near sigma -> 0), and checked only
against a loose absolute bound."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu
sa = pytest.importorskip("padding_aware_sigmoid_b200")


def _grid():
    x = np.concatenate([np.linspace(-80, 80, 160001), np.linspace(-12, -8, 40001)])
    return x.astype(np.float32)


def _exact(x):
    """sigma and sigma' = sigma(x) sigma(-x) from the oracle's sigma, which keeps
    relative accuracy in both tails (sigma(1 - sigma) in fp64 cancels for x > 20)."""
    orc = oracle.default()
    s = np.array([orc.sigmoid(float(v)) for v in x])
    sm = np.array([orc.sigmoid(-float(v)) for v in x])
    return s, s * sm


@pytest.fixture(scope="module")
def grid():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    x = _grid()
    s, g = _exact(x)
    return x, s, g


def _eval(x, mode):
    xt = torch.from_numpy(x).cuda()
    y, dy = sa.sigmoid_eval(xt, mode)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64), dy.cpu().numpy().astype(np.float64)


def test_exp_mode_relative_accuracy(grid):
    x, s, g = grid
    y, dy = _eval(x, sa.SIGMOID_EXP)
    tiny = s > 1e-30
    rel = np.abs(y - s)[tiny] / s[tiny]
    relg = np.abs(dy - g)[g > 1e-30] / g[g > 1e-30]
    print(f"EXP mode: max rel err sigma {rel.max():.3e}, sigma' {relg.max():.3e}")
    assert rel.max() < 4e-4
    assert relg.max() < 1e-3


def test_tanh_mode_error_report(grid):
    x, s, g = grid
    y, dy = _eval(x, sa.SIGMOID_TANH)
    abs_err = np.abs(y - s)
    sel = (x > -12) & (x < -8)
    rel_tail = (abs_err[sel] / s[sel]).max()
    print(f"TANH mode: max abs err sigma {abs_err.max():.3e}; max rel err on x in [-12,-8] "
          f"{rel_tail:.3e}; max abs err sigma' {np.abs(dy - g).max():.3e}")
    assert abs_err.max() < 1e-3
