"""The FMA-pipe 2^x approximation inside the attention softmax (Cody-Waite
split x = n + f, n = rint(x), f in [-1/2, 1/2]; 2^f from a fitted cubic; 2^n
added to the exponent field).  Stated bound: relative error <= 7.5e-5.

CPU: the cubic's coefficients, read from the kernel source, against numpy's
exp2 in fp64 over the whole reduced range.  GPU: the device function itself
over a dense grid, including the edge of the normal range and the clamp at
-126."""
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BOUND = 7.5e-5


def _coefficients():
    src = open(os.path.join(ROOT, "diffusion_transformer_block_flux_b200", "csrc", "common.cuh")).read()
    body = src[src.index("uint64_t exp2_poly2("):]
    body = body[:body.index("\n}\n")]
    # the packed constants of the body are the rounding constant 1.5 * 2^23 and the four coefficients
    c = [float(v) for v in re.findall(r"f2_pack\(([0-9.]+)f, \1f\)", body) if float(v) < 1.0]
    assert len(c) == 4, c
    return c  # c3, c2, c1, c0 in Horner order


def test_cubic_meets_its_stated_bound_on_the_reduced_range():
    c3, c2, c1, c0 = _coefficients()
    f = np.linspace(-0.5, 0.5, 200001)
    p = ((c3 * f + c2) * f + c1) * f + c0
    rel = np.abs(p / np.exp2(f) - 1.0)
    assert rel.max() <= BOUND, rel.max()
    # a fit, not a truncated series: the error is spread over the range
    assert rel.max() > 1e-6


@pytest.mark.gpu
def test_device_exp2_poly_against_exp2():
    import torch
    import diffusion_transformer_block_flux_b200 as dit
    grid = np.concatenate([np.linspace(-126.0, 8.0, 1 << 20),
                           np.arange(-126, 9) + 0.5, np.arange(-126, 9).astype(np.float64),
                           np.arange(-126, 9) - 0.4999, [-140.0, -1e30, -np.inf]]).astype(np.float32)
    x = torch.from_numpy(grid).cuda()
    y = torch.empty_like(x)
    dit.dit_selftest_exp2_poly(x, y)
    got = y.cpu().double().numpy()
    xs = grid.astype(np.float64)
    ref = np.exp2(np.maximum(xs, -126.0))
    rel = np.abs(got / ref - 1.0)
    normal = xs >= -125.999
    # the stated bound plus fp32 rounding of the evaluation, wherever the result is a normal number
    assert rel[normal].max() <= BOUND + 2e-7, rel[normal].max()
    # within 1e-3 of the clamp the exponent sum may leave the normal range: up to twice the bound
    edge = (xs >= -126.0) & ~normal
    assert rel[edge].max() <= 2 * BOUND + 2e-7, rel[edge].max()
    # below the clamp: exactly the value at -126, positive and finite
    at_clamp = got[xs == -126.0][0]
    low = got[xs < -126.0]
    assert at_clamp > 0 and np.all(low == at_clamp)
