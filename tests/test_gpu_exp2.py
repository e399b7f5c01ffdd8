"""The polynomial 2^x that the softmax can run on the FMA pipe
(tc::exp2_poly2: round-to-nearest range reduction, degree-3 minimax fit of
2^f on [-1/2, 1/2] in relative error, exp2_poly_fit.py) against CUDA's
exp2f on the same GPU: relative error within the fit's bound over the range
the softmax uses, and the clamp below -125."""
import numpy as np
import pytest
import torch

import mqa_attention_qkv_b200 as gqa

pytestmark = pytest.mark.gpu

FIT_BOUND = 7.5e-5      # the fit's maximum relative error on [-1/2, 1/2]


def _eval(x):
    xd = torch.from_numpy(np.asarray(x, dtype=np.float32)).cuda()
    poly, ref = torch.empty_like(xd), torch.empty_like(xd)
    gqa.gqa_debug_exp2_poly(xd, poly, ref)
    torch.cuda.synchronize()
    return poly.cpu().numpy().astype(np.float64), ref.cpu().numpy().astype(np.float64)


def test_exp2_poly_matches_exp2f_over_the_softmax_range():
    x = np.concatenate([np.linspace(-125.0, 8.0, 1 << 20), np.arange(-125, 9, dtype=np.float64),
                        np.arange(-125, 8) + 0.5, [0.0, -0.0]])
    poly, ref = _eval(x)
    rel = np.abs(poly - ref) / ref
    # the fit's bound plus a few float32 roundings of the evaluation
    assert float(rel.max()) <= FIT_BOUND + 4 * 2.0 ** -24, float(rel.max())
    # integers are reached through the exponent field: 2^n exactly up to the polynomial's value at f = 0
    ints = np.arange(-125, 9, dtype=np.float64)
    pi, ri = _eval(ints)
    assert np.all(np.abs(pi / ri - 1.0) <= FIT_BOUND)


def test_exp2_poly_clamps_below_minus_125():
    x = np.array([-126.0, -200.0, -1e30, -np.inf], dtype=np.float32)
    poly, _ = _eval(x)
    ref_at_clamp, _ = _eval([-125.0])
    assert np.all(poly == ref_at_clamp[0]) and 0.0 < poly[0] < 2.0 ** -124
