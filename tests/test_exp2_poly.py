"""The polynomial 2^x the attention kernels evaluate on the FMA pipe
(exp2_poly2 in csrc/common.cuh): its constants are the ones exp2_poly.py
derives (Chebyshev interpolation of 2^f on [-1/2, 1/2] after Cody-Waite
reduction), and its float32 arithmetic is within the derivation's error
bound of 2^x over the softmax argument range."""

import re

import numpy as np
import pytest

from gpt_decoder_lm_b200 import exp2_poly

SRC = "gpt_decoder_lm_b200/csrc/common.cuh"


def _source_coefficients():
    txt = open(SRC).read()
    body = txt[txt.index("uint64_t exp2_poly2("):]
    body = body[:body.index("\n}\n")]
    return [float(v) for v in re.findall(r"f2c\(([0-9.eE+-]+)f\)", body) if v not in ("12582912.0",)]


def test_source_constants_are_the_derivation():
    got = _source_coefficients()          # Horner order: c4, c3, c2, c1, c0
    want = exp2_poly.coefficients().astype(np.float32)[::-1]
    assert len(got) == exp2_poly.DEGREE + 1
    assert np.array_equal(np.float32(got), want), (got, want)


def test_interpolant_error_bound():
    f = np.linspace(-0.5, 0.5, 100001)
    c = exp2_poly.coefficients()
    p = np.polyval(c[::-1], f)
    assert np.abs(p / 2.0 ** f - 1).max() < 3.6e-6


def test_float32_evaluation_over_softmax_range():
    # probabilities are 2^(s - m) with s - m <= 0, and up to +8 under the
    # forward's lazy rescaling
    x = np.concatenate([np.linspace(-125, 8, 400001), np.arange(-125, 9, dtype=np.float64),
                        np.arange(-125, 9) + 0.5]).astype(np.float32)
    y = exp2_poly.evaluate_f32(x).astype(np.float64)
    ref = 2.0 ** x.astype(np.float64)
    assert np.all(np.isfinite(y)) and np.all(y > 0)
    assert np.abs(y / ref - 1).max() < 4e-6
    # below the clamp the result is ~2^-125, as negligible as the true value
    lo = exp2_poly.evaluate_f32(np.float32([-126.0, -200.0, -np.inf])).astype(np.float64)
    assert np.all((lo > 0) & (lo < 2.0 ** -124))


@pytest.mark.gpu
def test_device_polynomial_against_exp2f():

    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from gpt_decoder_lm_b200 import binding as gb
    x = np.concatenate([np.linspace(-125, 8, 1 << 20), np.arange(-125, 9), np.arange(-125, 9) + 0.5,
                        np.random.default_rng(0).uniform(-30, 0, 1 << 18)]).astype(np.float32)
    xd = torch.from_numpy(x).cuda()
    yp, yr = torch.empty_like(xd), torch.empty_like(xd)
    assert gb.STATUS[gb.test_exp2(xd, yp, yr, torch.cuda.current_stream().cuda_stream)] == "GPT_OK"
    yp, yr = yp.cpu().numpy().astype(np.float64), yr.cpu().numpy().astype(np.float64)
    assert np.abs(yp / yr - 1).max() < 4e-6
    # the device arithmetic is the derivation's float32 arithmetic (fused
    # multiply-adds; at most one unit in the last place apart)
    host = exp2_poly.evaluate_f32(x).astype(np.float64)
    assert np.abs(yp / host - 1).max() <= 2.0 ** -23
