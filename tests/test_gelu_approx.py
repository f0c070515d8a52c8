"""The bf16 layer path's GELU uses erf from Abramowitz & Stegun, Handbook of
Mathematical Functions, formula 7.1.26, whose published bound is |error| <=
1.5e-7. This reads the coefficients out of the kernel source and checks the
formula built from them against math.erf in double precision: a mistyped
coefficient breaks the bound."""
from __future__ import annotations

import math
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(__file__), "..", "blocked_attention_b200", "csrc", "rt_common.cuh")


def _coefficients():
    src = open(SRC).read()
    body = src[src.index("float erf_as7126(float x)"):]
    body = body[: body.index("\n}\n")]
    nums = [float(v) for v in re.findall(r"-?\d+\.\d+(?=f)", body)]
    # p, a5, a4, a3, a2, a1, log2(e), in the order the source uses them
    assert len(nums) == 7, nums
    return nums


def test_erf_coefficients_meet_the_published_bound():
    p, a5, a4, a3, a2, a1, log2e = _coefficients()
    assert abs(log2e - 1.0 / math.log(2.0)) < 1e-15
    x = np.linspace(0.0, 6.0, 60001)
    t = 1.0 / (1.0 + p * x)
    poly = t * (a1 + t * (a2 + t * (a3 + t * (a4 + t * a5))))
    approx = 1.0 - poly * np.exp2(-x * x * log2e)
    exact = np.array([math.erf(v) for v in x])
    err = np.max(np.abs(approx - exact))
    assert err <= 1.5e-7, err
    # and it is the published approximation, not some other: its error is
    # of that order, not far below it
    assert err > 1e-8


def test_gelu_from_it_is_within_bf16_rounding():
    p, a5, a4, a3, a2, a1, log2e = _coefficients()
    y = np.linspace(-8.0, 8.0, 16001)
    z = np.abs(y) / math.sqrt(2.0)
    t = 1.0 / (1.0 + p * z)
    erf = np.sign(y) * (1.0 - t * (a1 + t * (a2 + t * (a3 + t * (a4 + t * a5)))) * np.exp(-z * z))
    gelu = 0.5 * y * (1.0 + erf)
    exact = np.array([0.5 * v * (1.0 + math.erf(v / math.sqrt(2.0))) for v in y])
    # absolute error <= 0.5 |y| 1.5e-7: far below the bf16 storage step
    assert np.all(np.abs(gelu - exact) <= 0.5 * np.abs(y) * 1.5e-7 + 1e-12)
