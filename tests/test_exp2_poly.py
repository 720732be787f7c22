"""The software 2^x of the prefill softmax (prefill_sm100.cuh, exp2_poly):
its coefficients are the ones the Remez fit of csrc/gen_exp2_poly.py
produces, and its float32 evaluation stays within 2e-4 relative error of
2^x on the range the softmax feeds it (scores minus a reference max, at most
8 above it).  Checked against numpy's exp2 in float64, independently of the
kernel; the kernel's own use is covered by the GPU parity tests."""

import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "flashattention_attention_attn_b200", "csrc")
sys.path.insert(0, CSRC)
import gen_exp2_poly  # noqa: E402


def kernel_coefficients():
    text = open(os.path.join(CSRC, "prefill_sm100.cuh")).read()
    vals = dict(re.findall(r"kC(\d) = ([-+0-9.e]+)f", text))
    return [float(vals[str(i)]) for i in range(4)]


def test_kernel_constants_match_the_fit():
    fit = gen_exp2_poly.remez_relative()
    for a, b in zip(kernel_coefficients(), fit):
        assert abs(a - np.float32(b)) <= 2e-7 * max(1.0, abs(b))


def test_relative_error_bound_on_softmax_range():
    x = np.concatenate([np.linspace(-126.0, 8.0, 2_000_001), -np.arange(0, 126.25, 0.25), [0.0, 8.0, -0.5, 0.5]])
    got = gen_exp2_poly.eval_f32(kernel_coefficients(), x).astype(np.float64)
    rel = np.abs(got / np.exp2(x) - 1.0)
    assert rel.max() < 2e-4, rel.max()


def test_monotone_and_positive():
    x = np.linspace(-30.0, 8.0, 200_001)
    got = gen_exp2_poly.eval_f32(kernel_coefficients(), x)
    assert np.all(got > 0)
    # a bf16-rounded P cannot reorder: differences stay well within bf16 resolution
    assert np.all(np.diff(got.astype(np.float64)) > -2e-4 * got[1:])
