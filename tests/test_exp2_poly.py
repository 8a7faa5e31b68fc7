"""The cubic 2^x that the attention kernel evaluates on the FMA pipe: the
constants in isa_common.cuh are the ones the fitting script produces, and
their float32 evaluation (clamp, round-to-integer split, Horner, exponent
add) stays within 1e-4 relative error of 2^x on [-125, 0] -- far below the
2^-8 relative step of the bfloat16 probabilities it feeds."""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_attention_coarse_b200", "csrc")
sys.path.insert(0, CSRC)

import fit_exp2_poly as F  # noqa: E402


def kernel_constants():
    text = open(os.path.join(CSRC, "isa_common.cuh")).read()
    body = text[text.index("ex2_poly2"):]
    body = body[:body.index("\n}\n")]
    hexes = re.findall(r"__uint_as_float\((0x[0-9A-F]{8})u\)", body)
    # order in the source: c3, c2, c1, c0 (each listed twice, one per lane)
    uniq = list(dict.fromkeys(hexes))
    assert len(uniq) == 4
    c3, c2, c1, c0 = (np.uint32(int(h, 16)).view(np.float32) for h in uniq)
    return np.array([c0, c1, c2, c3], np.float32)


def test_constants_come_from_the_fit():
    c, err = F.fit()
    assert err < 8e-5
    np.testing.assert_array_equal(kernel_constants(), np.asarray(c, np.float32))


def test_float32_evaluation_error_bound():
    c = kernel_constants()
    xs = np.concatenate([np.linspace(-125, 0, 1_000_001, dtype=np.float32),
                         np.float32(-np.arange(0, 126)) + np.float32(0.5),
                         np.float32(-np.arange(0, 126))])
    got = F.eval_f32(c, xs).astype(np.float64)
    ref = np.exp2(xs.astype(np.float64))
    assert np.max(np.abs(got - ref) / ref) < 1e-4
    # below the clamp the result is a denormal, never a garbage normal number
    tiny = F.eval_f32(c, np.array([-126.0, -200.0, -np.inf], np.float32))
    assert np.all(tiny >= 0) and np.all(tiny < 1.2e-38)
