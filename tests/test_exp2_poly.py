"""The software 2^x of the attention softmax (part of the exponentials run on
the FMA pipes): its constants match the derivation script, and its fp32
arithmetic meets the error bound used for P (well under bf16 rounding, 2^-9)."""
import os
import re
import sys

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "linear_hybrid_attention_b200", "csrc")
sys.path.insert(0, CSRC)
import exp2_poly  # noqa: E402


def _kernel_constants():
    src = open(os.path.join(CSRC, "zb_common.cuh")).read()
    m = re.search(r"kC1 = ([0-9.e+-]+)f, kC2 = ([0-9.e+-]+)f, kC3 = ([0-9.e+-]+)f", src)
    return [1.0] + [float(v) for v in m.groups()]


def test_kernel_constants_match_derivation():
    coef, err = exp2_poly.remez_exp2()
    assert err < 1e-4
    k = _kernel_constants()
    assert np.allclose(np.float32(k), np.float32(coef), rtol=0, atol=2e-8)


def test_fp32_evaluation_error_bound():
    k = [np.float32(v) for v in _kernel_constants()]
    x = np.linspace(-126.0, 8.0, 2_000_001).astype(np.float32)
    y = exp2_poly.eval_f32(k, x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1.2e-4


def test_special_values():
    k = _kernel_constants()
    y = exp2_poly.eval_f32(k, np.array([-np.inf, -200.0, -127.0, 0.0, 1.0, 8.0, -3.0], dtype=np.float32))
    assert y.tolist() == [0.0, 0.0, 0.0, 1.0, 2.0, 256.0, 0.125]
