"""The FMA-pipe exp2 of the window kernel, checked on the CPU: the constants
compiled into window_tc.cu are those exp2_poly_fit.py derives, and the float32
evaluation the kernel performs stays within 1e-4 relative of 2^x (the softmax
weights are rounded to bf16 afterwards, a relative step of 2^-8)."""

import importlib.util
import os
import re

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "linear_attention_video_block_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("exp2_poly_fit", os.path.join(CSRC, "exp2_poly_fit.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _kernel_constants():
    src = open(os.path.join(CSRC, "window_tc.cu")).read()
    return np.array([float(re.search(rf"kExp2C{k} = ([0-9.eE+-]+)f;", src).group(1)) for k in range(4)],
                    dtype=np.float32)


def test_constants_match_the_fit():
    m = _fit_module()
    assert np.array_equal(_kernel_constants(), m.fit().astype(np.float32))


def test_float32_evaluation_error_bound():
    m = _fit_module()
    c = _kernel_constants()
    xs = np.concatenate([np.linspace(-125.0, 8.0, 4000001), np.arange(-125, 9)]).astype(np.float32)
    got = m.device_eval(c, xs).astype(np.float64)
    ref = np.exp2(xs.astype(np.float64))
    assert np.max(np.abs(got - ref) / ref) < 1e-4
    # below 2^-125 results turn subnormal; they only need to stay negligible
    tail = np.linspace(-200.0, -125.0, 10001).astype(np.float32)
    assert np.all(m.device_eval(c, tail) < 2.0 ** -124)
    # masked scores (-inf) clamp to 2^-126 ~ 1e-38, i.e. no weight
    assert m.device_eval(c, np.array([-np.inf], dtype=np.float32))[0] < 2e-38
