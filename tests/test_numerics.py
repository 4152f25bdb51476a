"""The FMA-pipe exponential the forward softmax uses for a quarter of its 2^x.

CPU: the coefficients compiled into the kernels are the ones the committed
Remez fit produces, and a float32 emulation of the device evaluation stays
within the fit's relative error bound. GPU: the device evaluation (and the
hardware ex2.approx it shares the work with) against exact 2^x.
"""

import importlib.util
import os
import re

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FIT = os.path.join(ROOT, "attention_sink_long_b200", "csrc", "exp2_poly_fit.py")
COMMON = os.path.join(ROOT, "attention_sink_long_b200", "csrc", "lg_common.cuh")
POLY_BOUND = 3e-6


def load_fit():
    spec = importlib.util.spec_from_file_location("exp2_poly_fit", FIT)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def header_coefficients():
    text = open(COMMON).read()
    body = text[text.index("float ex2_poly(float x)"):]
    body = body[: body.index("return")]
    vals = [float(v) for v in re.findall(r"([0-9]\.[0-9]+)f", body)]
    # p starts at C4, then fmaf(p, f, C3) ... C0
    c4, c3, c2, c1, c0 = vals[-5:]
    return np.array([c0, c1, c2, c3, c4], dtype=np.float32)


def test_compiled_coefficients_are_the_remez_fit():
    fit = load_fit()
    c = fit.remez_relative(fit.DEGREE).astype(np.float32)
    np.testing.assert_array_equal(header_coefficients(), c)


def test_float32_emulation_within_bound():
    fit = load_fit()
    c = header_coefficients()
    xs = np.linspace(-126.0, 64.0, 1_000_003).astype(np.float32)
    got = fit.eval_f32(c, xs).astype(np.float64)
    rel = np.abs(got / np.exp2(xs.astype(np.float64)) - 1.0)
    assert rel.max() < POLY_BOUND
    special = np.array([-np.inf, -1000.0, -127.0], dtype=np.float32)
    assert np.all(fit.eval_f32(c, special) == 0.0)


@pytest.mark.gpu
def test_device_exponentials_against_exact():
    import attention_sink_long_b200 as lg

    xs = torch.linspace(-126.0, 64.0, 2_000_003, dtype=torch.float32)
    xs = torch.cat([xs, torch.tensor([0.0, -0.5, 0.5, -1e-7, 1e-7, -8.0, 8.0])])
    x = xs.cuda()
    exact = torch.exp2(xs.double())
    ys = {}
    for method, bound in ((1, POLY_BOUND), (2, POLY_BOUND), (0, 2.0 ** -21)):
        y = torch.empty_like(x)
        ys[method] = y
        lg.lg_exp2_device(x, y, method)
        torch.cuda.synchronize()
        rel = (y.double().cpu() / exact - 1.0).abs()
        assert rel.max().item() < bound, (method, rel.max().item())
    # the paired form is the same arithmetic lane by lane
    assert torch.equal(ys[1], ys[2])
    for method in (0, 1, 2):
        z = torch.tensor([-float("inf"), -500.0], device="cuda")
        y = torch.empty_like(z)
        lg.lg_exp2_device(z, y, method)
        torch.cuda.synchronize()
        assert torch.all(y == 0), (method, y)
