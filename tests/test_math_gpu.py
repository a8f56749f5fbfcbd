"""The scalar functions the prefill softmax computes its weights with,
checked on the GPU over their whole input range against exact (fp64)
references (through the C ABI self-test hook fa_selftest_math).

- 2^x on the FMA pipe (exp2_fma_pair: round-to-nearest range reduction and
  the cubic of exp2_poly.cuh, generated with its error bound 7.485e-5):
  the relative error stays within that bound plus fp32 evaluation rounding
  for every x in [-125, 8] (the kernel's inputs are <= 8); below -125 (a
  masked score is -inf) the result is exactly 0, as the MUFU path gives 0
  below the normal range.
- 2^x by ex2.approx.ftz (MUFU): within 2^-21 relative on the same range,
  and 0 for -inf.
- the softcapped logit c * tanh(x * scale / c) in log2 units, computed as
  1 - 2 / (1 + 2^(2 y log2 e)): absolute error a few fp32 ulps of the cap,
  saturating to exactly +-cap for large |x|.
"""
import os
import re

import numpy as np
import pytest
import torch

from exact_io_aware_86_b200 import api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _poly_bound():
    """The cubic's relative-error bound, as its generator wrote it into the
    header the kernel is built from."""
    with open(os.path.join(ROOT, "exact_io_aware_86_b200", "csrc", "exp2_poly.cuh")) as f:
        m = re.search(r"kExp2PolyRelErr = ([0-9.eE+-]+)f;", f.read())
    return float(m.group(1))

pytestmark = pytest.mark.gpu

LOG2E = 1.4426950408889634


def _grid():
    """Dense grid over [-130, 8] plus the edges of the clamp and of the
    normal range, integers and half-integers (where the range reduction
    switches), and the masked value -inf."""
    x = np.linspace(-130.0, 8.0, 2_000_001, dtype=np.float64)
    edges = [-127.0, -126.5, -126.0, -125.75, -125.5, -125.25, -125.0, -124.999, -124.5, -0.5,
             0.0, 0.5, 1.0, 7.5, 8.0]
    e32 = np.array(edges, dtype=np.float32)
    near = np.concatenate([np.nextafter(e32, np.float32(-np.inf)),
                           np.nextafter(e32, np.float32(np.inf))])
    halves = np.arange(-130.0, 8.5, 0.5)
    x = np.concatenate([x, edges, near.astype(np.float64), halves]).astype(np.float32)
    return np.concatenate([x, np.array([-np.inf], dtype=np.float32)])


def _run(op, x, a=0.0, b=0.0):
    y = api.selftest_math(op, torch.from_numpy(x).cuda(), a, b)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


def test_exp2_on_the_fma_pipe_meets_its_bound():
    x = _grid()
    y = _run(api.MATH_EXP2_FMA, x)
    xd = x.astype(np.float64)
    normal = xd >= -125.0
    ref = np.exp2(xd[normal])
    rel = np.abs(y[normal] / ref - 1.0)
    # cubic's bound (from its generator) plus the fp32 rounding of the
    # Horner steps and of the reduced argument (a few units of 2^-24)
    bound = _poly_bound() + 8 * 2.0 ** -24
    worst = int(np.argmax(rel))
    assert rel[worst] <= bound, f"x={xd[normal][worst]!r}: rel err {rel[worst]:.3e} > {bound:.3e}"
    # masked, or below -125: exactly zero
    assert np.all(y[~normal] == 0.0), xd[~normal][y[~normal] != 0.0][:5]
    assert y[-1] == 0.0  # -inf


def test_exp2_on_mufu_is_accurate_and_flushes():
    x = _grid()
    y = _run(api.MATH_EXP2_MUFU, x)
    xd = x.astype(np.float64)
    normal = xd >= -126.0
    rel = np.abs(y[normal] / np.exp2(xd[normal]) - 1.0)
    assert rel.max() <= 2.0 ** -21, f"max rel err {rel.max():.3e}"
    assert y[-1] == 0.0
    # results below the normal range are flushed (ftz) to zero
    assert np.all(y[xd < -127.0] == 0.0)


@pytest.mark.parametrize("scale,cap", [(1.0 / np.sqrt(128.0), 50.0), (1.0, 50.0), (0.125, 0.5),
                                       (1.0 / np.sqrt(64.0), 5.0)])
def test_softcap_logit(scale, cap):
    x = np.concatenate([np.linspace(-300.0, 300.0, 1_000_001),
                        [0.0, 1e-6, -1e-6, 1e30, -1e30]]).astype(np.float32)
    a = np.float32(2.0 * LOG2E * scale / cap)
    b = np.float32(cap * LOG2E)
    y = _run(api.MATH_SOFTCAP_LOG2, x, float(a), float(b))
    # exact value for the fp32 constants the kernel receives
    ref = float(b) * np.tanh(x.astype(np.float64) * float(a) / (2.0 * LOG2E))
    err = np.abs(y - ref)
    # 1 - 2/(1 + e): one rounding of 1, rcp.approx and ex2.approx (2^-22
    # relative each, at most half of it reaching tanh), then the product by b
    bound = float(b) * 6.0 * 2.0 ** -24
    worst = int(np.argmax(err))
    assert err[worst] <= bound, f"x={x[worst]!r}: abs err {err[worst]:.3e} > {bound:.3e}"
    # saturation is exact
    assert y[-2] == float(b) and y[-1] == -float(b)
