"""The FMA-pipe 2^x polynomial of the attention softmax, evaluated on the CPU exactly as
the device code does it in fp32 (round-to-nearest add and subtract, fused multiply-add,
exponent added as an integer), with the coefficients read from the CUDA source: its
relative error over the softmax's range stays within the bound stated beside them.
The same function is checked on the device against exact 2^x in the GPU tests."""
from __future__ import annotations

import os
import re

import numpy as np
import pytest

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "hybrid_attention_ssm_head_b200", "csrc", "common.cuh")


def _coefficients():
    src = open(SRC).read()
    body = src[src.index("if constexpr (DEG == 5)"):src.index("// log(1 + e^x)")]
    five, three = body.split("} else {")
    get = lambda part: [float(v) for v in re.findall(r"make_float2\(([-0-9.e]+)f,", part)]  # noqa: E731
    return {5: get(five), 3: get(three)}


def _fma(a, b, c):
    # a*b is exact in fp64 for fp32 operands; the sum is rounded once to fp64, then to fp32
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _poly(x: np.ndarray, cs) -> np.ndarray:
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    rnd = np.float32(12582912.0)
    t = (x + rnd).astype(np.float32)
    f = (x - (t - rnd).astype(np.float32)).astype(np.float32)
    cs = [np.float32(c) for c in cs]
    p = _fma(np.full_like(f, cs[0]), f, np.full_like(f, cs[1]))
    for c in cs[2:]:
        p = _fma(p, f, np.full_like(f, c))
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23)))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


@pytest.mark.parametrize("degree,bound", [(3, 7.5e-5), (5, 2.4e-7)])
def test_polynomial_exp2_bound(degree, bound):
    cs = _coefficients()[degree]
    assert len(cs) == degree + 1
    x = np.concatenate([np.linspace(-125.0, 0.0, 1_000_003), -np.arange(0, 125.5, 0.5),
                        np.random.default_rng(0).uniform(-125, 0, 200_000)]).astype(np.float32)
    rel = np.abs(_poly(x, cs).astype(np.float64) - np.exp2(x.astype(np.float64))) / np.exp2(x.astype(np.float64))
    assert rel.max() <= bound, rel.max()
    # below the clamp the result is 2^-125
    np.testing.assert_allclose(_poly(np.array([-126.0, -1e4], np.float32), cs), 2.0 ** -125, rtol=bound)
