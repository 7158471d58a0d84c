"""CPU: the fine kernel's FMA-pipe exponential (poly_exp2_x2 in csrc/fine_tc.cu) emulated step
by step in fp32, against 2^x computed in fp64.  The constants are read from the kernel source,
so the test checks the arithmetic the kernel runs: max relative error below the 7.5e-5 its
comment states (far below the bf16 rounding of every P value) for x in [-125, 8], and tiny
values (at most 2^-124) for the masked arguments below -125."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "sparse_hierarchical_attention_pool_b200", "csrc", "fine_tc.cu")


def _constants():
    src = open(SRC).read()
    body = src[src.index("poly_exp2_x2(uint64_t x2)"):]
    body = body[:body.index("\n}\n")]
    names = {}
    for name in ("c3", "c2", "c1", "c0"):
        m = re.search(r"const uint64_t %s = f2_pack\(0x([0-9A-Fa-f]{8})u" % name, body)
        assert m, name
        names[name] = np.array([int(m.group(1), 16)], dtype=np.uint32).view(np.float32)[0]
    return names


def _f32(x):
    return np.asarray(x, dtype=np.float32)


def _fma(a, b, c):
    # one rounding: the fp32 product is exact in fp64
    return _f32(a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64))


def poly_exp2(x):
    c = _constants()
    a = np.maximum(_f32(x), np.float32(-125.0))
    magic = np.float32(12582912.0)                      # 1.5 * 2^23
    t = _f32(a + magic)
    f = _f32(a + (-(_f32(t + (-magic)))))
    p = _fma(_fma(_fma(np.full_like(f, c["c3"]), f, np.full_like(f, c["c2"])), f, np.full_like(f, c["c1"])),
             f, np.full_like(f, c["c0"]))
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001), np.linspace(-1.0, 1.0, 200_001)]).astype(np.float32)
    got = poly_exp2(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 7.5e-5 * 1.01, rel.max()


def test_masked_arguments_vanish():
    x = np.array([-126.0, -200.0, -1e30, -np.inf], dtype=np.float32)
    got = poly_exp2(x)
    assert np.all(got > 0) and np.all(got <= 2.0 ** -124)


def test_integer_arguments_are_near_exact_powers():
    x = np.arange(-30, 9, dtype=np.float32)
    got = poly_exp2(x).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(x.astype(np.float64)) - 1.0) < 1e-4)
