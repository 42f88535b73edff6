"""The FMA-pipe 2^x used for part of the softmax exponentials (sm100.cuh,
exp2_poly_x2) against numpy's exp2.

The constants are read from the CUDA header and the algorithm (floor by a
round-down add of 1.5*2^23, degree-3 polynomial in the fraction, integer add
of floor(x) into the exponent field) is replayed in float32 on the CPU.  The
result must stay within 1e-4 relative error everywhere the kernel uses it
(scores minus the running max: x in [-126, 8]); the bf16 rounding of P that
follows is 2^-9 relative.
"""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "grouped_differential_attention_gdla_b200", "csrc", "sm100.cuh")


def _constants():
    text = open(HDR).read()
    vals = {}
    for name in ("kExp2C0", "kExp2C1", "kExp2C2", "kExp2C3", "kRoundShift"):
        m = re.search(r"constexpr float %s = ([0-9.eE+-]+)f;" % name, text)
        assert m, name
        vals[name] = np.float32(float(m.group(1)))
    return vals


def _emulate(x):
    c = _constants()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    # add.rm: 1.5*2^23 + x rounded toward -inf is exactly 1.5*2^23 + floor(x)
    t = (np.float64(c["kRoundShift"]) + np.floor(x.astype(np.float64))).astype(np.float32)
    n = (t - c["kRoundShift"]).astype(np.float32)
    f = (x - n).astype(np.float32)
    q = np.float32(c["kExp2C3"]) * f + c["kExp2C2"]
    q = q.astype(np.float32) * f + c["kExp2C1"]
    q = q.astype(np.float32) * f + c["kExp2C0"]
    q = q.astype(np.float32)
    bits = q.view(np.uint32).astype(np.uint64) + ((t.view(np.uint32).astype(np.uint64) << 23)
                                                   & 0xFFFFFFFF)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_shift_constant_is_one_and_a_half_times_two_to_23():
    assert _constants()["kRoundShift"] == np.float32(1.5 * 2 ** 23)


def test_relative_error_over_softmax_range():
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32),
                        np.arange(-125, 9, dtype=np.float32),
                        np.arange(-125, 9, dtype=np.float32) - np.float32(1e-6)])
    y = _emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 1e-4, f"max relative error {rel.max():.3e} at x={x[np.argmax(rel)]}"


def test_clamps_very_negative_inputs():
    y = _emulate(np.array([-300.0, -1000.0, -125.0], dtype=np.float32))
    assert np.all(y > 0) and np.all(y < 2.4e-38)
