"""The hand-built edge rows of tests/quant_edges.py hit the quantizer branch
each kind names (llmdaily.org day-65, "From BF16 to INT8, INT4, or even fewer
bits", read with round half to even, the stored scale dividing, fp16
saturation at 65504 and an fp16 scale of 0 making a zero group).  Checked on
the CPU against the oracle's scalar quantizer, which the pin tests tie to the
pages; the GPU parity test then feeds the same rows to the CUDA kernels."""
import numpy as np
import pytest

from oracle import oracle as O
from tests.quant_edges import KINDS, fp8_values, group_values


@pytest.mark.parametrize("bits,asym,fp32", [(8, 0, 0), (8, 0, 1), (4, 0, 0), (4, 0, 1), (2, 0, 0),
                                             (2, 0, 1), (2, 1, 0), (4, 1, 0), (8, 1, 0)])
@pytest.mark.parametrize("kind", KINDS)
def test_edge_group_hits_its_branch(bits, asym, fp32, kind):
    rng = np.random.default_rng(bits * 10 + asym)
    n = 64
    x = group_values(kind, n, bits, asym, rng)
    Q, Qa = (1 << (bits - 1)) - 1, (1 << bits) - 1
    u = 2.0 ** -6 if bits == 8 else 2.0 ** -3
    if asym:
        s, z, q = O.quant_asym(x, bits, bool(fp32))
    else:
        s, q = O.quant_sym(x, bits, bool(fp32))
    # every code lies in the quantizer's range: [-Q, Q], or [0, 2^b - 1] with a zero-point
    assert q.min() >= (0 if asym else -Q) and q.max() <= (Qa if asym else Q)
    if kind == "zero":
        assert s == 0.0 and not q.any()
    elif kind == "constant":
        if asym:   # max == min: a zero-scale group whose zero-point holds the value
            assert s == 0.0 and z == -1.25 and not q.any()
        else:
            assert np.all(q == -Q)
    elif kind == "ties":
        assert s == u
        assert np.any(np.abs(x / u - np.floor(x / u)) == 0.5)
        want = np.rint(x.astype(np.float64) / u)   # numpy rounds half to even
        assert np.array_equal(q, want.astype(np.int32))
    elif kind == "saturate":
        if fp32:
            assert s > 65504.0
        else:
            assert s == 65504.0
            lim = Qa if asym else Q
            assert np.any(q == lim) and np.max(np.abs(x - (z if asym else 0.0))) / s > lim   # the clip fired
            if not asym:   # and at the negative end: elements below -(Q + 1/2) s take -Q exactly
                below = x / s < -(Q + 0.5)
                assert below.any() and np.all(q[below] == -Q)
    elif kind == "underflow":
        if not fp32:
            assert s == 0.0 and not q.any()
    elif kind == "subnormal":
        if not fp32:
            assert s == 2.0 ** -23   # an fp16 subnormal
            if bits == 4 or (bits == 2 and asym):
                lim = Qa if asym else Q
                assert q.max() == lim and x.max() / s > lim   # rounding lowered s, the clip fired
    else:
        assert s > 0.0


@pytest.mark.parametrize("kind", KINDS)
def test_fp8_edge_values(kind):
    rng = np.random.default_rng(3)
    x = fp8_values(kind, 64, rng)
    codes = [O.f32_to_e4m3(float(v)) for v in x]
    back = np.array([O.e4m3_to_f32(c) for c in codes])
    if kind == "ties":
        want = {1.0625: 1.0, -1.0625: -1.0, 1.1875: 1.25, -1.1875: -1.25, 9.5: 10.0, -9.5: -10.0,
                2.0 ** -10: 0.0, -(2.0 ** -10): 0.0, 3 * 2.0 ** -10: 2.0 ** -8}
        for a, b in zip(x, back):
            assert b == want[float(a)]
    elif kind == "saturate":
        assert np.all(np.abs(back) == 448.0)
    elif kind == "underflow":
        assert not back.any()
    elif kind == "subnormal":
        assert np.array_equal(back, x)
