"""The GPU-vs-oracle comparison helpers themselves, on the CPU: the asymmetric
group check accepts only the oracle's other rounding of a zero point that sits
exactly on a .5 tie, with the codes that go with it."""
import numpy as np
import pytest

from tests import parity


def test_asym_zero_point_tie(orc):
    # step 0.5 (exact in fp16), min -3.75 and max 3.75: (hi - lo) / 15 = 0.5 and
    # -lo / s = 7.5 exactly, which rounds to 8 (half to even); 7 is the other rounding
    x = np.linspace(-3.75, 3.75, 128)
    codes, s16, z16, pre = orc.quant_asym_int4(x, 1.0)
    assert s16 == 0x3800 and orc.f16_to_f64([z16])[0] == 8.0
    ref = orc.pack_nibbles(codes)
    alt_codes = np.clip(np.rint(x / 0.5) + 7, 0, 15).astype(np.int32)
    z7 = int(orc.f64_to_f16([7.0])[0])
    # the other rounding, with its codes: accepted
    assert parity.check_asym_group(orc, 1.0, orc.pack_nibbles(alt_codes), s16, z7, ref, s16, z16, pre, x, "tie") == 1
    # the other rounding with the first rounding's codes: rejected
    with pytest.raises(AssertionError):
        parity.check_asym_group(orc, 1.0, ref, s16, z7, ref, s16, z16, pre, x, "tie")
    # a zero point two away: rejected
    z6 = int(orc.f64_to_f16([6.0])[0])
    with pytest.raises(AssertionError):
        parity.check_asym_group(orc, 1.0, ref, s16, z6, ref, s16, z16, pre, x, "tie")
    # no tie: a different zero point is rejected
    y = np.linspace(-3.1, 4.4, 128)
    c2, s2, zz, p2 = orc.quant_asym_int4(y, 1.0)
    zother = int(orc.f64_to_f16([orc.f16_to_f64([zz])[0] + 1])[0])
    with pytest.raises(AssertionError):
        parity.check_asym_group(orc, 1.0, orc.pack_nibbles(c2), s2, zother, orc.pack_nibbles(c2), s2, zz, p2, y, "x")
    # identical results pass with nothing excused
    assert parity.check_asym_group(orc, 1.0, ref, s16, z16, ref, s16, z16, pre, x, "same") == 0
