"""The quantizer's refined division is the IEEE fp32 division, bit for bit,
for every divisor significand and every fp16 numerator with |x/s| < 64 (see
bq_check_division in include/bq.h for why one binade of divisors suffices)."""
import pytest

from quantized_gemm_group_b200 import bq

pytestmark = pytest.mark.gpu


def test_two_refinements_match_ieee_division_exhaustively():
    bad, checked, s_bad, x_bad = bq.bq_check_division(0x3F800000, 0x40000000, refinements=2)
    assert checked == (1 << 23) * 2 * 0x5400
    assert bad == 0, f"first mismatch s=0x{s_bad:08x} x=0x{x_bad:04x}"


def test_division_check_detects_differences():
    # a single refinement is not claimed exact; whatever it gives, the checker
    # must count consistently (pairs checked), and report a first mismatch iff any
    bad, checked, s_bad, x_bad = bq.bq_check_division(0x3F800000, 0x3F800000 + (1 << 16), refinements=1)
    assert checked == (1 << 16) * 2 * 0x5400
    assert (bad == 0) == (s_bad == 0)


@pytest.mark.parametrize("divisor", [3, 7, 15])
def test_constant_divisor_scale_matches_ieee_division_for_every_float(divisor):
    # every fp32 bit pattern of both signs, finite, infinite and NaN
    for lo, hi in ((0, 0x80000000), (0x80000000, 0x100000000 - 1)):
        bad, checked, x_bad, d_bad = bq.bq_check_const_division(divisor, lo, hi)
        assert checked == hi - lo
        assert bad == 0, f"first mismatch x=0x{x_bad:08x} / {d_bad}"
