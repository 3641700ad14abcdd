"""The quantizers' division shortcuts on the GPU, against IEEE binary32 bit for bit, exhaustively:
the MS-EDEN group scale's reciprocal RN(1/p) (hardware approximation plus one fused correction)
over every significand of every binade p can take (2^-103 <= p < 2^126: biased exponents
24..252), and RN(a/6) (FMA-corrected multiply) over every a the kernels divide
(2^-100 <= a < 2^128: 27..254)."""
import pytest

from nvfp4_quantized_b200 import qt2

pytestmark = pytest.mark.gpu


def test_reciprocal_is_ieee_exact_on_its_domain():
    assert qt2.qt2_selftest_division(24, 252)[0] == 0


def test_division_by_six_is_ieee_exact_on_its_domain():
    assert qt2.qt2_selftest_division(27, 254)[1] == 0


def test_selftest_refuses_a_bad_range():
    with pytest.raises(qt2.QT2Error):
        qt2.qt2_selftest_division(0, 3)
