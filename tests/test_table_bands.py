"""The band argument behind the kernels' code tables, checked on the oracle.

The table-based encoders (the streamed E4M3 kernels, the general
sliding-window kernels and the INT8 quantisers) compute the code of every
bf16 pattern only for a band of binades at and below amax's, and store the
zero code for everything smaller: 24 binades for E4M3 (x / s < 2^-13 there,
below half the smallest E4M3 subnormal 2^-9), 10 for INT8 (|x / s| < 1/2
there).  These tests check, with the oracle's own quantisers, that the largest
magnitude just below each band encodes to zero for every possible amax
exponent, and that binades well inside the band can still give a nonzero
code.
"""
import numpy as np

from oracle import sp24_oracle as O


def _bits(exp_field, mant):
    return np.uint16((exp_field << 7) | mant)


def _below_band(e_amax, band):
    """Largest bf16 magnitude whose exponent field lies below the band of
    `band` binades ending at amax's exponent field, or None."""
    e = e_amax - band
    return None if e < 0 else _bits(e, 127)


def test_e4m3_band_of_24_binades():
    for e_a in range(0, 255):
        for m_a in (0, 64, 127):
            amax_bits = _bits(e_a, m_a)
            if amax_bits == 0:
                continue
            s = O.scale_from_amax(O.bf16_to_f32(np.array([amax_bits]))[0])
            x = _below_band(e_a, 24)
            if x is not None:
                codes = O.quantize_with_scale(np.array([x, x | 0x8000], dtype=np.uint16), s)
                assert codes.tolist() == [0x00, 0x80], (e_a, m_a)
            # with amax at the bottom of its binade, the binade 19 below
            # amax's (inside the band) still reaches the smallest subnormal
            if m_a == 0 and e_a >= 19:
                top = _bits(e_a - 19, 127)
                assert O.quantize_with_scale(np.array([top], dtype=np.uint16), s)[0] == 0x01


def test_int8_band_of_10_binades():
    for e_a in range(0, 255):
        for m_a in (0, 64, 127):
            amax_bits = _bits(e_a, m_a)
            if amax_bits == 0:
                continue
            s = O.int8_scale_from_amax(O.bf16_to_f32(np.array([amax_bits]))[0])
            x = _below_band(e_a, 10)
            if x is not None:
                codes = O.int8_quantize_with_scale(np.array([x, x | 0x8000], dtype=np.uint16), s)
                assert codes.tolist() == [0, 0], (e_a, m_a)
            # with amax at the bottom of its binade, the binade 8 below
            # amax's (inside the band) reaches a nonzero code
            if m_a == 0 and e_a >= 8:
                top = _bits(e_a - 8, 127)
                assert O.int8_quantize_with_scale(np.array([top], dtype=np.uint16), s)[0] == 1
