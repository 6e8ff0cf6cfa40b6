"""The e4m3 storage used for the FP8 forward's inputs, pinned to values the OCP FP8 format
fixes (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; largest finite 448, smallest
subnormal 2^-9): encodings and round-to-nearest-even behaviour."""
import numpy as np

import synth_inputs as si


def test_e4m3_known_encodings():
    # scale is amax / 448, so include 448 to make the scale exactly 1
    vals = np.array([448.0, 1.0, 0.5, -2.0, 2.0 ** -9, 2.0 ** -6, 240.0, 0.0], dtype=np.float32)
    b, deq, scale = si.to_e4m3(vals)
    assert scale == 1.0
    assert b.tolist() == [0x7E, 0x38, 0x30, 0xC0, 0x01, 0x08, 0x77, 0x00]
    assert np.array_equal(deq, vals)


def test_e4m3_rounds_to_nearest_even():
    # between 1.0 (mantissa 000) and 1.125 (001) the midpoint 1.0625 goes to the even 1.0;
    # between 1.125 and 1.25 the midpoint 1.1875 goes to the even 1.25
    vals = np.array([448.0, 1.0625, 1.1875, 1.07], dtype=np.float32)
    _, deq, _ = si.to_e4m3(vals)
    assert deq[1:].tolist() == [1.0, 1.25, 1.125]


def test_tf32_rounding_to_nearest_even():
    # 1 + 2^-10 is a tf32 value; 1 + 2^-11 is the midpoint between 1 and it (ties to even: 1),
    # 1 + 3 * 2^-11 is the midpoint between 1 + 2^-10 and 1 + 2^-9 (ties to even: 1 + 2^-9)
    x = np.array([1 + 2.0 ** -10, 1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, 1 + 2.0 ** -11 + 2.0 ** -20, -3.0],
                 dtype=np.float32)
    assert si.round_tf32(x).tolist() == [1 + 2.0 ** -10, 1.0, 1 + 2.0 ** -9, 1 + 2.0 ** -10, -3.0]
