"""The e4m3 codec of the input generator (OCP E4M3: 1 sign, 4 exponent bits with bias 7, 3 mantissa
bits, no infinity, 0x7F / 0xFF NaN, largest finite 448). The FP8 parity tests take the exact
dequantised values from it, so it is pinned by values fixed by the format itself."""
import numpy as np

import synth


def test_known_codes():
    cases = {
        0.0: 0x00,
        1.0: 0x38,            # exponent 7 (bias 7), mantissa 0
        1.125: 0x39,          # mantissa 1/8
        1.875: 0x3F,
        2.0: 0x40,
        0.5: 0x30,
        448.0: 0x7E,          # 1.75 * 2^8, the largest finite value
        2.0 ** -6: 0x08,      # smallest normal
        2.0 ** -9: 0x01,      # smallest subnormal: 1/8 * 2^-6
        7.0 * 2.0 ** -9: 0x07,  # largest subnormal
        -2.0: 0xC0,
        -448.0: 0xFE,
    }
    for x, code in cases.items():
        assert int(synth.to_e4m3_bits(np.array([x]))[0]) == code, (x, hex(code))
        assert float(synth.e4m3_bits_to_f32(np.array([code], np.uint8))[0]) == x


def test_rounding_and_saturation():
    enc = lambda x: int(synth.to_e4m3_bits(np.array([x]))[0])  # noqa: E731
    assert enc(1.0625) == 0x38   # halfway between 1.0 (even code) and 1.125: ties to even
    assert enc(1.1875) == 0x3A   # halfway between 1.125 and 1.25 (even code 0x3A)
    assert enc(1.07) == 0x39     # nearer 1.125
    assert enc(2.0 ** -10) == 0x00  # halfway between 0 and the smallest subnormal: even code 0
    assert enc(500.0) == 0x7E and enc(1e30) == 0x7E and enc(-1e30) == 0xFE  # saturate to +-448


def test_every_finite_code_round_trips():
    codes = np.arange(256, dtype=np.uint8)
    codes = codes[(codes & 0x7F) != 0x7F]          # drop the two NaN codes
    vals = synth.e4m3_bits_to_f32(codes)
    back = synth.to_e4m3_bits(vals)
    nz = vals != 0                                 # +0 and -0 both decode to 0
    assert np.array_equal(back[nz], codes[nz])
    # values are exactly representable in bf16 (the FP8 oracle runs on their bf16 bits)
    assert np.array_equal(synth.bf16_bits_to_f32(synth.to_bf16_bits(vals)), vals)
