"""Pins of the oracle's MXFP8 quantiser (OCP Microscaling v1.0, E4M3
elements with E8M0 scales per 32 elements) against facts of the format:
the full table of E4M3 codes, exactly representable blocks round-tripping,
the scale exponent of a known maximum, saturation, rounding to nearest even
at halfway points, zero blocks and signed zero."""
import numpy as np

import oracle
from synth import f32_to_bf16_bits


def bf(x):
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def test_e4m3_code_table():
    # Normal codes: (1 + m/8) 2^(e-7) for e = 1..15; subnormals m 2^-9; 0x7e = 448 is the largest finite.
    v = oracle.e4m3_decode(np.arange(256, dtype=np.uint8))
    assert v[0x00] == 0 and v[0x01] == 2.0 ** -9 and v[0x07] == 7 * 2.0 ** -9
    assert v[0x08] == 2.0 ** -6 and v[0x38] == 1.0 and v[0x3c] == 1.5 and v[0x7e] == 448.0
    assert np.array_equal(v[0x80:0xff], -v[0x00:0x7f])


def test_representable_blocks_round_trip_exactly():
    # A block whose max is 448 * 2^k and whose values lie on the E4M3 grid
    # scaled by 2^k comes back exactly, with scale byte 127 + k.
    grid = oracle.e4m3_decode(np.arange(0, 0x7f, dtype=np.uint8))
    rng = np.random.default_rng(0)
    for k in (-20, -3, 0, 5, 30):
        vals = rng.choice(grid, size=(7, 64)) * rng.choice([-1.0, 1.0], size=(7, 64))
        vals[:, 0] = 448.0
        vals[:, 32] = -448.0
        x = vals * 2.0 ** k
        q, s = oracle.quantize_mxfp8(bf(x))
        assert np.all(s == 127 + k)
        assert np.array_equal(oracle.dequantize_mxfp8(q, s), x)


def test_scale_exponent_rounding_and_saturation():
    # max |x| = 100 -> floor(log2 100) = 6 -> e = -2: elements are x * 4.
    x = np.zeros((1, 32), np.float32)
    x[0, :7] = [100, 1.0, 3.125, 3.375, -0.0, 3 * 2.0 ** -11, 2.0 ** -12]
    q, s = oracle.quantize_mxfp8(bf(x))
    assert s[0, 0] == 127 - 2
    d = oracle.dequantize_mxfp8(q, s)[0]
    assert d[0] == 96                       # 400 is halfway between 384 and 416: the even mantissa (384)
    assert d[1] == 1.0
    assert d[2] == 3.0                      # 12.5 = halfway between 12 and 13: nearest even mantissa -> 12
    assert d[3] == 3.5                      # 13.5 = halfway between 13 and 14 -> 14
    assert q[0, 4] == 0x80                  # signed zero keeps its sign
    assert d[5] == 3 * 2.0 ** -11           # scaled 3 * 2^-9: the E4M3 subnormal code 3
    assert d[6] == 0                        # scaled 2^-10: halfway between 0 and 2^-9, rounds to the even 0
    # Saturation: within a block the max maps to [256, 512); values are never above 448.
    y = np.zeros((1, 32), np.float32)
    y[0, 0] = 1.9375 * 2.0 ** 10            # -> 1.9375 * 2^8 = 496 > 448: saturates
    q2, s2 = oracle.quantize_mxfp8(bf(y))
    assert s2[0, 0] == 127 + 2 and oracle.e4m3_decode(q2[0, 0]) == 448.0


def test_zero_block_takes_the_smallest_scale():
    q, s = oracle.quantize_mxfp8(bf(np.zeros((2, 64), np.float32)))
    assert np.all(s == 0) and np.all(q == 0)
