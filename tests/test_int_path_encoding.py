"""CPU checks of the integer decode path's encoding (one batch row, widths
8, 4, 2 on the u8 x s8 -> s32 tensor cores), from its definition alone:

* every bf16 input x of a unit whose exponents lie within 41 octaves of the
  unit's largest, E, is the integer X = |x| 2^(48 - E) (below 2^49) times a
  power of two, and seven signed 7-bit digits d_g = sign(x) ((X >> 7g) & 127)
  give back x exactly: sum_g d_g 2^(7g) 2^(E - 48) = x;
* the int32 sums of a unit stay below 2^24 in magnitude at every width, with
  the codes at their multiples (1, 16, 64 for r = 8, 4, 2), so their
  conversion to fp32 before the fold is exact;
* each width's K unit makes every plane row a whole number of 16-byte units.

Plain integer arithmetic; nothing here is shared with the oracle or the
library."""
import numpy as np
import pytest

import synth


def _bf16_fields(bits):
    bits = int(bits)
    sign = -1 if bits & 0x8000 else 1
    e = (bits >> 7) & 0xFF
    m = bits & 0x7F
    if e == 0:
        return sign, m, 1 - 134          # subnormal: no implicit bit
    return sign, 0x80 | m, e - 134       # x = sign * m * 2^f, m < 256


def _top_exponent(m, f):
    return f + int(m).bit_length() - 1


@pytest.mark.parametrize("seed", range(6))
def test_seven_digits_reconstruct_every_input_exactly(seed):
    rng = np.random.default_rng(seed)
    k = 512
    x = rng.standard_normal(k).astype(np.float32)
    # spread over many octaves, with exact zeros and the unit's extremes
    x *= np.float32(2.0) ** rng.integers(-30, 10, size=k).astype(np.float32)
    x[::37] = 0.0
    bits = synth.bf16_bits_from_f32(x)
    fields = [_bf16_fields(b) for b in bits]
    E = max(_top_exponent(m, f) for s, m, f in fields if m)
    for (s, m, f), b in zip(fields, bits):
        if m == 0:
            continue
        if f < E - 48:                    # beyond the window: the unit takes the bf16 path
            continue
        X = m << (f + 48 - E)
        assert X < 2 ** 49
        digits = [s * ((X >> (7 * g)) & 127) for g in range(7)]
        assert all(-127 <= d <= 127 for d in digits)
        back = sum(d * 2 ** (7 * g) for g, d in enumerate(digits))
        value = synth.f32_from_bf16_bits(np.array([b], dtype=np.uint16))[0]
        assert back * 2.0 ** (E - 48) == float(value)


def test_window_is_where_the_digits_stay_exact():
    """X = m 2^(f + 48 - E) is an integer for every significand m exactly when
    f >= E - 48; one place lower an odd m would lose its last bit, which is
    why such a unit takes the bf16 path. With 8 significant bits, the lowest
    exact input sits 48 - 7 = 41 octaves below the unit's top octave."""
    for E in (-60, 0, 90):
        for m in (1, 3, 0x81, 0xFF):
            f = E - 48
            assert (m * 2 ** (f + 48 - E)) == m                 # an integer, held by the digits
            f = E - 49
            assert (m * 2.0 ** (f + 48 - E)) % 1 != 0           # odd m: half a unit lost
        top_of_lowest = (E - 48) + 7
        assert E - top_of_lowest == 41


@pytest.mark.parametrize("r,code_multiple,codes_per_unit", [(8, 1, 128), (4, 16, 256), (2, 64, 512)])
def test_unit_sums_stay_exact_in_fp32(r, code_multiple, codes_per_unit):
    max_code = ((1 << r) - 1) * code_multiple          # the A operand byte, unsigned
    assert max_code <= 255
    worst = codes_per_unit * max_code * 127            # every digit at its largest magnitude
    assert worst < 2 ** 24, (r, worst)
    assert worst < 2 ** 31


@pytest.mark.parametrize("r,planes,unit", [(8, (8,), 32), (4, (4,), 32), (6, (4, 2), 64), (2, (2,), 64),
                                           (3, (2, 1), 128)])
def test_k_unit_gives_whole_16_byte_plane_rows(r, planes, unit):
    for k in (unit, 3 * unit, 4096 + unit):
        for b in planes:
            assert (k * b // 8) % 16 == 0, (r, k, b)
    # and a K off the unit by half would break a plane's row pitch; at r = 8
    # a byte plane only needs K % 16, and the unit is the pages' K % 32
    if r != 8:
        k = unit // 2 if unit > 32 else unit + 16
        assert any((k * b / 8) % 16 != 0 for b in planes)
