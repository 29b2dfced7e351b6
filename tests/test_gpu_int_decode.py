"""GPU parity of the decode at one batch row for r = 8, 4, 2, which runs on the
integer tensor cores: the codes are u8, and the prep kernel writes each input
of a unit as the exact integer x 2^(48 - E) (E the unit's largest exponent) in
seven signed 7-bit digits, one per MMA column. Inputs more than 41 octaves
below the unit's largest, non-finite inputs, or a unit whose largest exponent
lies outside [-72, 100] send that unit down the bf16 path instead. Either way
y = x . W_r^T must hold within |y - y_ref| <= 1e-3 sum|x||W_r| + 1e-6 against
the float64 oracle, whatever the spread of the inputs."""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import check_linear, gpu_linear, gpu_pack, to_dev, weights

pytestmark = pytest.mark.gpu

WIDTHS = [8, 4, 2]


def _bf16(x: np.ndarray):
    bits = synth.bf16_bits_from_f32(np.asarray(x, dtype=np.float32))
    return bits, synth.f32_from_bf16_bits(bits).astype(np.float64)


def _run(x: np.ndarray, r: int, n=384, seed=21, law="gauss"):
    k = x.shape[1]
    _, w_vals = weights(law, n, k, seed, "bf16")
    q, a, z = oracle.quantize_minmax(w_vals)
    packed = gpu_pack(to_dev(q), r)
    bits, vals = _bf16(x)
    y = gpu_linear(bits, packed, to_dev(a), to_dev(z), n, r)
    return check_linear(y, vals, oracle.dequant_slice(q, a, z, r), f"integer path r={r} M=1")


@pytest.mark.parametrize("r", WIDTHS)
def test_gaussian_inputs(r):
    rng = np.random.default_rng(1)
    _run(rng.standard_normal((1, 4096)), r)


@pytest.mark.parametrize("r", WIDTHS)
@pytest.mark.parametrize("span", [7, 8, 20, 33, 40])
def test_inputs_spanning_many_octaves_inside_a_unit(r, span):
    """Inputs down to 2^-span of the unit's largest (at most 41 octaves: the
    digits hold them exactly, from digit 0 up to digit 6)."""
    rng = np.random.default_rng(span + 10 * r)
    k = 2048
    x = np.sign(rng.standard_normal((1, k))) * (1 + rng.random((1, k))) * 2.0 ** -rng.integers(0, span + 1, size=(1, k))
    x[0, ::128] = 4.0  # the largest of every unit sits at 2^2
    _run(x, r)


@pytest.mark.parametrize("r", WIDTHS)
@pytest.mark.parametrize("span", [42, 60, 200])
def test_units_beyond_41_octaves_take_the_bf16_path(r, span):
    rng = np.random.default_rng(100 + span + r)
    k = 2048
    x = rng.standard_normal((1, k))
    # one unit spans `span` octaves, the others stay Gaussian
    x[0, 1024:1152] *= 2.0 ** -rng.integers(0, min(span, 120) + 1, size=128)
    x[0, 1024] = 8.0
    x[0, 1100] = 8.0 * 2.0 ** -min(span, 120)
    _run(x, r)


@pytest.mark.parametrize("r", WIDTHS)
def test_zeros_subnormals_and_single_nonzero(r):
    k = 1536
    x = np.zeros((1, k))
    x[0, 3] = 1.0                               # one input
    x[0, 512 + 7] = 2.0 ** -130                 # bf16 subnormals only
    x[0, 512 + 100] = -3 * 2.0 ** -133
    x[0, 1024 + 5] = -2.0 ** -120               # a normal next to subnormals
    x[0, 1024 + 9] = 2.0 ** -133
    _run(x, r)


@pytest.mark.parametrize("r", WIDTHS)
@pytest.mark.parametrize("e", [-90, -74, -70, 90, 105])
def test_extreme_scales(r, e):
    """Units whose largest input is near the ends of the bf16 range: inside
    [2^-72, 2^100] the digit weights stay normal fp32; outside, the unit falls
    back to the bf16 path."""
    rng = np.random.default_rng(7)
    x = rng.standard_normal((1, 1024)) * 2.0 ** e
    _run(x, r, n=200)


@pytest.mark.parametrize("r", WIDTHS)
def test_inputs_on_every_bf16_significand(r):
    """Every 8-bit significand at several exponents, so every digit pattern
    and both signs occur."""
    sig = 1.0 + np.arange(128) / 128.0
    x = np.concatenate([sig * 2.0 ** e for e in (-20, -9, -3, 0, 5, 13)])[None, :]
    x[0, 1::2] *= -1
    _run(x, r, n=256)


@pytest.mark.parametrize("r", WIDTHS)
def test_heavy_tailed_weights_ragged_rows(r):
    rng = np.random.default_rng(3)
    _run(rng.standard_normal((1, 14336)), r, n=1000, seed=301, law="t")
