"""Pins of the oracle's MXFP8 quantiser (E4M3 elements, E8M0 block scales).

The article names MXFP8 (§02) without defining it; these pins come from the OCP MX v1.0
format definition: hand-derived codes, an exhaustive nearest-value search, round trips,
and a cross-check against torch's float8_e4m3fn conversion (a library routine, used only
as a check on in-range values).
"""
import numpy as np
import pytest

from oracle import mxfp8 as mx


def _all_e4m3_values():
    codes = np.arange(256, dtype=np.uint8)
    vals = mx.e4m3_decode(codes)
    return codes, vals


@pytest.mark.parametrize("value,code", [
    (1.0, 0x38), (-1.0, 0xB8), (448.0, 0x7E), (-448.0, 0xFE), (2.0 ** -9, 0x01),
    (2.0 ** -10, 0x00),          # tie between 0 and 2**-9 -> even (0)
    (3 * 2.0 ** -10, 0x02),      # tie between 1 and 2 quanta -> even (2)
    (464.0, 0x7E),               # tie between 448 and 480 -> even (448)
    (480.0, 0x7E), (511.0, 0x7E),  # saturate
    (2.0 ** -6, 0x08),           # smallest normal
    (1.0625, 0x38),              # tie between 1.0 (m=0) and 1.125 (m=1) -> m=0
    (1.1875, 0x3A),              # tie between 1.125 (m=1) and 1.25 (m=2) -> m=2
    (0.0, 0x00), (-0.0, 0x80), (-(2.0 ** -11), 0x80),
    (7 * 2.0 ** -9, 0x07), (15 * 2.0 ** -10, 0x08),   # subnormal max, tie into the normals
    (240.0, 0x77), (256.0, 0x78),
])
def test_e4m3_hand_derived(value, code):
    assert int(mx.e4m3_encode(np.array([value]))[0]) == code


def test_e4m3_decode_table():
    codes, vals = _all_e4m3_values()
    assert np.isnan(vals[0x7F]) and np.isnan(vals[0xFF])
    pos = vals[:0x7F]
    assert pos[0] == 0 and np.all(np.diff(pos) > 0)            # strictly increasing
    assert pos[-1] == 448.0 and vals[0x01] == 2.0 ** -9
    assert np.array_equal(vals[0x80:0xFF], -vals[:0x7F])


def test_e4m3_round_trip_every_code():
    codes, vals = _all_e4m3_values()
    ok = ~np.isnan(vals)
    back = mx.e4m3_encode(vals[ok])
    assert np.array_equal(back, codes[ok])


def test_e4m3_matches_nearest_search():
    """Exhaustive nearest representable value, ties to the even code, saturating."""
    codes, vals = _all_e4m3_values()
    rep = vals[:0x7F]                      # non-negative finite values, codes 0..0x7E
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.uniform(-520, 520, 4000), rng.uniform(-0.05, 0.05, 4000),
                        rng.uniform(-2.0 ** -5, 2.0 ** -5, 2000),
                        (rep[1:] + rep[:-1]) / 2,          # exact midpoints
                        -(rep[1:] + rep[:-1]) / 2])
    got = mx.e4m3_encode(v)
    a = np.minimum(np.abs(v), 448.0)
    dist = np.abs(a[:, None] - rep[None, :])
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    # among equidistant candidates choose the even code
    even = (np.arange(0x7F) % 2 == 0)[None, :]
    pick = np.where(cand.sum(1) > 1, np.argmax(cand & even, axis=1), np.argmax(cand, axis=1))
    expect = pick.astype(np.uint8) | np.where(np.signbit(v), 0x80, 0).astype(np.uint8)
    assert np.array_equal(got, expect)


def test_e4m3_against_torch_in_range():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.uniform(-448, 448, 20000), rng.normal(0, 1, 20000),
                        rng.normal(0, 1e-2, 5000)]).astype(np.float32)
    t = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = mx.e4m3_encode(v.astype(np.float64))
    nz = v != 0
    assert np.array_equal(got[nz], t[nz])


def test_scale_rule_and_saturation():
    # amax in [256, 512) * 2**s after scaling; 2**s is the largest power with amax*2**-s < 512
    x = np.zeros((5, 32))
    x[0, 0] = 1.0          # s = -8 -> 1.0 * 2**8 = 256 exactly
    x[1, :] = 511.0        # s = 0, every element saturates to 448
    x[2, 3] = 2.0 ** 130   # s clamps to 127 - 8 = ... floor(log2) = 130 -> s = 122
    x[3, 5] = 2.0 ** -140  # s would be -148: clamps to -127
    codes, scales = mx.quantize_mx(x)
    assert scales[0, 0] == 127 - 8 and codes[0, 0] == 0x78
    assert scales[1, 0] == 127 and np.all(codes[1] == 0x7E)
    assert scales[2, 0] == 127 + 122
    assert scales[3, 0] == 0
    assert scales[4, 0] == 0 and np.all(codes[4] == 0)       # all-zero block


def test_power_of_two_block_exact_and_round_trip_bound():
    rng = np.random.default_rng(3)
    p2 = np.ldexp(1.0, rng.integers(-20, 20, (64, 32))) * rng.choice([-1, 1], (64, 32))
    p2[:, 0] = np.ldexp(1.0, 19)   # keep all elements within the E4M3 range of the block
    p2 = np.where(np.abs(p2) < 2.0 ** 2, 2.0 ** 2, p2)
    assert np.array_equal(mx.fake_quantize_mx(p2), p2)
    x = rng.normal(0, 3, (128, 256))
    codes, scales = mx.quantize_mx(x)
    xh = mx.dequantize_mx(codes, scales)
    s = np.repeat(scales.astype(np.int64) - 127, 32, axis=1)
    v = np.abs(x) * np.ldexp(1.0, -s)
    _, e2 = np.frexp(v)
    q = np.ldexp(1.0, np.maximum(e2 - 1, -6) - 3) * np.ldexp(1.0, s)
    sat = v > 448
    assert np.all(np.abs(x - xh)[~sat] <= q[~sat] / 2 + 1e-300)
    assert np.all(np.abs(xh[sat]) == 448.0 * np.ldexp(1.0, s[sat]))


def test_token_direction_quantiser_pads_with_zeros():
    rng = np.random.default_rng(4)
    x = rng.normal(size=(45, 64))
    codes, scales = mx.quantize_mx_axis0_segment(x)
    assert codes.shape == (64, 64) and scales.shape == (2, 64)
    assert np.all(codes[45:] == 0)
    ref_c, ref_s = mx.quantize_mx(np.vstack([x, np.zeros((19, 64))]).T)
    assert np.array_equal(codes, ref_c.T) and np.array_equal(scales, ref_s.T)
