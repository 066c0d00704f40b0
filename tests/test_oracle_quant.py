"""Pins of the oracle's per-token, per-group quantiser (SPECTRA technical summary,
"SPECTRA pipeline" stage 3: tokens are projected down and quantised per token;
fp16 min-max scale and zero per group, round half to even)."""
import itertools
import struct

import numpy as np
import pytest

import oracle


def _f32(v: float) -> float:
    return struct.unpack("<f", struct.pack("<f", v))[0]


def _f16(v: float) -> float:
    v = max(-65504.0, min(65504.0, v))
    return float(np.float16(v))  # float64 -> float16 rounds once, to nearest even


def _python_route(x, b):
    """Second route: Python fp64 arithmetic rounded to fp32 after every op.

    Rounding an exact fp64 sum or quotient of two fp32 values to fp32 gives the
    correctly rounded fp32 result (53 >= 2*24 + 2), so this reproduces IEEE fp32
    arithmetic without numpy's float32 kernels.
    """
    x = [_f32(float(v)) for v in x]
    mn, mx = min(x), max(x)
    rng = _f32(mx - mn)
    s = _f16(_f32(rng / float(2 ** b - 1)))
    z = _f16(mn)
    if s == 0.0:
        return [0] * len(x), s, z
    out = []
    for v in x:
        t = _f32(_f32(v - z) / s)
        k = round(t)  # Python round(): half to even
        out.append(int(min(max(k, 0), 2 ** b - 1)))
    return out, s, z


@pytest.mark.parametrize("b", [1, 2, 3, 4, 8])
def test_matches_python_fp32_route(b):
    rng = np.random.default_rng(b)
    for scale in (1e-3, 1.0, 37.0):
        x = (rng.standard_normal((200, 16)) * scale).astype(np.float32)
        codes, s, z = oracle.quantize_groups(x, b)
        for i in range(x.shape[0]):
            c2, s2, z2 = _python_route(x[i], b)
            assert list(codes[i]) == c2
            assert float(s[i]) == s2 and float(z[i]) == z2


def test_round_half_to_even_on_exact_ties():
    # s = 1 and z = 0 exactly; x - z = k + 0.5 exactly -> even neighbour
    x = np.array([[0.0, 0.5, 1.5, 2.5, 3.0, 7.0, 4.5, 5.5]], dtype=np.float32)
    codes, s, z = oracle.quantize_groups(x, 3)
    assert float(s[0]) == 1.0 and float(z[0]) == 0.0
    assert list(codes[0]) == [0, 0, 2, 2, 3, 7, 4, 6]


@pytest.mark.parametrize("g,b", [(2, 1), (3, 2), (4, 2), (3, 3), (4, 3)])
def test_brute_force_best_codes(g, b):
    """On the grid {z + k s}, the codes minimise ||x - x_hat||^2 (nearest point)."""
    rng = np.random.default_rng(10 * g + b)
    x = (rng.standard_normal((300, g)) * 3).astype(np.float32)
    codes, s, z = oracle.quantize_groups(x, b)
    for i in range(x.shape[0]):
        sf, zf = float(s[i]), float(z[i])
        if sf == 0:
            continue
        best = min(sum((float(x[i, k]) - (zf + c[k] * sf)) ** 2 for k in range(g))
                   for c in itertools.product(range(2 ** b), repeat=g))
        mine = sum((float(x[i, k]) - (zf + int(codes[i, k]) * sf)) ** 2 for k in range(g))
        assert mine <= best * (1 + 1e-9) + 1e-30


def test_one_bit_dequant_values():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((100, 16)).astype(np.float32)
    codes, s, z = oracle.quantize_groups(x, 1)
    dq = oracle.dequantize_groups(codes, s, z)
    lo = z.astype(np.float64)[:, None]
    hi = lo + s.astype(np.float64)[:, None]
    assert np.all((dq == lo) | (dq == hi))


@pytest.mark.parametrize("b", [1, 2, 3, 4, 8])
def test_endpoints(b):
    rng = np.random.default_rng(20 + b)
    x = rng.standard_normal((200, 16)).astype(np.float32)
    codes, s, z = oracle.quantize_groups(x, b)
    amin, amax = np.argmin(x, axis=1), np.argmax(x, axis=1)
    r = np.arange(x.shape[0])
    assert np.all(codes[r, amin] == 0)
    assert np.all(codes[r, amax] >= 2 ** b - 2)
    dq = oracle.dequantize_groups(codes, s, z)
    err = np.abs(dq[r, amax] - x[r, amax])
    bound = s.astype(np.float64) / 2 + (2 ** b) * np.abs(s.astype(np.float64)) * 2 ** -11 \
        + np.abs(z.astype(np.float64)) * 2 ** -11 + 1e-30
    assert np.all(err <= bound)


def test_constant_group_gives_zero_scale():
    x = np.full((3, 8), 1.2345, dtype=np.float32)
    codes, s, z = oracle.quantize_groups(x, 4)
    assert np.all(codes == 0) and np.all(s == 0)
    assert np.all(oracle.dequantize_groups(codes, s, z) == np.float64(np.float16(1.2345)))


def test_fp16_saturation():
    x = np.array([[-70000.0, 70000.0] + [0.0] * 6], dtype=np.float32)
    codes, s, z = oracle.quantize_groups(x, 1)
    assert float(z[0]) == -65504.0 and float(s[0]) == 65504.0


def test_sixteen_bit_reconstruction_bound():
    """With 16-bit widths every unclamped coordinate is within s/2 of its value
    (plus the fp32 rounding of (x - z)/s); clamped ones within s/2 plus the drift
    of the grid's top end caused by the fp16 rounding of s and z."""
    rng = np.random.default_rng(7)
    x = rng.standard_normal((500, 16)).astype(np.float32)
    codes, s, z = oracle.quantize_groups(x, 16, any_width=True)
    dq = oracle.dequantize_groups(codes, s, z)
    sf = s.astype(np.float64)[:, None]
    zf = z.astype(np.float64)[:, None]
    x64 = x.astype(np.float64)
    t = (x64 - zf) / sf
    err = np.abs(dq - x64)
    unclamped = (t <= 2 ** 16 - 1) & (t >= 0)
    tight = sf / 2 + 2.0 ** -23 * np.abs(x64 - zf) + 1e-300
    assert np.all(err[unclamped] <= np.broadcast_to(tight, err.shape)[unclamped])
    # fp16 rounding of s: half an ulp, 2^-11 relative, or 2^-25 once s is subnormal
    loose = sf / 2 + np.abs(x.min(axis=1).astype(np.float64))[:, None] * 2 ** -11 \
        + (2 ** 16) * (sf * 2 ** -11 + 2.0 ** -25)
    assert np.all(err <= loose)
