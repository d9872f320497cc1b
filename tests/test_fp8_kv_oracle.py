"""Pins of the oracle's FP8 (E4M3) KV-cache codec against what the format and
the arithmetic fix: exact representables round-trip, the half-spacing bound
(spacing from the E4M3 exponent/mantissa definition, not from the oracle's
tables), ties to the even mantissa, saturation at +-448, signed zero,
monotonicity, and the calibrated scale's closed forms."""
import math

import numpy as np

import oracle


def _spacing(a: float) -> float:
    """Gap between adjacent E4M3 magnitudes around a (|a| <= 448): 3 mantissa
    bits, exponent bias 7, subnormals below 2^-6 spaced 2^-9."""
    a = abs(a)
    if a < 2.0 ** -6:
        return 2.0 ** -9
    return 2.0 ** (math.floor(math.log2(a)) - 3)


def _finite_bytes():
    return [b for b in range(256) if (b & 0x7F) != 0x7F]


def test_representables_round_trip():
    for b in _finite_bytes():
        v = oracle.e4m3_decode(b)
        assert oracle.e4m3_encode_signed(v) == b, hex(b)


def test_half_spacing_bound_and_sign():
    rng = np.random.default_rng(7)
    ys = np.concatenate([rng.uniform(-448, 448, 4000), rng.normal(0, 0.05, 4000),
                         rng.uniform(-2 ** -6, 2 ** -6, 2000)]).astype(np.float32)
    for y in ys:
        b = oracle.e4m3_encode_signed(float(y))
        v = oracle.e4m3_decode(b)
        assert abs(v - float(y)) <= 0.5 * _spacing(float(y)) * (1 + 2 ** -20), (y, hex(b))
        assert (b >> 7) == int(np.signbit(y))


def test_ties_go_to_even_mantissa():
    mags = sorted(oracle.e4m3_decode(b) for b in range(0x7F))
    for lo, hi in zip(mags[:-1], mags[1:]):
        mid = np.float32((lo + hi) / 2)
        if float(mid) != (lo + hi) / 2:
            continue  # midpoint not representable in fp32 (never here, but be safe)
        b = oracle.e4m3_encode_signed(float(mid))
        assert b & 1 == 0, (lo, hi, hex(b))
        assert oracle.e4m3_decode(b) in (lo, hi)
        assert oracle.e4m3_encode_signed(-float(mid)) == (b | 0x80)


def test_saturation_and_zero():
    for y in (448.0, 449.0, 480.0, 1e6, 3.0e38):
        assert oracle.e4m3_encode_signed(y) == 0x7E
        assert oracle.e4m3_encode_signed(-y) == 0xFE
    assert oracle.e4m3_encode_signed(0.0) == 0x00
    assert oracle.e4m3_encode_signed(-0.0) == 0x80
    # below half the smallest subnormal (2^-10): rounds to zero, sign kept
    assert oracle.e4m3_encode_signed(2.0 ** -11) == 0x00
    assert oracle.e4m3_encode_signed(-(2.0 ** -11)) == 0x80
    # exactly half the smallest subnormal is a tie: zero (even) wins
    assert oracle.e4m3_encode_signed(2.0 ** -10) == 0x00


def test_monotone():
    ys = np.sort(np.random.default_rng(3).uniform(-500, 500, 5000).astype(np.float32))
    vals = [oracle.e4m3_decode(oracle.e4m3_encode_signed(float(y))) for y in ys]
    assert all(a <= b for a, b in zip(vals[:-1], vals[1:]))


def test_calibrated_scale_closed_forms():
    assert oracle.fp8_kv_scale(448.0) == 1.0
    assert oracle.fp8_kv_scale(896.0) == 2.0
    assert oracle.fp8_kv_scale(0.0) == 1.0
    a = np.float32(3.7)
    assert oracle.fp8_kv_scale(float(a)) == float(np.float32(a / np.float32(448.0)))
    # the calibrated scale maps amax onto the top of the grid
    for a in (0.01, 1.0, 37.5, 1000.0):
        s = oracle.fp8_kv_scale(a)
        b = oracle.e4m3_encode_signed(float(np.float32(np.float32(a) / np.float32(s))))
        assert b in (0x7E, 0x7D)


def test_tensor_quantize_exact_for_representables():
    """x = v * s with s a power of two and v on the E4M3 grid: every code is
    exact, so the decoded tensor times s reproduces x."""
    rng = np.random.default_rng(11)
    bytes_ = rng.choice(_finite_bytes(), size=(37, 53))
    for s in (1.0, 0.25, 8.0):
        v = np.vectorize(oracle.e4m3_decode)(bytes_)
        x = (v * s).astype(np.float32)
        x_bits = (x.view(np.uint32) >> 16).astype(np.uint16)
        # every E4M3 value has <= 4 significant bits, so x is exact in bf16
        assert np.array_equal(x_bits.astype(np.uint32) << 16, x.view(np.uint32))
        q = oracle.fp8_kv_quantize(x_bits, s)
        assert np.array_equal(np.vectorize(oracle.e4m3_decode)(q) * s, v * s)


def test_tensor_quantize_dequant_bound():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((64, 96)) * 3).astype(np.float32)
    x_bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    xb = oracle.bf16_bits_to_f32(x_bits).astype(np.float64)
    s = oracle.fp8_kv_scale(float(np.abs(xb).max()))
    q = oracle.fp8_kv_quantize(x_bits, s)
    xhat = np.vectorize(oracle.e4m3_decode)(q) * s
    y = xb / s
    bound = np.array([0.5 * _spacing(t) for t in y.ravel()]).reshape(y.shape) * s * (1 + 2 ** -20)
    assert np.all(np.abs(xhat - xb) <= bound)
