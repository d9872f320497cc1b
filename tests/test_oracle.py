"""Pins for the CPU oracle (no GPU).  Each test checks the oracle against
something other than itself: the format definitions the pages name, a library
conversion (torch's float8_e4m3fn), an independent rounding method (integer
banker's rounding per binade), closed forms, invariants and brute force."""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_act_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _fmt():
    return {r[0]: [float(v) for v in r[1:]] for r in _golden("nvfp4_format.txt")}


# ------------------------------------------------------------------ formats

def test_e2m1_grid_matches_format():
    fmt = _fmt()
    mags = [oracle.e2m1_decode(c) for c in range(8)]
    assert mags == fmt["e2m1_magnitudes"]
    for c in range(8):
        assert oracle.e2m1_decode(c | 8) == -mags[c]
    assert math.copysign(1.0, oracle.e2m1_decode(8)) == -1.0


def test_e4m3_table_matches_torch_float8():
    tab = oracle.e4m3_table()
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    both_nan = np.isnan(tab) & np.isnan(ref)
    assert np.all(both_nan | (tab == ref))
    fmt = _fmt()
    assert tab[0x7E] == fmt["e4m3_max_finite"][0]
    assert tab[0x01] == fmt["e4m3_min_subnormal"][0]
    assert np.isnan(tab[0x7F]) and np.isnan(tab[0xFF])
    assert np.all(np.diff(tab[:0x7F]) > 0)


def _torch_e4m3(v):
    return torch.tensor(np.asarray(v, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_encode_matches_torch_rounding():
    tab = oracle.e4m3_table()[:0x7F]
    mids = (tab[:-1] + tab[1:]) / 2
    vals = [np.float32(m) for m in mids]
    vals += [np.nextafter(np.float32(m), np.float32(0)) for m in mids]
    vals += [np.nextafter(np.float32(m), np.float32(1e9)) for m in mids]
    vals += list(np.float32(tab))
    rng = np.random.default_rng(5)
    vals += list((rng.uniform(0, 1, 3000) ** 6 * 463.9).astype(np.float32))
    vals += list(np.float32(2.0) ** rng.uniform(-14, 8.8, 3000).astype(np.float32))
    vals = np.array([v for v in vals if v < 464], dtype=np.float32)
    got = np.array([oracle.e4m3_encode(v) for v in vals], dtype=np.uint8)
    assert np.array_equal(got, _torch_e4m3(vals))


def test_e4m3_saturates_at_448():
    for v in [448.0, 460.0, 464.0, 1e6, float("inf")]:
        assert oracle.e4m3_encode(v) == 0x7E


def _banker_e2m1(y):
    """E2M1 value by per-binade integer banker's rounding (an independent
    method): step 0.5 below 2, 1 on [2,4), 2 on [4,6], saturate at 6."""
    a = abs(float(y))
    if a >= 6:
        v = 6.0
    elif a < 2:
        v = round(a * 2) / 2
    elif a < 4:
        v = float(round(a))
    else:
        v = round(a / 2) * 2.0
    return -v if math.copysign(1.0, y) < 0 else v


def test_e2m1_golden_ties():
    for x, want in _golden("e2m1_ties.txt"):
        got = oracle.e2m1_decode(oracle.e2m1_encode(float(x)))
        assert got == float(want) and math.copysign(1, got) == math.copysign(1, float(want)), (x, got)


def test_e2m1_encode_matches_banker_rounding():
    grid = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    pts = set()
    for a, b in zip(grid[:-1], grid[1:]):
        m = np.float32((a + b) / 2)
        pts |= {m, np.nextafter(m, np.float32(0)), np.nextafter(m, np.float32(10))}
    rng = np.random.default_rng(11)
    pts |= set(rng.uniform(0, 8, 4000).astype(np.float32))
    pts |= {np.float32(0), np.float32(1e-30), np.float32(6), np.float32(7), np.float32(1e30)}
    for p in pts:
        for y in (p, -p):
            y = np.float32(y)
            got = oracle.e2m1_decode(oracle.e2m1_encode(y))
            want = _banker_e2m1(y)
            assert got == want and math.copysign(1, got) == math.copysign(1, want), (y, got, want)


# -------------------------------------------------------------- quantizer

def _blocks(x_bits):
    return oracle.bf16_bits_to_f32(x_bits).astype(np.float64)


def _codes_unpacked(codes):
    lo = codes & 15
    hi = codes >> 4
    return np.stack([lo, hi], -1).reshape(codes.shape[0], -1)


def _values(codes_unpacked):
    return oracle.e2m1_table()[codes_unpacked]


@pytest.mark.parametrize("which", ["tiny", "student_t"])
def test_half_ulp_bound_and_saturation(which):
    if which == "tiny":
        X, _ = wl.tiny_linear(0)
    else:
        X = wl.activation_student_t(96, 512, 4)
    xb = wl.bf16_bits(X)
    codes, scales, g = oracle.quantize_tensor(xb)
    x = _blocks(xb)
    s = oracle.e4m3_table()[scales].repeat(16, axis=1)
    d = (s.astype(np.float32) * np.float32(g)).astype(np.float64)
    v = _values(_codes_unpacked(codes))
    assert np.all(scales <= 0x7E)
    ok = d > 0
    y = np.where(ok, x / np.where(ok, d, 1), 0)
    gap = np.where(np.abs(y) < 2, 0.5, np.where(np.abs(y) < 4, 1.0, 2.0))
    inside = ok & (np.abs(y) <= 6)
    err = np.abs(x - v * d)
    assert np.all(err[inside] <= 0.5 * gap[inside] * d[inside] * (1 + 2.0 ** -22))
    sat = ok & (np.abs(y) > 6)
    assert np.all(np.abs(v[sat]) == 6) and np.all(np.sign(v[sat]) == np.sign(x[sat]))


def test_amax_element_is_six_at_scale_448():
    """With g = amax / 2688 the element holding the tensor amax lands on the
    top of both grids: scale 448 and code +-6."""
    for seed in range(6):
        X = wl.activation_normal(32, 128, seed, n_outliers=2, scale=37.0 + seed)
        xb = wl.bf16_bits(X)
        codes, scales, g = oracle.quantize_tensor(xb)
        x = _blocks(xb)
        r, k = np.unravel_index(np.argmax(np.abs(x)), x.shape)
        assert scales[r, k // 16] == 0x7E
        c = _codes_unpacked(codes)[r, k]
        assert c & 7 == 7 and (c >> 3) == (x[r, k] < 0)
        assert g == np.float32(np.float32(np.abs(x).max()) / np.float32(2688))


def test_zero_tensor_and_zero_blocks():
    x = np.zeros((4, 64), dtype=np.float32)
    x[1, :] = -0.0
    xb = wl.bf16_bits(wl.to_bf16(x))
    codes, scales, g = oracle.quantize_tensor(xb)
    assert g == 1.0
    assert np.all(scales == 0)
    c = _codes_unpacked(codes)
    assert np.all(c[0] == 0) and np.all(c[1] == 8)
    # one live block, the rest zero: zero blocks get scale 0 and +-0 codes
    x = np.zeros((2, 64), dtype=np.float32)
    x[0, 20] = 3.0
    codes, scales, g = oracle.quantize_tensor(wl.bf16_bits(wl.to_bf16(x)))
    assert scales[0, 1] == 0x7E and np.count_nonzero(scales) == 1


def test_packing_low_nibble_first():
    x = np.zeros((1, 16), dtype=np.float32)
    x[0, :4] = [6.0, -0.5, 1.0, -3.0]
    g = np.float32(1.0 / 448.0)
    codes, scales = oracle.quantize(wl.bf16_bits(wl.to_bf16(x)), g)
    d = np.float32(np.float32(oracle.e4m3_decode(scales[0, 0])) * g)
    c = _codes_unpacked(codes)[0]
    for k in range(4):
        assert oracle.e2m1_decode(c[k]) == _banker_e2m1(np.float32(np.float32(x[0, k]) / d))
    assert codes[0, 0] == (c[0] | (c[1] << 4)) and codes[0, 0] == (7 | (9 << 4))
    assert codes[0, 1] == (c[2] | (c[3] << 4))


def test_exhaustive_bf16_against_numpy_pipeline():
    """Every finite bf16 value, placed in blocks whose amax is fixed by a pivot
    element, against the scale/element pipeline recomputed with numpy fp32
    arithmetic, torch's E4M3 conversion and banker's rounding."""
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = oracle.bf16_bits_to_f32(allbits)
    finite = np.isfinite(vals)
    for pivot, g in [(448.0, 1.0), (6.0, 1.0), (3.0, 0.01), (1e-3, 1e-6), (100.0, 0.3), (2.0 ** -20, 2.0 ** -30)]:
        pivot = np.float32(pivot)
        g = np.float32(g)
        sel = allbits[finite & (np.abs(vals) <= pivot)]
        n = len(sel)
        nblk = (n + 14) // 15
        blk = np.zeros((nblk, 16), dtype=np.uint16)
        blk[:, 0] = wl.bf16_bits(wl.to_bf16(np.array([pivot])))[0]
        flat = np.zeros(nblk * 15, dtype=np.uint16)
        flat[:n] = sel
        blk[:, 1:] = flat.reshape(nblk, 15)
        codes, scales = oracle.quantize(blk, g)
        s32 = np.float32(np.float32(pivot / np.float32(6)) / g)
        if s32 < 464:
            assert np.all(scales == _torch_e4m3([s32])[0])
        else:
            assert np.all(scales == 0x7E)
        s = np.float32(oracle.e4m3_decode(int(scales[0, 0])))
        d = np.float32(s * g)
        xs = oracle.bf16_bits_to_f32(blk)
        c = _codes_unpacked(codes)
        tab = oracle.e2m1_table()
        got = tab[c]
        if d == 0:
            assert np.all((c & 7) == 0)
            continue
        y = (xs / d).astype(np.float32)
        want = np.vectorize(_banker_e2m1)(y)
        assert np.array_equal(got, want)
        assert np.array_equal(np.signbit(got), np.signbit(want))


def _e4m3_of_f32(s32: np.ndarray) -> np.ndarray:
    """E4M3 byte of non-negative fp32 values: torch's round-to-nearest-even
    conversion below 464 (the midpoint above 448), 448 (0x7E) from there."""
    out = np.full(s32.shape, 0x7E, dtype=np.uint8)
    low = s32 < 464
    out[low] = _torch_e4m3(s32[low])
    return out


def test_scale_byte_follows_the_r2_operation_order():
    """The block scale byte is E4M3(fl32(fl32(bamax / 6) / g)) (R2).  Global
    scales are chosen so that the scale lands within a few fp32 ulps of an
    E4M3 rounding midpoint, where forming it as bamax / fl32(6 g) instead
    rounds to the other neighbour for some pairs; every pair is checked on
    a block with one live element against numpy fp32 arithmetic and torch's
    E4M3 conversion."""
    rng = np.random.default_rng(5)
    tab = oracle.e4m3_table()[:0x7F].astype(np.float64)
    mids = ((tab[:-1] + tab[1:]) / 2)[8:]                    # normal-range midpoints
    b_bits = rng.integers(0x3C00, 0x4700, 400).astype(np.uint16)  # bf16 block amax, ~2^-7 .. 2^15
    bam = oracle.bf16_bits_to_f32(b_bits).astype(np.float32)
    pairs_b, pairs_g = [], []
    for m in mids:
        t = (bam / np.float32(6)).astype(np.float32)
        g0 = (t / np.float32(m)).astype(np.float32)
        for g in (g0, np.nextafter(g0, np.float32(0)), np.nextafter(g0, np.float32(np.inf))):
            ok = np.isfinite(g) & (g > 0)
            pairs_b.append(b_bits[ok])
            pairs_g.append(g[ok])
    pb = np.concatenate(pairs_b)
    pg = np.concatenate(pairs_g).astype(np.float32)
    bv = oracle.bf16_bits_to_f32(pb).astype(np.float32)
    s32 = ((bv / np.float32(6)).astype(np.float32) / pg).astype(np.float32)
    alt = (bv / (np.float32(6) * pg).astype(np.float32)).astype(np.float32)
    want = _e4m3_of_f32(s32)
    discriminating = want != _e4m3_of_f32(alt)
    assert discriminating.sum() > 0  # the pairs do tell the two orders apart
    pick = np.unique(np.concatenate([np.flatnonzero(discriminating), rng.integers(0, len(pb), 2000)]))
    for i in pick:
        blk = np.zeros((1, 16), dtype=np.uint16)
        blk[0, 3] = pb[i]
        _, scales = oracle.quantize(blk, pg[i])
        assert scales[0, 0] == want[i], (hex(pb[i]), float(pg[i]))


def test_on_grid_blocks_are_reproduced_exactly():
    """g = 1 and blocks whose largest code is 6: quantize(dequant(q)) == q
    and the reconstruction error is zero (scale identity)."""
    rng = np.random.default_rng(3)
    rows, K = 8, 256
    codes_u = rng.integers(0, 16, size=(rows, K))
    codes_u[:, ::16] = rng.choice([7, 15], size=(rows, K // 16))  # max |code| = 6 in each block
    sbytes = rng.integers(0x20, 0x60, size=(rows, K // 16)).astype(np.uint8)
    v = oracle.e2m1_table()[codes_u] * oracle.e4m3_table()[sbytes].repeat(16, axis=1)
    xb = wl.bf16_bits(wl.to_bf16(v))
    assert np.array_equal(oracle.bf16_bits_to_f32(xb).astype(np.float64), v)  # exactly representable
    codes, scales = oracle.quantize(xb, np.float32(1.0))
    assert np.array_equal(scales, sbytes)
    cu = _codes_unpacked(codes)
    # +0 / -0 codes may differ only in the sign of zero values, which round-trip as signed zeros
    assert np.array_equal(oracle.e2m1_table()[cu], oracle.e2m1_table()[codes_u])
    assert np.array_equal(oracle.dequant(codes, scales, 1.0), v)


# ------------------------------------------------------- scale-factor layout

def test_sf_layout_is_bijection_of_512_byte_tiles():
    # (300, 80) and (260, 48): several row tiles with K / 16 not a multiple
    # of 4, where the padded K-tile count sets the row tiles' stride
    for rows, K in [(1, 64), (130, 256), (256, 320), (64, 16), (300, 80), (260, 48)]:
        total = oracle.sf_bytes(rows, K)
        rpad = (rows + 127) // 128 * 128
        cpad = (K // 16 + 3) // 4 * 4
        assert total == rpad * cpad
        seen = np.zeros(total, dtype=np.int64)
        for r in range(rpad):
            for c in range(cpad):
                seen[oracle.sf_offset(r, c, K)] += 1
        assert np.all(seen == 1)
        # four consecutive blocks of one row share one 4-byte word
        for r in (0, 37, rpad - 1):
            base = oracle.sf_offset(r, 0, K)
            assert base % 4 == 0
            assert [oracle.sf_offset(r, c, K) for c in range(4)] == [base + i for i in range(4)]


def _documented_sf_positions(rows, K):
    """Byte position of every logical scale (r, c) in the block-scaled MMA's
    scale layout, built the way NVIDIA's cuBLAS documentation describes it
    (section "1D Block Scaling Factors Layout"): pad the [rows, K/16] scale
    matrix to whole 128 x 4 tiles; store the tiles one after another, K-tiles
    fastest, 512 bytes each; inside a tile, split the 128 rows into four
    groups of 32 and interleave them, so that 16 consecutive bytes hold the
    4 scales of rows j, j+32, j+64 and j+96.  Expressed here with array
    reshapes, not with the oracle's modular arithmetic."""
    rpad = (rows + 127) // 128 * 128
    cpad = (K // 16 + 3) // 4 * 4
    idx = np.arange(rpad * cpad).reshape(rpad, cpad)            # logical position ids
    tiles = idx.reshape(rpad // 128, 128, cpad // 4, 4).transpose(0, 2, 1, 3)
    inter = tiles.reshape(rpad // 128, cpad // 4, 4, 32, 4).transpose(0, 1, 3, 2, 4)
    stored = inter.reshape(-1)                                   # stored[byte] = logical id
    pos = np.empty_like(stored)
    pos[stored] = np.arange(stored.size)
    return pos.reshape(rpad, cpad)


def test_sf_layout_matches_documented_interleave():
    for rows, K in [(1, 64), (128, 64), (130, 256), (300, 1344), (64, 16), (300, 80), (260, 48)]:
        pos = _documented_sf_positions(rows, K)
        got = np.array([[oracle.sf_offset(r, c, K) for c in range(pos.shape[1])] for r in range(pos.shape[0])])
        assert np.array_equal(got, pos), (rows, K)
    # the documented example: row 33, block 2 sits in the second 16-byte group
    # at the second 4-byte slot
    assert oracle.sf_offset(33, 2, 64) == 1 * 16 + 1 * 4 + 2


def test_swizzle_roundtrip():
    rng = np.random.default_rng(9)
    for rows, K in [(200, 320), (64, 256), (5, 16)]:
        logical = rng.integers(0, 127, size=(rows, K // 16)).astype(np.uint8)
        sw = oracle.swizzle(logical, K)
        assert np.array_equal(oracle.unswizzle(sw, rows, K), logical)
        mask = np.zeros_like(sw, dtype=bool)
        for r in range(rows):
            for c in range(K // 16):
                mask[oracle.sf_offset(r, c, K)] = True
        assert np.all(sw[~mask] == 0)


# --------------------------------------------------------------------- GEMM

def _int_codes(rng, shape):
    # codes for 0, +-1, +-2, +-4
    return rng.choice([0, 2, 4, 6, 10, 12, 14], size=shape)


def _pack(cu):
    return (cu[:, 0::2] | (cu[:, 1::2] << 4)).astype(np.uint8)


def test_gemm_exact_integer_case():
    rng = np.random.default_rng(1)
    M, N, K = 24, 40, 128
    ca, cw = _int_codes(rng, (M, K)), _int_codes(rng, (N, K))
    one = 0x38  # E4M3 1.0
    sa = np.full((M, K // 16), one, np.uint8)
    sw = np.full((N, K // 16), one, np.uint8)
    ia = oracle.e2m1_table()[ca].astype(np.int64)
    iw = oracle.e2m1_table()[cw].astype(np.int64)
    want = ia @ iw.T
    C, B = oracle.linear_full(_pack(ca), sa, 1.0, _pack(cw), sw, np.float32(1.0))
    assert np.array_equal(C, want.astype(np.float64))
    assert np.array_equal(B, (np.abs(ia) @ np.abs(iw).T).astype(np.float64))
    ms, ns = rng.integers(0, M, 50), rng.integers(0, N, 50)
    Cs, Bs = oracle.linear_sampled(_pack(ca), sa, 1.0, _pack(cw), sw, np.float32(1.0), ms, ns)
    assert np.array_equal(Cs, want[ms, ns].astype(np.float64))


def test_gemm_selector_weights_pick_columns():
    """W with one code-1 entry per row selects a column of A^, times g_w."""
    X, _ = wl.tiny_linear(0)
    ca, sa, ga = oracle.quantize_tensor(wl.bf16_bits(X))
    M, K = X.shape
    N = 32
    picks = np.random.default_rng(2).integers(0, K, N)
    cw = np.zeros((N, K), dtype=np.int64)
    cw[np.arange(N), picks] = 2  # value 1.0
    sw = np.full((N, K // 16), 0x38, np.uint8)
    gw = np.float32(0.125)
    C, _ = oracle.linear_full(ca, sa, ga, _pack(cw), sw, gw)
    A = oracle.dequant(ca, sa, ga)
    assert np.array_equal(C, A[:, picks] * float(gw))


def test_sampled_matches_full_and_bound_dominates():
    X, W = wl.tiny_linear(0)
    ca, sa, ga = oracle.quantize_tensor(wl.bf16_bits(X))
    cw, sw, gw = oracle.quantize_tensor(wl.bf16_bits(W))
    C, B = oracle.linear_full(ca, sa, ga, cw, sw, gw)
    assert np.all(B >= np.abs(C))
    rng = np.random.default_rng(0)
    ms, ns = rng.integers(0, 64, 200), rng.integers(0, 128, 200)
    Cs, Bs = oracle.linear_sampled(ca, sa, ga, cw, sw, gw, ms, ns)
    assert np.allclose(Cs, C[ms, ns], rtol=1e-12, atol=1e-12 * B[ms, ns].max())
    assert np.allclose(Bs, B[ms, ns], rtol=1e-12)
    # the quantized GEMM stays near the bf16 product (NVFP4 error, a loose sanity check)
    ref = oracle.bf16_bits_to_f32(wl.bf16_bits(X)).astype(np.float64) @ \
        oracle.bf16_bits_to_f32(wl.bf16_bits(W)).astype(np.float64).T
    rel = np.linalg.norm(C - ref) / np.linalg.norm(ref)
    assert rel < 0.25


def test_fused_equals_per_module_and_mismatch_factor():
    """Per-segment global scales: the fused weight quantizes exactly like its
    modules one by one, and its GEMM is their concatenation.  Using the first
    module's scale for every segment (the fused-kernel mismatch) scales
    segment m by exactly g_0 / g_m."""
    rng = np.random.default_rng(4)
    K = 128
    widths, sig = [24, 40, 8], [0.005, 0.05, 0.02]
    parts = [wl.weight_normal(w, K, s, 10 + i) for i, (w, s) in enumerate(zip(widths, sig))]
    Wf = torch.cat(parts, 0)
    segs = wl.segments_from_widths(widths)
    cf, sf, gseg = oracle.quantize_segments(wl.bf16_bits(Wf), segs)
    X = wl.activation_normal(16, K, 7)
    ca, sa, ga = oracle.quantize_tensor(wl.bf16_bits(X))
    grow = oracle.rows_scale(segs, gseg, Wf.shape[0])
    Cf, _ = oracle.linear_full(ca, sa, ga, cf, sf, grow)
    for (a, b), p in zip(segs, parts):
        cm, sm, gm = oracle.quantize_tensor(wl.bf16_bits(p))
        assert np.array_equal(cm, cf[a:b]) and np.array_equal(sm, sf[a:b])
        Cm, _ = oracle.linear_full(ca, sa, ga, cm, sm, gm)
        assert np.array_equal(Cm, Cf[:, a:b])
    assert len(set(gseg.tolist())) == 3
    Cbad, _ = oracle.linear_full(ca, sa, ga, cf, sf, np.float32(gseg[0]))
    for (a, b), gm in zip(segs, gseg):
        ratio = float(np.float32(gseg[0])) / float(np.float32(gm))
        assert np.allclose(Cbad[:, a:b], Cf[:, a:b] * ratio, rtol=1e-12, atol=0)


# ---------------------------------------------------------------- SwiGLU

def test_double_to_bf16_matches_torch_on_fp32_values():
    rng = np.random.default_rng(8)
    v = np.concatenate([rng.standard_normal(3000) * 10.0 ** rng.uniform(-30, 30, 3000),
                        [0.0, -0.0, 1e-40, -3e-39, 3.3e38]]).astype(np.float32)
    want = wl.bf16_bits(torch.from_numpy(v).to(torch.bfloat16))
    got = np.array([oracle.double_to_bf16(float(x)) for x in v], dtype=np.uint16)
    assert np.array_equal(got, want)


def test_double_to_bf16_ties_go_to_even():
    """fp32 values exactly halfway between two bf16 neighbours (low 16 bits
    0x8000), over every exponent, both signs and both parities of the bf16
    mantissa's last bit, subnormals included: round to the even neighbour,
    as torch's fp32 -> bf16 conversion does."""
    hi = np.arange(0, 0x7F7F, dtype=np.uint32)                   # every finite bf16 magnitude below the top
    bits = np.concatenate([hi, hi | 0x8000]) << 16 | 0x8000
    v = bits.astype(np.uint32).view(np.float32)
    want = wl.bf16_bits(torch.from_numpy(v.copy()).to(torch.bfloat16))
    got = np.array([oracle.double_to_bf16(float(x)) for x in v], dtype=np.uint16)
    assert np.array_equal(got, want)
    assert np.all((got & 1) == 0)                                # the even neighbour every time


def test_swiglu_against_torch_float64():
    rng = np.random.default_rng(6)
    gu = wl.to_bf16(rng.standard_normal((8, 64)) * 3)
    h = oracle.swiglu(wl.bf16_bits(gu))
    g = gu[:, :32].double()
    u = gu[:, 32:].double()
    ref = (torch.nn.functional.silu(g) * u).numpy()
    hv = oracle.bf16_bits_to_f32(h).astype(np.float64)
    # within half a bf16 ulp of the fp64 value
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-38))) - 7)
    assert np.all(np.abs(hv - ref) <= 0.5 * ulp * (1 + 1e-9))
    assert np.all(hv[gu[:, :32].float().numpy() == 0] == 0)


# ------------------------------------------------- gated MLP weight layout

def test_gated_layout_alternates_gate_and_up_blocks():
    F = 384
    rows = [oracle.gated_stored_row(r, F) for r in range(2 * F)]
    assert sorted(rows) == list(range(2 * F))                     # a permutation
    assert rows[0] == 0 and rows[127] == 127 and rows[128] == 256  # gate blocks at even 128-row slots
    assert rows[F] == 128 and rows[F + 127] == 255 and rows[2 * F - 1] == 2 * F - 1  # up blocks at odd slots
    data = np.arange(2 * F)
    inter = oracle.interleave_gate_up(data, F)
    for t in range(2 * F // 256):
        assert np.array_equal(inter[256 * t: 256 * t + 128], data[128 * t: 128 * t + 128])
        assert np.array_equal(inter[256 * t + 128: 256 * t + 256], data[F + 128 * t: F + 128 * t + 128])


def test_silu_mul_against_torch():
    rng = np.random.default_rng(17)
    g = rng.standard_normal(1000) * 8
    u = rng.standard_normal(1000)
    ref = (torch.nn.functional.silu(torch.from_numpy(g)) * torch.from_numpy(u)).numpy()
    assert np.allclose(oracle.silu_mul(g, u), ref, rtol=1e-14, atol=1e-300)
    assert oracle.silu_mul(0.0, 3.0) == 0.0
