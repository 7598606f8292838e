"""Pins of the oracle's quantized radius (levels uniform on [0, thr], L = 24 S,
b-bit codes packed like the indices) against brute force, closed forms and
the already-pinned fp16-radius decode."""
import numpy as np
import pytest


def all_f16_up_to(limit):
    """Every non-negative finite fp16 bit pattern whose value is <= limit."""
    bits = np.arange(0, 0x7C00, dtype=np.uint16)
    vals = bits.view(np.float16).astype(np.float64)
    return bits[vals <= limit], vals[vals <= limit]


@pytest.mark.parametrize("S,thr", [(8, 3.0), (32, 5.4972), (1, 0.37), (3, 1000.25)])
def test_level_is_the_nearest_grid_point(oracle, S, thr):
    """Brute force over every fp16 radius up to 1.2 thr: the level is the
    nearest point of the decoded grid k * delta (within one fp32 rounding of a
    tie), and radii at or above thr take the top level."""
    L = 24 * S
    thr = float(np.float32(thr))
    grid = np.array([oracle.radius_of_level(k, thr, S) for k in range(L)])
    bits, vals = all_f16_up_to(1.2 * thr)
    sample = np.linspace(0, len(bits) - 1, min(len(bits), 6000)).astype(int)
    delta = thr / (L - 1)
    for bi, v in zip(bits[sample], vals[sample]):
        k = oracle.radius_level(bi, thr, S)
        assert 0 <= k < L
        if v >= thr:
            assert k == L - 1
            continue
        d = np.abs(v - grid)
        assert d[k] <= d.min() + 1e-6 * delta, (v, k, int(np.argmin(d)))
        assert abs(v - grid[k]) <= 0.5 * delta * (1 + 1e-5) + 1e-7 * thr


def test_end_points_nan_and_degenerate_thresholds(oracle):
    S, L = 8, 192
    assert oracle.radius_level(0x0000, 3.0, S) == 0
    assert oracle.radius_level(0x4200, 3.0, S) == L - 1              # 3.0 exactly
    assert oracle.radius_level(0x7BFF, 3.0, S) == L - 1              # 65504
    assert oracle.radius_level(0x7E00, 3.0, S) == 0                  # NaN radius
    for thr in (0.0, -1.0, float("inf"), float("nan")):
        assert oracle.radius_level(0x3C00, thr, S) == 0
        assert oracle.radius_of_level(5, thr, S) == 0.0
    assert oracle.radius_of_level(0, 3.0, S) == 0.0


def test_levels_are_monotone(oracle):
    bits, vals = all_f16_up_to(10.0)
    ks = np.array([oracle.radius_level(b_, 7.25, 32) for b_ in bits[::7]])
    assert np.all(np.diff(ks) >= 0)


def test_packing_matches_an_independent_unpack(oracle):
    rng = np.random.default_rng(0)
    B, H, T, D, S = 2, 3, 64, 128, 32
    b = oracle.index_bits(S)
    thr = np.array([2.0, 0.5, 9.0], np.float32)
    r = (rng.random(B * H * T * D // 4) * 10).astype(np.float16).view(np.uint16)
    words = oracle.quantize_radius(r, thr, B, H, T, D, S)
    assert words.size == B * H * T * D // 128 * b
    w = words.reshape(-1, b)
    bitsarr = np.unpackbits(w.view(np.uint8), bitorder="little").reshape(w.shape[0], 32, b)
    codes = (bitsarr.astype(np.uint32) << np.arange(b, dtype=np.uint32)).sum(2).reshape(-1)
    heads = (np.arange(r.size) // (T * D // 4)) % H
    want = np.array([oracle.radius_level(r[j], thr[heads[j]], S) for j in range(r.size)])
    np.testing.assert_array_equal(codes, want)


def test_decode_on_the_grid_equals_the_fp16_radius_decode(oracle):
    """With delta a power of two, radii k * delta are exact fp16 values, their
    level is k and the decoded radius is the radius itself: the
    quantized-radius decode equals the pinned fp16-radius decode bit for bit
    (both granularities' lists included)."""
    rng = np.random.default_rng(1)
    B, H, T, D, S = 1, 2, 32, 128, 8
    L = 24 * S
    thr = np.full(H, (L - 1) * 2.0 ** -6, np.float32)           # delta = 2^-6 exactly
    n = B * H * T * D // 4
    k = rng.integers(0, L, n)
    radius = (k * 2.0 ** -6).astype(np.float16).view(np.uint16)
    idx = rng.integers(0, 24 * S, n).astype(np.uint32)
    b = oracle.index_bits(S)
    words = np.zeros(n // 32 * b, np.uint32)
    for j in range(n):                                            # LSB-first packing, by hand
        for i in range(b):
            if (idx[j] >> i) & 1:
                bit = (j % 32) * b + i
                words[(j // 32) * b + bit // 32] |= np.uint32(1 << (bit % 32))
    cb = oracle.make_codebook(3, S, H)
    rw = oracle.quantize_radius(radius, thr, B, H, T, D, S)
    for gran, out_idx, out_val in ((0, np.array([5, 77], np.uint32),
                                    rng.integers(0, 0x7000, (2, 4)).astype(np.uint16)),
                                   (1, np.array([9, 301], np.uint32),
                                    rng.integers(0, 0x7000, 2).astype(np.uint16))):
        for dt in (oracle.BF16, oracle.F32):
            y0, _ = oracle.decode(words, radius, cb, S, B, H, T, D, out_idx, out_val, gran, dt)
            y1, _ = oracle.decode_qradius(words, rw, thr, cb, S, B, H, T, D, out_idx, out_val,
                                          gran, dt)
            np.testing.assert_array_equal(y0.view(np.uint8), y1.view(np.uint8))
