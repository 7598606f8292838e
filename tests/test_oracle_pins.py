"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these checks re-types an oracle formula: each compares the oracle
with an independent fact -- a group-theoretic identity, a textbook or library
routine (numpy sort/partition, numpy float16, torch bfloat16, complex 2x2
matrices as a model of the quaternions), a published known-answer vector, a
hand-worked example, or a figure printed on the pages (tests/golden/).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers
def cmat(q):
    """Quaternion a+bi+cj+dk as the complex 2x2 matrix [[a+bi, c+di], [-c+di, a-bi]].
    Matrix multiplication of these is the quaternion product (H is isomorphic
    to this subalgebra of M2(C)), an independent model of the Hamilton product."""
    a, b, c, d = [float(v) for v in q]
    return np.array([[a + 1j * b, c + 1j * d], [-c + 1j * d, a - 1j * b]], dtype=np.complex128)


def from_cmat(m):
    return np.array([m[0, 0].real, m[0, 0].imag, m[0, 1].real, m[0, 1].imag])


def qmul_ref(a, b):
    return from_cmat(cmat(a) @ cmat(b))


def hurwitz_units_independent():
    """The 24 Hurwitz units built from their description: the 8 quaternions
    +-1, +-i, +-j, +-k and the 16 of the form (+-1 +- i +- j +- k)/2."""
    out = []
    for a in range(4):
        for sg in (1.0, -1.0):
            v = np.zeros(4)
            v[a] = sg
            out.append(v)
    for signs in itertools.product((0.5, -0.5), repeat=4):
        out.append(np.array(signs))
    return np.array(out)


# ---------------------------------------------------------------- 2T table
def test_2t_is_the_hurwitz_unit_group(oracle):
    t = oracle.table_2t()
    ref = hurwitz_units_independent()
    # same 24 vectors (the pages: the 24 unit Hurwitz quaternions, the
    # vertices of the 24-cell, i.e. the binary tetrahedral group 2T)
    key = lambda a: sorted(map(tuple, np.round(a, 12)))
    assert key(t) == key(ref)
    assert len({tuple(v) for v in t}) == 24
    assert np.allclose(np.linalg.norm(t, axis=1), 1.0, atol=0, rtol=0)


def test_2t_closed_under_product(oracle):
    t = oracle.table_2t()
    rows = {tuple(v) for v in t}
    for a in t:
        for b in t:
            p = qmul_ref(a, b)
            assert tuple(p) in rows          # exact: entries are 0, +-1/2, +-1
            assert tuple(oracle.qmul(a, b)) in rows
    # identity and inverses (conjugates) present
    assert (1.0, 0.0, 0.0, 0.0) in rows
    for a in t:
        assert (a[0], -a[1], -a[2], -a[3]) in rows


def test_2t_min_pairwise_angle_is_60_degrees(oracle):
    t = oracle.table_2t()
    g = t @ t.T
    off = g[~np.eye(24, dtype=bool)]
    # distinct vertices: inner products only -1, -1/2, 0, 1/2
    assert set(np.round(off, 12)) == {-1.0, -0.5, 0.0, 0.5}
    assert math.degrees(math.acos(off.max())) == pytest.approx(60.0, abs=1e-12)


def test_2t_enumeration_convention(oracle):
    # p = 2a + sign for the 8 axis units, 8 + m for the 16 half units
    assert list(oracle.element_2t(0)) == [1, 0, 0, 0]
    assert list(oracle.element_2t(3)) == [0, -1, 0, 0]
    assert list(oracle.element_2t(6)) == [0, 0, 0, 1]
    assert list(oracle.element_2t(8)) == [0.5, 0.5, 0.5, 0.5]
    assert list(oracle.element_2t(8 + 0b1010)) == [0.5, -0.5, 0.5, -0.5]


# ---------------------------------------------------------------- algebra
def test_hamilton_defining_relations(oracle):
    one, i, j, k = np.eye(4)
    m1 = -one
    q = oracle.qmul
    for u in (i, j, k):
        assert np.array_equal(q(u, u), m1)
    assert np.array_equal(q(q(i, j), k), m1)
    assert np.array_equal(q(i, j), k)
    assert np.array_equal(q(j, k), i)
    assert np.array_equal(q(k, i), j)
    assert np.array_equal(q(j, i), -k)


def test_hamilton_matches_matrix_model(oracle):
    rng = np.random.default_rng(5)
    for _ in range(200):
        a, b = rng.standard_normal(4), rng.standard_normal(4)
        assert np.allclose(oracle.qmul(a, b), qmul_ref(a, b), rtol=0, atol=1e-13)


def test_left_multiplication_is_an_isometry(oracle):
    # the pages' argument for calibration-free codebooks: left multiplication
    # by a unit quaternion preserves norms and inner products on S^3
    rng = np.random.default_rng(6)
    for _ in range(200):
        q = rng.standard_normal(4)
        q /= np.linalg.norm(q)
        a, b = rng.standard_normal(4), rng.standard_normal(4)
        qa, qb = oracle.qmul(q, a), oracle.qmul(q, b)
        assert np.linalg.norm(qa) == pytest.approx(np.linalg.norm(a), rel=1e-13)
        assert qa @ qb == pytest.approx(a @ b, rel=1e-12, abs=1e-12)


def test_inner_product_identity_used_by_the_search(oracle):
    # <x, q_p q_s> = <x conj(q_s), q_p> for unit q_s: scoring the 24 products
    # of one secondary codeword reduces to scoring y = x conj(q_s) against 2T
    rng = np.random.default_rng(7)
    t = oracle.table_2t()
    for _ in range(100):
        qs = rng.standard_normal(4)
        qs /= np.linalg.norm(qs)
        x = rng.standard_normal(4)
        y = qmul_ref(x, qs * np.array([1, -1, -1, -1]))
        for qp in t:
            assert x @ qmul_ref(qp, qs) == pytest.approx(y @ qp, abs=1e-12)


def test_codeword_f32_is_the_rounded_product(oracle):
    rng = np.random.default_rng(8)
    t = oracle.table_2t()
    for _ in range(50):
        qs = rng.standard_normal(4).astype(np.float32)
        qs /= np.linalg.norm(qs)
        qs = qs.astype(np.float32)
        for p in range(24):
            c = oracle.codeword(p, qs).astype(np.float64)
            ref = qmul_ref(t[p], qs.astype(np.float64))
            # at most 3 roundings of values <= 2 in magnitude
            assert np.abs(c - ref).max() <= 3 * 2.0 ** -24 * 2
            if p < 8:  # axis units: a signed permutation, exact
                assert np.array_equal(c, ref)


# ---------------------------------------------------------------- RNG / codebook
def test_philox4x32_10_known_answers(oracle):
    # known-answer vectors published with the Philox definition (Random123)
    kat = [
        ([0, 0, 0, 0], [0, 0], [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8]),
        ([0xFFFFFFFF] * 4, [0xFFFFFFFF] * 2, [0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD]),
        ([0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344], [0xA4093822, 0x299F31D0],
         [0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1]),
    ]
    for ctr, key, want in kat:
        assert list(oracle.philox4x32_10(ctr, key)) == want


def test_codebook_unit_norm_and_deterministic(oracle):
    cb = oracle.make_codebook(1, 32, 64)
    n = np.linalg.norm(cb.astype(np.float64), axis=-1)
    assert np.abs(n - 1).max() < 2e-7
    assert np.array_equal(cb, oracle.make_codebook(1, 32, 64))
    assert not np.array_equal(cb, oracle.make_codebook(2, 32, 64))
    # a sub-range of groups is the same rows as the full draw
    assert np.array_equal(cb[10:20], oracle.make_codebook(1, 32, 10, group0=10))


def test_codebook_is_haar_uniform_on_s3(oracle):
    # a normalised Gaussian 4-vector is uniform on S^3: each coordinate w has
    # density (2/pi) sqrt(1 - w^2), so E[w] = 0, E[w^2] = 1/4, E|w| = 4/(3 pi)
    cb = oracle.make_codebook(1, 1000, 60).reshape(-1, 4).astype(np.float64)
    n = cb.shape[0]
    se = 1.0 / math.sqrt(n)
    assert np.abs(cb.mean(0)).max() < 5 * 0.5 * se
    assert np.abs((cb ** 2).mean(0) - 0.25).max() < 5 * 0.2 * se
    assert np.abs(np.abs(cb).mean(0) - 4 / (3 * math.pi)).max() < 5 * 0.27 * se
    # coordinates uncorrelated
    c = np.corrcoef(cb.T)
    assert np.abs(c - np.eye(4)).max() < 5 * se


@pytest.mark.parametrize("S", [8, 32])
def test_24S_distinct_codewords(oracle, S):
    # 24 S effective codewords from S stored parameters
    cb = oracle.make_codebook(1, S, 16)
    t = oracle.table_2t()
    for g in range(16):
        words = np.array([qmul_ref(t[p], cb[g, s].astype(np.float64))
                          for s in range(S) for p in range(24)])
        assert words.shape == (24 * S, 4)
        gram = words @ words.T
        np.fill_diagonal(gram, -2)
        assert gram.max() < 1 - 1e-9        # no two codewords coincide


# ---------------------------------------------------------------- formats
def test_f16_matches_numpy_round_to_nearest_even(oracle):
    rng = np.random.default_rng(9)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-9, 5, 20000),
        np.array([0.0, -0.0, 1.0, 65504.0, 65519.0, -65519.99, 6.1035156e-05, 5.96e-08,
                  2.98e-08, 2.9802322e-08, 8.940697e-08, 1.0009766, 1.0004883, 1.0014648,
                  2049.0, 2051.0, -3.0e-6], np.float32)])
    got, nsat = oracle.f32_to_f16_sat(vals)
    assert nsat == 0
    want = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, want)
    back = oracle.f16_to_f32(got)
    assert np.array_equal(back.view(np.uint32), want.view(np.float16).astype(np.float32).view(np.uint32))


def test_f16_saturation_and_specials(oracle):
    vals = np.array([65520.0, -1e30, np.inf, -np.inf, np.nan], np.float32)
    got, nsat = oracle.f32_to_f16_sat(vals)
    assert list(got[:4]) == [0x7BFF, 0xFBFF, 0x7C00, 0xFC00]
    assert got[4] & 0x7FFF == 0x7E00
    assert nsat == 2


def test_bf16_matches_torch(oracle):
    rng = np.random.default_rng(10)
    vals = (rng.standard_normal(50000) * 10.0 ** rng.integers(-30, 30, 50000)).astype(np.float32)
    vals = np.concatenate([vals, np.array([0.0, -0.0, 3.0e38, 3.4e38, np.inf, -np.inf], np.float32)])
    # ties: values exactly halfway between two bf16 numbers
    ties = (np.arange(1, 2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    vals = np.concatenate([vals, ties, -ties])
    got = oracle.f32_to_bf16(vals)
    want = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)
    assert np.array_equal(oracle.bf16_to_f32(got),
                          torch.from_numpy(got.view(np.int16)).view(torch.bfloat16).float().numpy())


def test_chunk_norm_error_bound(oracle):
    rng = np.random.default_rng(11)
    x = rng.standard_normal((100000, 4)).astype(np.float32)
    r = oracle.chunk_norm(x).astype(np.float64).ravel()
    ref = np.sqrt((x.astype(np.float64) ** 2).sum(1))
    ulp = np.spacing(ref.astype(np.float32)).astype(np.float64)
    err = np.abs(r - ref) / ulp
    # three roundings in r^2 (relative error <= 1.5 * 2^-24, halved by the
    # square root) plus the rounding of sqrt: at most ~1.25 ulp, typically < 0.5
    assert err.max() <= 1.5
    assert err.mean() < 0.35
    assert np.array_equal(oracle.chunk_norm(np.zeros((3, 4), np.float32)).ravel(), np.zeros(3, np.float32))


# ---------------------------------------------------------------- packing
def test_packing_worked_example_b8(oracle):
    # S=8: 24*8 = 192 codewords -> 8 bits; chunk k's index in bits 8k..8k+7
    assert oracle.index_bits(8) == 8
    words = np.array([0x03020100, 0x07060504, 0x0B0A0908, 0x0F0E0D0C,
                      0x13121110, 0x17161514, 0x1B1A1918, 0x1F1E1D1C], np.uint32)
    assert list(oracle.get_index(words, 8, np.arange(32))) == list(range(32))


def test_packing_worked_example_b10(oracle):
    # S=32: 768 codewords -> 10 bits.  Chunk 0 = 0x3FF fills bits 0..9; chunk 3
    # = 1 sets bit 30; chunk 4 = 0x201 sets bits 40 and 49 (word 1 bits 8, 17);
    # chunk 31 = 0x200 sets bit 319 (word 9 bit 31).
    assert oracle.index_bits(32) == 10
    words = np.zeros(10, np.uint32)
    words[0] = 0x3FF | (1 << 30)
    words[1] = (1 << 8) | (1 << 17)
    words[9] = 1 << 31
    idx = oracle.get_index(words, 32, np.arange(32))
    want = np.zeros(32, np.uint32)
    want[0], want[3], want[4], want[31] = 0x3FF, 1, 0x201, 0x200
    assert np.array_equal(idx, want)


@pytest.mark.parametrize("S,b", [(1, 5), (8, 8), (11, 9), (32, 10), (43, 11), (1000, 15), (65535, 21)])
def test_index_bits(oracle, S, b):
    assert oracle.index_bits(S) == b == math.ceil(math.log2(24 * S))


# ---------------------------------------------------------------- search
def _ref_pick(x, qs_head):
    """fp64 brute force over the 24 S products built with complex matrices."""
    t = hurwitz_units_independent()
    u = x.astype(np.float64) / np.linalg.norm(x.astype(np.float64))
    words = []
    for s in range(qs_head.shape[0]):
        for qp in t:
            words.append(qmul_ref(qp, qs_head[s].astype(np.float64)))
    words = np.array(words)
    sc = words @ u
    order = np.argsort(-sc)
    return words, sc, order


def test_search_matches_independent_brute_force(oracle):
    rng = np.random.default_rng(12)
    S = 8
    cb = oracle.make_codebook(3, S, 1)
    x = rng.standard_normal((1, 1, 64, 128)).astype(np.float32)
    words, radius, best, second, st = oracle.encode(x, cb, S)
    idx = oracle.get_index(words, S, np.arange(64 * 32))
    chunks = x.reshape(-1, 4)
    n_tie = 0
    for j in range(chunks.shape[0]):
        W, sc, order = _ref_pick(chunks[j], cb[0])
        c = oracle.codeword(idx[j] % 24, cb[0, idx[j] // 24]).astype(np.float64)
        picked = int(np.argmin(np.abs(W - c).sum(1)))
        gap = sc[order[0]] - sc[picked]
        if picked != order[0]:
            n_tie += 1
            assert gap <= 1e-6 * abs(sc[order[0]])
    assert n_tie <= 2


def test_search_S1_identity_is_nearest_24cell_vertex(oracle):
    # S = 1 with q_s = 1 reduces to "nearest vertex of the 24-cell"
    rng = np.random.default_rng(13)
    cb = np.array([[[1.0, 0.0, 0.0, 0.0]]], np.float32)
    x = rng.standard_normal((1, 1, 8, 128)).astype(np.float32)
    words, radius, best, second, st = oracle.encode(x, cb, 1)
    idx = oracle.get_index(words, 1, np.arange(8 * 32))
    units = hurwitz_units_independent()
    t = oracle.table_2t()
    for j, ch in enumerate(x.reshape(-1, 4).astype(np.float64)):
        want = units[np.argmax(units @ ch)]
        assert np.array_equal(t[idx[j]], want)


def test_codewords_reencode_to_themselves(oracle):
    S = 32
    cb = oracle.make_codebook(1, S, 1)
    cw = np.array([oracle.codeword(i % 24, cb[0, i // 24]) for i in range(24 * S)], np.float32)
    x = np.zeros((1, 1, 24 * S // 32, 128), np.float32)
    x.reshape(-1, 4)[:] = cw
    words, radius, best, second, st = oracle.encode(x, cb, S)
    idx = oracle.get_index(words, S, np.arange(24 * S))
    hit = idx == np.arange(24 * S)
    # a miss is allowed only for an exact or near tie in fp32
    for j in np.nonzero(~hit)[0]:
        assert best[j] - second[j] <= 1e-6
    assert hit.mean() > 0.99


def test_ties_go_to_lowest_index(oracle):
    # x = (1, 1, 0, 0)/sqrt2 is equally close to +1 (p=0) and +i (p=2) and to
    # the half units with signs (+,+,*,*): p=0 must win
    cb = np.array([[[1.0, 0.0, 0.0, 0.0], [0.0, 1.0, 0.0, 0.0]]], np.float32)
    x = np.zeros((1, 1, 1, 128), np.float32)
    x.reshape(-1, 4)[0] = [1.0, 1.0, 0.0, 0.0]
    x.reshape(-1, 4)[1] = [0.0, 0.0, 0.0, -2.0]   # -k: p = 7 (s=0) beats s=1 copies
    words, radius, *_ = oracle.encode(x, cb, 2)
    idx = oracle.get_index(words, 2, np.arange(32))
    assert idx[0] == 0
    assert idx[1] == 7
    assert np.all(idx[2:] == 0)          # zero chunks -> index 0
    assert np.all(radius[2:] == 0)


def test_angular_error_falls_like_the_covering_rate(oracle):
    # random multiplicative packing: covering radius O((24 S)^(-1/3)); the mean
    # quantisation angle should shrink by about 8^(1/3) = 2 from S=4 to S=32
    rng = np.random.default_rng(14)
    x = rng.standard_normal((1, 1, 128, 128)).astype(np.float32)
    ang = {}
    for S in (4, 32):
        cb = oracle.make_codebook(1, S, 1)
        words, radius, best, second, st = oracle.encode(x, cb, S)
        ang[S] = np.degrees(np.arccos(np.clip(best.astype(np.float64), -1, 1))).mean()
    ratio = ang[4] / ang[32]
    assert 1.7 < ratio < 2.3


# ---------------------------------------------------------------- Med3x
def test_lower_median_worked_example(oracle):
    # 4 chunks with norms 4, 1, 3, 2 (one per axis): lower median = 2, thr = 6
    x = np.zeros((1, 1, 1, 128), np.float32)
    c = x.reshape(-1, 4)
    c[0, 0], c[1, 1], c[2, 2], c[3, 3] = 4, 1, 3, 2
    c[4:, 0] = 0.0
    # 32 chunks: 28 zeros + {1,2,3,4}: sorted = 28 zeros, 1, 2, 3, 4 -> rank 15 = 0
    rmed, thr = oracle.med3_threshold(x)
    assert rmed[0] == 0.0 and thr[0] == 0.0
    c[4:, 0] = 1.5
    # now: 1, 1.5 x28, 2, 3, 4 -> rank 15 is 1.5
    rmed, thr = oracle.med3_threshold(x)
    assert rmed[0] == np.float32(1.5) and thr[0] == np.float32(4.5)


@pytest.mark.parametrize("gran", [0, 1])
def test_median_matches_numpy_partition(oracle, gran):
    rng = np.random.default_rng(15)
    x = (rng.standard_t(3, (2, 3, 96, 128))).astype(np.float32)
    rmed, thr = oracle.med3_threshold(x, 3.0, gran)
    for h in range(3):
        xh = x[:, h]
        v = oracle.chunk_norm(xh).ravel() if gran == 0 else np.abs(xh).ravel()
        k = v.size // 2 - 1
        assert rmed[h] == np.partition(v, k)[k]
        assert thr[h] == np.float32(3.0) * rmed[h]


def test_extract_finds_planted_outliers_in_order(oracle):
    rng = np.random.default_rng(16)
    B, H, T, D = 2, 2, 64, 128
    x = rng.standard_normal((B, H, T, D)).astype(np.float32) * 0.1
    n = B * H * T * D // 4
    planted = np.sort(rng.choice(n, 40, replace=False))
    xc = x.reshape(-1, 4)
    xc[planted] *= 1000.0
    rmed, thr = oracle.med3_threshold(x)
    idx, val, slab_off, cnt, st = oracle.extract(x, thr)
    assert cnt == 40 and np.array_equal(idx, planted)
    assert np.array_equal(val, xc[planted].astype(np.float16).view(np.uint16))
    per_slab = T * D // 4
    for s in range(B * H):
        want = np.sum((planted >= s * per_slab) & (planted < (s + 1) * per_slab))
        assert slab_off[s + 1] - slab_off[s] == want
    # capacity overflow: first `cap` entries written, required count reported
    idx2, val2, _, cnt2, st2 = oracle.extract(x, thr, cap=10)
    assert cnt2 == 40 and np.array_equal(idx2, planted[:10]) and st2["flags"] & 1
    # encode with thr zeroes them: index 0, radius 0
    cb = oracle.make_codebook(1, 8, H)
    words, radius, *_ = oracle.encode(x, cb, 8, thr=thr)
    assert np.all(radius[planted] == 0)
    assert np.all(oracle.get_index(words, 8, planted) == 0)


def test_element_mode_extract_and_add_back(oracle):
    rng = np.random.default_rng(17)
    x = rng.standard_normal((1, 1, 32, 128)).astype(np.float32)
    e = np.array([5, 77, 1000, 4095])
    x.reshape(-1)[e] = [50.0, -40.0, 60.0, 45.0]
    rmed, thr = oracle.med3_threshold(x, 3.0, 1)
    idx, val, slab_off, cnt, st = oracle.extract(x, thr, gran=1)
    big = np.nonzero(np.abs(x.reshape(-1)) > thr[0])[0]
    assert np.array_equal(idx, big) and set(e) <= set(idx.tolist())
    cb = oracle.make_codebook(1, 32, 1)
    words, radius, *_ = oracle.encode(x, cb, 32, thr=thr, gran=1)
    y, _ = oracle.decode(words, radius, cb, 32, 1, 1, 32, 128, out_idx=idx, out_val=val,
                         gran=1, out_dtype=1)
    # restored elements carry their fp16 value plus the codeword's share
    assert np.allclose(y.reshape(-1)[e], x.reshape(-1)[e], rtol=0.02, atol=0.5)


# ---------------------------------------------------------------- decode
def test_decode_is_radius_times_codeword(oracle):
    rng = np.random.default_rng(18)
    S = 8
    cb = oracle.make_codebook(4, S, 1)
    x = rng.standard_normal((1, 1, 32, 128)).astype(np.float32)
    words, radius, best, second, st = oracle.encode(x, cb, S)
    y, _ = oracle.decode(words, radius, cb, S, 1, 1, 32, 128, out_dtype=1)
    idx = oracle.get_index(words, S, np.arange(32 * 32))
    rr = radius.view(np.float16).astype(np.float64)
    tt = oracle.table_2t()
    for j in range(32 * 32):
        c = qmul_ref(tt[idx[j] % 24], cb[0, idx[j] // 24].astype(np.float64))
        assert np.allclose(y.reshape(-1, 4)[j], rr[j] * c, rtol=1e-6, atol=1e-6)
    # norm preserved up to the fp16 radius and fp32 codeword rounding
    yn = np.linalg.norm(y.reshape(-1, 4).astype(np.float64), axis=1)
    xn = np.linalg.norm(x.reshape(-1, 4).astype(np.float64), axis=1)
    assert np.allclose(yn, xn, rtol=1e-3)
    # bf16 output is the RN-even rounding of the fp32 output
    yb, _ = oracle.decode(words, radius, cb, S, 1, 1, 32, 128, out_dtype=0)
    assert np.array_equal(yb, torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))


def test_decode_flags_bad_index(oracle):
    words = np.full(8, 0xFFFFFFFF, np.uint32)          # every index 255 >= 192
    radius = np.full(32, 0x3C00, np.uint16)
    cb = oracle.make_codebook(1, 8, 1)
    y, st = oracle.decode(words, radius, cb, 8, 1, 1, 1, 128, out_dtype=1)
    assert st["flags"] & 8 and np.all(y == 0)


def test_nonfinite_chunks(oracle):
    x = np.zeros((1, 1, 1, 128), np.float32)
    c = x.reshape(-1, 4)
    c[0] = [np.nan, 1, 0, 0]
    c[1] = [np.inf, 0, 0, 0]
    c[2] = [1e20, 0, 0, 0]        # r^2 overflows fp32 -> r = inf
    c[3] = [70000.0, 0, 0, 0]     # radius saturates to 65504
    cb = oracle.make_codebook(1, 8, 1)
    words, radius, best, second, st = oracle.encode(x, cb, 8)
    assert list(radius[:3]) == [0x7E00] * 3 and radius[3] == 0x7BFF
    assert st["n_nonfinite"] == 3 and st["n_saturated"] == 1 and st["flags"] == 6
    assert np.all(oracle.get_index(words, 8, np.arange(3)) == 0)


# ---------------------------------------------------------------- pages' figures
def test_pages_figures():
    with open(os.path.join(GOLDEN, "pages_figures.json")) as f:
        g = json.load(f)
    fig = {e["id"]: e for e in g["figures"]}
    # 24 S effective codewords: 192 at S=8, 768 at S=32
    assert 24 * 8 == fig["codewords_S8"]["value"]
    assert 24 * 32 == fig["codewords_S32"]["value"]
    # bits per element: log2(24 S) / 2 reproduces 3.79 at S=8 and ~5 at S=32
    assert round(math.log2(24 * 8) / 2, 2) == fig["bits_S8"]["value"]
    assert abs(math.log2(24 * 32) / 2 - fig["bits_S32"]["value"]) < 0.25
    # Llama-3-70B, 128k tokens, K+V fp16: 80 layers x 8 KV heads x 128 x 2 B x 2
    gb = 80 * 8 * 128 * 2 * 2 * 131072 / 1e9
    assert round(gb) == fig["cache_70b_128k_gb"]["value"]
    assert fig["med3_C"]["value"] == 3
    assert fig["min_angle_deg"]["value"] == 60


# ---------------------------------------------------------------- the near-tie arbiter
# Every GPU index that differs from the oracle's is excused or failed by the
# oracle's own scores (score_chunks: the fp32 score of a given codeword; best /
# second of encode and encode_chunks).  These pins tie those functions to an
# independent fp64 model: codewords built from complex 2x2 matrices in the
# enumeration order the pages' set is given in (8 axis units p = 2a + sign,
# then the 16 half units p = 8 + m), scored against x / |x| in fp64.
def _units_enumerated():
    out = []
    for p in range(24):
        if p < 8:
            v = np.zeros(4)
            v[p // 2] = -1.0 if p % 2 else 1.0
        else:
            v = np.array([-0.5 if ((p - 8) >> c) & 1 else 0.5 for c in range(4)])
        out.append(v)
    return np.array(out)


def _fp64_scores(chunk, cb_head):
    """fp64 <x/|x|, q_p q_s> for every global index s*24 + p."""
    units = _units_enumerated()
    W = np.array([qmul_ref(units[p], cb_head[s].astype(np.float64))
                  for s in range(cb_head.shape[0]) for p in range(24)])
    x = chunk.astype(np.float64)
    n = np.linalg.norm(x)
    return W @ (x / n) if n > 0 else np.zeros(W.shape[0])


def _zeroed(chunk, thr_h, gran):
    """The chunk as the search sees it after Med3x zeroing (pages, section 3):
    chunk mode zeroes a chunk whose fp32 norm exceeds thr, element mode zeroes
    each element with |x| > thr."""
    c = chunk.astype(np.float32).copy()
    if thr_h is None:
        return c
    if gran == 0:
        r = np.sqrt(np.sum(c.astype(np.float64) ** 2))
        return np.zeros(4, np.float32) if r > thr_h else c
    c[np.abs(c) > thr_h] = 0.0
    return c


def _arbiter_case(oracle):
    # three heads with distinct codebooks, two batches, a few planted large
    # chunks so that Med3x zeroes something in both granularities
    rng = np.random.default_rng(21)
    B, H, T, D, S = 2, 3, 8, 128, 8
    x = rng.standard_normal((B, H, T, D)).astype(np.float32)
    xc = x.reshape(-1, 4)
    big = rng.choice(xc.shape[0], 24, replace=False)
    xc[big] *= 9.0
    xc[big[:6], 1] = 40.0                  # one large element in some chunks
    cb = oracle.make_codebook(4, S, H)
    return x, cb, S


# (fp32 score vs fp64: |u| = |c| = 1 up to rounding; u_i is a rounded quotient
# of a rounded norm, c_i a sum of 4 exact terms rounded 3 times, the dot product
# 4 rounded products and 3 rounded sums: well under 24 units of 2^-24)
SCORE_ABS_TOL = 24 * 2.0 ** -24


@pytest.mark.parametrize("gran,use_thr", [(0, False), (0, True), (1, True)])
def test_score_chunks_matches_independent_fp64_scores(oracle, gran, use_thr):
    x, cb, S = _arbiter_case(oracle)
    B, H, T, D = x.shape
    thr = oracle.med3_threshold(x, 3.0, gran)[1] if use_thr else None
    rng = np.random.default_rng(22)
    chunks = np.sort(rng.choice(B * H * T * D // 4, 60, replace=False)).astype(np.int64)
    per_slab = T * D // 4
    n_words = 24 * S
    all_idx = np.tile(np.arange(n_words, dtype=np.uint32), chunks.size)
    rep = np.repeat(chunks, n_words)
    sc = oracle.score_chunks(x, cb, S, rep, all_idx, thr=thr, gran=gran).reshape(-1, n_words)
    xc = x.reshape(-1, 4)
    for q, j in enumerate(chunks):
        h = (j // per_slab) % H
        c = _zeroed(xc[j], None if thr is None else thr[h], gran)
        ref = _fp64_scores(c, cb[h])
        if not np.any(c):
            assert np.all(sc[q] == 0.0)          # a zero chunk has no search
            continue
        assert np.abs(sc[q].astype(np.float64) - ref).max() <= SCORE_ABS_TOL, (j, h)


@pytest.mark.parametrize("gran,use_thr", [(0, False), (0, True), (1, True)])
def test_best_and_second_are_the_top_two_scores(oracle, gran, use_thr):
    x, cb, S = _arbiter_case(oracle)
    B, H, T, D = x.shape
    thr = oracle.med3_threshold(x, 3.0, gran)[1] if use_thr else None
    words, radius, best, second, _ = oracle.encode(x, cb, S, thr=thr, gran=gran)
    n = B * H * T * D // 4
    idx = oracle.get_index(words, S, np.arange(n))
    per_slab = T * D // 4
    n_words = 24 * S
    xc = x.reshape(-1, 4)
    chunks = np.arange(0, n, 7, dtype=np.int64)
    sc = oracle.score_chunks(x, cb, S, np.repeat(chunks, n_words),
                             np.tile(np.arange(n_words, dtype=np.uint32), chunks.size),
                             thr=thr, gran=gran).reshape(-1, n_words)
    at_pick = oracle.score_chunks(x, cb, S, chunks, idx[chunks], thr=thr, gran=gran)
    for q, j in enumerate(chunks):
        h = (j // per_slab) % H
        c = _zeroed(xc[j], None if thr is None else thr[h], gran)
        if not np.any(c):
            assert idx[j] == 0 and best[j] == 0.0 and second[j] == 0.0
            continue
        # the score of the oracle's own pick is its best, bit for bit
        assert at_pick[q].view(np.uint32) == best[j].view(np.uint32)
        # best and second are the two largest of the 24 S scores (second may
        # equal best on an exact tie), and the pick is the lowest index of best
        srt = np.sort(sc[q])[::-1]
        assert best[j] == srt[0] and second[j] == srt[1], j
        assert idx[j] == int(np.nonzero(sc[q] == srt[0])[0][0])
        # and against the independent fp64 scores
        ref = np.sort(_fp64_scores(c, cb[h]))[::-1]
        assert abs(float(best[j]) - ref[0]) <= SCORE_ABS_TOL
        assert abs(float(second[j]) - ref[1]) <= SCORE_ABS_TOL


@pytest.mark.parametrize("gran,use_thr", [(0, False), (0, True), (1, True)])
def test_encode_chunks_equals_the_whole_call_encode(oracle, gran, use_thr):
    # the sampled form used at full size must give what the whole-call encode
    # gives on the same chunks (head selection, zeroing, radius, scores)
    x, cb, S = _arbiter_case(oracle)
    B, H, T, D = x.shape
    thr = oracle.med3_threshold(x, 3.0, gran)[1] if use_thr else None
    words, radius, best, second, _ = oracle.encode(x, cb, S, thr=thr, gran=gran)
    n = B * H * T * D // 4
    rng = np.random.default_rng(23)
    chunks = rng.permutation(n)[:300].astype(np.int64)      # any order, all heads
    i2, r2, b2, s2 = oracle.encode_chunks(x, cb, S, chunks, thr=thr, gran=gran)
    assert np.array_equal(i2, oracle.get_index(words, S, chunks))
    assert np.array_equal(r2, radius[chunks])
    assert np.array_equal(b2.view(np.uint32), best[chunks].view(np.uint32))
    assert np.array_equal(s2.view(np.uint32), second[chunks].view(np.uint32))
