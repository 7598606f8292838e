"""Pins of the oracle's joint (index, radius level) code and outlier flags.

The joint code restates the pages' bit budget (3.79 bits per element at
S = 8, about 5 at S = 32: two log2(24 S)-bit digits per chunk of four
elements) as a mixed-radix number: per chunk the digit D = idx * L + k in
base L^2 (L = 24 S), n chunks of a slab per block value V = sum D_c L^(2c).
The checks compare the oracle with Python's arbitrary-precision integers
(an independent model of the same definition), with round trips, with the
pages' printed figures and with numpy bit operations for the flags."""
import json
import math
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def pack_fields(vals, b):
    """LSB-first b-bit fields in groups of 32 (the index-word layout), by numpy."""
    vals = np.asarray(vals, np.uint64)
    n = vals.size
    bits = ((vals[:, None] >> np.arange(b, dtype=np.uint64)) & 1).astype(np.uint8)
    bits = bits.reshape(n // 32, 32 * b)
    return np.packbits(bits, axis=1, bitorder="little").view(np.uint32).reshape(-1)


def big_int_runs(idx, k, B, H, T, D, S):
    """The joint code by Python integers: per slab one integer whose bits are
    the blocks' values at offsets q * w, cut into 32-bit words."""
    L = 24 * S
    m = L * L
    n = 0
    while m ** (n + 1) < 2 ** 64:
        n += 1
    w = (m ** n - 1).bit_length()
    cps = T * D // 4
    nb = -(-cps // n)
    wps = -(-(nb * w) // 32)
    out = []
    for s in range(B * H):
        stream = 0
        for q in range(nb):
            v = 0
            for c in range(n):
                j = q * n + c
                d = int(idx[s * cps + j]) * L + int(k[s * cps + j]) if j < cps else 0
                v += d * m ** c
            stream |= v << (q * w)
        out += [(stream >> (32 * i)) & 0xFFFFFFFF for i in range(wps)]
    return np.array(out, np.uint32), n, w


@pytest.mark.parametrize("S", [1, 2, 8, 11, 32, 48, 1000, 65535])
def test_block_size_is_the_largest_that_fits_64_bits(oracle, S):
    m = (24 * S) ** 2
    n = max(i for i in range(1, 64) if m ** i < 2 ** 64)
    assert oracle.joint_block_chunks(S) == n
    assert oracle.joint_block_bits(S) == (m ** n - 1).bit_length()


def test_bits_per_element_against_the_pages(oracle):
    figs = {f["id"]: f["value"] for f in
            json.load(open(os.path.join(GOLDEN, "pages_figures.json")))["figures"]}
    # S = 8: 4 chunks in 61 bits, 3.8125 bits per element; the pages' 3.79 is
    # the unblocked log2(192^2) / 4 = 3.7925
    assert oracle.joint_block_chunks(8) == 4 and oracle.joint_block_bits(8) == 61
    b8 = 61 / 16
    assert abs(b8 - math.log2(192 ** 2) / 4) < 0.025
    assert abs(b8 - figs["bits_S8"]) < 0.025
    # S = 32: 3 chunks in 58 bits, 4.833 bits per element ("about 5")
    assert oracle.joint_block_chunks(32) == 3 and oracle.joint_block_bits(32) == 58
    assert 58 / 12 < 4.85 and abs(58 / 12 - figs["bits_S32"]) < 0.2


@pytest.mark.parametrize("S,shape", [(8, (2, 1, 10, 128)), (32, (1, 2, 11, 128)),
                                     (32, (2, 3, 32, 4)), (1, (1, 1, 64, 16)), (1000, (1, 1, 3, 128))])
def test_pack_equals_the_big_integer_definition(oracle, S, shape):
    B, H, T, D = shape
    n_chunks = B * H * T * D // 4
    rng = np.random.default_rng(S + T)
    L = 24 * S
    idx = rng.integers(0, L, n_chunks)
    k = rng.integers(0, L, n_chunks)
    idx[:3] = [0, L - 1, L - 1]          # the extreme digits
    k[:3] = [0, L - 1, 0]
    b = oracle.index_bits(S)
    joint, bad = oracle.pack_joint(pack_fields(idx, b), pack_fields(k, b), B, H, T, D, S)
    want, n, w = big_int_runs(idx, k, B, H, T, D, S)
    assert bad == 0
    assert np.array_equal(joint, want)
    i2, k2 = oracle.unpack_joint(joint, B, H, T, D, S)
    assert np.array_equal(i2, idx) and np.array_equal(k2, k)


def test_out_of_range_pairs_are_counted_and_stored_as_zero(oracle):
    B, H, T, D, S = 1, 1, 4, 128, 8
    n_chunks = T * 32
    idx = np.zeros(n_chunks, np.uint32)
    k = np.ones(n_chunks, np.uint32)
    idx[5] = 200                          # >= L = 192 (8 bits hold up to 255)
    k[7] = 255
    b = oracle.index_bits(S)
    joint, bad = oracle.pack_joint(pack_fields(idx, b), pack_fields(k, b), B, H, T, D, S)
    assert bad == 2
    i2, k2 = oracle.unpack_joint(joint, B, H, T, D, S)
    assert i2[5] == 0 and k2[5] == 0 and i2[7] == 0 and k2[7] == 0
    assert np.all(k2[np.r_[0:5, 6, 8:n_chunks]] == 1)


def test_flags_are_the_list_as_a_bitmap(oracle):
    rng = np.random.default_rng(3)
    n_chunks = 32 * 50
    lst = np.sort(rng.choice(n_chunks, 123, replace=False)).astype(np.uint32)
    flags = oracle.list_flags(lst, n_chunks)
    want = np.zeros(n_chunks // 32, np.uint32)
    np.bitwise_or.at(want, lst // 32, (np.uint32(1) << (lst % 32).astype(np.uint32)))
    assert np.array_equal(flags, want)
    back, n = oracle.list_from_flags(flags, n_chunks)
    assert n == lst.size and np.array_equal(back, lst)
