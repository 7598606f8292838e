"""The C ABI library loads here (no GPU needed), exports every entry point
include/hqmq.h declares, and rejects bad arguments synchronously before any
CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hqmq.h")


@pytest.fixture(scope="module")
def lib():
    from kv_cache_quantization_hqmq_b200 import build
    build.build()
    from kv_cache_quantization_hqmq_b200 import hqmq
    return hqmq.lib()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"HQMQ_API\s+[\w\s\*]*?\b(hqmq_\w+)\s*\(", text)


def test_header_declares_the_four_calls_of_the_path():
    names = declared_functions()
    for n in ("hqmq_make_codebook", "hqmq_outlier_extract", "hqmq_encode", "hqmq_decode"):
        assert n in names
    assert len(names) == len(set(names)) >= 9


def test_every_declared_symbol_is_exported(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_only_declared_symbols_are_exported():
    import subprocess
    from kv_cache_quantization_hqmq_b200 import build
    out = subprocess.check_output(["nm", "-D", "--defined-only", build.LIB], text=True)
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l and "hqmq" in l}
    assert exported == set(declared_functions())


def test_host_queries(lib):
    from kv_cache_quantization_hqmq_b200 import hqmq
    assert hqmq.hqmq_version().startswith("hqmq-b200")
    assert hqmq.hqmq_index_bits(8) == 8 and hqmq.hqmq_index_bits(32) == 10
    assert hqmq.hqmq_index_bits(0) == 0 and hqmq.hqmq_index_bits(65536) == 0
    # 70B call: 1 x 8 x 131072 x 128 -> 1,048,576 groups x 10 words
    assert hqmq.hqmq_index_words(1, 8, 131072, 128, 32) == 1048576 * 10
    assert hqmq.hqmq_index_words(1, 1, 3, 128, 8) == 24       # 3 groups x 8 words
    assert hqmq.hqmq_index_words(1, 1, 3, 12, 8) == 0         # 9 chunks: not whole groups
    assert hqmq.hqmq_index_words(1, 1, 8, 6, 8) == 0          # D % 4 != 0
    assert hqmq.hqmq_outlier_workspace_size(1, 8, 131072, 128) > 8 * 2048 * 4
    assert hqmq.hqmq_outlier_workspace_size(1, 8, 131072, 128, 2) == 0


def test_bad_arguments_rejected_without_cuda(lib):
    P = ctypes.c_void_p
    good = P(1 << 20)                   # never dereferenced: validation fails first
    st = None
    # S out of range / bad shapes / unknown enums -> HQMQ_ERR_ARG (1)
    assert lib.hqmq_make_codebook(1, 0, 4, 0, good, None) == 1
    assert lib.hqmq_make_codebook(1, 8, 0, 0, good, None) == 1
    assert lib.hqmq_make_codebook(1, 8, 2, 0xFFFFFFFF, good, None) == 1
    assert lib.hqmq_encode(good, 0, 1, 1, 8, 6, good, 8, None, 0, good, good, st, None) == 1
    assert lib.hqmq_encode(good, 0, 1, 1, 3, 12, good, 8, None, 0, good, good, st, None) == 1
    assert lib.hqmq_encode(good, 2, 1, 1, 8, 128, good, 8, None, 0, good, good, st, None) == 1
    assert lib.hqmq_encode(good, 0, 1, 1, 8, 128, good, 70000, None, 0, good, good, st, None) == 1
    assert lib.hqmq_encode(good, 0, 1, 1, 8, 128, good, 8, None, 5, good, good, st, None) == 1
    assert lib.hqmq_encode(None, 0, 1, 1, 8, 128, good, 8, None, 0, good, good, st, None) == 1
    assert lib.hqmq_encode(good, 0, 300, 300, 8, 128, good, 8, None, 0, good, good, st, None) == 1
    # misaligned pointers -> HQMQ_ERR_ALIGN (2)
    assert lib.hqmq_encode(P((1 << 20) + 8), 0, 1, 1, 8, 128, good, 8, None, 0, good, good, st,
                           None) == 2
    assert lib.hqmq_decode(good, P((1 << 20) + 2), good, 8, None, None, None, None, 0, 0, 1, 1, 8,
                           128, good, 0, st, None) == 2
    # outlier extract: C must be positive and finite; workspace must be large enough
    assert lib.hqmq_outlier_extract(good, 0, 1, 1, 8, 128, ctypes.c_float(0.0), 0, good, good,
                                    good, good, good, None, 16, good, 1 << 20, st, None) == 1
    assert lib.hqmq_outlier_extract(good, 0, 1, 1, 8, 128, ctypes.c_float(float("inf")), 0, good,
                                    good, good, good, good, None, 16, good, 1 << 20, st, None) == 1
    assert lib.hqmq_outlier_extract(good, 0, 1, 1, 8, 128, ctypes.c_float(3.0), 0, good, good,
                                    good, good, good, None, 16, good, 16, st, None) == 4


def test_next_row_queries_and_argument_checks(lib):
    """The attention, quantized-radius, given-threshold and batched-append
    entry points: size queries, and synchronous rejection of bad arguments
    (no CUDA call is made)."""
    from kv_cache_quantization_hqmq_b200 import hqmq
    P = ctypes.c_void_p
    good = P(1 << 20)
    # workspace sizes
    assert hqmq.hqmq_attention_workspace_size(1, 8) > 1024 * 8 * 130 * 4
    assert hqmq.hqmq_attention_workspace_size(0, 8) == 0
    assert hqmq.hqmq_outlier_extract_given_thr_workspace_size(1, 8, 1, 128) > 0
    assert hqmq.hqmq_outlier_extract_given_thr_workspace_size(1, 8, 1, 6) == 0
    # attention: D must be 128, G <= 8, Hq a multiple of Hk, a finite scale
    codes = hqmq.KVCodes(good, good, good, None, None, None, 0, 0, None, None)
    ref = ctypes.byref(codes)
    F = ctypes.c_float
    ws = 1 << 30
    assert lib.hqmq_attention_decode(good, None, ref, ref, 8, 1, 8, 8, 64, 64, F(0.1), good, 1,
                                     good, ws, None, None) == 1          # D = 64
    assert lib.hqmq_attention_decode(good, None, ref, ref, 8, 1, 72, 8, 64, 128, F(0.1), good, 1,
                                     good, ws, None, None) == 1          # G = 9
    assert lib.hqmq_attention_decode(good, None, ref, ref, 8, 1, 12, 8, 64, 128, F(0.1), good, 1,
                                     good, ws, None, None) == 1          # Hq % Hk != 0
    assert lib.hqmq_attention_decode(good, None, ref, ref, 8, 1, 8, 8, 64, 128, F(float("nan")),
                                     good, 1, good, ws, None, None) == 1  # scale NaN
    assert lib.hqmq_attention_decode(good, None, ref, ref, 8, 1, 8, 8, 64, 128, F(0.1), good, 1,
                                     good, 16, None, None) == 4          # workspace too small
    qr = hqmq.KVCodes(good, None, good, None, None, None, 0, 0, good, good)
    assert lib.hqmq_attention_decode(good, None, ref, ctypes.byref(qr), 8, 1, 8, 8, 64, 128,
                                     F(0.1), good, 1, good, ws, None, None) == 1  # mixed formats
    noradius = hqmq.KVCodes(good, None, good, None, None, None, 0, 0, None, None)
    assert lib.hqmq_attention_decode(good, None, ctypes.byref(noradius), ctypes.byref(noradius),
                                     8, 1, 8, 8, 64, 128, F(0.1), good, 1, good, ws, None,
                                     None) == 1                         # no radius of any form
    # quantized radius
    assert lib.hqmq_quantize_radius(good, good, 1, 1, 32, 128, 0, good, None) == 1
    assert lib.hqmq_quantize_radius(None, good, 1, 1, 32, 128, 8, good, None) == 1
    assert lib.hqmq_decode_qradius(good, good, good, good, 8, good, good, None, 16, 0, 1, 1, 32,
                                   128, good, 0, None, None) == 1       # a list needs tile_off
    # given-threshold list: workspace too small, misaligned threshold
    assert lib.hqmq_outlier_extract_given_thr(good, 0, 1, 8, 1, 128, good, 0, good, good, good,
                                              None, 64, good, 16, None, None) == 4
    assert lib.hqmq_outlier_extract_given_thr(good, 0, 1, 8, 1, 128, P((1 << 20) + 2), 0, good,
                                              good, good, None, 64, good, 1 << 20, None, None) == 2
    # batched append: codebooks of a call must fit in shared memory; cap < 2^32
    assert lib.hqmq_append_batch(good, 0, 4, 1, 64, 1, 128, good, 0, good, 1000, good, good, good,
                                 good, good, None, 64, None, None) == 1
    assert lib.hqmq_append_batch(good, 0, 4, 1, 8, 1, 128, good, 0, good, 32, good, good, good,
                                 good, good, None, 1 << 33, None, None) == 1
    assert lib.hqmq_append_batch(good, 0, 0, 1, 8, 1, 128, good, 0, good, 32, good, good, good,
                                 good, good, None, 64, None, None) == 1


def test_joint_code_queries_and_argument_errors(lib):
    from kv_cache_quantization_hqmq_b200 import hqmq
    assert hqmq.hqmq_joint_block(8) == (4, 61) and hqmq.hqmq_joint_block(32) == (3, 58)
    assert hqmq.hqmq_joint_block(0) == (0, 0) and hqmq.hqmq_joint_block(2731) == (0, 0)
    # 70B call at S = 32: 8 slabs, each ceil(4194304 / 3) blocks of 58 bits
    nb = -(-4194304 // 3)
    assert hqmq.hqmq_joint_words(1, 8, 131072, 128, 32) == 8 * ((nb * 58 + 31) // 32)
    assert hqmq.hqmq_joint_words(1, 8, 131072, 128, 2731) == 0
    good = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 2)
    # rejected before any CUDA call: bad S, missing pointers, misalignment
    assert lib.hqmq_pack_joint(good, good, 0, 1, 1, 32, 128, good, None, None) == hqmq.HQMQ_ERR_ARG
    assert lib.hqmq_pack_joint(None, good, 8, 1, 1, 32, 128, good, None, None) == hqmq.HQMQ_ERR_ARG
    assert lib.hqmq_pack_joint(odd, good, 8, 1, 1, 32, 128, good, None, None) == hqmq.HQMQ_ERR_ALIGN
    assert lib.hqmq_list_flags(good, None, 16, 1, 1, 32, 128, good, None) == hqmq.HQMQ_ERR_ARG
    assert lib.hqmq_list_flags(odd, good, 16, 1, 1, 32, 128, good, None) == hqmq.HQMQ_ERR_ALIGN
    y4 = ctypes.c_void_p((1 << 20) + 4)       # 4-byte aligned: not enough for bf16 chunks
    assert lib.hqmq_decode_joint(good, good, good, 8, None, None, None, 0, 1, 1, 32, 128, y4, 0,
                                 None) == hqmq.HQMQ_ERR_ALIGN
    assert lib.hqmq_decode_joint(good, good, good, 8, good, None, None, 16, 1, 1, 32, 128, good, 0,
                                 None) == hqmq.HQMQ_ERR_ARG      # flags without tile offsets
