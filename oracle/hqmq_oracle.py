"""ctypes front end of the plain C oracle (``hqmq_oracle.c``).

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and the
cpu_baseline / reference leg of ``bench.py`` are the only users.  The product
library never imports this module, and this module imports nothing from the
product package.

Every function here marshals numpy arrays into the C oracle; the arithmetic
lives in ``hqmq_oracle.c``, where each function cites the passage of the pages
it follows.  Arrays of bf16 values are carried as ``np.uint16`` bit patterns,
fp16 the same way.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hqmq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_hqmq.so")

BF16, F32 = 0, 1
CHUNK, ELEMENT = 0, 1

FLAG_OVERFLOW, FLAG_SATURATED, FLAG_NONFINITE, FLAG_BAD_INDEX = 1, 2, 4, 8

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-Wall", "-Wextra"]


class Status(ctypes.Structure):
    _fields_ = [
        ("flags", ctypes.c_uint32),
        ("reserved", ctypes.c_uint32),
        ("n_outliers", ctypes.c_uint64),
        ("n_saturated", ctypes.c_uint64),
        ("n_nonfinite", ctypes.c_uint64),
    ]

    def as_dict(self):
        return {k: int(getattr(self, k)) for k, _ in self._fields_}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no FMA contraction) into liboracle_hqmq.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_U32 = ctypes.c_uint32
_U64 = ctypes.c_uint64
_I64 = ctypes.c_int64
_F = ctypes.c_float

_SIGS = {
    "oracle_bf16_to_f32": (_F, [ctypes.c_uint16]),
    "oracle_f32_to_bf16": (ctypes.c_uint16, [_F]),
    "oracle_f16_to_f32": (_F, [ctypes.c_uint16]),
    "oracle_f32_to_f16_sat": (ctypes.c_uint16, [_F, _P]),
    "oracle_qmul_f64": (None, [_P, _P, _P]),
    "oracle_2t_element": (None, [_I, _P]),
    "oracle_codeword_f32": (None, [_I, _P, _P]),
    "oracle_philox4x32_10": (None, [_P, _P, _P]),
    "oracle_codeword_secondary": (None, [_U64, _U32, _U32, _P]),
    "oracle_make_codebook": (None, [_U64, _U32, _U32, _U32, _P]),
    "oracle_chunk_norm": (_F, [_P]),
    "oracle_score": (_F, [_P, _P, _U32, _U32]),
    "oracle_index_bits": (_U32, [_U32]),
    "oracle_get_index": (_U32, [_P, _U32, ctypes.c_size_t]),
    "oracle_encode": (None, [_P, _I, _I, _I, _I, _I, _P, _U32, _P, _I, _P, _P, _P, _P, _P]),
    "oracle_encode_chunks": (None, [_P, _I, _I, _I, _I, _I, _P, _U32, _P, _I, _P, _I64, _P, _P, _P, _P]),
    "oracle_med3_threshold": (None, [_P, _I, _I, _I, _I, _I, _F, _I, _P, _P]),
    "oracle_extract": (_I64, [_P, _I, _I, _I, _I, _I, _P, _I, _P, _P, _P, _U64, _P]),
    "oracle_decode": (None, [_P, _P, _P, _U32, _P, _P, _I64, _I, _I, _I, _I, _I, _P, _I, _P]),
    "oracle_f32_to_bf16_array": (None, [_P, _P, _I64]),
    "oracle_bf16_to_f32_array": (None, [_P, _P, _I64]),
    "oracle_f32_to_f16_sat_array": (_I64, [_P, _P, _I64]),
    "oracle_f16_to_f32_array": (None, [_P, _P, _I64]),
    "oracle_chunk_norm_array": (None, [_P, _P, _I64]),
    "oracle_get_index_array": (None, [_P, _U32, _P, _I64, _P]),
    "oracle_score_chunks": (None, [_P, _I, _I, _I, _I, _I, _P, _U32, _P, _I, _P, _P, _I64, _P]),
    "oracle_radius_level": (_U32, [ctypes.c_uint16, _F, _U32]),
    "oracle_radius_of_level": (_F, [_U32, _F, _U32]),
    "oracle_quantize_radius": (None, [_P, _P, _I, _I, _I, _I, _U32, _P]),
    "oracle_decode_qradius": (None, [_P, _P, _P, _P, _U32, _P, _P, _I64, _I, _I, _I, _I, _I, _P,
                                     _I, _P]),
    "oracle_joint_block_chunks": (_U32, [_U32]),
    "oracle_joint_block_bits": (_U32, [_U32]),
    "oracle_joint_slab_words": (_U64, [_I, _I, _U32]),
    "oracle_pack_joint": (_U64, [_P, _P, _I, _I, _I, _I, _U32, _P]),
    "oracle_unpack_joint": (None, [_P, _I, _I, _I, _I, _U32, _P, _P]),
    "oracle_list_flags": (None, [_P, _I64, _U64, _P]),
    "oracle_list_from_flags": (_I64, [_P, _U64, _P, _I64]),
}


def lib():
    """The loaded oracle.  HQMQ_ORACLE_LIB may name another build of the same
    source; the mutation tests use it to load an oracle with a planted bug."""
    global _lib
    if _lib is None:
        path = os.environ.get("HQMQ_ORACLE_LIB") or build()
        l = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(l, name)
            fn.restype = res
            fn.argtypes = args
        _lib = l
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _x_dtype(x):
    if x.dtype == np.uint16:
        return BF16
    if x.dtype == np.float32:
        return F32
    raise TypeError("x must be uint16 (bf16 bits) or float32, got %s" % x.dtype)


# ---------------------------------------------------------------- scalars
def f32_to_bf16(a):
    a = _c(a, np.float32)
    out = np.empty(a.shape, np.uint16)
    lib().oracle_f32_to_bf16_array(_ptr(a), _ptr(out), a.size)
    return out


def bf16_to_f32(a):
    a = _c(a, np.uint16)
    out = np.empty(a.shape, np.float32)
    lib().oracle_bf16_to_f32_array(_ptr(a), _ptr(out), a.size)
    return out


def f32_to_f16_sat(a):
    """Returns (fp16 bit patterns, number of saturated values)."""
    a = _c(a, np.float32)
    out = np.empty(a.shape, np.uint16)
    n = lib().oracle_f32_to_f16_sat_array(_ptr(a), _ptr(out), a.size)
    return out, int(n)


def f16_to_f32(a):
    a = _c(a, np.uint16)
    out = np.empty(a.shape, np.float32)
    lib().oracle_f16_to_f32_array(_ptr(a), _ptr(out), a.size)
    return out


# ---------------------------------------------------------------- algebra
def qmul(a, b):
    a = _c(a, np.float64); b = _c(b, np.float64)
    out = np.empty(4, np.float64)
    lib().oracle_qmul_f64(_ptr(a), _ptr(b), _ptr(out))
    return out


def element_2t(p):
    out = np.empty(4, np.float64)
    lib().oracle_2t_element(int(p), _ptr(out))
    return out


def table_2t():
    return np.stack([element_2t(p) for p in range(24)])


def codeword(p, qs):
    qs = _c(qs, np.float32)
    out = np.empty(4, np.float32)
    lib().oracle_codeword_f32(int(p), _ptr(qs), _ptr(out))
    return out


def philox4x32_10(ctr, key):
    ctr = _c(ctr, np.uint32); key = _c(key, np.uint32)
    out = np.empty(4, np.uint32)
    lib().oracle_philox4x32_10(_ptr(ctr), _ptr(key), _ptr(out))
    return out


def make_codebook(seed, S, n_groups, group0=0):
    """[n_groups, S, 4] fp32 secondary codebooks of groups group0.."""
    out = np.empty((n_groups, S, 4), np.float32)
    lib().oracle_make_codebook(int(seed), int(S), int(n_groups), int(group0), _ptr(out))
    return out


def chunk_norm(x):
    """fp32 norms of the 4-element chunks of x (last axis multiple of 4)."""
    x = _c(x, np.float32)
    n = x.size // 4
    out = np.empty(n, np.float32)
    lib().oracle_chunk_norm_array(_ptr(x), _ptr(out), n)
    return out.reshape(x.shape[:-1] + (x.shape[-1] // 4,))


def index_bits(S):
    return int(lib().oracle_index_bits(int(S)))


def index_words(B, H, T, D, S):
    return (B * H * T * D // 128) * index_bits(S)


# ---------------------------------------------------------------- the path
def med3_threshold(x, C=3.0, gran=CHUNK):
    """Per-head lower-median r_med and thr = fl32(C * r_med); x: [B,H,T,D]."""
    B, H, T, D = x.shape
    x = np.ascontiguousarray(x)
    rmed = np.empty(H, np.float32)
    thr = np.empty(H, np.float32)
    lib().oracle_med3_threshold(_ptr(x), _x_dtype(x), B, H, T, D, float(C), gran,
                                _ptr(rmed), _ptr(thr))
    return rmed, thr


def extract(x, thr, gran=CHUNK, cap=None):
    """Ordered outlier list: (idx u32[n], val u16[n,4] or [n], slab_off u32[B*H+1],
    required count, status dict)."""
    B, H, T, D = x.shape
    x = np.ascontiguousarray(x)
    thr = _c(thr, np.float32)
    if cap is None:
        cap = B * H * T * D // 4 if gran == CHUNK else B * H * T * D
    idx = np.zeros(max(cap, 1), np.uint32)
    vw = 4 if gran == CHUNK else 1
    val = np.zeros((max(cap, 1), vw), np.uint16)
    slab_off = np.zeros(B * H + 1, np.uint32)
    st = Status()
    n = lib().oracle_extract(_ptr(x), _x_dtype(x), B, H, T, D, _ptr(thr), gran,
                             _ptr(idx), _ptr(val), _ptr(slab_off), int(cap), ctypes.byref(st))
    k = min(n, cap)
    v = val[:k] if gran == CHUNK else val[:k, 0]
    return idx[:k], v, slab_off, int(n), st.as_dict()


def encode(x, codebook, S, thr=None, gran=CHUNK):
    """Whole-call encode.  Returns (words u32, radius u16 [chunks], best f32,
    second f32, status dict)."""
    B, H, T, D = x.shape
    x = np.ascontiguousarray(x)
    cb = _c(codebook, np.float32)
    assert cb.size == H * S * 4
    n_chunks = B * H * T * D // 4
    words = np.zeros(index_words(B, H, T, D, S), np.uint32)
    radius = np.zeros(n_chunks, np.uint16)
    best = np.zeros(n_chunks, np.float32)
    second = np.zeros(n_chunks, np.float32)
    thr_a = None if thr is None else _c(thr, np.float32)
    st = Status()
    lib().oracle_encode(_ptr(x), _x_dtype(x), B, H, T, D, _ptr(cb), int(S), _ptr(thr_a), gran,
                        _ptr(words), _ptr(radius), _ptr(best), _ptr(second), ctypes.byref(st))
    return words, radius, best, second, st.as_dict()


def encode_chunks(x, codebook, S, chunks, thr=None, gran=CHUNK):
    """Encode only the listed flat chunk indices: (idx, radius, best, second)."""
    B, H, T, D = x.shape
    x = np.ascontiguousarray(x)
    cb = _c(codebook, np.float32)
    chunks = _c(chunks, np.int64)
    n = chunks.size
    idx = np.zeros(n, np.uint32)
    radius = np.zeros(n, np.uint16)
    best = np.zeros(n, np.float32)
    second = np.zeros(n, np.float32)
    thr_a = None if thr is None else _c(thr, np.float32)
    lib().oracle_encode_chunks(_ptr(x), _x_dtype(x), B, H, T, D, _ptr(cb), int(S), _ptr(thr_a),
                               gran, _ptr(chunks), n, _ptr(idx), _ptr(radius), _ptr(best),
                               _ptr(second))
    return idx, radius, best, second


def score_chunks(x, codebook, S, chunks, idx, thr=None, gran=CHUNK):
    """fp32 oracle score of the given codeword index for each listed chunk."""
    B, H, T, D = x.shape
    x = np.ascontiguousarray(x)
    cb = _c(codebook, np.float32)
    chunks = _c(chunks, np.int64)
    idx = _c(idx, np.uint32)
    out = np.zeros(chunks.size, np.float32)
    thr_a = None if thr is None else _c(thr, np.float32)
    lib().oracle_score_chunks(_ptr(x), _x_dtype(x), B, H, T, D, _ptr(cb), int(S), _ptr(thr_a),
                              gran, _ptr(chunks), _ptr(idx), chunks.size, _ptr(out))
    return out


def get_index(words, S, chunks):
    words = _c(words, np.uint32)
    chunks = _c(chunks, np.int64)
    out = np.zeros(chunks.size, np.uint32)
    lib().oracle_get_index_array(_ptr(words), index_bits(S), _ptr(chunks), chunks.size, _ptr(out))
    return out


def decode(words, radius, codebook, S, B, H, T, D, out_idx=None, out_val=None,
           gran=CHUNK, out_dtype=BF16):
    """Whole-call decode; returns (y [B,H,T,D] as uint16 bf16 bits or float32,
    status dict)."""
    words = _c(words, np.uint32)
    radius = _c(radius, np.uint16)
    cb = _c(codebook, np.float32)
    n_out = 0
    oi = ov = None
    if out_idx is not None and len(out_idx) > 0:
        oi = _c(out_idx, np.uint32)
        ov = _c(out_val, np.uint16)
        n_out = oi.size
    y = np.zeros((B, H, T, D), np.uint16 if out_dtype == BF16 else np.float32)
    st = Status()
    lib().oracle_decode(_ptr(words), _ptr(radius), _ptr(cb), int(S), _ptr(oi), _ptr(ov), n_out,
                        gran, B, H, T, D, _ptr(y), out_dtype, ctypes.byref(st))
    return y, st.as_dict()


def radius_level(radius_f16, thr, S):
    """Level k of one fp16 radius (bits) for threshold thr: the quantized-radius
    reading (uniform on [0, thr], L = 24 S levels); see hqmq_oracle.c."""
    return int(lib().oracle_radius_level(int(radius_f16), float(thr), 24 * int(S)))


def radius_of_level(k, thr, S):
    return float(lib().oracle_radius_of_level(int(k), float(thr), 24 * int(S)))


def quantize_radius(radius, thr, B, H, T, D, S):
    """Radius codes of a whole call (uint32 words laid out like the index words)."""
    radius = _c(radius, np.uint16)
    thr = _c(thr, np.float32)
    words = np.zeros(index_words(B, H, T, D, S), np.uint32)
    lib().oracle_quantize_radius(_ptr(radius), _ptr(thr), B, H, T, D, int(S), _ptr(words))
    return words


def decode_qradius(words, rcode_words, thr, codebook, S, B, H, T, D, out_idx=None, out_val=None,
                   gran=CHUNK, out_dtype=BF16):
    """decode() with each chunk's radius taken from its radius code."""
    words = _c(words, np.uint32)
    rw = _c(rcode_words, np.uint32)
    thr = _c(thr, np.float32)
    cb = _c(codebook, np.float32)
    n_out = 0
    oi = ov = None
    if out_idx is not None and len(out_idx) > 0:
        oi = _c(out_idx, np.uint32)
        ov = _c(out_val, np.uint16)
        n_out = oi.size
    y = np.zeros((B, H, T, D), np.uint16 if out_dtype == BF16 else np.float32)
    st = Status()
    lib().oracle_decode_qradius(_ptr(words), _ptr(rw), _ptr(thr), _ptr(cb), int(S), _ptr(oi),
                                _ptr(ov), n_out, gran, B, H, T, D, _ptr(y), out_dtype,
                                ctypes.byref(st))
    return y, st.as_dict()


def attention_decode(q_bits, k_hat, v_hat, scale, G, seq_len=None):
    """Decode-phase attention over decoded caches, in fp64 (numpy).

    The pages run their decoder inside the attention kernel
    (gist.science/nl, Technische Samenvatting, "Memory en Latentie"); what
    that kernel feeds is plain scaled dot-product attention of one new query
    token per sequence over the decoded keys and values.  Written out:
      q      = the bf16 query values, q_bits uint16 [B, Hq, D];
      K, V   = k_hat / v_hat [B, Hk, T, D] (the decoded values, any float type);
      len_b  = seq_len[b] clamped to [0, T] (None: T);
      for query head h the KV head is h // G (G consecutive query heads share
      one KV head);
      s_t    = scale * <q[b, h], K[b, h // G, t]>, t < len_b;
      o[b, h] = sum_t exp(s_t) V[b, h // G, t] / sum_t exp(s_t)   (0 if len_b = 0).
    The maximum of s is subtracted before exp (the ratio is unchanged)."""
    q = bf16_to_f32(np.asarray(q_bits, np.uint16)).astype(np.float64)
    B, Hq, D = q.shape
    T = k_hat.shape[2]
    o = np.zeros((B, Hq, D), np.float64)
    for b in range(B):
        n = T if seq_len is None else min(max(int(seq_len[b]), 0), T)
        if n == 0:
            continue
        for h in range(Hq):
            K = np.asarray(k_hat[b, h // G, :n], np.float64)
            V = np.asarray(v_hat[b, h // G, :n], np.float64)
            s = scale * (K @ q[b, h])
            w = np.exp(s - s.max())
            o[b, h] = (w @ V) / w.sum()
    return o


def joint_block_chunks(S):
    """Chunks per block of the joint (index, radius level) code."""
    return int(lib().oracle_joint_block_chunks(int(S)))


def joint_block_bits(S):
    """Bits per block of the joint code."""
    return int(lib().oracle_joint_block_bits(int(S)))


def joint_words(B, H, T, D, S):
    return B * H * int(lib().oracle_joint_slab_words(T, D, int(S)))


def pack_joint(words, rcode_words, B, H, T, D, S):
    """Joint code of a call from its index and radius-code words: (uint32
    words of the B*H slab runs, number of chunks stored as digit 0 because
    their index or level was out of range)."""
    words = _c(words, np.uint32)
    rw = _c(rcode_words, np.uint32)
    out = np.zeros(joint_words(B, H, T, D, S), np.uint32)
    bad = lib().oracle_pack_joint(_ptr(words), _ptr(rw), B, H, T, D, int(S), _ptr(out))
    return out, int(bad)


def unpack_joint(joint, B, H, T, D, S):
    """(index, level) of every chunk of a call from its joint code."""
    joint = _c(joint, np.uint32)
    n = B * H * T * D // 4
    idx = np.zeros(n, np.uint32)
    k = np.zeros(n, np.uint32)
    lib().oracle_unpack_joint(_ptr(joint), B, H, T, D, int(S), _ptr(idx), _ptr(k))
    return idx, k


def list_flags(out_idx, n_chunks):
    """Per packing group of 32 chunks, the flag word of its listed outliers."""
    oi = _c(out_idx, np.uint32)
    flags = np.zeros(n_chunks // 32, np.uint32)
    lib().oracle_list_flags(_ptr(oi), oi.size, int(n_chunks), _ptr(flags))
    return flags


def list_from_flags(flags, n_chunks, cap=None):
    flags = _c(flags, np.uint32)
    cap = int(n_chunks) if cap is None else int(cap)
    out = np.zeros(max(cap, 1), np.uint32)
    n = lib().oracle_list_from_flags(_ptr(flags), int(n_chunks), _ptr(out), cap)
    return out[:min(n, cap)], int(n)
