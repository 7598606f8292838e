"""Thin Python binding of libhqmq (include/hqmq.h).

Argument marshalling only: every step of the HQMQ path runs in the CUDA
kernels of libhqmq.so.  torch provides device memory and streams.  There is no
fallback: if the library is missing or fails to load, importing this module
raises.

Entry points keep the C names.  Tensors are passed where the C ABI takes
device pointers; shapes and dtypes are read from them; `stream` defaults to
torch's current stream.  Non-zero return codes raise HQMQError.

A serving flow, per (layer, role) cache x [B, H, T, 128] (bf16):

    hqmq_make_codebook(seed, S, n_groups, 0, cb)          # once per model
    hqmq_make_search_table(cb_call, S, H, table)          # once per model (S <= 48)
    hqmq_encode_med3(x, 3.0, HQMQ_GRAN_CHUNK, cb_call, S, table, words, radius, rmed,
                     thr, out_idx, out_val, slab_off, cap, ws, tile_off=tile_off)
    # optional 2b bits per chunk: hqmq_quantize_radius(radius, thr, x.shape, S, rwords)
    # decode step, every (layer, role) at once, against the prefill's thr:
    hqmq_append_batch(x_new, thr_all, HQMQ_GRAN_CHUNK, cb_all, S, words_new, radius_new,
                      oi_new, ov_new, so_new, cap_new, tile_off=to_new)
    # attention of the new queries straight from the codes:
    k = kv_codes(words_k, radius_k, cb_k, out_idx_k, out_val_k, tile_off_k, cap, 0)
    v = kv_codes(words_v, radius_v, cb_v, out_idx_v, out_val_v, tile_off_v, cap, 0)
    hqmq_attention_decode(q, k, v, S, H, T, o, alloc_attention_ws(B, H), seq_len=lens)
    # or the dense cache: hqmq_decode(words, radius, cb_call, S, out_idx, out_val,
    #                                  slab_off, cap, 0, y, tile_off=tile_off)
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhqmq.so")

HQMQ_OK, HQMQ_ERR_ARG, HQMQ_ERR_ALIGN, HQMQ_ERR_CUDA, HQMQ_ERR_WORKSPACE = 0, 1, 2, 3, 4
HQMQ_BF16, HQMQ_F32 = 0, 1
HQMQ_GRAN_CHUNK, HQMQ_GRAN_ELEMENT = 0, 1
FLAG_OUTLIER_OVERFLOW, FLAG_SATURATED, FLAG_NONFINITE, FLAG_BAD_INDEX = 1, 2, 4, 8
FLAG_MED3_FALLBACK = 16


class HQMQError(RuntimeError):
    def __init__(self, fn, rc):
        super().__init__("%s failed: %s (%d)" % (fn, _lib.hqmq_error_string(rc).decode(), rc))
        self.rc = rc


if not os.path.exists(LIB_PATH):
    raise ImportError("libhqmq.so is not built (%s); run "
                      "`python -m kv_cache_quantization_hqmq_b200.build`" % LIB_PATH)

_lib = ctypes.CDLL(LIB_PATH)
_P, _I, _U32, _U64, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_float
_SIGS = {
    "hqmq_version": (ctypes.c_char_p, []),
    "hqmq_error_string": (ctypes.c_char_p, [_I]),
    "hqmq_index_bits": (_U32, [_U32]),
    "hqmq_index_words": (_U64, [_I, _I, _I, _I, _U32]),
    "hqmq_make_codebook": (_I, [_U64, _U32, _U32, _U32, _P, _P]),
    "hqmq_outlier_workspace_size": (_U64, [_I, _I, _I, _I, _I]),
    "hqmq_outlier_extract": (_I, [_P, _I, _I, _I, _I, _I, _F, _I, _P, _P, _P, _P, _P, _P, _U64,
                                  _P, _U64, _P, _P]),
    "hqmq_list_tiles": (_U64, [_I, _I, _I, _I]),
    "hqmq_encode": (_I, [_P, _I, _I, _I, _I, _I, _P, _U32, _P, _I, _P, _P, _P, _P]),
    "hqmq_decode": (_I, [_P, _P, _P, _U32, _P, _P, _P, _P, _U64, _I, _I, _I, _I, _I, _P, _I, _P,
                         _P]),
    "hqmq_outlier_extract_noalloc": (_I, [_P, _I, _I, _I, _I, _I, _F, _I, _P, _P, _P, _P, _P,
                                          _U64, _P, _P]),
    "hqmq_encode_med3_workspace_size": (_U64, [_I, _I, _I, _I, _I]),
    "hqmq_encode_med3": (_I, [_P, _I, _I, _I, _I, _I, _F, _I, _P, _U32, _P, _P, _P, _P, _P, _P,
                              _P, _P, _P, _U64, _P, _U64, _P, _P]),
    "hqmq_search_table_bytes": (_U64, [_U32]),
    "hqmq_make_search_table": (_I, [_P, _U32, _U32, _P, _P]),
    "hqmq_encode_lut": (_I, [_P, _I, _I, _I, _I, _I, _P, _U32, _P, _P, _I, _P, _P, _P, _P]),
    "hqmq_quantize_radius": (_I, [_P, _P, _I, _I, _I, _I, _U32, _P, _P]),
    "hqmq_append_batch": (_I, [_P, _I, _I, _I, _I, _I, _I, _P, _I, _P, _U32, _P, _P, _P, _P, _P,
                               _P, _U64, _P, _P]),
    "hqmq_outlier_extract_given_thr_workspace_size": (_U64, [_I, _I, _I, _I]),
    "hqmq_outlier_extract_given_thr": (_I, [_P, _I, _I, _I, _I, _I, _P, _I, _P, _P, _P, _P, _U64,
                                            _P, _U64, _P, _P]),
    "hqmq_decode_qradius": (_I, [_P, _P, _P, _P, _U32, _P, _P, _P, _U64, _I, _I, _I, _I, _I, _P,
                                 _I, _P, _P]),
    "hqmq_joint_block": (None, [_U32, _P, _P]),
    "hqmq_joint_words": (_U64, [_I, _I, _I, _I, _U32]),
    "hqmq_pack_joint": (_I, [_P, _P, _U32, _I, _I, _I, _I, _P, _P, _P]),
    "hqmq_list_flags": (_I, [_P, _P, _U64, _I, _I, _I, _I, _P, _P]),
    "hqmq_decode_joint": (_I, [_P, _P, _P, _U32, _P, _P, _P, _U64, _I, _I, _I, _I, _P, _I, _P]),
    "hqmq_attention_workspace_size": (_U64, [_I, _I]),
    "hqmq_attention_decode": (_I, [_P, _P, _P, _P, _U32, _I, _I, _I, _I, _I, _F, _P, _I, _P,
                                   _U64, _P, _P]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def lib():
    return _lib


def _check(name, rc):
    if rc != HQMQ_OK:
        raise HQMQError(name, rc)


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return HQMQ_BF16
    if t.dtype == torch.float32:
        return HQMQ_F32
    raise TypeError("HQMQ tensors are bf16 or fp32, got %s" % t.dtype)


def _shape4(x):
    if x.dim() != 4:
        raise ValueError("expected a [B, H, T, D] tensor, got shape %s" % (tuple(x.shape),))
    if not x.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return tuple(int(v) for v in x.shape)


# ---------------------------------------------------------------- queries
def hqmq_version():
    return _lib.hqmq_version().decode()


def hqmq_index_bits(S):
    return int(_lib.hqmq_index_bits(S))


def hqmq_index_words(B, H, T, D, S):
    return int(_lib.hqmq_index_words(B, H, T, D, S))


def hqmq_outlier_workspace_size(B, H, T, D, gran=HQMQ_GRAN_CHUNK):
    return int(_lib.hqmq_outlier_workspace_size(B, H, T, D, gran))


def hqmq_encode_med3_workspace_size(B, H, T, D, gran=HQMQ_GRAN_CHUNK):
    return int(_lib.hqmq_encode_med3_workspace_size(B, H, T, D, gran))


# ---------------------------------------------------------------- calls
def hqmq_make_codebook(seed, S, n_groups, group0, codebook, stream=None):
    """codebook: fp32 device tensor of n_groups * S * 4 elements."""
    assert codebook.dtype == torch.float32 and codebook.numel() == n_groups * S * 4
    _check("hqmq_make_codebook", _lib.hqmq_make_codebook(seed, S, n_groups, group0,
                                                         _ptr(codebook), _stream(stream)))
    return codebook


def hqmq_outlier_extract(x, C, gran, rmed, thr, out_idx, out_val, slab_off, cap, ws,
                         status=None, stream=None, tile_off=None):
    """tile_off: optional uint32 [hqmq_list_tiles(B, H, T, D) + 1] output."""
    B, H, T, D = _shape4(x)
    _check("hqmq_outlier_extract", _lib.hqmq_outlier_extract(
        _ptr(x), _dtype_code(x), B, H, T, D, float(C), gran, _ptr(rmed), _ptr(thr),
        _ptr(out_idx), _ptr(out_val), _ptr(slab_off), _ptr(tile_off), int(cap), _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(status), _stream(stream)))


def hqmq_list_tiles(B, H, T, D):
    return int(_lib.hqmq_list_tiles(B, H, T, D))


def hqmq_outlier_extract_noalloc(x, C, gran, rmed, thr, out_idx, out_val, slab_off, cap,
                                 status=None, stream=None):
    """Med3x with the library's fixed 1 MiB device scratch instead of a
    caller workspace, for callers that cannot allocate device memory.  Calls
    on one device share that scratch: do not let two of them overlap."""
    B, H, T, D = _shape4(x)
    _check("hqmq_outlier_extract_noalloc", _lib.hqmq_outlier_extract_noalloc(
        _ptr(x), _dtype_code(x), B, H, T, D, float(C), gran, _ptr(rmed), _ptr(thr),
        _ptr(out_idx), _ptr(out_val), _ptr(slab_off), int(cap), _ptr(status), _stream(stream)))


def hqmq_encode(x, codebook, S, thr, gran, idx_words, radius, status=None, stream=None):
    B, H, T, D = _shape4(x)
    _check("hqmq_encode", _lib.hqmq_encode(
        _ptr(x), _dtype_code(x), B, H, T, D, _ptr(codebook), S, _ptr(thr), gran,
        _ptr(idx_words), _ptr(radius), _ptr(status), _stream(stream)))


def hqmq_search_table_bytes(S):
    return int(_lib.hqmq_search_table_bytes(S))


def hqmq_make_search_table(codebook, S, n_groups, table, stream=None):
    """table: uint8 device tensor of n_groups * hqmq_search_table_bytes(S) bytes."""
    assert table.numel() * table.element_size() >= n_groups * hqmq_search_table_bytes(S)
    _check("hqmq_make_search_table", _lib.hqmq_make_search_table(
        _ptr(codebook), S, n_groups, _ptr(table), _stream(stream)))
    return table


def hqmq_encode_lut(x, codebook, S, table, thr, gran, idx_words, radius, status=None,
                    stream=None):
    B, H, T, D = _shape4(x)
    _check("hqmq_encode_lut", _lib.hqmq_encode_lut(
        _ptr(x), _dtype_code(x), B, H, T, D, _ptr(codebook), S, _ptr(table), _ptr(thr), gran,
        _ptr(idx_words), _ptr(radius), _ptr(status), _stream(stream)))


def hqmq_encode_med3(x, C, gran, codebook, S, table, idx_words, radius, rmed, thr, out_idx,
                     out_val, slab_off, cap, ws, status=None, stream=None, tile_off=None):
    """Med3x + encode (table may be None: S-codeword loop); tile_off: optional
    uint32 [hqmq_list_tiles(B, H, T, D) + 1] output."""
    B, H, T, D = _shape4(x)
    _check("hqmq_encode_med3", _lib.hqmq_encode_med3(
        _ptr(x), _dtype_code(x), B, H, T, D, float(C), gran, _ptr(codebook), S, _ptr(table),
        _ptr(idx_words), _ptr(radius), _ptr(rmed), _ptr(thr), _ptr(out_idx), _ptr(out_val),
        _ptr(slab_off), _ptr(tile_off), int(cap), _ptr(ws), ws.numel() * ws.element_size(),
        _ptr(status), _stream(stream)))


def hqmq_decode(idx_words, radius, codebook, S, out_idx, out_val, slab_off, cap, gran, y,
                status=None, stream=None, tile_off=None):
    """tile_off: the list's tile offsets (applied in the main pass), or None."""
    B, H, T, D = _shape4(y)
    _check("hqmq_decode", _lib.hqmq_decode(
        _ptr(idx_words), _ptr(radius), _ptr(codebook), S, _ptr(out_idx), _ptr(out_val),
        _ptr(slab_off), _ptr(tile_off), int(cap), gran, B, H, T, D, _ptr(y), _dtype_code(y),
        _ptr(status), _stream(stream)))


def hqmq_outlier_extract_given_thr_workspace_size(B, H, T, D):
    return int(_lib.hqmq_outlier_extract_given_thr_workspace_size(B, H, T, D))


def hqmq_outlier_extract_given_thr(x, thr, gran, out_idx, out_val, slab_off, cap, ws,
                                   status=None, stream=None, tile_off=None):
    """Med3x list of x under a given threshold thr [H] (no median of its own):
    the streaming form for decode-phase tokens."""
    B, H, T, D = _shape4(x)
    _check("hqmq_outlier_extract_given_thr", _lib.hqmq_outlier_extract_given_thr(
        _ptr(x), _dtype_code(x), B, H, T, D, _ptr(thr), gran, _ptr(out_idx), _ptr(out_val),
        _ptr(slab_off), _ptr(tile_off), int(cap), _ptr(ws), ws.numel() * ws.element_size(),
        _ptr(status), _stream(stream)))


def hqmq_append_batch(x, thr, gran, codebook, S, idx_words, radius, out_idx, out_val, slab_off,
                      cap, tile_off=None, status=None, stream=None):
    """n_calls small calls in one launch; x: [n_calls, B, H, T, D]; every other
    array holds the calls' arrays back to back (see include/hqmq.h)."""
    if x.dim() != 5 or not x.is_contiguous():
        raise ValueError("x must be a contiguous [n_calls, B, H, T, D] tensor")
    C, B, H, T, D = (int(v) for v in x.shape)
    _check("hqmq_append_batch", _lib.hqmq_append_batch(
        _ptr(x), _dtype_code(x), C, B, H, T, D, _ptr(thr), gran, _ptr(codebook), S,
        _ptr(idx_words), _ptr(radius), _ptr(out_idx), _ptr(out_val), _ptr(slab_off),
        _ptr(tile_off), int(cap), _ptr(status), _stream(stream)))


def hqmq_quantize_radius(radius, thr, shape, S, rcode_words, stream=None):
    """Radius codes (b bits per chunk, uniform on [0, thr_h], 24 S levels) of a
    call's fp16 radii; shape = (B, H, T, D)."""
    B, H, T, D = shape
    _check("hqmq_quantize_radius", _lib.hqmq_quantize_radius(
        _ptr(radius), _ptr(thr), B, H, T, D, S, _ptr(rcode_words), _stream(stream)))
    return rcode_words


def hqmq_decode_qradius(idx_words, rcode_words, thr, codebook, S, out_idx, out_val, tile_off,
                        cap, gran, y, status=None, stream=None):
    """hqmq_decode with the radii taken from their codes; a list needs tile_off."""
    B, H, T, D = _shape4(y)
    _check("hqmq_decode_qradius", _lib.hqmq_decode_qradius(
        _ptr(idx_words), _ptr(rcode_words), _ptr(thr), _ptr(codebook), S, _ptr(out_idx),
        _ptr(out_val), _ptr(tile_off), int(cap), gran, B, H, T, D, _ptr(y), _dtype_code(y),
        _ptr(status), _stream(stream)))


def hqmq_joint_block(S):
    """(chunks per block, bits per block) of the joint (index, level) code."""
    n, w = ctypes.c_uint32(0), ctypes.c_uint32(0)
    _lib.hqmq_joint_block(S, ctypes.byref(n), ctypes.byref(w))
    return n.value, w.value


def hqmq_joint_words(B, H, T, D, S):
    return int(_lib.hqmq_joint_words(B, H, T, D, S))


def alloc_joint(B, H, T, D, S, device="cuda"):
    n = hqmq_joint_words(B, H, T, D, S)
    if n == 0:
        raise ValueError("bad shape/S for the joint code")
    return torch.empty(n, dtype=torch.int32, device=device)


def hqmq_pack_joint(idx_words, rcode_words, S, shape, joint, status=None, stream=None):
    """The joint code of a call (shape = (B, H, T, D)) from its index and
    radius-code words."""
    B, H, T, D = shape
    _check("hqmq_pack_joint", _lib.hqmq_pack_joint(
        _ptr(idx_words), _ptr(rcode_words), S, B, H, T, D, _ptr(joint), _ptr(status),
        _stream(stream)))
    return joint


def hqmq_list_flags(out_idx, slab_off, cap, shape, flags, stream=None):
    """The 1-bit outlier flags (uint32 [B*H*T*D/128]) of a chunk-mode list."""
    B, H, T, D = shape
    _check("hqmq_list_flags", _lib.hqmq_list_flags(
        _ptr(out_idx), _ptr(slab_off), int(cap), B, H, T, D, _ptr(flags), _stream(stream)))
    return flags


def hqmq_decode_joint(joint, thr, codebook, S, flags, out_val, tile_off, cap, y, stream=None):
    """Decode from the joint code; flags (with the list's values and tile
    offsets) restore the chunk-mode outliers, or None."""
    B, H, T, D = _shape4(y)
    _check("hqmq_decode_joint", _lib.hqmq_decode_joint(
        _ptr(joint), _ptr(thr), _ptr(codebook), S, _ptr(flags), _ptr(out_val), _ptr(tile_off),
        int(cap), B, H, T, D, _ptr(y), _dtype_code(y), _stream(stream)))


class KVCodes(ctypes.Structure):
    """hqmq_kv_codes: one coded K or V cache (device pointers)."""
    _fields_ = [("idx_words", _P), ("radius", _P), ("codebook", _P), ("out_idx", _P),
                ("out_val", _P), ("tile_off", _P), ("cap", _U64), ("gran", _I),
                ("rcode_words", _P), ("thr", _P)]


def kv_codes(idx_words, radius, codebook, out_idx=None, out_val=None, tile_off=None, cap=0,
             gran=HQMQ_GRAN_CHUNK, rcode_words=None, thr=None):
    """The hqmq_kv_codes record of one coded cache (the tensors must outlive
    the calls that use it).  rcode_words + thr: the quantized-radius format
    (radius may then be None)."""
    c = KVCodes(_ptr(idx_words), _ptr(radius), _ptr(codebook), _ptr(out_idx), _ptr(out_val),
                _ptr(tile_off), int(cap) if out_idx is not None else 0, int(gran),
                _ptr(rcode_words), _ptr(thr))
    c._keep = (idx_words, radius, codebook, out_idx, out_val, tile_off, rcode_words, thr)
    return c


def hqmq_attention_workspace_size(B, Hk):
    return int(_lib.hqmq_attention_workspace_size(B, Hk))


def hqmq_attention_decode(q, k, v, S, Hk, T, o, ws, scale=None, seq_len=None, status=None,
                          stream=None):
    """o[b, h] = softmax(scale q[b, h] K^T) V over the first seq_len[b] tokens
    of the coded caches k, v (KVCodes from kv_codes; [B, Hk, T, 128]).
    q: bf16 [B, Hq, 128]; o: bf16 or fp32 [B, Hq, 128]; seq_len: int32 [B]
    or None; scale defaults to 1/sqrt(128)."""
    if q.dim() != 3 or q.dtype != torch.bfloat16 or not q.is_contiguous():
        raise ValueError("q must be a contiguous bf16 [B, Hq, D] tensor")
    B, Hq, D = (int(v_) for v_ in q.shape)
    if scale is None:
        scale = D ** -0.5
    _check("hqmq_attention_decode", _lib.hqmq_attention_decode(
        _ptr(q), _ptr(seq_len), ctypes.byref(k), ctypes.byref(v), S, B, Hq, Hk, T, D,
        float(scale), _ptr(o), _dtype_code(o), _ptr(ws), ws.numel() * ws.element_size(),
        _ptr(status), _stream(stream)))
    return o


def alloc_attention_ws(B, Hk, device="cuda"):
    return torch.empty(hqmq_attention_workspace_size(B, Hk), dtype=torch.uint8, device=device)


# ---------------------------------------------------------------- buffers
def new_status(device="cuda"):
    """A zeroed device hqmq_status (4 x 64-bit words)."""
    return torch.zeros(4, dtype=torch.int64, device=device)


def read_status(status):
    v = status.cpu().numpy().view("uint64")
    return {"flags": int(v[0] & 0xFFFFFFFF), "n_outliers": int(v[1]),
            "n_saturated": int(v[2]), "n_nonfinite": int(v[3])}


def alloc_codes(B, H, T, D, S, device="cuda"):
    """(idx_words uint32 as int32, radius fp16 bits as int16) for one call."""
    nw = hqmq_index_words(B, H, T, D, S)
    if nw == 0:
        raise ValueError("bad shape/S")
    words = torch.empty(nw, dtype=torch.int32, device=device)
    radius = torch.empty(B * H * T * D // 4, dtype=torch.int16, device=device)
    return words, radius


def alloc_tile_off(B, H, T, D, device="cuda"):
    """uint32 (as int32) [hqmq_list_tiles + 1]: a call's list tile offsets."""
    n = hqmq_list_tiles(B, H, T, D)
    if n == 0:
        raise ValueError("bad shape")
    return torch.empty(n + 1, dtype=torch.int32, device=device)


def alloc_outliers(B, H, T, D, cap, gran=HQMQ_GRAN_CHUNK, device="cuda"):
    """(rmed, thr, out_idx, out_val, slab_off, ws) for one call's Med3x step."""
    rmed = torch.empty(H, dtype=torch.float32, device=device)
    thr = torch.empty(H, dtype=torch.float32, device=device)
    out_idx = torch.empty(max(cap, 1), dtype=torch.int32, device=device)
    out_val = torch.empty(max(cap, 1) * (4 if gran == HQMQ_GRAN_CHUNK else 1), dtype=torch.int16,
                          device=device)
    slab_off = torch.empty(B * H + 1, dtype=torch.int32, device=device)
    ws = torch.empty(hqmq_outlier_workspace_size(B, H, T, D, gran), dtype=torch.uint8,
                     device=device)
    return rmed, thr, out_idx, out_val, slab_off, ws
