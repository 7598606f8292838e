"""Helpers of the GPU parity tests: run the CUDA path through the C ABI and
compare it with the CPU oracle on the same seeded inputs.

Tolerances (the method's own bar):
* codeword indices: bit-exact, except where the oracle's fp32 score of the
  GPU's pick is within NEAR_TIE_REL (relative) of the oracle's best score; such
  near-ties are counted and reported;
* radius, Med3x thresholds, outlier lists, decoded values from the same codes:
  bit-exact (NaN equals NaN, +0 equals -0);
* decoded values end to end (GPU encode + decode vs oracle encode + decode):
  within DECODE_ABS_TOL absolute, outside the exempt near-tie chunks.
"""
import numpy as np
import torch

from kv_cache_quantization_hqmq_b200 import hqmq
from kv_cache_quantization_hqmq_b200.workloads import as_numpy_bits

NEAR_TIE_REL = 1e-6
DECODE_ABS_TOL = 1e-3


def unpack_indices(words, S, n_chunks):
    """Vectorised LSB-first unpack of the packed index words (numpy)."""
    b = hqmq.hqmq_index_bits(S)
    w = np.ascontiguousarray(np.asarray(words).view(np.uint32)).reshape(-1, b)
    bits = np.unpackbits(w.view(np.uint8), bitorder="little").reshape(w.shape[0], 32 * b)
    bits = bits.reshape(w.shape[0], 32, b).astype(np.uint32)
    idx = (bits << np.arange(b, dtype=np.uint32)).sum(axis=2, dtype=np.uint32)
    return idx.reshape(-1)[:n_chunks]


def to_host(t):
    return t.detach().cpu().numpy()


def same_f16_or_bf16_bits(a, b, bf16):
    a = np.asarray(a).view(np.uint16)
    b = np.asarray(b).view(np.uint16)
    inf = 0x7F80 if bf16 else 0x7C00
    nan_a, nan_b = (a & 0x7FFF) > inf, (b & 0x7FFF) > inf
    zero = ((a & 0x7FFF) == 0) & ((b & 0x7FFF) == 0)
    return (a == b) | (nan_a & nan_b) | zero


def same_f32(a, b):
    a = np.asarray(a, np.float32)
    b = np.asarray(b, np.float32)
    return (a.view(np.uint32) == b.view(np.uint32)) | (np.isnan(a) & np.isnan(b)) | \
        ((a == 0) & (b == 0))


# ------------------------------------------------------------------ GPU path
def gpu_codebook(seed, S, n_groups, group0=0):
    cb = torch.empty(n_groups * S * 4, dtype=torch.float32, device="cuda")
    hqmq.hqmq_make_codebook(seed, S, n_groups, group0, cb)
    return cb


def gpu_med3(x_dev, C=3.0, gran=0, cap=None):
    B, H, T, D = x_dev.shape
    n = B * H * T * D // 4 if gran == 0 else B * H * T * D
    cap = n if cap is None else cap
    st = hqmq.new_status()
    rmed, thr, oi, ov, so, ws = hqmq.alloc_outliers(B, H, T, D, cap, gran)
    to = hqmq.alloc_tile_off(B, H, T, D)
    hqmq.hqmq_outlier_extract(x_dev, C, gran, rmed, thr, oi, ov, so, cap, ws, st, tile_off=to)
    torch.cuda.synchronize()
    return dict(rmed=rmed, thr=thr, out_idx=oi, out_val=ov, slab_off=so, tile_off=to, cap=cap,
                status=hqmq.read_status(st))


LIST_TILE_CHUNKS = 1024


def list_tile_off(idx, B, H, T, D, gran=0):
    """The list's tile offsets from their definition: for every tile (1024
    consecutive chunks of a slab, the slab's last tile possibly shorter) the
    number of list entries before its first chunk, then the total."""
    cps = T * D // 4
    tps = -(-cps // LIST_TILE_CHUNKS)
    starts = (np.arange(B * H)[:, None] * cps +
              np.minimum(np.arange(tps)[None, :] * LIST_TILE_CHUNKS, cps)).reshape(-1)
    chunk = np.asarray(idx, np.int64) // (4 if gran else 1)
    off = np.searchsorted(chunk, starts, side="left")
    return np.concatenate([off, [len(chunk)]]).astype(np.uint32)


def gpu_search_table(cb_dev, S, n_groups):
    t = torch.empty(n_groups * hqmq.hqmq_search_table_bytes(S), dtype=torch.uint8, device="cuda")
    hqmq.hqmq_make_search_table(cb_dev, S, n_groups, t)
    return t


def gpu_encode(x_dev, cb_dev, S, thr_dev=None, gran=0, encoder="sloop"):
    """encoder: "sloop" (hqmq_encode) or "lut" (hqmq_encode_lut with tables
    built here from the same codebook)."""
    B, H, T, D = x_dev.shape
    words, radius = hqmq.alloc_codes(B, H, T, D, S)
    st = hqmq.new_status()
    if encoder == "lut":
        table = gpu_search_table(cb_dev, S, H)
        hqmq.hqmq_encode_lut(x_dev, cb_dev, S, table, thr_dev, gran, words, radius, st)
    else:
        hqmq.hqmq_encode(x_dev, cb_dev, S, thr_dev, gran, words, radius, st)
    torch.cuda.synchronize()
    return words, radius, hqmq.read_status(st)


def gpu_decode(words, radius, cb_dev, S, shape, out_dtype=torch.bfloat16, med=None, gran=0,
               tiles=False):
    """tiles: apply the list through med["tile_off"] (in the main pass)."""
    y = torch.empty(shape, dtype=out_dtype, device="cuda")
    st = hqmq.new_status()
    if med is None:
        hqmq.hqmq_decode(words, radius, cb_dev, S, None, None, None, 0, gran, y, st)
    else:
        hqmq.hqmq_decode(words, radius, cb_dev, S, med["out_idx"], med["out_val"],
                         med["slab_off"], med["cap"], gran, y, st,
                         tile_off=med["tile_off"] if tiles else None)
    torch.cuda.synchronize()
    return y, hqmq.read_status(st)


# ------------------------------------------------------------------ checks
def check_codes(oracle, x_np, cb_np, S, gpu_idx, gpu_radius, thr=None, gran=0, chunks=None):
    """Compare GPU indices / radii with the oracle on all chunks or a sample.
    Returns (n_checked, n_exempt_mismatch, n_near_tie)."""
    if chunks is None:
        words, rad_o, best, second, _ = oracle.encode(x_np, cb_np, S, thr=thr, gran=gran)
        idx_o = unpack_indices(words, S, rad_o.size)
        chunks = np.arange(rad_o.size, dtype=np.int64)
        gi, gr = gpu_idx, gpu_radius
    else:
        chunks = np.asarray(chunks, np.int64)
        idx_o, rad_o, best, second = oracle.encode_chunks(x_np, cb_np, S, chunks, thr=thr,
                                                          gran=gran)
        gi, gr = gpu_idx[chunks], gpu_radius[chunks]
    assert np.array_equal(np.asarray(gr).view(np.uint16), rad_o), "radius mismatch"
    mm = np.nonzero(gi != idx_o)[0]
    if mm.size:
        sg = oracle.score_chunks(x_np, cb_np, S, chunks[mm], gi[mm], thr=thr, gran=gran)
        gap = best[mm].astype(np.float64) - sg.astype(np.float64)
        bad = gap > NEAR_TIE_REL * np.abs(best[mm].astype(np.float64))
        assert not bad.any(), "non-tie index mismatch at chunks %s (gap %s)" % (
            chunks[mm][bad][:10], gap[bad][:10])
    nz = best > 0          # zero (or zeroed outlier) chunks have no search
    near = int(np.sum(nz & (best.astype(np.float64) - second.astype(np.float64)
                            <= NEAR_TIE_REL * np.abs(best.astype(np.float64)))))
    return chunks.size, int(mm.size), near


def check_med3(oracle, x_np, g, C=3.0, gran=0):
    """Thresholds and the whole outlier list bit-exact against the oracle."""
    rmed_o, thr_o = oracle.med3_threshold(x_np, C, gran)
    assert same_f32(to_host(g["rmed"]), rmed_o).all(), (to_host(g["rmed"]), rmed_o)
    assert same_f32(to_host(g["thr"]), thr_o).all()
    idx_o, val_o, so_o, n_o, st_o = oracle.extract(x_np, thr_o, gran=gran, cap=g["cap"])
    so = to_host(g["slab_off"]).view(np.uint32)
    assert np.array_equal(so, so_o)
    assert g["status"]["n_outliers"] == n_o
    k = min(n_o, g["cap"])
    assert np.array_equal(to_host(g["out_idx"]).view(np.uint32)[:k], idx_o[:k])
    vw = 4 if gran == 0 else 1
    gv = to_host(g["out_val"]).view(np.uint16)[:k * vw].reshape(-1, vw) if gran == 0 else \
        to_host(g["out_val"]).view(np.uint16)[:k]
    assert same_f16_or_bf16_bits(gv, val_o, bf16=False).all()
    if g.get("tile_off") is not None:
        full = idx_o if k == n_o else oracle.extract(x_np, thr_o, gran=gran)[0]
        B, H, T, D = x_np.shape
        assert np.array_equal(to_host(g["tile_off"]).view(np.uint32),
                              list_tile_off(full, B, H, T, D, gran))
    return thr_o, idx_o, val_o, so_o, n_o
