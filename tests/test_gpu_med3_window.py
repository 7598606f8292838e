"""Med3x against the oracle: hqmq_outlier_extract's window pipeline (two reads
of x) and the fused hqmq_encode_med3 (one read of x in chunk mode with search
tables: speculative encode plus fix-up pass; two reads otherwise), including
inputs built to defeat the sample window (so the exact fallback decides) and
to overflow its buffers, and the status counts of the fused call."""
import numpy as np
import pytest
import torch

from _parity import (check_codes, check_med3, gpu_search_table, same_f16_or_bf16_bits, same_f32,
                     to_host, unpack_indices)

pytestmark = pytest.mark.gpu
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

from kv_cache_quantization_hqmq_b200 import hqmq  # noqa: E402
from kv_cache_quantization_hqmq_b200 import workloads as W  # noqa: E402


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def x_dev(x):
    return dev(x.view(np.int16)).view(torch.bfloat16) if x.dtype == np.uint16 else dev(x)


def sampled_chunks(cps):
    """Mask of the chunks of a slab of cps chunks that the Med3x sample reads:
    quad q (one per 128 chunks) is chunks 4 (q mod 32) .. + 3 of the first
    128 of the (q div 32)-th run of 4096 chunks, or the first 4 of its own 128
    chunks when that lies past the slab."""
    mask = np.zeros(cps, dtype=bool)
    for q in range((cps + 127) // 128):
        j0 = (q // 32) * 4096 + 4 * (q % 32)
        if j0 + 4 > cps:
            j0 = q * 128
        mask[j0:j0 + 4] = True
    return mask


def fused(x_np, cb_np, S, gran, use_table, C=3.0, cap=None):
    B, H, T, D = x_np.shape
    xd = x_dev(x_np)
    cbd = dev(cb_np.reshape(-1))
    n = B * H * T * D // 4 if gran == 0 else B * H * T * D
    cap = n if cap is None else cap
    table = gpu_search_table(cbd, S, H) if use_table else None
    words, radius = hqmq.alloc_codes(B, H, T, D, S)
    rmed, thr, oi, ov, so, _ = hqmq.alloc_outliers(B, H, T, D, cap, gran)
    ws = torch.empty(hqmq.hqmq_encode_med3_workspace_size(B, H, T, D, gran), dtype=torch.uint8,
                     device="cuda")
    st = hqmq.new_status()
    to = hqmq.alloc_tile_off(B, H, T, D)
    hqmq.hqmq_encode_med3(xd, C, gran, cbd, S, table, words, radius, rmed, thr, oi, ov, so, cap,
                          ws, st, tile_off=to)
    torch.cuda.synchronize()
    return dict(words=words, radius=radius, rmed=rmed, thr=thr, out_idx=oi, out_val=ov,
                slab_off=so, tile_off=to, cap=cap, status=hqmq.read_status(st))


def check_fused(oracle, x_np, S, gran, use_table, seed=1, cap=None):
    B, H, T, D = x_np.shape
    cb = oracle.make_codebook(seed, S, H)
    g = fused(x_np, cb, S, gran, use_table, cap=cap)
    thr_o, *_ = check_med3(oracle, x_np, g, 3.0, gran)
    gi = unpack_indices(to_host(g["words"]), S, B * H * T * D // 4)
    n, mm, near = check_codes(oracle, x_np, cb, S, gi, to_host(g["radius"]), thr=thr_o, gran=gran)
    print("[fused] %s gran %d table %d: %d chunks, %d near-tie mismatches, %d outliers"
          % (x_np.shape, gran, use_table, n, mm, g["status"]["n_outliers"]))
    return g


@pytest.mark.parametrize("use_table", [True, False])
@pytest.mark.parametrize("gran", [0, 1])
def test_fused_qwen(oracle, gran, use_table):
    w = W.WORKLOADS["qwen_outlier"]
    x = W.as_numpy_bits(W.make_call_input(w, 4, 1, tokens=1024))
    g = check_fused(oracle, x, w.S, gran, use_table)
    if gran == 0:   # chunk norms: the sample window holds (element mode may fall back here)
        assert not g["status"]["flags"] & hqmq.FLAG_MED3_FALLBACK


@pytest.mark.parametrize("shape", [(1, 1, 32, 4), (2, 3, 8, 64), (3, 2, 200, 128),
                                   (1, 1, 4100, 128), (8, 2, 96, 128)])
def test_fused_shapes(oracle, shape):
    rng = np.random.default_rng(sum(shape) + 7)
    x = (rng.standard_t(3, shape) * 1.5).astype(np.float32)
    x = W.as_numpy_bits(torch.from_numpy(x).to(torch.bfloat16))
    check_fused(oracle, x, 8, 0, True)
    check_fused(oracle, x, 8, 1, True)


def test_fused_fp32_input(oracle):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((2, 2, 64, 128)).astype(np.float32)
    x.reshape(-1, 4)[::37] *= 20.0
    check_fused(oracle, x, 32, 0, True)


def test_window_miss_takes_the_exact_fallback(oracle):
    # make exactly the chunks the sample reads huge, so that the sampled
    # median is far above the true one
    rng = np.random.default_rng(4)
    x = rng.standard_normal((1, 2, 512, 128)).astype(np.float32)
    c = x.reshape(1, 2, -1, 4)
    c[:, :, sampled_chunks(c.shape[2])] *= 1000.0
    x = W.as_numpy_bits(torch.from_numpy(x).to(torch.bfloat16))
    g = check_fused(oracle, x, 8, 0, True)
    assert g["status"]["flags"] & hqmq.FLAG_MED3_FALLBACK
    check_fused(oracle, x, 8, 1, False)


def test_uncertain_band_overflow_takes_the_exact_fallback(oracle):
    # half of the chunks at norm 1, half just around 3: every chunk of the
    # second half sits in the threshold's uncertainty band
    rng = np.random.default_rng(5)
    n = 1 * 1 * 2048 * 32
    u = rng.standard_normal((n, 4))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    r = np.where(np.arange(n) % 2 == 0, 1.0, 3.0 * (1 + 1e-3 * rng.standard_normal(n)))
    x = (u * r[:, None]).astype(np.float32).reshape(1, 1, 2048, 128)
    g = check_fused(oracle, x, 8, 0, True)
    assert g["status"]["flags"] & hqmq.FLAG_MED3_FALLBACK


def test_fused_capacity_overflow(oracle):
    w = W.WORKLOADS["qwen_outlier"]
    x = W.as_numpy_bits(W.make_call_input(w, 0, 0, tokens=256))
    g = check_fused(oracle, x, w.S, 0, True, cap=50)
    assert g["status"]["flags"] & hqmq.FLAG_OUTLIER_OVERFLOW


def test_fused_equals_separate_calls_full_size_70b(oracle):
    # one full 70B call: fused (one read) vs hqmq_outlier_extract +
    # hqmq_encode_lut (two reads): bit-identical codes, list, offsets and
    # status; then the decode with the list applied inside the main pass
    # equals the decode with the separate list kernel
    w = W.WORKLOADS["llama3_70b_128k"]
    B, H, T, D = w.call_shape
    xd = W.make_call_input(w, 11, 0, device="cuda")
    cb = torch.empty(H * w.S * 4, dtype=torch.float32, device="cuda")
    hqmq.hqmq_make_codebook(w.codebook_seed, w.S, H, W.group0(11, 0, H), cb)
    table = gpu_search_table(cb, w.S, H)
    cap = B * H * T * D // 4 // 10
    words, radius = hqmq.alloc_codes(B, H, T, D, w.S)
    rmed, thr, oi, ov, so, ws = hqmq.alloc_outliers(B, H, T, D, cap)
    st = hqmq.new_status()
    to = hqmq.alloc_tile_off(B, H, T, D)
    hqmq.hqmq_encode_med3(xd, w.C, 0, cb, w.S, table, words, radius, rmed, thr, oi, ov, so, cap,
                          ws, st, tile_off=to)
    words2, radius2 = hqmq.alloc_codes(B, H, T, D, w.S)
    rmed2, thr2, oi2, ov2, so2, ws2 = hqmq.alloc_outliers(B, H, T, D, cap)
    st2 = hqmq.new_status()
    to2 = hqmq.alloc_tile_off(B, H, T, D)
    hqmq.hqmq_outlier_extract(xd, w.C, 0, rmed2, thr2, oi2, ov2, so2, cap, ws2, st2, tile_off=to2)
    hqmq.hqmq_encode_lut(xd, cb, w.S, table, thr2, 0, words2, radius2, st2)
    torch.cuda.synchronize()
    for a, b in ((words, words2), (radius, radius2), (thr, thr2), (so, so2), (to, to2)):
        assert torch.equal(a, b)
    ys = []
    for tiles in (False, True):
        y = torch.empty(B, H, T, D, dtype=torch.bfloat16, device="cuda")
        hqmq.hqmq_decode(words, radius, cb, w.S, oi, ov, so, cap, 0, y, hqmq.new_status(),
                         tile_off=to if tiles else None)
        ys.append(y)
    torch.cuda.synchronize()
    assert torch.equal(ys[0].view(torch.int16), ys[1].view(torch.int16))
    n = int(so[-1])
    assert torch.equal(oi[:n], oi2[:n]) and torch.equal(ov[:4 * n], ov2[:4 * n])
    assert hqmq.read_status(st) == hqmq.read_status(st2)
    assert not hqmq.read_status(st)["flags"] & hqmq.FLAG_MED3_FALLBACK
    # and the median / threshold equal the oracle's
    x = W.as_numpy_bits(xd)
    rmed_o, thr_o = oracle.med3_threshold(x, w.C, 0)
    assert same_f32(to_host(thr), thr_o).all()


def expected_status(oracle, x_np, cb, S, gran, cap):
    """The oracle's status of Med3x + encode: outliers, list and radius
    saturations, non-finite chunks, and the flags they raise."""
    _, thr_o = oracle.med3_threshold(x_np, 3.0, gran)
    _, _, _, n_o, st_x = oracle.extract(x_np, thr_o, gran=gran, cap=cap)
    *_, st_e = oracle.encode(x_np, cb, S, thr=thr_o, gran=gran)
    return {"n_outliers": n_o, "n_saturated": st_x["n_saturated"] + st_e["n_saturated"],
            "n_nonfinite": st_e["n_nonfinite"], "flags": st_x["flags"] | st_e["flags"]}


def status_mix_input(rng, T=512):
    """fp32 (1, 2, T, 128): head 0 with a median chunk norm near 40000 (bulk
    radii above 65504 saturate, outlier values above 65504 saturate in the
    list) and a dense band of norms around 3x the median; head 1 N(0, 1)
    with NaN and inf chunks and planted outliers."""
    x = rng.standard_normal((1, 2, T, 128)).astype(np.float32)
    c = x.reshape(1, 2, -1, 4)
    n = c.shape[2]
    u = c[0, 0] / np.linalg.norm(c[0, 0], axis=1, keepdims=True)
    r = np.full(n, 40000.0) * (1 + 0.3 * rng.standard_normal(n))
    band = rng.random(n) < 0.05
    r[band] = np.median(r) * rng.uniform(2.95, 3.05, band.sum())
    big = rng.random(n) < 0.01
    r[big] = 1e6
    c[0, 0] = u * np.abs(r)[:, None]
    k = rng.choice(n, 12, replace=False)
    c[0, 1, k[:4], 1] = np.nan
    c[0, 1, k[4:8], 2] = np.inf
    c[0, 1, k[8:], :] *= 50.0
    return x


@pytest.mark.parametrize("seed", [0, 1])
def test_fused_status_counts_match_the_oracle(oracle, seed):
    x = status_mix_input(np.random.default_rng(40 + seed))
    B, H, T, D = x.shape
    cb = oracle.make_codebook(seed + 3, 8, H)
    g = check_fused(oracle, x, 8, 0, True, seed=seed + 3)
    want = expected_status(oracle, x, cb, 8, 0, g["cap"])
    got = g["status"]
    assert not got["flags"] & hqmq.FLAG_MED3_FALLBACK
    assert got["n_saturated"] > 0 and got["n_nonfinite"] == 4
    for k in ("n_outliers", "n_saturated", "n_nonfinite"):
        assert got[k] == want[k], (k, got, want)
    assert got["flags"] & ~hqmq.FLAG_MED3_FALLBACK == want["flags"]


def test_fused_status_counts_after_a_window_miss(oracle):
    # the sampled quads made huge (see test_window_miss_takes_the_exact_fallback)
    # plus non-finite and saturating chunks: the fallback head's status must
    # come from the exact re-encode only
    rng = np.random.default_rng(9)
    x = rng.standard_normal((1, 2, 512, 128)).astype(np.float32)
    c = x.reshape(1, 2, -1, 4)
    c[:, :, sampled_chunks(c.shape[2])] *= 1000.0
    c[0, 0, 5, 0] = np.nan
    c[0, 1, 9, 3] = np.inf
    c[0, 0, 700] = 3e4
    cb = oracle.make_codebook(2, 8, 2)
    g = check_fused(oracle, x, 8, 0, True, seed=2)
    assert g["status"]["flags"] & hqmq.FLAG_MED3_FALLBACK
    want = expected_status(oracle, x, cb, 8, 0, g["cap"])
    for k in ("n_outliers", "n_saturated", "n_nonfinite"):
        assert g["status"][k] == want[k], (k, g["status"], want)


# ------------------------------------------------------------------ full sizes
# The fused call the bench times (chunk mode, search tables, tile offsets), at
# the full call shape of each Med3x workload, against the oracle directly:
# r_med and thr, the whole ordered list, slab and tile offsets and the status
# bit-exact; indices and radii on a sample that includes every listed
# chunk's neighbourhood of the threshold.
FULL_SIZE_FUSED = [("llama3_70b_128k", 40, 1), ("mha7b_s8", 5, 1), ("mha7b_s32", 3, 0),
                   ("qwen_outlier", 27, 1)]


def threshold_band_chunks(x_np, thr, H, T, D, k, rng):
    """Up to k chunks whose norm lies within 5% of their head's threshold
    (the chunks whose outlier decision is the closest), chosen at random."""
    xc = x_np.reshape(-1, 4)
    if x_np.dtype == np.uint16:
        xc = (xc.astype(np.uint32) << 16).view(np.float32)
    r = np.sqrt(np.sum(xc.astype(np.float64) ** 2, axis=1))
    head = (np.arange(r.size) // (T * D // 4)) % H
    t = thr.astype(np.float64)[head]
    band = np.nonzero(np.abs(r - t) <= 0.05 * t)[0]
    return rng.choice(band, min(k, band.size), replace=False) if band.size else band


@pytest.mark.parametrize("name,layer,role", FULL_SIZE_FUSED,
                         ids=["%s-L%d-r%d" % f for f in FULL_SIZE_FUSED])
def test_fused_full_size_against_the_oracle(oracle, name, layer, role):
    w = W.WORKLOADS[name]
    B, H, T, D = w.call_shape
    n_chunks = B * H * T * D // 4
    x = W.as_numpy_bits(W.make_call_input(w, layer, role, device="cuda"))
    cb = oracle.make_codebook(w.codebook_seed, w.S, H, W.group0(layer, role, H))
    g = fused(x, cb, w.S, 0, True, cap=n_chunks // 5)
    thr_o, idx_o, val_o, so_o, n_o = check_med3(oracle, x, g, w.C, 0)
    # status: the list's count and saturations (bulk chunks have r <= thr, far
    # below the fp16 limit, and the inputs are finite), no fallback
    _, _, _, _, st_x = oracle.extract(x, thr_o, gran=0, cap=g["cap"])
    assert g["status"] == {"flags": st_x["flags"], "n_outliers": n_o,
                           "n_saturated": st_x["n_saturated"], "n_nonfinite": 0}, g["status"]
    rng = np.random.default_rng(layer * 2 + role + 17)
    chunks = np.concatenate([rng.choice(n_chunks, 12000, replace=False),
                             threshold_band_chunks(x, thr_o, H, T, D, 3000, rng),
                             idx_o[rng.choice(idx_o.size, min(1000, idx_o.size), replace=False)],
                             np.array([0, n_chunks - 1])]).astype(np.int64)
    chunks = np.unique(chunks)
    gi = unpack_indices(to_host(g["words"]), w.S, n_chunks)
    n, mm, near = check_codes(oracle, x, cb, w.S, gi, to_host(g["radius"]), thr=thr_o, gran=0,
                              chunks=chunks)
    assert n >= 10000
    print("[fused full size] %s L%d role %d: %d outliers (%.3f%%), %d sampled chunks, "
          "%d near-tie index differences, %d near-tie pairs"
          % (name, layer, role, n_o, 100.0 * n_o / n_chunks, n, mm, near))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_fused_every_chunk_inside_the_window(oracle, dtype):
    # Chunk norms within 0.1% of 1 (all in one bin of the sample's histogram,
    # so every chunk is a window key and goes through the encode pass's event
    # queue, which then fills up inside a unit), a contiguous run of 100
    # outliers (more than one unit's candidate-value slots), 2% scattered
    # outliers and 1% of chunks around the threshold 3 r_med (its band).
    rng = np.random.default_rng(11)
    B, H, T, D = 1, 2, 256, 128
    n = B * H * T * D // 4
    u = rng.standard_normal((n, 4))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    r = 1.0 + 1e-3 * rng.random(n)
    pick = rng.random(n)
    r = np.where(pick < 0.02, 50.0, r)
    r = np.where((pick >= 0.02) & (pick < 0.03), 3.0015 * (1 + 2e-4 * rng.standard_normal(n)), r)
    r[5000:5100] = 20.0
    x = (u * r[:, None]).astype(np.float32).reshape(B, H, T, D)
    if dtype == "bf16":
        x = W.as_numpy_bits(torch.from_numpy(x).to(torch.bfloat16))
    g = check_fused(oracle, x, 32, 0, True)
    assert not g["status"]["flags"] & hqmq.FLAG_MED3_FALLBACK
    assert g["status"]["n_outliers"] > 0.02 * n
