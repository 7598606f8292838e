"""GPU parity: the CUDA path, called through the C ABI, against the CPU oracle
on the same seeded inputs.  Small cases are compared element by element over
every output; full-size calls of the bench workloads (same kernels, same
launch configuration as bench.py) are compared exactly where the oracle is
cheap (Med3x thresholds and outlier lists, decode) and on sampled chunks for
the search."""
import numpy as np
import pytest
import torch

from _parity import (list_tile_off, DECODE_ABS_TOL, NEAR_TIE_REL, check_codes, check_med3, gpu_codebook,
                     gpu_decode, gpu_encode, gpu_med3, same_f16_or_bf16_bits, same_f32, to_host,
                     unpack_indices)

pytestmark = pytest.mark.gpu

cuda = pytest.importorskip("torch").cuda
if not cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

from kv_cache_quantization_hqmq_b200 import hqmq  # noqa: E402
from kv_cache_quantization_hqmq_b200 import workloads as W  # noqa: E402


def report(name, n, mm, near):
    print("[parity] %s: %d chunks, %d index mismatches (all near-ties), %d near-ties"
          % (name, n, mm, near))


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bf16_dev(x_np_u16):
    return torch.from_numpy(x_np_u16.view(np.int16)).cuda().view(torch.bfloat16)


def x_to_dev(x_np):
    return bf16_dev(x_np) if x_np.dtype == np.uint16 else dev(x_np)


ENCODERS = ["sloop", "lut"]


def full_call(oracle, x_np, S, cb_np, med3=False, C=3.0, gran=0, name="", check_e2e=True,
              encoder="sloop"):
    """Whole-call parity: Med3x (optional), encode (S-loop or table search), decode."""
    B, H, T, D = x_np.shape
    xd = x_to_dev(x_np)
    cbd = dev(cb_np.reshape(-1))
    med = thr_o = None
    if med3:
        med = gpu_med3(xd, C, gran)
        thr_o, oi_o, ov_o, so_o, n_o = check_med3(oracle, x_np, med, C, gran)
    words, radius, st = gpu_encode(xd, cbd, S, med["thr"] if med3 else None, gran, encoder)
    n_chunks = B * H * T * D // 4
    gi = unpack_indices(to_host(words), S, n_chunks)
    n, mm, near = check_codes(oracle, x_np, cb_np, S, gi, to_host(radius), thr=thr_o, gran=gran)
    report("%s [%s]" % (name, encoder), n, mm, near)
    # decode parity on the ORACLE's codes: bit-exact, bf16 and fp32 outputs
    ow, orad, _, _, _ = oracle.encode(x_np, cb_np, S, thr=thr_o, gran=gran)
    owd, orad_d = dev(ow.view(np.int32)), dev(orad.view(np.int16))
    med_o = None
    if med3:
        k = oi_o.size
        med_o = dict(out_idx=dev(oi_o.view(np.int32)) if k else torch.zeros(1, dtype=torch.int32, device="cuda"),
                     out_val=dev(ov_o.reshape(-1).view(np.int16)) if k else torch.zeros(4, dtype=torch.int16, device="cuda"),
                     slab_off=dev(so_o.view(np.int32)), cap=k,
                     tile_off=dev(list_tile_off(oi_o, B, H, T, D, gran).view(np.int32)))
    for out_dt, od in ((torch.bfloat16, 0), (torch.float32, 1)):
        yo, _ = oracle.decode(ow, orad, cb_np, S, B, H, T, D,
                              out_idx=oi_o if med3 else None, out_val=ov_o if med3 else None,
                              gran=gran, out_dtype=od)
        # the list applied by a second kernel, and inside the main pass
        for tiles in ((False, True) if med3 else (False,)):
            y, _ = gpu_decode(owd, orad_d, cbd, S, (B, H, T, D), out_dt, med_o, gran, tiles)
            if od == 0:
                ok = same_f16_or_bf16_bits(to_host(y.view(torch.int16)), yo, bf16=True)
            else:
                ok = same_f32(to_host(y), yo)
            assert ok.all(), "decode (tiles %d) mismatch at %s" % (tiles, np.argwhere(~ok)[:5])
    if check_e2e:
        # end to end: GPU encode + GPU decode vs oracle encode + decode
        yo, _ = oracle.decode(ow, orad, cb_np, S, B, H, T, D,
                              out_idx=oi_o if med3 else None, out_val=ov_o if med3 else None,
                              gran=gran, out_dtype=1)
        exempt = gi != unpack_indices(ow, S, n_chunks)
        for tiles in ((False, True) if med3 else (False,)):
            y, _ = gpu_decode(words, radius, cbd, S, (B, H, T, D), torch.float32,
                              med if med3 else None, gran, tiles)
            diff = np.abs(to_host(y).reshape(-1, 4) - yo.reshape(-1, 4)).max(axis=1)
            assert np.all(diff[~exempt] <= DECODE_ABS_TOL)
    return dict(words=words, radius=radius, status=st, med=med)


# ------------------------------------------------------------------ codebook
@pytest.mark.parametrize("S,G", [(8, 512), (32, 1280), (1, 7), (1000, 3)])
def test_codebook_matches_oracle(oracle, S, G):
    cb = to_host(gpu_codebook(1, S, G)).reshape(G, S, 4)
    want = oracle.make_codebook(1, S, G)
    ulp = np.abs(cb.view(np.int32).astype(np.int64) - want.view(np.int32).astype(np.int64))
    n_diff = int((ulp != 0).sum())
    print("[parity] codebook S=%d G=%d: %d of %d values differ (max %d ulp)"
          % (S, G, n_diff, cb.size, ulp.max()))
    assert ulp.max() <= 1 and n_diff <= max(2, cb.size // 10000)
    sub = to_host(gpu_codebook(1, S, 2, group0=G - 2)).reshape(2, S, 4)
    assert np.array_equal(sub, cb[G - 2:])


# ------------------------------------------------------------------ whole calls
@pytest.mark.parametrize("encoder", ENCODERS)
def test_tiny_config(oracle, encoder):
    w = W.WORKLOADS["tiny"]
    cb = oracle.make_codebook(w.codebook_seed, w.S, w.n_groups)
    for role in (0, 1):
        x = W.as_numpy_bits(W.make_call_input(w, 0, role))
        g0 = W.group0(0, role, w.heads)
        full_call(oracle, x, w.S, cb[g0:g0 + w.heads], name="tiny role %d" % role,
                  encoder=encoder)


@pytest.mark.parametrize("encoder", ENCODERS)
@pytest.mark.parametrize("layer", [0, 31])
def test_llama8b_short(oracle, layer, encoder):
    w = W.WORKLOADS["llama3_8b"]
    x = W.as_numpy_bits(W.make_call_input(w, layer, 1, tokens=256))
    cb = oracle.make_codebook(w.codebook_seed, w.S, w.heads, W.group0(layer, 1, w.heads))
    full_call(oracle, x, w.S, cb, name="llama8b L%d T256" % layer, encoder=encoder)


@pytest.mark.parametrize("encoder", ENCODERS)
@pytest.mark.parametrize("gran", [0, 1])
def test_qwen_med3_short(oracle, gran, encoder):
    w = W.WORKLOADS["qwen_outlier"]
    x = W.as_numpy_bits(W.make_call_input(w, 3, 0, tokens=512))
    cb = oracle.make_codebook(w.codebook_seed, w.S, w.heads, W.group0(3, 0, w.heads))
    r = full_call(oracle, x, w.S, cb, med3=True, gran=gran, name="qwen T512 gran %d" % gran,
                  encoder=encoder)
    assert r["med"]["status"]["n_outliers"] > 0


@pytest.mark.parametrize("encoder", ENCODERS)
@pytest.mark.parametrize("S", [8, 32])
def test_mha_batched_med3_short(oracle, S, encoder):
    w = W.WORKLOADS["mha7b_s8"]
    x = W.as_numpy_bits(W.make_call_input(w, 5, 1, tokens=64, batch=3))
    cb = oracle.make_codebook(w.codebook_seed, S, w.heads, W.group0(5, 1, w.heads))
    full_call(oracle, x, S, cb, med3=True, name="mha B3 T64 S%d" % S, encoder=encoder)


# ------------------------------------------------------------------ edge cases
@pytest.mark.parametrize("S", [1, 3, 170, 171, 1000, 7000])
def test_codebook_sizes(oracle, S):
    # S=171 and S=1000 take the decode path without a shared codeword table;
    # S=7000 the encode path with the codebook in global memory
    rng = np.random.default_rng(S)
    x = rng.standard_normal((1, 2, 32, 128)).astype(np.float32)
    cb = oracle.make_codebook(9, S, 2)
    full_call(oracle, x, S, cb, name="S=%d" % S, check_e2e=S < 1000)


@pytest.mark.parametrize("S", [1, 2, 3, 8, 17, 32, 48])
def test_search_table_codebook_sizes(oracle, S):
    rng = np.random.default_rng(100 + S)
    x = rng.standard_normal((1, 2, 64, 128)).astype(np.float32)
    cb = oracle.make_codebook(11, S, 2)
    full_call(oracle, x, S, cb, name="S=%d" % S, encoder="lut")


def test_search_table_rejects_large_S():
    assert hqmq.hqmq_search_table_bytes(49) == 0
    assert hqmq.hqmq_search_table_bytes(48) == 8 * 32 ** 3 * 16


@pytest.mark.parametrize("encoder", ENCODERS)
@pytest.mark.parametrize("shape", [(1, 1, 32, 4), (2, 3, 8, 64), (1, 2, 40, 256), (3, 1, 200, 128),
                                   (1, 1, 4100, 128)])
def test_shapes_and_ragged_tails(oracle, shape, encoder):
    # ragged: 4100 tokens -> 131200 chunks per slab, not a multiple of the
    # 2048-chunk decode range nor of the 4096-chunk extraction tile
    rng = np.random.default_rng(sum(shape))
    x = (rng.standard_t(3, shape) * 2).astype(np.float32)
    x = W.as_numpy_bits(torch.from_numpy(x).to(torch.bfloat16))
    cb = oracle.make_codebook(2, 8, shape[1])
    full_call(oracle, x, 8, cb, med3=True, name="shape %s" % (shape,), encoder=encoder)


@pytest.mark.parametrize("encoder", ENCODERS)
def test_zero_nonfinite_and_saturating_chunks(oracle, encoder):
    x = np.random.default_rng(1).standard_normal((1, 1, 32, 128)).astype(np.float32)
    c = x.reshape(-1, 4)
    c[0] = 0.0
    c[1] = [np.nan, 1, 0, 0]
    c[2] = [np.inf, 0, 0, 0]
    c[3] = [1e20, 0, 0, 0]
    c[4] = [7e4, 0, 0, 0]
    c[5] = [-0.0, 0.0, -0.0, 0.0]
    cb = oracle.make_codebook(1, 8, 1)
    xd, cbd = dev(x), dev(cb.reshape(-1))
    words, radius, st = gpu_encode(xd, cbd, 8, encoder=encoder)
    gi = unpack_indices(to_host(words), 8, 1024)
    check_codes(oracle, x, cb, 8, gi, to_host(radius))
    assert st["n_nonfinite"] == 3 and st["n_saturated"] == 1 and st["flags"] == 6


@pytest.mark.parametrize("encoder", ENCODERS)
def test_exact_ties_go_to_lowest_index(oracle, encoder):
    cb = np.array([[[1.0, 0.0, 0.0, 0.0], [0.0, 1.0, 0.0, 0.0], [0.5, 0.5, 0.5, 0.5]]],
                  np.float32)
    x = np.zeros((1, 1, 1, 128), np.float32)
    c = x.reshape(-1, 4)
    c[0] = [1, 1, 0, 0]
    c[1] = [0, 0, 0, -2]
    c[2] = [1, 1, 1, 1]
    c[3] = [-1, 0, 0, 0]
    c[4] = [1, -1, 1, -1]
    xd, cbd = dev(x), dev(cb.reshape(-1))
    words, radius, st = gpu_encode(xd, cbd, 3, encoder=encoder)
    gi = unpack_indices(to_host(words), 3, 32)
    words_o, rad_o, *_ = oracle.encode(x, cb, 3)
    assert np.array_equal(gi, unpack_indices(words_o, 3, 32))


def test_outlier_capacity_overflow(oracle):
    w = W.WORKLOADS["qwen_outlier"]
    x = W.as_numpy_bits(W.make_call_input(w, 0, 0, tokens=256))
    xd = bf16_dev(x)
    g = gpu_med3(xd, 3.0, 0, cap=100)
    assert g["status"]["flags"] & hqmq.FLAG_OUTLIER_OVERFLOW
    check_med3(oracle, x, g, 3.0, 0)
    assert g["status"]["n_outliers"] > 100


@pytest.mark.parametrize("shape", [(2, 3, 1, 128), (1, 2, 3, 128), (2, 1, 9, 128), (3, 2, 32, 4)])
def test_decode_odd_group_counts(oracle, shape):
    # slabs with an odd number of 32-chunk packing groups (one-token decode
    # steps, D = 4): the last pair of groups of a slab is half empty; nothing
    # may be written past the slab (the next slab, or past the tensor)
    B, H, T, D = shape
    rng = np.random.default_rng(sum(shape))
    x = rng.standard_normal(shape).astype(np.float32)
    x.reshape(-1, 4)[::7] *= 6.0
    S = 8
    cb = oracle.make_codebook(2, S, H)
    cbd = dev(cb.reshape(-1))
    _, thr_o = oracle.med3_threshold(x, 3.0, 0)
    oi_o, ov_o, so_o, n_o, _ = oracle.extract(x, thr_o)
    assert n_o > 0
    ow, orad, _, _, _ = oracle.encode(x, cb, S, thr=thr_o)
    n = B * H * T * D
    for listed in ("none", "kernel", "tiles"):
        yo, _ = oracle.decode(ow, orad, cb, S, B, H, T, D,
                              out_idx=None if listed == "none" else oi_o,
                              out_val=None if listed == "none" else ov_o, out_dtype=0)
        guard = torch.full((n + 8192,), 0x5A5A, dtype=torch.int16, device="cuda")
        y = guard[:n].view(torch.bfloat16).view(B, H, T, D)
        st = hqmq.new_status()
        if listed == "none":
            hqmq.hqmq_decode(dev(ow.view(np.int32)), dev(orad.view(np.int16)), cbd, S, None, None,
                             None, 0, 0, y, st)
        else:
            to = dev(list_tile_off(oi_o, B, H, T, D, 0).view(np.int32))
            hqmq.hqmq_decode(dev(ow.view(np.int32)), dev(orad.view(np.int16)), cbd, S,
                             dev(oi_o.view(np.int32)), dev(ov_o.reshape(-1).view(np.int16)),
                             dev(so_o.view(np.int32)), n_o, 0, y, st,
                             tile_off=to if listed == "tiles" else None)
        torch.cuda.synchronize()
        g = to_host(guard)
        assert np.all(g[n:] == 0x5A5A), "decode wrote past the tensor (%s)" % listed
        ok = same_f16_or_bf16_bits(g[:n].view(np.uint16), yo.reshape(-1), bf16=True)
        assert ok.all(), (listed, np.argwhere(~ok.reshape(-1))[:5])
        assert hqmq.read_status(st)["flags"] == 0


def test_decode_bad_index_flag(oracle):
    words = torch.full((8,), -1, dtype=torch.int32, device="cuda")
    radius = torch.full((32,), 0x3C00, dtype=torch.int16, device="cuda")
    cbd = dev(oracle.make_codebook(1, 8, 1).reshape(-1))
    y, st = gpu_decode(words, radius, cbd, 8, (1, 1, 1, 128), torch.float32)
    assert st["flags"] & hqmq.FLAG_BAD_INDEX
    assert torch.all(y == 0)


def test_arguments_rejected(oracle):
    x = torch.zeros((1, 1, 8, 6), dtype=torch.bfloat16, device="cuda")
    cb = torch.zeros(32, dtype=torch.float32, device="cuda")
    with pytest.raises(hqmq.HQMQError):
        hqmq.hqmq_encode(x, cb, 8, None, 0, cb, cb)


# ------------------------------------------------------------------ full sizes
def _full_size_call(oracle, name, layer, role, n_sample=20000, gran=0, encoder="sloop"):
    w = W.WORKLOADS[name]
    B, H, T, D = w.call_shape
    xd = W.make_call_input(w, layer, role, device="cuda")
    x = W.as_numpy_bits(xd)
    g0 = W.group0(layer, role, H)
    cbd = gpu_codebook(w.codebook_seed, w.S, H, g0)
    cb = oracle.make_codebook(w.codebook_seed, w.S, H, g0)
    assert np.abs(to_host(cbd).reshape(cb.shape).view(np.int32).astype(np.int64)
                  - cb.view(np.int32).astype(np.int64)).max() <= 1
    cbd = dev(cb.reshape(-1))        # both sides score the same codebook bytes
    thr_o = None
    med = None
    if w.med3:
        med = gpu_med3(xd, w.C, gran)
        thr_o, oi_o, ov_o, so_o, n_o = check_med3(oracle, x, med, w.C, gran)
        print("[parity] %s L%d role %d: %d outliers (%.3f%%), status flags %d" % (
            name, layer, role, n_o, 100.0 * n_o / (B * H * T * D / (4 if gran == 0 else 1)),
            med["status"]["flags"]))
        if gran == 0:
            assert not med["status"]["flags"] & hqmq.FLAG_MED3_FALLBACK
    words, radius, st = gpu_encode(xd, cbd, w.S, med["thr"] if med else None, gran, encoder)
    n_chunks = B * H * T * D // 4
    gi = unpack_indices(to_host(words), w.S, n_chunks)
    rng = np.random.default_rng(layer * 2 + role)
    chunks = np.sort(rng.choice(n_chunks, n_sample, replace=False))
    # always include the first/last chunks and some outlier chunks
    extra = [0, n_chunks - 1]
    if med is not None and gran == 0 and len(oi_o):
        extra += list(oi_o[:50])
    chunks = np.unique(np.concatenate([chunks, np.array(extra, np.int64)]))
    n, mm, near = check_codes(oracle, x, cb, w.S, gi, to_host(radius), thr=thr_o, gran=gran,
                              chunks=chunks)
    report("%s L%d role %d (sampled) [%s]" % (name, layer, role, encoder), n, mm, near)
    # decode at full size: seeded random codes + the oracle's outlier list
    rs = np.random.default_rng(99)
    b = hqmq.hqmq_index_bits(w.S)
    idx_r = rs.integers(0, 24 * w.S, n_chunks, dtype=np.uint32)
    bits = ((idx_r[:, None] >> np.arange(b, dtype=np.uint32)) & 1).astype(np.uint8)
    wr = np.packbits(bits.reshape(n_chunks // 32, 32 * b), axis=1, bitorder="little")
    wr = np.ascontiguousarray(wr).view(np.uint32)
    del bits
    assert np.array_equal(unpack_indices(wr.reshape(-1), w.S, 4096), idx_r[:4096])
    rad_r = (rs.standard_normal(n_chunks).astype(np.float32) * 2).astype(np.float16).view(np.uint16)
    med_o = None
    if med is not None:
        k = len(oi_o)
        med_o = dict(out_idx=dev(oi_o.view(np.int32)), out_val=dev(ov_o.reshape(-1).view(np.int16)),
                     slab_off=dev(so_o.view(np.int32)), cap=k,
                     tile_off=dev(list_tile_off(oi_o, B, H, T, D, gran).view(np.int32)))
    yo, _ = oracle.decode(wr.reshape(-1), rad_r, cb, w.S, B, H, T, D,
                          out_idx=oi_o if med is not None else None,
                          out_val=ov_o if med is not None else None, gran=gran, out_dtype=0)
    for tiles in ((False, True) if med is not None else (False,)):
        y, _ = gpu_decode(dev(wr.reshape(-1).view(np.int32)), dev(rad_r.view(np.int16)), cbd,
                          w.S, (B, H, T, D), torch.bfloat16, med_o, gran, tiles)
        ok = same_f16_or_bf16_bits(to_host(y.view(torch.int16)), yo, bf16=True)
        assert ok.all(), (tiles, np.argwhere(~ok.reshape(-1))[:5])


@pytest.mark.parametrize("encoder", ENCODERS)
def test_full_size_llama8b_call(oracle, encoder):
    _full_size_call(oracle, "llama3_8b", 7, 0, encoder=encoder)


@pytest.mark.parametrize("encoder", ENCODERS)
def test_full_size_qwen_call(oracle, encoder):
    _full_size_call(oracle, "qwen_outlier", 27, 1, encoder=encoder)


@pytest.mark.parametrize("encoder", ENCODERS)
def test_full_size_mha_call(oracle, encoder):
    _full_size_call(oracle, "mha7b_s32", 0, 0, n_sample=5000, encoder=encoder)


@pytest.mark.parametrize("encoder", ENCODERS)
def test_full_size_llama70b_call(oracle, encoder):
    _full_size_call(oracle, "llama3_70b_128k", 40, 1, n_sample=10000, encoder=encoder)


def test_full_size_llama70b_call_element_mode(oracle):
    _full_size_call(oracle, "llama3_70b_128k", 79, 0, n_sample=5000, gran=1)
