"""Parity of the quantized-radius calls (hqmq_quantize_radius,
hqmq_decode_qradius) with the oracle: bit-exact radius codes and decoded
values.  Inputs are written by the oracle (Med3x threshold, list, encode) from
seeded tensors, or are seeded synthetic fp16 radii; none comes from the CUDA
path."""
import numpy as np
import pytest
import torch

from _parity import list_tile_off, to_host
from kv_cache_quantization_hqmq_b200 import hqmq
from kv_cache_quantization_hqmq_b200.workloads import WORKLOADS, as_numpy_bits, group0, make_call_input

pytestmark = pytest.mark.gpu
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


def dev(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a).view(dtype)).cuda()


def gpu_qcodes(radius_u16, thr, shape, S):
    B, H, T, D = shape
    rw = torch.empty(hqmq.hqmq_index_words(B, H, T, D, S), dtype=torch.int32, device="cuda")
    hqmq.hqmq_quantize_radius(dev(radius_u16, np.int16), dev(np.asarray(thr, np.float32), np.float32),
                              shape, S, rw)
    torch.cuda.synchronize()
    return rw, to_host(rw).view(np.uint32)


@pytest.mark.parametrize("name,gran", [("qwen_outlier", 0), ("mha7b_s8", 0),
                                       ("llama3_70b_128k", 1), ("qwen_outlier", 1)])
def test_codes_and_decode_match_the_oracle(oracle, name, gran):
    w = WORKLOADS[name].with_(heads=2)
    B, T, D, S, H = 2, 256, 128, w.S, 2
    shape = (B, H, T, D)
    x = as_numpy_bits(make_call_input(w, 0, 0, tokens=T, batch=B))
    cb = oracle.make_codebook(w.codebook_seed, S, H, group0(0, 0, H))
    _, thr = oracle.med3_threshold(x, w.C, gran)
    idx, val, _, _, _ = oracle.extract(x, thr, gran)
    words, radius, _, _, _ = oracle.encode(x, cb, S, thr, gran)
    want = oracle.quantize_radius(radius, thr, B, H, T, D, S)
    rw_dev, got = gpu_qcodes(radius, thr, shape, S)
    np.testing.assert_array_equal(got, want)
    to = list_tile_off(idx, B, H, T, D, gran)
    for out_dt, odt in ((torch.bfloat16, oracle.BF16), (torch.float32, oracle.F32)):
        y = torch.empty(shape, dtype=out_dt, device="cuda")
        st = hqmq.new_status()
        has = len(idx) > 0
        hqmq.hqmq_decode_qradius(dev(words, np.int32), rw_dev, dev(thr, np.float32),
                                 torch.from_numpy(cb.reshape(-1)).cuda(), S,
                                 dev(idx, np.int32) if has else None,
                                 dev(val.reshape(-1), np.int16) if has else None,
                                 dev(to, np.int32) if has else None, len(idx), gran, y, st)
        torch.cuda.synchronize()
        ref, _ = oracle.decode_qradius(words, want, thr, cb, S, B, H, T, D, idx, val, gran, odt)
        g = to_host(y.view(torch.int16) if out_dt == torch.bfloat16 else y)
        np.testing.assert_array_equal(g.view(np.uint8), ref.view(np.uint8))
        assert hqmq.read_status(st)["flags"] == 0
    print("[qradius] %s gran=%d: %d codes, %d list entries, bits/elem %.2f"
          % (name, gran, radius.size, len(idx), 2 * oracle.index_bits(S) / 4))


def test_codes_full_size_70b_shape(oracle):
    """The 70B call shape (1 x 8 x 131072 x 128, S = 32) on seeded synthetic
    fp16 radii in [0, 1.3 thr] with zeros, NaN and 65504 mixed in; heads with a
    zero, infinite and NaN threshold."""
    B, H, T, D, S = 1, 8, 131072, 128, 32
    n = B * H * T * D // 4
    rng = np.random.default_rng(2)
    thr = np.array([3.0, 2.5, 0.0, np.inf, 7.75, np.nan, 1e-3, 40.0], np.float32)
    heads = (np.arange(n) // (T * D // 4)) % H
    scale = np.where(np.isfinite(thr) & (thr > 0), thr, 1.0)[heads]
    r = (rng.random(n) * 1.3 * scale).astype(np.float16)
    r[rng.integers(0, n, 1000)] = 0
    r[rng.integers(0, n, 1000)] = np.float16(65504)
    r = r.view(np.uint16).copy()
    r[rng.integers(0, n, 1000)] = 0x7E00
    want = oracle.quantize_radius(r, thr, B, H, T, D, S)
    _, got = gpu_qcodes(r, thr, (B, H, T, D), S)
    np.testing.assert_array_equal(got, want)


def test_rejects_bad_arguments():
    rw = torch.empty(64, dtype=torch.int32, device="cuda")
    r = torch.zeros(1024, dtype=torch.int16, device="cuda")
    thr = torch.ones(1, device="cuda")
    with pytest.raises(hqmq.HQMQError):
        hqmq.hqmq_quantize_radius(r, thr, (1, 1, 32, 130), 8, rw)       # D % 4 != 0
    with pytest.raises(hqmq.HQMQError):
        hqmq.hqmq_quantize_radius(r, thr, (1, 1, 32, 128), 0, rw)       # S = 0
