"""Streaming Med3x for decode-phase tokens (hqmq_outlier_extract_given_thr):
the outlier list of a batch of new tokens under the threshold of an earlier
batch (the prefill), then the encode of the new tokens with that threshold.
Parity with the oracle (extract and encode with the same threshold):
bit-exact lists, offsets and radii; indices bit-exact up to counted
near-ties.  The threshold comes from the oracle's median of the prefill."""
import numpy as np
import pytest
import torch

from _parity import check_codes, gpu_codebook, list_tile_off, to_host, unpack_indices
from kv_cache_quantization_hqmq_b200 import hqmq
from kv_cache_quantization_hqmq_b200.workloads import WORKLOADS, as_numpy_bits, group0, make_call_input

pytestmark = pytest.mark.gpu
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


def gpu_list_given_thr(x_dev, thr, gran):
    B, H, T, D = x_dev.shape
    n = B * H * T * D // 4 * (4 if gran else 1)
    oi = torch.zeros(n, dtype=torch.int32, device="cuda")
    ov = torch.zeros(n * (4 if gran == 0 else 1), dtype=torch.int16, device="cuda")
    so = torch.empty(B * H + 1, dtype=torch.int32, device="cuda")
    to = hqmq.alloc_tile_off(B, H, T, D)
    ws = torch.empty(hqmq.hqmq_outlier_extract_given_thr_workspace_size(B, H, T, D),
                     dtype=torch.uint8, device="cuda")
    st = hqmq.new_status()
    hqmq.hqmq_outlier_extract_given_thr(x_dev, torch.from_numpy(thr).cuda(), gran, oi, ov, so, n,
                                        ws, st, tile_off=to)
    torch.cuda.synchronize()
    k = int(to_host(so)[-1])
    return (to_host(oi)[:k].view(np.uint32), to_host(ov).view(np.uint16), to_host(so).view(np.uint32),
            to_host(to).view(np.uint32), hqmq.read_status(st))


@pytest.mark.parametrize("T", [1, 7, 300])
@pytest.mark.parametrize("gran", [0, 1])
def test_list_under_a_given_threshold(oracle, T, gran):
    w = WORKLOADS["qwen_outlier"]
    B, H, D = 2, w.heads, w.head_dim
    prefill = as_numpy_bits(make_call_input(w, 1, 0, tokens=256, batch=B))
    _, thr = oracle.med3_threshold(prefill, w.C, gran)
    xw = w.with_(input_seed=w.input_seed + 77 + T)
    x = make_call_input(xw, 1, 0, tokens=T, batch=B)
    want_idx, want_val, want_so, n_req, _ = oracle.extract(as_numpy_bits(x), thr, gran)
    idx, val, so, to, st = gpu_list_given_thr(x.cuda(), thr, gran)
    np.testing.assert_array_equal(idx, want_idx)
    vw = 4 if gran == 0 else 1
    np.testing.assert_array_equal(val[:len(idx) * vw], np.asarray(want_val).reshape(-1))
    np.testing.assert_array_equal(so, want_so)
    np.testing.assert_array_equal(to, list_tile_off(want_idx, B, H, T, D, gran))
    assert st["n_outliers"] == n_req and st["flags"] == 0
    print("[stream] T=%d gran=%d: %d entries" % (T, gran, len(idx)))


def test_one_token_decode_steps(oracle):
    """A prefill's threshold, then three decode steps of one token per
    sequence: list and encode of each step against the oracle."""
    w = WORKLOADS["llama3_70b_128k"]
    B, H, D, S = 2, w.heads, w.head_dim, w.S
    prefill = as_numpy_bits(make_call_input(w, 0, 1, tokens=512, batch=B))
    _, thr = oracle.med3_threshold(prefill, w.C, 0)
    cb = oracle.make_codebook(w.codebook_seed, S, H, group0(0, 1, H))
    cb_dev = gpu_codebook(w.codebook_seed, S, H, group0(0, 1, H))
    table = torch.empty(H * hqmq.hqmq_search_table_bytes(S), dtype=torch.uint8, device="cuda")
    hqmq.hqmq_make_search_table(cb_dev, S, H, table)
    thr_dev = torch.from_numpy(thr).cuda()
    for step in range(3):
        xs = make_call_input(w.with_(input_seed=1000 + step), 0, 1, tokens=1, batch=B)
        x_np = as_numpy_bits(xs)
        idx, val, so, to, st = gpu_list_given_thr(xs.cuda(), thr, 0)
        want_idx, want_val, _, _, _ = oracle.extract(x_np, thr, 0)
        np.testing.assert_array_equal(idx, want_idx)
        np.testing.assert_array_equal(val[:len(idx) * 4], np.asarray(want_val).reshape(-1))
        words, radius = hqmq.alloc_codes(B, H, 1, D, S)
        hqmq.hqmq_encode_lut(xs.cuda(), cb_dev, S, table, thr_dev, 0, words, radius)
        torch.cuda.synchronize()
        n = B * H * D // 4
        check_codes(oracle, x_np, cb, S, unpack_indices(to_host(words), S, n), to_host(radius),
                    thr=thr, gran=0)
        print("[stream] step %d: %d outlier chunks of %d" % (step, len(idx), B * H * D // 4))
