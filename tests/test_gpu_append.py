"""hqmq_append_batch: n_calls small calls (a decode step's new tokens of every
(layer, role)) in one launch.  Each call's list, offsets, radii and indices
against the oracle's extract and encode under that call's threshold:
bit-exact, indices up to counted near-ties.  Thresholds come from the
oracle's median of a prefill per call."""
import numpy as np
import pytest
import torch

from _parity import check_codes, list_tile_off, to_host, unpack_indices
from kv_cache_quantization_hqmq_b200 import hqmq
from kv_cache_quantization_hqmq_b200.workloads import WORKLOADS, as_numpy_bits, group0, make_call_input

pytestmark = pytest.mark.gpu
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


@pytest.mark.parametrize("name,T,gran", [("llama3_70b_128k", 1, 0), ("qwen_outlier", 3, 0),
                                         ("qwen_outlier", 1, 1), ("mha7b_s8", 2, 0)])
def test_batched_calls_match_the_oracle(oracle, name, T, gran):
    w = WORKLOADS[name].with_(heads=4)
    B, H, D, S = 2, 4, w.head_dim, w.S
    calls = [(l, r) for l in range(3) for r in range(2)]
    C = len(calls)
    xs, thrs, cbs = [], [], []
    for l, r in calls:
        pre = as_numpy_bits(make_call_input(w, l, r, tokens=128, batch=B))
        thrs.append(oracle.med3_threshold(pre, w.C, gran)[1])
        xs.append(make_call_input(w.with_(input_seed=500 + l), l, r, tokens=T, batch=B))
        cbs.append(oracle.make_codebook(w.codebook_seed, S, H, group0(l, r, H)))
    x = torch.stack(xs).cuda()
    n_chunks = B * H * T * D // 4
    n_units = n_chunks * (4 if gran else 1)
    cap = n_units
    nw = hqmq.hqmq_index_words(B, H, T, D, S)
    n_tiles = hqmq.hqmq_list_tiles(B, H, T, D)
    words = torch.zeros(C * nw, dtype=torch.int32, device="cuda")
    radius = torch.zeros(C * n_chunks, dtype=torch.int16, device="cuda")
    oi = torch.zeros(C * cap, dtype=torch.int32, device="cuda")
    ov = torch.zeros(C * cap * (1 if gran else 4), dtype=torch.int16, device="cuda")
    so = torch.zeros(C * (B * H + 1), dtype=torch.int32, device="cuda")
    to = torch.zeros(C * (n_tiles + 1), dtype=torch.int32, device="cuda")
    st = hqmq.new_status()
    hqmq.hqmq_append_batch(x, torch.from_numpy(np.stack(thrs)).cuda(), gran,
                           torch.from_numpy(np.stack(cbs).reshape(-1)).cuda(), S, words, radius, oi,
                           ov, so, cap, tile_off=to, status=st)
    torch.cuda.synchronize()
    words_h = to_host(words).view(np.uint32).reshape(C, nw)
    radius_h = to_host(radius).view(np.uint16).reshape(C, n_chunks)
    oi_h = to_host(oi).view(np.uint32).reshape(C, cap)
    ov_h = to_host(ov).view(np.uint16).reshape(C, -1)
    so_h = to_host(so).view(np.uint32).reshape(C, B * H + 1)
    to_h = to_host(to).view(np.uint32).reshape(C, n_tiles + 1)
    total = 0
    for c in range(C):
        x_np = as_numpy_bits(xs[c])
        idx_o, val_o, so_o, n_o, _ = oracle.extract(x_np, thrs[c], gran)
        total += n_o
        np.testing.assert_array_equal(so_h[c], so_o)
        np.testing.assert_array_equal(oi_h[c, :n_o], idx_o)
        vw = 1 if gran else 4
        np.testing.assert_array_equal(ov_h[c, :n_o * vw], np.asarray(val_o).reshape(-1))
        np.testing.assert_array_equal(to_h[c], list_tile_off(idx_o, B, H, T, D, gran))
        check_codes(oracle, x_np, cbs[c], S, unpack_indices(words_h[c], S, n_chunks),
                    radius_h[c], thr=thrs[c], gran=gran)
    s = hqmq.read_status(st)
    assert s["n_outliers"] == total and (s["flags"] & ~2) == 0, s
    print("[append] %s T=%d gran=%d: %d calls, %d list entries" % (name, T, gran, C, total))
