"""hqmq_outlier_extract_noalloc: the Med3x entry point for callers that
cannot allocate device memory (a serving engine whose GPU memory is all
reserved by its own pool, or a hook where cudaMalloc/cudaFree may not run).
It keeps its scratch in the library's fixed device array instead of a
caller workspace; its results must equal those of hqmq_outlier_extract.

This file sorts last so that a run stopping at the first failure has already
run every other test; it also passes when run alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

from kv_cache_quantization_hqmq_b200 import hqmq  # noqa: E402
from kv_cache_quantization_hqmq_b200 import workloads as W  # noqa: E402


def _run(x, gran, cap, noalloc):
    B, H, T, D = x.shape
    st = hqmq.new_status()
    rmed, thr, oi, ov, so, ws = hqmq.alloc_outliers(B, H, T, D, cap, gran)
    oi.fill_(-1)
    ov.fill_(-1)
    if noalloc:
        del ws
        hqmq.hqmq_outlier_extract_noalloc(x, 3.0, gran, rmed, thr, oi, ov, so, cap, st)
    else:
        hqmq.hqmq_outlier_extract(x, 3.0, gran, rmed, thr, oi, ov, so, cap, ws, st)
    torch.cuda.synchronize()
    return [t.cpu().numpy() for t in (rmed, thr, oi, ov, so)], hqmq.read_status(st)


@pytest.mark.parametrize("gran", [0, 1])
def test_noalloc_matches_workspace_entry_point_twice(gran):
    w = W.WORKLOADS["qwen_outlier"]
    # two calls in a row on different inputs (K then V), the second reusing
    # the scratch the first left behind
    for role in (0, 1):
        x = W.make_call_input(w, 2, role, device="cuda", tokens=1024)
        n = x.numel() // 4 if gran == 0 else x.numel()
        cap = n // 5
        a, sa = _run(x, gran, cap, noalloc=True)
        b, sb = _run(x, gran, cap, noalloc=False)
        for u, v in zip(a, b):
            assert np.array_equal(u.view(np.uint8), v.view(np.uint8))
        # the workspace entry point may report that its sampled median window
        # fell back to the exact path (a diagnostic bit this one never sets)
        sb["flags"] &= ~hqmq.FLAG_MED3_FALLBACK
        assert sa == sb and sa["n_outliers"] > 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    lib = hqmq.lib()
    need = hqmq.hqmq_outlier_workspace_size(1, 160, 64, 128)
    assert need > (1 << 20)
    p = ctypes.c_void_p(1 << 20)
    rc = lib.hqmq_outlier_extract_noalloc(p, 0, 1, 160, 64, 128, ctypes.c_float(3.0), 0, p, p, p,
                                          p, p, 16, None, None)
    assert rc == hqmq.HQMQ_ERR_WORKSPACE
