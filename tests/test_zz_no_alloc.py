"""hqmq_outlier_extract_noalloc: the Med3x entry point for callers that
cannot allocate device memory (a serving engine whose GPU memory is all
reserved by its own pool, or a hook where cudaMalloc/cudaFree may not run).
It keeps its scratch in the library's fixed device array instead of a
caller workspace; its results must equal those of hqmq_outlier_extract.

This file sorts last so that a run stopping at the first failure has already
run every other test; it also passes when run alone in a fresh process."""
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


# The three-pass selection's scratch for a call [B, H, T, D]: a 2048-bin
# histogram per head (8 KB), 8 bytes of selection state per head and two
# uint32 counts per 4096-chunk tile, each region rounded up to 256 bytes.
# With T*D/4 <= 4096 (one tile per slab) and B = 1 that is
# 8192 H + 2 * ceil256(4 H) + ceil256(8 H): H = 127 fits the 1 MiB array
# (1,042,432 bytes), H = 128 does not (1,050,624).
H_FITS = 127


def _noalloc_shape(H):
    return (1, H, 32, 128)          # 1024 chunks per slab: one tile


def test_noalloc_largest_shape_that_fits_matches_workspace_entry_point():
    # the last 256-byte regions of the array are in use here: an off-by-one
    # or misaligned region at the end of the scratch would show up as a
    # difference from the workspace entry point
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    x = torch.randn(_noalloc_shape(H_FITS), generator=g, device="cuda").to(torch.bfloat16)
    x.view(-1, 4)[::97] *= 20.0                     # some outliers in every head
    for gran in (0, 1):
        n = x.numel() // 4 if gran == 0 else x.numel()
        for _ in range(2):                          # twice in a row
            a, sa = _run(x, gran, n, noalloc=True)
            b, sb = _run(x, gran, n, noalloc=False)
            for u, v in zip(a, b):
                assert np.array_equal(u.view(np.uint8), v.view(np.uint8))
            sb["flags"] &= ~hqmq.FLAG_MED3_FALLBACK
            assert sa == sb and sa["n_outliers"] > 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # real buffers of the rejected shape: if the size check ever let this
    # shape through, the call would run on valid memory and fail an assert
    # below instead of touching memory it does not own
    B, H, T, D = _noalloc_shape(H_FITS + 1)
    x = torch.zeros((B, H, T, D), dtype=torch.bfloat16, device="cuda")
    cap = B * H * T * D // 4
    rmed, thr, oi, ov, so, ws = hqmq.alloc_outliers(B, H, T, D, cap, 0)
    st = hqmq.new_status()
    with pytest.raises(hqmq.HQMQError) as e:
        hqmq.hqmq_outlier_extract_noalloc(x, 3.0, 0, rmed, thr, oi, ov, so, cap, st)
    assert e.value.rc == hqmq.HQMQ_ERR_WORKSPACE
    # twice as many heads, several batches and tiles: rejected as well
    B, H, T, D = 2, 2 * (H_FITS + 1), 160, 128
    x = torch.zeros((B, H, T, D), dtype=torch.bfloat16, device="cuda")
    cap = B * H * T * D // 4
    rmed, thr, oi, ov, so, ws = hqmq.alloc_outliers(B, H, T, D, cap, 0)
    with pytest.raises(hqmq.HQMQError) as e:
        hqmq.hqmq_outlier_extract_noalloc(x, 3.0, 0, rmed, thr, oi, ov, so, cap, st)
    assert e.value.rc == hqmq.HQMQ_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert hqmq.read_status(st)["flags"] == 0       # nothing ran
