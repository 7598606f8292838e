"""The bench's roofline accounting, worked by hand for the Llama-3-70B 128k
call (1 x 8 x 131072 x 128 bf16, S = 32, Med3x chunk mode): the scope's
algorithmic bytes of the encode call (x read twice, codes, 12 B per outlier),
the one-read figure, the decode's bytes, and the HBM fraction the line
reports from a per-call time."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from kv_cache_quantization_hqmq_b200 import workloads as W  # noqa: E402


def test_70b_call_bytes_by_hand():
    w = W.WORKLOADS["llama3_70b_128k"]
    assert w.call_shape == (1, 8, 131072, 128) and w.S == 32 and w.med3
    n_out = 901_499                               # outlier chunks of one call
    ab = bench.algorithmic_bytes(w, n_out, table=True)
    x = 8 * 131072 * 128 * 2                      # bf16 input: 268,435,456 B
    chunks = 8 * 131072 * 128 // 4                # 33,554,432
    codes = chunks * (10 + 16) // 8               # 10-bit index + fp16 radius per chunk
    lst = n_out * (4 + 8)                         # u32 index + 4 fp16 values
    assert ab["med3_encode"] == 2 * x + codes + lst
    assert ab["med3_encode_one_read"] == x + codes + lst
    assert ab["decode"] == codes + lst + x        # codes and list in, bf16 y out
    # 268,435,456 (x) + 109,051,904 (codes) + 10,817,988 (list)
    assert int(ab["med3_encode_one_read"]) == 388_305_348


def test_hbm_fraction_from_a_call_time():
    w = W.WORKLOADS["llama3_70b_128k"]
    peaks = {"hbm_gbs": 6553.9}
    kern = bench.kernel_stats(w, {"med3_encode": 0.334, "decode": 0.0868}, peaks, 901_499, True)
    ab = bench.algorithmic_bytes(w, 901_499, True)
    e = kern["med3_encode"]
    assert e["hbm_gbs"] == pytest.approx(ab["med3_encode"] / 0.334e-3 / 1e9, rel=1e-3)
    assert e["hbm_frac"] == pytest.approx(e["hbm_gbs"] / 6553.9, abs=1e-4)
    assert e["one_read_hbm_frac"] == pytest.approx(
        ab["med3_encode_one_read"] / 0.334e-3 / 1e9 / 6553.9, abs=1e-4)
    assert kern["decode"]["hbm_frac"] == pytest.approx(ab["decode"] / 0.0868e-3 / 1e9 / 6553.9,
                                                       abs=1e-4)
    assert e["calls_per_step"] == w.n_calls == 160
