"""Parity of hqmq_attention_decode (attention read straight from the codes)
with the oracle.

Inputs: seeded K/V tensors and queries of the workloads (reduced token counts);
the codes, radii and Med3x lists are written by the ORACLE (encode, extract),
so no input of the oracle comes from the CUDA path.  Expected: the oracle's
bf16 decode of those codes, then its fp64 attention.

Tolerance (derived from the kernel's arithmetic, per batch b and query head h;
u = 2^-24):
* a score enters exp2 as x = sl2 * s with s the fp32 tensor-core sum of 128
  exact bf16 products: |dx| <= sl2 * 128 * 2u * max_t sum_d |q_d k_td|
  plus one rounding of x;
* exp2 (<= 2^-21 relative), the split P = P_hi + P_lo (<= 2^-17);
* the normalised weights then err by at most d = 2 (ln2 |dx| + 2^-21 + 2^-17)
  relative, so |do| <= d * max_{t,i} |v_ti - o_i|;
* fp32 accumulation over the blocks and the merges: n_add * u * max|v| with
  n_add = T / 16 + 64.
The test asserts |o_gpu - o_ref| <= 2 x that bound (and reports the largest
ratio), and bf16 outputs within one bf16 rounding of it.

The full-size cases use the bench's shapes and launch configuration: the
inputs repeat with a period of P tokens along T (the codes and the Med3x
list of one period, written by the oracle, tiled to T; the per-head median of
k identical copies is the median of one copy, so the tiled list is the
oracle's list of the whole tensor), and softmax over k identical copies of a
period equals softmax over one period, so the expected output is the oracle's
attention over one period.
"""
import numpy as np
import pytest
import torch

from _parity import list_tile_off
from kv_cache_quantization_hqmq_b200 import hqmq
from kv_cache_quantization_hqmq_b200.workloads import (WORKLOADS, as_numpy_bits, group0,
                                                       make_call_input, make_query)

pytestmark = pytest.mark.gpu
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

U = 2.0 ** -24


def oracle_cache(oracle, w, layer, role, B, T, gran=0, med3=None, rq=False):
    """Oracle-written codes (and list) of one cache, and its bf16 decode as fp32
    (rq: with the radius quantized on [0, range], range = thr in chunk mode and
    2 thr in element mode)."""
    S = w.S
    H, D = w.heads, w.head_dim
    x = as_numpy_bits(make_call_input(w, layer, role, tokens=T, batch=B))
    cb = oracle.make_codebook(w.codebook_seed, S, H, group0(layer, role, H))
    thr = idx = val = None
    if (w.med3 if med3 is None else med3):
        _, thr = oracle.med3_threshold(x, w.C, gran)
        idx, val, _, _, _ = oracle.extract(x, thr, gran)
    words, radius, _, _, _ = oracle.encode(x, cb, S, thr, gran)
    rw = rng_ = None
    if rq:
        rng_ = (thr * (2 if gran else 1)).astype(np.float32)
        rw = oracle.quantize_radius(radius, rng_, B, H, T, D, S)
        y, _ = oracle.decode_qradius(words, rw, rng_, cb, S, B, H, T, D, idx, val, gran,
                                     oracle.BF16)
    else:
        y, _ = oracle.decode(words, radius, cb, S, B, H, T, D, idx, val, gran, oracle.BF16)
    return dict(words=words, radius=radius, cb=cb, idx=idx, val=val, gran=gran, rw=rw, rrange=rng_,
                y=oracle.bf16_to_f32(y).reshape(B, H, T, D))


def device_codes(c, B, H, T, D, reps=1):
    """Uploads a cache's codes (tiled reps times along T) as hqmq_kv_codes."""
    b = hqmq.hqmq_index_bits(int(c["cb"].size // (H * 4)))
    words = c["words"].reshape(B * H, -1)
    radius = c["radius"].reshape(B * H, -1)
    wd = torch.from_numpy(np.ascontiguousarray(np.tile(words, (1, reps))).view(np.int32).reshape(-1))
    rd = torch.from_numpy(np.ascontiguousarray(np.tile(radius, (1, reps))).view(np.int16).reshape(-1))
    assert wd.numel() == B * H * T * reps * D // 128 * b
    dev = dict(words=wd.cuda(), radius=rd.cuda(), cb=torch.from_numpy(c["cb"].reshape(-1)).cuda())
    qr = {}
    if c.get("rw") is not None:
        rw = c["rw"].reshape(B * H, -1)
        dev["rw"] = torch.from_numpy(np.ascontiguousarray(np.tile(rw, (1, reps))).view(np.int32)
                                     .reshape(-1)).cuda()
        dev["rrange"] = torch.from_numpy(c["rrange"]).cuda()
        dev["radius"] = None
        qr = dict(rcode_words=dev["rw"], thr=dev["rrange"])
    idx, val = c["idx"], c["val"]
    if idx is None or len(idx) == 0:
        return hqmq.kv_codes(dev["words"], dev["radius"], dev["cb"], **qr), dev
    el = 4 if c["gran"] else 1                       # list units per chunk
    cps = T * D // 4 * el                            # units per slab, one period
    slab, off = np.asarray(idx, np.int64) // cps, np.asarray(idx, np.int64) % cps
    tiled = np.concatenate([slab * cps * reps + r * cps + off for r in range(reps)])
    order = np.argsort(tiled, kind="stable")
    tiled = tiled[order].astype(np.uint32)
    v = np.asarray(val).reshape(len(idx), -1)
    vt = np.concatenate([v] * reps)[order]
    to = list_tile_off(tiled, B, H, T * reps, D, c["gran"])
    dev.update(idx=torch.from_numpy(tiled.view(np.int32)).cuda(),
               val=torch.from_numpy(np.ascontiguousarray(vt).view(np.int16).reshape(-1)).cuda(),
               to=torch.from_numpy(to.view(np.int32)).cuda())
    return hqmq.kv_codes(dev["words"], dev["radius"], dev["cb"], dev["idx"], dev["val"],
                         dev["to"], len(tiled), c["gran"], **qr), dev


def bound(q_bits, k, v, o_ref, scale, G, seq_len, T):
    """Per (b, h) error bound of the fp32 kernel (see the module docstring)."""
    q = hqmq_bf16(q_bits)
    B, Hq, D = q.shape
    sl2 = scale / np.log(2.0)
    out = np.zeros((B, Hq))
    for b in range(B):
        n = T if seq_len is None else min(max(int(seq_len[b]), 0), T)
        if n == 0:
            continue
        for h in range(Hq):
            K, V = k[b, h // G, :n].astype(np.float64), v[b, h // G, :n].astype(np.float64)
            sq = np.abs(K * q[b, h]).sum(1).max()
            x = np.abs(sl2 * (K @ q[b, h])).max()
            dx = sl2 * 128 * 2 * U * sq + 2 * U * x
            d = 2 * (np.log(2.0) * dx + 2.0 ** -21 + 2.0 ** -17)
            dv = np.abs(V - o_ref[b, h]).max()
            out[b, h] = d * dv + (T / 16 + 64) * U * np.abs(V).max()
    return out


def hqmq_bf16(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def run_case(oracle, w, B, T, seq_len=None, gran=0, out_dtype=torch.float32, layer=0, reps=1,
             med3=None, rq=False):
    H, D, Hq = w.heads, w.head_dim, w.n_q_heads
    G = Hq // H
    kc = oracle_cache(oracle, w, layer, 0, B, T, gran, med3, rq)
    vc = oracle_cache(oracle, w, layer, 1, B, T, gran, med3, rq)
    kd, keep_k = device_codes(kc, B, H, T, D, reps)
    vd, keep_v = device_codes(vc, B, H, T, D, reps)
    q = make_query(w, layer, batch=B)
    qb = as_numpy_bits(q)
    scale = D ** -0.5
    sl = None if seq_len is None else torch.tensor(seq_len, dtype=torch.int32).cuda()
    o = torch.full((B, Hq, D), float("nan"), dtype=out_dtype, device="cuda")
    ws = hqmq.alloc_attention_ws(B, H)
    st = hqmq.new_status()
    hqmq.hqmq_attention_decode(q.cuda(), kd, vd, w.S, H, T * reps, o, ws, scale=scale,
                               seq_len=sl, status=st)
    torch.cuda.synchronize()
    # the expected output over one period (seq_len scaled back for tiled inputs)
    assert reps == 1 or seq_len is None or all(s_ % T == 0 for s_ in seq_len)
    sl_p = None if seq_len is None else [min(max(s, 0), T * reps) for s in seq_len]
    if reps > 1 and sl_p is not None:            # k whole periods: one period
        sl_p = [T if s_ > 0 else 0 for s_ in sl_p]
    ref = oracle.attention_decode(qb, kc["y"], vc["y"], scale, G, sl_p)
    tol = 2 * bound(qb, kc["y"], vc["y"], ref, scale, G, sl_p, T * reps)
    got = o.float().cpu().numpy().astype(np.float64)
    if out_dtype == torch.bfloat16:
        tol = tol[:, :, None] + 2.0 ** -8 * np.abs(ref)
    else:
        tol = tol[:, :, None]
    err = np.abs(got - ref)
    assert np.isfinite(got).all()
    ratio = (err / np.maximum(tol, 1e-30)).max()
    print("[attn] %s B=%d T=%d reps=%d G=%d gran=%d list=%d/%d: max err %.3g, err/tol %.3g"
          % (w.name, B, T, reps, G, gran, 0 if kc["idx"] is None else len(kc["idx"]),
             0 if vc["idx"] is None else len(vc["idx"]), err.max(), ratio))
    assert (err <= tol).all(), "max err/tol %.3g" % ratio
    assert hqmq.read_status(st)["flags"] == 0
    return ratio


@pytest.mark.parametrize("T", [16, 48, 1000])
def test_attention_no_list(oracle, T):
    run_case(oracle, WORKLOADS["llama3_8b"], B=2, T=T)


def test_attention_gqa7_outlier_list(oracle):
    run_case(oracle, WORKLOADS["qwen_outlier"], B=2, T=600, seq_len=[600, 257])


def test_attention_mha_ragged_lengths(oracle):
    w = WORKLOADS["mha7b_s8"].with_(heads=3, q_heads=3)
    run_case(oracle, w, B=4, T=100, seq_len=[0, 1, 100, 37])


def test_attention_lengths_clamped(oracle):
    run_case(oracle, WORKLOADS["llama3_8b"].with_(heads=2, q_heads=8), B=3, T=64,
             seq_len=[-5, 5, 1000])


def test_attention_element_mode(oracle):
    w = WORKLOADS["llama3_70b_128k"].with_(heads=2, q_heads=16)
    run_case(oracle, w, B=1, T=512, gran=1)


def test_attention_g8_bf16_out(oracle):
    w = WORKLOADS["llama3_70b_128k"].with_(heads=2, q_heads=16)
    run_case(oracle, w, B=2, T=2048, out_dtype=torch.bfloat16)


def test_attention_full_size_70b_128k(oracle):
    """B=1, Hk=8, Hq=64, T=131072, S=32, Med3x chunk list: the bench's launch."""
    w = WORKLOADS["llama3_70b_128k"]
    run_case(oracle, w, B=1, T=1024, reps=128)


def test_attention_full_size_8b(oracle):
    """B=1, Hk=8, Hq=32, T=8192, S=8, no list."""
    w = WORKLOADS["llama3_8b"]
    run_case(oracle, w, B=1, T=512, reps=16, seq_len=[512 * 13])


def test_attention_rejects_bad_arguments():
    w = WORKLOADS["llama3_8b"]
    B, H, T, D = 1, 2, 32, 128
    words, radius = hqmq.alloc_codes(B, H, T, D, 8)
    cb = torch.zeros(H * 8 * 4, dtype=torch.float32, device="cuda")
    kv = hqmq.kv_codes(words, radius, cb)
    ws = hqmq.alloc_attention_ws(B, H)
    q = torch.zeros(B, 2 * 9, D, dtype=torch.bfloat16, device="cuda")     # G = 9 > 8
    o = torch.zeros(B, 2 * 9, D, dtype=torch.float32, device="cuda")
    with pytest.raises(hqmq.HQMQError):
        hqmq.hqmq_attention_decode(q, kv, kv, 8, H, T, o, ws)
    q = torch.zeros(B, 4, D, dtype=torch.bfloat16, device="cuda")
    o = torch.zeros(B, 4, D, dtype=torch.float32, device="cuda")
    with pytest.raises(hqmq.HQMQError):                                    # workspace too small
        hqmq.hqmq_attention_decode(q, kv, kv, 8, H, T, o, ws[:1024])
    del w


def test_attention_dense_list_past_staging(oracle):
    """Tiles with more list entries than the kernel stages (192 per tile):
    the rest is found in global memory."""
    w = WORKLOADS["qwen_outlier"].with_(channel_frac=0.4, heads=2, q_heads=14)
    run_case(oracle, w, B=1, T=256, seq_len=[250])


@pytest.mark.parametrize("S", [3, 16, 100])
def test_attention_other_codebook_sizes(oracle, S):
    """Index widths other than 8 and 10 bits (generic kernels; S = 100 with
    fewer table copies)."""
    w = WORKLOADS["qwen_outlier"].with_(S=S, heads=2, q_heads=6)
    run_case(oracle, w, B=2, T=96, seq_len=[96, 40])


def test_attention_list_truncated_at_cap(oracle):
    """A list whose writer ran out of room: only the entries below cap exist
    (the tile offsets still count all of them); the chunks past cap keep
    their zeroed codes, exactly as hqmq_decode reads them."""
    w = WORKLOADS["qwen_outlier"].with_(heads=2, q_heads=6)
    B, T, D, H = 1, 256, 128, 2
    G = w.n_q_heads // H
    kc = oracle_cache(oracle, w, 0, 0, B, T)
    vc = oracle_cache(oracle, w, 0, 1, B, T)
    kd, keep_k = device_codes(kc, B, H, T, D)
    vd, keep_v = device_codes(vc, B, H, T, D)
    cap_k, cap_v = len(kc["idx"]) // 2, len(vc["idx"]) // 3
    kd.cap, vd.cap = cap_k, cap_v                     # the tile offsets keep the full counts
    q = make_query(w, 0, batch=B)
    o = torch.empty(B, w.n_q_heads, D, dtype=torch.float32, device="cuda")
    hqmq.hqmq_attention_decode(q.cuda(), kd, vd, w.S, H, T, o, hqmq.alloc_attention_ws(B, H))
    torch.cuda.synchronize()

    def trunc_decode(c, cap):
        y, _ = oracle.decode(c["words"], c["radius"], c["cb"], w.S, B, H, T, D, c["idx"][:cap],
                             c["val"][:cap], 0, oracle.BF16)
        return oracle.bf16_to_f32(y).reshape(B, H, T, D)

    kt, vt = trunc_decode(kc, cap_k), trunc_decode(vc, cap_v)
    qb = as_numpy_bits(q)
    ref = oracle.attention_decode(qb, kt, vt, D ** -0.5, G)
    tol = 2 * bound(qb, kt, vt, ref, D ** -0.5, G, None, T)[:, :, None]
    err = np.abs(o.cpu().numpy() - ref)
    assert (err <= tol).all(), (err / tol).max()
    full = oracle.attention_decode(qb, kc["y"], vc["y"], D ** -0.5, G)
    assert np.abs(full - ref).max() > 10 * tol.max()    # the truncation does change the result


def test_attention_quantized_radius_gqa7_list(oracle):
    """K and V with radius codes (5 bits per element with the index at S = 32)."""
    run_case(oracle, WORKLOADS["qwen_outlier"], B=2, T=600, seq_len=[600, 257], rq=True)


def test_attention_quantized_radius_element_mode(oracle):
    w = WORKLOADS["llama3_70b_128k"].with_(heads=2, q_heads=16)
    run_case(oracle, w, B=1, T=512, gran=1, rq=True)


def test_attention_quantized_radius_full_size_70b_128k(oracle):
    run_case(oracle, WORKLOADS["llama3_70b_128k"], B=1, T=1024, reps=128, rq=True)


def test_attention_many_sequences(oracle):
    """160 (b, hk) heads: one CTA per head writes the output directly (no CTA
    partials); ragged lengths."""
    w = WORKLOADS["llama3_8b"].with_(heads=4, q_heads=16)
    B = 40
    lens = [(7 * i) % 97 + 1 for i in range(B)]
    run_case(oracle, w, B=B, T=96, seq_len=lens)
