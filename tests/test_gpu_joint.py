"""The joint (index, radius level) block code and the 1-bit outlier flags on
the GPU against the oracle: packed words bit for bit, flags bit for bit, and
the decode from joint code + flags equal to the oracle's quantized-radius
decode of the same codes and list, bit for bit; at the full 70B call shape,
the whole chain against the GPU's quantized-radius decode."""
import numpy as np
import pytest
import torch

from _parity import list_tile_off, same_f16_or_bf16_bits, same_f32, to_host, unpack_indices

pytestmark = pytest.mark.gpu
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

from kv_cache_quantization_hqmq_b200 import hqmq  # noqa: E402
from kv_cache_quantization_hqmq_b200 import workloads as W  # noqa: E402


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def oracle_codes(oracle, x, S, seed=1):
    """The oracle's codes of a call: Med3x (chunk mode), encode, radius levels."""
    B, H, T, D = x.shape
    cb = oracle.make_codebook(seed, S, H)
    _, thr = oracle.med3_threshold(x, 3.0, 0)
    oi, ov, so, n_o, _ = oracle.extract(x, thr)
    words, rad, _, _, _ = oracle.encode(x, cb, S, thr=thr)
    rw = oracle.quantize_radius(rad, thr, B, H, T, D, S)
    return cb, thr, oi, ov, so, n_o, words, rw


CASES = [("qwen_outlier", 1024), ("qwen_outlier", 1000), ("mha7b_s8", 256), ("tiny", 256)]


@pytest.mark.parametrize("name,tokens", CASES, ids=["%s-T%d" % c for c in CASES])
def test_joint_pack_flags_and_decode_match_the_oracle(oracle, name, tokens):
    w = W.WORKLOADS[name]
    x = W.as_numpy_bits(W.make_call_input(w, 3, 1, tokens=tokens, batch=min(w.batch, 2)))
    B, H, T, D = x.shape
    S = w.S
    cb, thr, oi, ov, so, n_o, words, rw = oracle_codes(oracle, x, S)
    # pack: bit for bit
    joint_o, bad = oracle.pack_joint(words, rw, B, H, T, D, S)
    assert bad == 0
    joint = hqmq.alloc_joint(B, H, T, D, S)
    st = hqmq.new_status()
    hqmq.hqmq_pack_joint(dev(words.view(np.int32)), dev(rw.view(np.int32)), S, (B, H, T, D),
                         joint, st)
    torch.cuda.synchronize()
    assert np.array_equal(to_host(joint).view(np.uint32), joint_o)
    assert hqmq.read_status(st)["flags"] == 0
    # flags: bit for bit
    n_chunks = B * H * T * D // 4
    flags = torch.empty(n_chunks // 32, dtype=torch.int32, device="cuda")
    cap = max(n_o, 1)
    oid = dev(oi.view(np.int32)) if n_o else torch.zeros(1, dtype=torch.int32, device="cuda")
    hqmq.hqmq_list_flags(oid, dev(so.view(np.int32)), cap, (B, H, T, D), flags)
    torch.cuda.synchronize()
    assert np.array_equal(to_host(flags).view(np.uint32), oracle.list_flags(oi, n_chunks))
    # decode from joint code + flags = the oracle's quantized-radius decode
    ovd = dev(ov.reshape(-1).view(np.int16)) if n_o else torch.zeros(4, dtype=torch.int16,
                                                                     device="cuda")
    to = dev(list_tile_off(oi, B, H, T, D, 0).view(np.int32))
    for out_dt, od in ((torch.bfloat16, 0), (torch.float32, 1)):
        for with_list in (False, True):
            yo, _ = oracle.decode_qradius(words, rw, thr, cb, S, B, H, T, D,
                                          out_idx=oi if with_list else None,
                                          out_val=ov if with_list else None, out_dtype=od)
            y = torch.empty((B, H, T, D), dtype=out_dt, device="cuda")
            hqmq.hqmq_decode_joint(joint, dev(thr), dev(cb.reshape(-1)), S,
                                   flags if with_list else None, ovd if with_list else None,
                                   to if with_list else None, n_o, y)
            torch.cuda.synchronize()
            if od == 0:
                ok = same_f16_or_bf16_bits(to_host(y.view(torch.int16)), yo, bf16=True)
            else:
                ok = same_f32(to_host(y), yo)
            assert ok.all(), (out_dt, with_list, np.argwhere(~ok.reshape(-1))[:5])
    n, wbits = hqmq.hqmq_joint_block(S)
    print("[joint] %s T%d: %d chunks, %d outliers, %d words (%.4f bits/elem codes)"
          % (name, tokens, n_chunks, n_o, joint.numel(), joint.numel() * 32 / (n_chunks * 4)))


def test_joint_full_size_70b_call_equals_the_qradius_decode(oracle):
    # the whole chain at the benched call shape: Med3x + encode, levels,
    # joint code, flags, decode -- equal to hqmq_decode_qradius on the same
    # codes and list, bit for bit; the joint code unpacks (oracle) to the
    # GPU's index and level fields on a sample
    w = W.WORKLOADS["llama3_70b_128k"]
    B, H, T, D = w.call_shape
    S = w.S
    xd = W.make_call_input(w, 17, 0, device="cuda")
    cb = torch.empty(H * S * 4, dtype=torch.float32, device="cuda")
    hqmq.hqmq_make_codebook(w.codebook_seed, S, H, W.group0(17, 0, H), cb)
    table = torch.empty(H * hqmq.hqmq_search_table_bytes(S), dtype=torch.uint8, device="cuda")
    hqmq.hqmq_make_search_table(cb, S, H, table)
    n_chunks = B * H * T * D // 4
    cap = n_chunks // 10
    words, radius = hqmq.alloc_codes(B, H, T, D, S)
    rmed, thr, oi, ov, so, _ = hqmq.alloc_outliers(B, H, T, D, cap)
    ws = torch.empty(hqmq.hqmq_encode_med3_workspace_size(B, H, T, D, 0), dtype=torch.uint8,
                     device="cuda")
    to = hqmq.alloc_tile_off(B, H, T, D)
    hqmq.hqmq_encode_med3(xd, w.C, 0, cb, S, table, words, radius, rmed, thr, oi, ov, so, cap, ws,
                          hqmq.new_status(), tile_off=to)
    rw = torch.empty_like(words)
    hqmq.hqmq_quantize_radius(radius, thr, (B, H, T, D), S, rw)
    joint = hqmq.alloc_joint(B, H, T, D, S)
    st = hqmq.new_status()
    hqmq.hqmq_pack_joint(words, rw, S, (B, H, T, D), joint, st)
    flags = torch.empty(n_chunks // 32, dtype=torch.int32, device="cuda")
    hqmq.hqmq_list_flags(oi, so, cap, (B, H, T, D), flags)
    y_joint = torch.empty((B, H, T, D), dtype=torch.bfloat16, device="cuda")
    hqmq.hqmq_decode_joint(joint, thr, cb, S, flags, ov, to, cap, y_joint)
    y_qr = torch.empty_like(y_joint)
    hqmq.hqmq_decode_qradius(words, rw, thr, cb, S, oi, ov, to, cap, 0, y_qr)
    torch.cuda.synchronize()
    assert hqmq.read_status(st)["flags"] == 0
    assert torch.equal(y_joint.view(torch.int16), y_qr.view(torch.int16))
    # the packed words against the oracle's unpack on a sample of slabs' runs
    n, wbits = hqmq.hqmq_joint_block(S)
    jh = to_host(joint).view(np.uint32)
    wps = jh.size // (B * H)
    rng = np.random.default_rng(5)
    gi = unpack_indices(to_host(words), S, n_chunks)
    gk = unpack_indices(to_host(rw), S, n_chunks)
    for s in rng.choice(B * H, 2, replace=False):
        idx_o, k_o = oracle.unpack_joint(jh[s * wps:(s + 1) * wps], 1, 1, T, D, S)
        c = T * D // 4
        assert np.array_equal(idx_o, gi[s * c:(s + 1) * c])
        assert np.array_equal(k_o, gk[s * c:(s + 1) * c])
    # flags: exactly the list's chunks
    n_o = int(so[-1])
    lst = to_host(oi[:n_o]).view(np.uint32)
    assert np.array_equal(to_host(flags).view(np.uint32), oracle.list_flags(lst, n_chunks))
