"""Pins of the oracle's decode-phase attention (oracle.attention_decode)
against things other than itself: torch's scaled_dot_product_attention in
fp64 (a library routine), closed forms (one token, equal keys, zero scale, a
dominant key), the GQA head mapping and token-permutation invariance."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F


def bf16_bits(x):
    """bf16 bit patterns (RN-even) of a float array, via torch."""
    t = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def q_values(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def sdpa(q, k, v, scale, G, seq_len):
    """torch SDPA (fp64, CPU), GQA by repeating each KV head G times, the
    tokens >= seq_len[b] masked out."""
    B, Hq, D = q.shape
    T = k.shape[2]
    qt = torch.from_numpy(q).view(B, Hq, 1, D)
    kt = torch.from_numpy(k.astype(np.float64)).repeat_interleave(G, dim=1)
    vt = torch.from_numpy(v.astype(np.float64)).repeat_interleave(G, dim=1)
    mask = torch.arange(T)[None, None, None, :] < torch.tensor(seq_len)[:, None, None, None]
    o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    return o.view(B, Hq, D).numpy()


def test_matches_torch_sdpa_gqa_masked(oracle):
    rng = np.random.default_rng(0)
    B, Hk, G, T, D = 3, 2, 3, 37, 128
    qb = bf16_bits(rng.standard_normal((B, Hk * G, D)))
    k = rng.standard_normal((B, Hk, T, D)).astype(np.float32) * 2
    v = rng.standard_normal((B, Hk, T, D)).astype(np.float32)
    seq_len = [37, 5, 0]
    scale = D ** -0.5
    got = oracle.attention_decode(qb, k, v, scale, G, seq_len)
    ref = sdpa(q_values(qb), k, v, scale, G, seq_len)
    np.testing.assert_allclose(got[:2], ref[:2], rtol=1e-12, atol=1e-12)
    assert np.all(got[2] == 0.0)                               # empty sequence: 0


def test_full_length_default_equals_explicit(oracle):
    rng = np.random.default_rng(1)
    qb = bf16_bits(rng.standard_normal((2, 4, 128)))
    k = rng.standard_normal((2, 2, 9, 128))
    v = rng.standard_normal((2, 2, 9, 128))
    a = oracle.attention_decode(qb, k, v, 0.1, 2)
    b = oracle.attention_decode(qb, k, v, 0.1, 2, [9, 100])     # clamped to T
    np.testing.assert_array_equal(a, b)


def test_one_token_returns_its_value(oracle):
    rng = np.random.default_rng(2)
    qb = bf16_bits(rng.standard_normal((1, 2, 128)))
    k = rng.standard_normal((1, 1, 5, 128))
    v = rng.standard_normal((1, 1, 5, 128))
    o = oracle.attention_decode(qb, k, v, 0.3, 2, [1])
    np.testing.assert_array_equal(o[0, 0], v[0, 0, 0])
    np.testing.assert_array_equal(o[0, 1], v[0, 0, 0])


def test_equal_keys_or_zero_scale_give_the_mean(oracle):
    rng = np.random.default_rng(3)
    qb = bf16_bits(rng.standard_normal((1, 1, 128)))
    v = rng.standard_normal((1, 1, 20, 128))
    k_same = np.repeat(rng.standard_normal((1, 1, 1, 128)), 20, axis=2)
    o = oracle.attention_decode(qb, k_same, v, 0.2, 1, [13])
    np.testing.assert_allclose(o[0, 0], v[0, 0, :13].mean(0), rtol=0, atol=1e-13)
    k = rng.standard_normal((1, 1, 20, 128))
    o = oracle.attention_decode(qb, k, v, 0.0, 1)
    np.testing.assert_allclose(o[0, 0], v[0, 0].mean(0), rtol=0, atol=1e-13)


def test_dominant_key_selects_its_value(oracle):
    rng = np.random.default_rng(4)
    q = rng.standard_normal(128)
    qb = bf16_bits(q[None, None])
    k = rng.standard_normal((1, 1, 30, 128)) * 0.01
    k[0, 0, 17] = q_values(qb)[0, 0] * 10.0                    # score ~ 10 |q|^2 >> others
    v = rng.standard_normal((1, 1, 30, 128))
    o = oracle.attention_decode(qb, k, v, 1.0, 1)
    np.testing.assert_allclose(o[0, 0], v[0, 0, 17], rtol=0, atol=1e-12)


def test_gqa_head_mapping(oracle):
    """Query head h reads KV head h // G: with V of KV head j equal to j + 1
    everywhere, o[b, h] = h // G + 1 exactly."""
    rng = np.random.default_rng(5)
    B, Hk, G, T = 2, 3, 4, 11
    qb = bf16_bits(rng.standard_normal((B, Hk * G, 128)))
    k = rng.standard_normal((B, Hk, T, 128))
    v = np.broadcast_to(np.arange(1, Hk + 1, dtype=np.float64)[None, :, None, None],
                        (B, Hk, T, 128)).copy()
    o = oracle.attention_decode(qb, k, v, 0.5, G)
    want = (np.arange(Hk * G) // G + 1).astype(np.float64)
    np.testing.assert_allclose(o, np.broadcast_to(want[None, :, None], o.shape), rtol=1e-15)


def test_token_order_does_not_matter(oracle):
    rng = np.random.default_rng(6)
    qb = bf16_bits(rng.standard_normal((1, 2, 128)))
    k = rng.standard_normal((1, 1, 25, 128))
    v = rng.standard_normal((1, 1, 25, 128))
    perm = rng.permutation(25)
    a = oracle.attention_decode(qb, k, v, 0.2, 2)
    b = oracle.attention_decode(qb, k[:, :, perm], v[:, :, perm], 0.2, 2)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("bad", ["kv_head_mod", "no_max_shift_scale", "drop_last_token"])
def test_planted_mistakes_are_caught(oracle, bad, monkeypatch):
    """Plausible mistakes planted in a copy of the oracle's attention fail the
    SDPA comparison above."""
    rng = np.random.default_rng(7)
    B, Hk, G, T, D = 2, 2, 3, 16, 128
    qb = bf16_bits(rng.standard_normal((B, Hk * G, D)))
    k = rng.standard_normal((B, Hk, T, D))
    v = rng.standard_normal((B, Hk, T, D))
    scale = D ** -0.5

    def mutated(q_bits, k_hat, v_hat, scale_, G_, seq_len=None):
        q = q_values(np.asarray(q_bits, np.uint16))
        o = np.zeros(q.shape)
        for b in range(q.shape[0]):
            n = k_hat.shape[2] - (1 if bad == "drop_last_token" else 0)
            for h in range(q.shape[1]):
                hk = h % Hk if bad == "kv_head_mod" else h // G_
                s = (1.0 if bad == "no_max_shift_scale" else scale_) * (k_hat[b, hk, :n] @ q[b, h])
                w = np.exp(s - s.max())
                o[b, h] = (w @ v_hat[b, hk, :n]) / w.sum()
        return o

    ref = sdpa(q_values(qb), k, v, scale, G, [T] * B)
    np.testing.assert_allclose(oracle.attention_decode(qb, k, v, scale, G), ref, rtol=1e-12,
                               atol=1e-12)
    assert not np.allclose(mutated(qb, k, v, scale, G), ref, rtol=1e-6, atol=1e-6)
