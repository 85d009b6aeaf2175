"""Pins of the verifier-attention oracle (oracle/attention.py): rotary
embedding properties, closed forms of softmax attention, causality, the cache
writes."""
import numpy as np

import oracle
from oracle.attention import HEAD_DIM, N_HEADS, attn_verify, rope

H = N_HEADS * HEAD_DIM


def _bits(a):
    return oracle.round_bf16_bits(np.asarray(a, dtype=np.float64))


def test_rope_rotates_pairs_and_depends_on_relative_position():
    rng = np.random.default_rng(1)
    q, k = rng.normal(0, 1, (1, H)), rng.normal(0, 1, (1, H))
    assert np.array_equal(rope(q, [0]), q)  # position 0: identity
    r = rope(q, [37])
    pair_norm = lambda a: np.hypot(a.reshape(-1, 2)[:, 0], a.reshape(-1, 2)[:, 1])
    assert np.allclose(pair_norm(r), pair_norm(q), rtol=1e-12)
    # per head, <rope(q, m), rope(k, n)> depends on m - n only
    for m, n, s in [(5, 2, 100), (0, 9, 31), (1000, 3, 7)]:
        a = (rope(q, [m]) * rope(k, [n])).reshape(N_HEADS, HEAD_DIM).sum(1)
        b = (rope(q, [m + s]) * rope(k, [n + s])).reshape(N_HEADS, HEAD_DIM).sum(1)
        assert np.allclose(a, b, rtol=1e-9, atol=1e-9)
    # the first pair turns by the full position angle, the last by 10000^(-126/128) of it
    e = np.zeros((1, H))
    e[0, 0] = 1.0
    assert np.allclose(rope(e, [2.0])[0, :2], [np.cos(2.0), np.sin(2.0)])


def _eye_qkv(q_scale=0.0):
    """W_qkv with q = q_scale * x, k = x, v = x."""
    return _bits(np.concatenate([np.eye(H) * q_scale, np.eye(H), np.eye(H)]))


def test_single_position_returns_its_own_value():
    """L = 0, K = 0: the one key is the row itself, softmax weight 1, o = v = x
    (W_v = I), and with W_o = I the output is bf16(x + x) = 2x exactly."""
    rng = np.random.default_rng(2)
    x = _bits(rng.normal(0, 1, (3, H)))
    cache = np.zeros((3, 2, 4, H), dtype=np.uint16)
    out, _, mid = attn_verify(x, _eye_qkv(0.3), _bits(np.eye(H)), cache, [0, 0, 0], 0)
    assert np.array_equal(mid["o"], x)
    assert np.array_equal(oracle.widen(out), 2 * oracle.widen(x))


def test_zero_query_averages_the_visible_values():
    """W_q = 0: every score is 0, so row i's output is the mean of the values at
    positions 0 .. L+i (cached ones, then the new rows' own)."""
    rng = np.random.default_rng(3)
    B, K, L = 2, 3, 5
    x = _bits(rng.normal(0, 1, (B * (K + 1), H)))
    cache = np.zeros((B, 2, 16, H), dtype=np.uint16)
    cache[:, 1, :L] = _bits(rng.normal(0, 1, (B, L, H)))
    _, new_cache, mid = attn_verify(x, _eye_qkv(0.0), _bits(np.eye(H)), cache, [L, L], K)
    for b in range(B):
        for i in range(K + 1):
            vals = oracle.widen(new_cache[b, 1, : L + i + 1])
            assert np.allclose(oracle.widen(mid["o"][b * (K + 1) + i]), vals.mean(0), rtol=2 ** -8, atol=1e-6)


def test_causal_and_cache_writes():
    """Row i never sees the new rows after it; the cache gets the rotated k and
    the v of the new rows at positions L..L+K and nothing else."""
    rng = np.random.default_rng(4)
    B, K, L = 1, 3, 7
    wqkv = _bits(rng.normal(0, 0.03, (3 * H, H)))
    wo = _bits(rng.normal(0, 0.03, (H, H)))
    x = _bits(rng.normal(0, 1, (K + 1, H)))
    cache = _bits(rng.normal(0, 1, (B, 2, 16, H)))
    out, new_cache, mid = attn_verify(x, wqkv, wo, cache, [L], K)
    x2 = x.copy()
    x2[1:] = _bits(rng.normal(0, 1, (K, H)))  # change every row after the first
    out2, _, _ = attn_verify(x2, wqkv, wo, cache, [L], K)
    assert np.array_equal(out[0], out2[0]) and not np.array_equal(out[1], out2[1])
    assert np.array_equal(new_cache[:, :, :L], cache[:, :, :L])
    assert np.array_equal(new_cache[:, :, L + K + 1:], cache[:, :, L + K + 1:])
    assert np.array_equal(new_cache[0, 0, L: L + K + 1], mid["k"])
    v_new = oracle.round_bf16_bits(oracle.widen(x) @ oracle.widen(wqkv)[2 * H:].T)
    assert np.array_equal(new_cache[0, 1, L: L + K + 1], v_new)


def test_one_dominant_key_is_copied():
    """q = 4x and one cached key along the query in every head: its weight is ~1
    and o is that position's value."""
    rng = np.random.default_rng(5)
    L = 6
    x = _bits(rng.normal(0, 1, (1, H)))
    cache = np.zeros((1, 2, 8, H), dtype=np.uint16)
    cache[0, 1, :L] = _bits(rng.normal(0, 1, (L, H)))
    # position 2's cached key is twice the (rotated) query: its score per head is
    # 2 |q_h|^2 / sqrt(128), in the hundreds; the other cached keys are 0
    q_at = rope(4.0 * oracle.widen(x), [L])  # the query as attn_verify rotates it
    cache[0, 0, 2] = _bits(2.0 * q_at)
    wqkv = _eye_qkv(4.0)
    _, _, mid = attn_verify(x, wqkv, _bits(np.eye(H)), cache, [L], 0)
    assert np.allclose(oracle.widen(mid["o"][0]), oracle.widen(cache[0, 1, 2]), rtol=2 ** -7, atol=1e-3)


def test_rope_frequencies_follow_roformer():
    """RoFormer's theta_i = 10000^(-2(i-1)/d) for the i-th pair (i from 1): the
    second pair of a head turns by p * 10000^(-1/64), the last by p * 10000^(-63/64)."""
    p = 3.0
    for i, theta in [(2, 10000.0 ** (-2.0 / 128)), (64, 10000.0 ** (-126.0 / 128))]:
        e = np.zeros((1, H))
        e[0, 2 * (i - 1)] = 1.0
        r = rope(e, [p])[0, 2 * (i - 1): 2 * i]
        assert np.allclose(r, [np.cos(p * theta), np.sin(p * theta)], rtol=0, atol=1e-12)


def test_two_keys_softmax_by_hand():
    """Head 0 only: x = e_0, q = 8 x (rotated to position 2), cached key 0 = 3 q/8
    and key 1 = 0, the new row's own key rope(x, 2): scores 24, 0 and 8, divided
    by sqrt(128); head 0's output is the softmax-weighted mix of the values
    written by hand."""
    L = 2
    x = np.zeros((1, H))
    x[0, 0] = 1.0
    xb = _bits(x)
    cache = np.zeros((1, 2, 4, H), dtype=np.uint16)
    qdir = rope(x, [L])[0]  # (cos 2, sin 2) on pair 0
    cache[0, 0, 0] = _bits(3.0 * qdir)
    v0, v1 = np.zeros(H), np.zeros(H)
    v0[:HEAD_DIM], v1[:HEAD_DIM] = 1.0, -1.0
    cache[0, 1, 0], cache[0, 1, 1] = _bits(v0), _bits(v1)
    wqkv = _eye_qkv(8.0)
    _, new_cache, mid = attn_verify(xb, wqkv, _bits(np.eye(H)), cache, [L], 0)
    s = np.array([24.0, 0.0, 8.0]) / np.sqrt(128.0)
    w = np.exp(s - s.max())
    w /= w.sum()
    vs = np.stack([v0, v1, oracle.widen(new_cache[0, 1, 2])])[:, :HEAD_DIM]
    want = w @ vs
    assert np.allclose(oracle.widen(mid["o"][0, :HEAD_DIM]), want, rtol=2 ** -7, atol=2 ** -9)
