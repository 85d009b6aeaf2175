"""Pins for the oracle's router, top-k and permutation (CPU only)."""
import ctypes
import ctypes.util

import numpy as np
import pytest

import oracle
import synth_inputs as si


def _random_bf16_bits(g, n, exp_lo=1, exp_hi=160, zero_frac=0.05, sub_frac=0.05):
    """bf16 bit patterns with exponent fields spread over [exp_lo, exp_hi],
    plus zeros and subnormals, random signs; no inf/nan."""
    sign = g.integers(0, 2, n).astype(np.uint16) << 15
    expo = g.integers(exp_lo, exp_hi + 1, n).astype(np.uint16)
    mant = g.integers(0, 128, n).astype(np.uint16)
    r = g.random(n)
    expo = np.where(r < zero_frac + sub_frac, 0, expo).astype(np.uint16)
    mant = np.where(r < zero_frac, 0, mant).astype(np.uint16)
    return (sign | (expo << 7) | mant).astype(np.uint16)


def test_bf16_rounding_matches_independent_fp32_path():
    g = np.random.default_rng(1)
    a = (g.standard_normal(20000) * np.exp(g.uniform(-60, 60, 20000))).astype(np.float32)
    # exact ties and near-ties around 1
    ties = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -20, -(1 + 2 ** -8), 2 ** -130, 3 * 2 ** -134], dtype=np.float32)
    a = np.concatenate([a, ties])
    assert np.array_equal(oracle.round_bf16_bits(a.astype(np.float64)), si.f32_to_bf16_bits(a))
    # hand values
    assert oracle.round_bf16_bits(np.array([1.0]))[0] == 0x3F80
    assert oracle.round_bf16_bits(np.array([1 + 2 ** -8]))[0] == 0x3F80          # tie -> even
    assert oracle.round_bf16_bits(np.array([1 + 3 * 2 ** -8]))[0] == 0x3F82      # tie -> even (up)
    assert oracle.round_bf16_bits(np.array([1 + 2 ** -8 + 2 ** -40]))[0] == 0x3F81  # above the tie (fp64 only)


def test_router_logits_match_libm_fmaf_chain():
    """The fp64 emulation of the fp32 fma chain equals C's fmaf, term by term,
    on inputs whose exponents span subnormals to 2^33 (exercises the
    inexact-in-fp64 branch of the argument in router_logits)."""
    libm = ctypes.CDLL(ctypes.util.find_library("m"))
    libm.fmaf.restype = ctypes.c_float
    libm.fmaf.argtypes = [ctypes.c_float, ctypes.c_float, ctypes.c_float]
    g = np.random.default_rng(7)
    T, E, H = 3, 5, 61
    xb = _random_bf16_bits(g, T * H).reshape(T, H)
    wb = _random_bf16_bits(g, E * H).reshape(E, H)
    # the last token/expert pair is tiny: its products fall in fp32's subnormal
    # range, where a rounded product followed by an add differs from fma
    xb[-1] = _random_bf16_bits(g, H, exp_lo=50, exp_hi=64, zero_frac=0, sub_frac=0)
    wb[-1] = _random_bf16_bits(g, H, exp_lo=50, exp_hi=64, zero_frac=0, sub_frac=0)
    bias = g.standard_normal(E).astype(np.float32)
    bias[-1] = 0.0
    got = oracle.router_logits(xb, wb, bias)
    xf = si.bf16_bits_to_f32(xb)
    wf = si.bf16_bits_to_f32(wb)
    f32 = np.float32
    for t in range(T):
        for e in range(E):
            q = []
            for h0, h1 in [(0, 15), (15, 30), (30, 45), (45, 61)]:  # quarters of 61, floor(q*61/4)
                acc = 0.0
                for h in range(h0, h1):
                    acc = libm.fmaf(float(xf[t, h]), float(wf[e, h]), acc)
                q.append(f32(acc))
            want = f32(f32(f32(q[0] + q[1]) + f32(q[2] + q[3])) + bias[e])
            assert np.float32(got[t, e]).view(np.uint32) == want.view(np.uint32), (t, e)


def test_router_logits_fma_at_a_double_rounding_boundary():
    """A hand-made case where fma and a rounded product followed by an add
    disagree: acc = 2^-125 after the first term, then the product
    1.5 * (255/256) * 2^-149 lies just below 1.5 units of 2^-149. Rounded on its
    own it becomes 1 unit, and acc + 1 unit is a tie that rounds back to 2^-125;
    fma rounds the exact sum up to 2^-125 + 2^-148."""
    f = np.array
    # H = 8: both terms sit in the first quarter (h = 0, 1); the rest are zero
    x = si.f32_to_bf16_bits(f([[2.0 ** -62, 1.5 * 2.0 ** -75] + [0.0] * 6], dtype=np.float32))
    w = si.f32_to_bf16_bits(f([[2.0 ** -63, (255 / 256) * 2.0 ** -74] + [0.0] * 6], dtype=np.float32))
    got = oracle.router_logits(x, w)[0, 0]
    assert got == np.float32(2.0 ** -125 + 2.0 ** -148)
    libm = ctypes.CDLL(ctypes.util.find_library("m"))
    libm.fmaf.restype = ctypes.c_float
    libm.fmaf.argtypes = [ctypes.c_float, ctypes.c_float, ctypes.c_float]
    acc = libm.fmaf(2.0 ** -62, 2.0 ** -63, 0.0)
    assert np.float32(libm.fmaf(1.5 * 2.0 ** -75, (255 / 256) * 2.0 ** -74, acc)) == got


def test_router_summation_order_is_the_quarter_tree():
    """A case that separates the quarter tree from one sequential chain (H = 8,
    quarters {0,1} {2,3} {4,5} {6,7}): with x = [2^-30, 0, 0, 0, 1, 0, -1, 0]
    and w = 1, the tree gives (2^-30 + 0) + (1 + -1) = 2^-30, while a single
    chain absorbs 2^-30 into 1 and ends at 0."""
    H = 8
    tiny = 2.0 ** -30
    x = si.f32_to_bf16_bits(np.array([[tiny, 0, 0, 0, 1.0, 0, -1.0, 0]], dtype=np.float32))
    w = si.f32_to_bf16_bits(np.ones((1, H), dtype=np.float32))
    assert oracle.router_logits(x, w)[0, 0] == np.float32(tiny)
    assert oracle.segment_bounds(1280) == [(0, 320), (320, 640), (640, 960), (960, 1280)]
    assert oracle.segment_bounds(61) == [(0, 15), (15, 30), (30, 45), (45, 61)]


def test_topk_matches_bruteforce_with_ties():
    g = np.random.default_rng(3)
    for E, k in [(8, 2), (16, 6), (64, 6)]:
        # logits drawn from a small set so that ties are frequent
        l = g.choice(np.array([-1.5, -0.25, 0.0, 0.5, 2.0], dtype=np.float32), size=(40, E))
        idx, gates = oracle.route(l, k)
        for t in range(l.shape[0]):
            want = sorted(range(E), key=lambda e: (-float(l[t, e]), e))[:k]
            assert list(idx[t]) == want
        p = oracle.softmax_gates(l)
        assert np.allclose(p.sum(axis=1), 1.0)
        assert np.allclose(gates, np.take_along_axis(p, idx.astype(np.int64), axis=1))


def test_router_zero_weights_closed_form():
    d = si.Dims(H=64, I=8, E=64, S=2, k=6, V=32)
    x = si.hidden_states(0, 0, 5, d.H)
    w = np.zeros((d.E, d.H), dtype=np.uint16)
    l = oracle.router_logits(x, w)
    assert np.all(l == 0)
    idx, gates = oracle.route(l, d.k)
    assert np.array_equal(idx, np.tile(np.arange(6, dtype=np.int32), (5, 1)))
    assert np.allclose(gates, 1 / 64)
    assert np.allclose(gates.sum(axis=1), 6 / 64)


def test_route_invariants_random():
    d = si.Dims(H=128, I=8, E=64, S=2, k=6, V=32)
    x = si.hidden_states(0, 9, 50, d.H)
    w = si.normal_bf16(si.rng(0, 9, 1), (d.E, d.H), 0.02)
    l = oracle.router_logits(x, w)
    idx, gates = oracle.route(l, d.k)
    for t in range(50):
        assert len(set(idx[t].tolist())) == 6
        assert np.all(np.diff(l[t, idx[t]]) <= 0)
        outside = np.setdiff1d(np.arange(64), idx[t])
        assert l[t, idx[t]].min() >= l[t, outside].max()
    assert np.all(np.diff(gates, axis=1) <= 0)
    assert np.all(gates.sum(axis=1) < 1)


def test_bias_added_in_fp32_after_the_chain():
    d = si.Dims(H=32, I=8, E=8, S=1, k=2, V=16)
    x = si.hidden_states(1, 2, 4, d.H)
    w = si.normal_bf16(si.rng(1, 2, 1), (d.E, d.H), 0.02)
    b = si.zipf_router_bias(d.E)
    assert np.allclose(b, [-2 * np.log(e + 1) for e in range(d.E)], atol=1e-6)
    assert np.array_equal(oracle.router_logits(x, w, b), (oracle.router_logits(x, w) + b).astype(np.float32))


def test_permutation_invariants():
    g = np.random.default_rng(5)
    for T, E, k in [(1, 8, 2), (37, 64, 6), (500, 64, 6)]:
        idx = np.stack([g.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
        counts, offsets, perm, inv = oracle.expert_permutation(idx, E)
        N = T * k
        assert counts.sum() == N and offsets[0] == 0 and offsets[-1] == N
        assert np.array_equal(np.sort(perm), np.arange(N))          # bijection
        assert np.array_equal(perm[inv], np.arange(N))              # inv o perm = id
        keys = idx.reshape(-1)[perm]
        assert np.all(np.diff(keys) >= 0)                           # grouped by expert
        for e in range(E):
            seg = perm[offsets[e]:offsets[e + 1]]
            assert np.all(keys[offsets[e]:offsets[e + 1]] == e)
            assert np.all(np.diff(seg) > 0)                         # stable
