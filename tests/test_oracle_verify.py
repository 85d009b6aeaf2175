"""Pins for the oracle's LM-head argmax, prefix accept, metrics and the lossless
property (CPU only)."""
import json
import math
import os
import struct

import numpy as np
import pytest

import oracle
import synth_inputs as si

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _fp32(v: float) -> float:
    return struct.unpack("f", struct.pack("f", v))[0]


def test_argmax_bruteforce_exact_sums():
    """Tiny vocabulary: exact sums by math.fsum, one rounding to fp32, first
    maximum — against the chunked fp64 matmul of the oracle."""
    g = np.random.default_rng(11)
    V, H, R = 53, 24, 9
    lm = si.normal_bf16(g, (V, H), 0.02)
    hid = si.normal_bf16(g, (R, H), 1.0)
    lm[17] = lm[5]  # duplicate row: an exact tie, resolved to the lower index
    hid[0] = si.f32_to_bf16_bits(si.bf16_bits_to_f32(lm[5]) * 50)  # row 0 prefers rows 5 and 17
    arg, best = oracle.lm_head_argmax(hid, lm, chunk=7)
    hf, lf = si.bf16_bits_to_f32(hid).astype(float), si.bf16_bits_to_f32(lm).astype(float)
    for r in range(R):
        z = [_fp32(math.fsum(hf[r] * lf[v])) for v in range(V)]
        m = max(z)
        assert arg[r] == z.index(m)
        assert best[r] == np.float32(m)
    assert arg[0] == 5


def test_argmax_chunking_invariant_and_one_hot():
    g = np.random.default_rng(12)
    V, H = 300, 16
    lm = si.normal_bf16(g, (V, H), 0.02)
    hid = si.normal_bf16(g, (20, H), 1.0)
    a1, _ = oracle.lm_head_argmax(hid, lm, chunk=1)
    a2, _ = oracle.lm_head_argmax(hid, lm, chunk=8192)
    assert np.array_equal(a1, a2)
    # one-hot closed form: LM[v] = (v+1)/1024 * e_{v mod H} (exact in bf16 for
    # v < 256); hid = e_h -> the largest v with v mod H == h wins
    V1 = 200
    lm1 = np.zeros((V1, H), dtype=np.float32)
    for v in range(V1):
        lm1[v, v % H] = (v + 1) / 1024
    eye = np.eye(H, dtype=np.float32)
    a3, b3 = oracle.lm_head_argmax(si.f32_to_bf16_bits(eye), si.f32_to_bf16_bits(lm1))
    for h in range(H):
        want = max(v for v in range(V1) if v % H == h)
        assert a3[h] == want and b3[h] == np.float32((want + 1) / 1024)


def test_prefix_accept_closed_forms():
    K, B = 3, 5
    arg = np.arange(B * (K + 1)).reshape(B, K + 1) + 100
    d = np.zeros((B, K), dtype=np.int64)
    d[0] = arg[0, :K]                         # all correct -> a = K, K+1 tokens
    d[1] = [-7, arg[1, 1], arg[1, 2]]         # first wrong -> a = 0 even if later ones agree
    d[2] = [arg[2, 0], 10 ** 9, arg[2, 2]]    # second wrong (out of range) -> a = 1
    d[3] = [arg[3, 0], arg[3, 1], -1]         # last wrong -> a = 2
    d[4] = [arg[4, 1], arg[4, 2], arg[4, 3]]  # shifted by one position -> a = 0
    acc, out = oracle.prefix_accept(arg.ravel(), d, B, K)
    assert acc.tolist() == [3, 0, 1, 2, 0]
    assert out[0].tolist() == arg[0].tolist()
    assert out[1].tolist() == [arg[1, 0], -1, -1, -1]
    assert out[2].tolist() == [arg[2, 0], arg[2, 1], -1, -1]
    assert out[3].tolist() == [arg[3, 0], arg[3, 1], arg[3, 2], -1]
    assert out[4].tolist() == [arg[4, 0], -1, -1, -1]
    # K = 0 is plain greedy: nothing drafted, the verifier's token is committed
    acc0, out0 = oracle.prefix_accept(np.array([42, 43]), np.zeros((2, 0), dtype=np.int64), 2, 0)
    assert acc0.tolist() == [0, 0] and out0.tolist() == [[42], [43]]


@pytest.mark.parametrize("K,p", [(3, 0.576), (1, 0.576), (3, 0.751)])
def test_accept_length_statistics(K, p):
    """Drafts equal to the argmax with probability p, independently per
    position: P(a >= j) = p^j, so E[tau] = sum_{j=0..K} p^j."""
    B, V = 20000, 129280
    g = np.random.default_rng(K)
    arg = g.integers(0, V, B * (K + 1))
    d = si.drafts_from_argmax(arg, B, K, p, V, seed=0, cfg=K)
    acc, _ = oracle.prefix_accept(arg, d, B, K)
    want = sum(p ** j for j in range(K + 1))
    sd = np.std(acc + 1) / math.sqrt(B)
    assert abs(oracle.tau(acc) - want) < 4 * sd
    hist = np.bincount(acc, minlength=K + 1) / B
    for j in range(K):
        assert abs(hist[j] - p ** j * (1 - p)) < 0.02


def test_pages_speculative_numbers_pin_the_metric_definitions():
    """tests/golden/l4_speculative.json holds the L4 figures the pages print.
    They fix acceptance rate = (tau - 1)/K (not a/(K+1) or tau/(K+1)) and the
    relation speed-up S = tau / c."""
    with open(os.path.join(GOLDEN, "l4_speculative.json")) as f:
        gold = json.load(f)
    K, tau_pg, acc_pg = gold["K"], gold["tau_eager"], gold["acceptance_rate"]
    # a run of 1000 steps with 1728 accepted drafts prints as tau 2.73 and 57.6%
    acc = np.array([2] * 728 + [1] * 272, dtype=np.int64)
    assert acc.sum() == 1728
    assert round(oracle.tau(acc), 2) == tau_pg
    assert round(oracle.acceptance_rate(acc, K) * 100, 1) == acc_pg
    # the two printed figures are consistent under (tau-1)/K within their rounding
    lo, hi = (tau_pg - 0.005 - 1) / K, (tau_pg + 0.005 - 1) / K
    assert lo <= acc_pg / 100 + 0.0005 and acc_pg / 100 - 0.0005 <= hi
    assert not (abs(tau_pg / (K + 1) - acc_pg / 100) < 0.01)
    S = gold["spec_tok_s_eager"] / gold["ar_tok_s_eager"]
    assert round(S, 2) == gold["speedup_eager"]
    assert round(tau_pg / S, 2) == gold["cost_eager"]
    # under CUDA graphs K=3 would give AR * tau / c below the K=1 figure
    k3_graphs = gold["ar_tok_s_graphs"] * gold["tau_graphs"] / gold["cost_graphs"]
    assert k3_graphs < gold["k1_tok_s_graphs"]
    # per-step overhead (c - 1) / AR rate, both modes near the printed ~9 ms
    for c, ar in [(gold["cost_eager"], gold["ar_tok_s_eager"]), (gold["cost_graphs"], gold["ar_tok_s_graphs"])]:
        assert abs((c - 1) / ar * 1000 - gold["overhead_ms"]) < 0.6


def test_lossless_speculative_equals_greedy():
    """Token identity of draft-and-verify decoding with plain greedy decoding on
    a synthetic Markov decoder, for several depths and draft qualities."""
    d = si.Dims(H=32, I=16, E=8, S=1, k=2, V=61)
    layers = [si.layer_weights(0, 60, l, d, std=0.1) for l in range(2)]
    dec = oracle.MarkovDecoder(emb=si.normal_bf16(si.rng(0, 60, 9), (d.V, d.H), 1.0), layers=layers,
                               lm=si.normal_bf16(si.rng(0, 60, 10), (d.V, d.H), 0.1), k=d.k, I=d.I)
    n = 40
    ref = oracle.greedy_decode(dec, start=3, n=n)
    assert len(set(ref)) > 1
    for K, p in [(3, 0.7), (1, 0.5), (3, 0.0), (4, 1.0), (0, 0.0)]:
        got, steps = oracle.speculative_decode(dec, start=3, n=n, K=K, p=p, seed=K)
        assert got == ref, (K, p)
        if p == 1.0:
            assert all(a == K for a in steps)
        if p == 0.0 and K > 0:
            assert sum(steps) <= 2  # a uniform draft matches only by chance
