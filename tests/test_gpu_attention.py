"""Verifier attention over a KV cache on the GPU against the oracle
(oracle/attention.py): outputs, the rows written to the cache, the positions
left alone, and the bounds check on the cache length."""
import numpy as np
import pytest
import torch

import greedy_speculative_verify_b200 as vgv
import oracle
import synth_inputs as si

from gpu_common import ACT_TOL, D, dev, ensure_lib, row_rel_err

pytestmark = pytest.mark.gpu
H = D.H


@pytest.fixture(scope="module")
def weights():
    ensure_lib()
    g = np.random.default_rng(17)
    wqkv = oracle.round_bf16_bits(g.normal(0, 0.02, (3 * H, H)))
    wo = oracle.round_bf16_bits(g.normal(0, 0.05, (H, H)))
    return wqkv, wo


def _run(weights, B, K, lens, L_max, seed):
    wqkv, wo = weights
    g = np.random.default_rng(seed)
    x = oracle.round_bf16_bits(g.normal(0, 1, (B * (K + 1), H)))
    cache = np.zeros((B, 2, L_max, H), dtype=np.uint16)
    for b, L in enumerate(lens):
        cache[b, :, :L] = oracle.round_bf16_bits(g.normal(0, 0.7, (2, L, H)))
    cache_d = dev(cache)
    out = torch.empty(B * (K + 1), H, dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(out)
    ws = torch.empty(vgv.vg_attn_workspace_bytes(B, K, L_max), dtype=torch.uint8, device="cuda")
    lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
    vgv.vg_attn_verify(B, K, dev(x), dev(wqkv), dev(wo), cache_d, lens_d, out, ws, o_out=o)
    torch.cuda.synchronize()
    return x, cache, si.torch_to_bits(out), si.torch_to_bits(cache_d), si.torch_to_bits(o)


@pytest.mark.parametrize("B,K,lens", [(2, 3, [0, 5]), (4, 0, [300, 17, 0, 1000]), (3, 7, [255, 256, 1]),
                                      (2, 3, [2044, 777])])
def test_attention_matches_oracle(weights, B, K, lens):
    L_max = max(lens) + K + 1 + 3
    x, cache, out, new_cache, o = _run(weights, B, K, lens, L_max, seed=B * 100 + K)
    st, info = vgv.vg_get_device_status()
    assert st == 0, (st, info)
    ref_out, ref_cache, mid = oracle.attn_verify(x, weights[0], weights[1], cache, lens, K)
    assert row_rel_err(oracle.widen(out), oracle.widen(ref_out)) <= ACT_TOL
    assert row_rel_err(oracle.widen(o), oracle.widen(mid["o"])) <= ACT_TOL  # the heads' output itself
    for b, L in enumerate(lens):
        assert np.array_equal(new_cache[b, :, :L], cache[b, :, :L])                  # old positions untouched
        assert np.array_equal(new_cache[b, :, L + K + 1:], cache[b, :, L + K + 1:])  # nothing beyond the new rows
        for kv in (0, 1):  # the new rows, within rounding of the projection
            assert row_rel_err(oracle.widen(new_cache[b, kv, L: L + K + 1]),
                               oracle.widen(ref_cache[b, kv, L: L + K + 1])) <= ACT_TOL


def test_cache_overflow_is_reported_and_leaves_x(weights):
    B, K, L_max = 2, 3, 16
    x, cache, out, new_cache, o = _run(weights, B, K, [3, 13], L_max, seed=5)  # 13 + 4 > 16
    st, info = vgv.vg_get_device_status()  # reads and clears
    assert st == 6, (st, info)
    assert np.array_equal(out[4:], x[4:])            # o = 0 for the overflowing sequence: out = x
    assert np.array_equal(new_cache[1], cache[1])    # and its cache is not written


def test_attention_bench_shape(weights):
    """The bench's attention launch (B = 32, K = 3, caches of 2,048 + 4
    positions): every row against the oracle, half the sequences at the full
    2,048 cached positions, the others ragged below it."""
    B, K, L = 32, 3, 2048
    lens = [L if b % 2 == 0 else L - 1 - (97 * b) % L for b in range(B)]
    x, cache, out, new_cache, o = _run(weights, B, K, lens, L + K + 1, seed=2048)
    st, info = vgv.vg_get_device_status()
    assert st == 0, (st, info)
    ref_out, ref_cache, mid = oracle.attn_verify(x, weights[0], weights[1], cache, lens, K)
    assert row_rel_err(oracle.widen(o), oracle.widen(mid["o"])) <= ACT_TOL
    assert row_rel_err(oracle.widen(out), oracle.widen(ref_out)) <= ACT_TOL
    for b in (0, 1, B - 1):
        L_b = lens[b]
        assert np.array_equal(new_cache[b, :, :L_b], cache[b, :, :L_b])
        for kv in (0, 1):
            assert row_rel_err(oracle.widen(new_cache[b, kv, L_b: L_b + K + 1]),
                               oracle.widen(ref_cache[b, kv, L_b: L_b + K + 1])) <= ACT_TOL


def test_attention_longest_cache(weights):
    """The largest cache the call takes (L_max = 32,768 positions, the decoder's
    position limit) with the most new rows (K = 7): one sequence filling it to
    the last position, one nearly empty."""
    B, K, L_max = 2, 7, 32768
    lens = [L_max - K - 1, 5]
    x, cache, out, new_cache, o = _run(weights, B, K, lens, L_max, seed=32768)
    st, info = vgv.vg_get_device_status()
    assert st == 0, (st, info)
    ref_out, ref_cache, mid = oracle.attn_verify(x, weights[0], weights[1], cache, lens, K)
    assert row_rel_err(oracle.widen(o), oracle.widen(mid["o"])) <= ACT_TOL
    assert row_rel_err(oracle.widen(out), oracle.widen(ref_out)) <= ACT_TOL
    for b, L in enumerate(lens):
        for kv in (0, 1):
            assert row_rel_err(oracle.widen(new_cache[b, kv, L: L + K + 1]),
                               oracle.widen(ref_cache[b, kv, L: L + K + 1])) <= ACT_TOL
    assert np.array_equal(new_cache[0, :, :lens[0]], cache[0, :, :lens[0]])
