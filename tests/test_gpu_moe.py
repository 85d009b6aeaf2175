"""GPU parity of the MoE layer (vg_moe_ffn) against the CPU oracle.

Routing ids, expert offsets, permutation and its inverse are compared bit for
bit; activations, expert outputs and the layer output within ACT_TOL per row.
Sizes span one token to the 36,992-token prefill shape, ragged tails, both
router kernels and both grouping paths.
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from gpu_common import ACT_TOL, D, assert_device_ok, dev, ensure_lib, f32, row_rel_err, run_moe

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def layer():
    ensure_lib()
    return si.layer_weights(0, 1, 0, D)


def _compare(g, r, T, check_act=True):
    assert np.array_equal(g["idx"], r["idx"]), "routing ids differ"
    assert np.allclose(g["g"], r["g"], rtol=1e-5, atol=1e-8)
    assert np.array_equal(g["offsets"], r["offsets"])
    assert np.array_equal(g["perm"], r["perm"])
    assert np.array_equal(g["inv"], r["inv"])
    N = T * D.k
    if check_act:
        assert row_rel_err(g["act"][:N], r["act"]) <= ACT_TOL
        assert row_rel_err(g["expert_out"][:N], r["expert_out"]) <= ACT_TOL
        sa = g["act"][N:].reshape(D.S, T, D.I)
        so = g["expert_out"][N:].reshape(D.S, T, D.H)
        for s in range(D.S):
            assert row_rel_err(sa[s], r["shared_act"][s]) <= ACT_TOL
            assert row_rel_err(so[s], r["shared_out"][s]) <= ACT_TOL
    assert row_rel_err(g["out"], r["out"]) <= ACT_TOL


@pytest.mark.parametrize("T", [1, 2, 4, 16, 63, 64, 128, 200, 296, 297, 1100, 2000])
def test_layer_parity(layer, T):
    """T=16: the tiny verify shape; 128: one decode layer at B=32, K=3; 2 and
    4: batch-1 K=1 / K=3; up to 296 the two-token entry kernel (an odd T leaves
    one CTA a single token; 296 fills 148 CTAs); from 64 on the expert kernel's
    fixed first units (63 just below); 200: several token tiles per shared
    expert with a ragged tail; 297 and 1100: the entry kernel with several
    tokens per CTA; 2000: 12,000 assignments take the tiled router and the
    multi-kernel grouping path."""
    x = si.hidden_states(0, 1, T, D.H, tensor_id=100 + T)
    r = oracle.moe_ffn(x, layer["router_w"], layer["expert_w"], layer["shared_w"], k=D.k, I=D.I, add_residual=False)
    g = run_moe(x, layer, add_residual=False)
    _compare(g, r, T)
    g1 = run_moe(x, layer, add_residual=True)
    assert np.array_equal(g1["idx"], r["idx"])
    assert row_rel_err(g1["out"], f32(x) + r["out"]) <= ACT_TOL


def test_layer_skewed_routing(layer):
    """T=4096 with the per-expert bias 2 ln(1/(e+1)): expert 0 takes every token
    (32 token tiles), experts past ~30 take none."""
    T = 4096
    bias = si.zipf_router_bias(D.E)
    x = si.hidden_states(0, 4, T, D.H)
    r = oracle.moe_ffn(x, layer["router_w"], layer["expert_w"], layer["shared_w"], k=D.k, I=D.I, bias=bias,
                       add_residual=False)
    assert r["counts"][0] > 4000 and (r["counts"] == 0).sum() > 10
    g = run_moe(x, layer, bias=bias, add_residual=False)
    _compare(g, r, T)


@pytest.mark.parametrize("T", [64, 128, 295])
def test_decode_skewed_routing(layer, T):
    """Decode sizes with the per-expert bias 2 ln(1/(e+1)): most experts get no
    token, so the expert kernel's fixed first units of unused experts only
    release their pipeline stages, and their further units are skipped; at 128
    and 295 tokens some routed experts take more than one 64-token tile, whose
    further token rows follow the 64 x 64 rows of the fixed first tiles."""
    bias = si.zipf_router_bias(D.E)
    x = si.hidden_states(0, 9, T, D.H, tensor_id=300 + T)
    r = oracle.moe_ffn(x, layer["router_w"], layer["expert_w"], layer["shared_w"], k=D.k, I=D.I, bias=bias,
                       add_residual=False)
    assert (r["counts"] == 0).sum() > 20
    if T >= 128:
        assert (r["counts"] > 64).sum() >= 4
    g = run_moe(x, layer, bias=bias, add_residual=False)
    _compare(g, r, T)


def test_layer_prefill_sampled(layer):
    """The prefill shape, T = 32 pages x 1,156 visual tokens = 36,992, run in
    full on the GPU; the oracle recomputes 192 sampled tokens (every per-token
    quantity is independent of the other tokens), and the full-size grouping
    is checked as a stable sort of the routing ids."""
    T = 36992
    x = si.hidden_states(0, 3, T, D.H)
    g = run_moe(x, layer, add_residual=True)
    rng = np.random.default_rng(3)
    rows = np.sort(rng.choice(T, 192, replace=False))
    r = oracle.moe_ffn(x[rows], layer["router_w"], layer["expert_w"], layer["shared_w"], k=D.k, I=D.I,
                       add_residual=True)
    assert np.array_equal(g["idx"][rows], r["idx"])
    assert np.allclose(g["g"][rows], r["g"], rtol=1e-5, atol=1e-8)
    assert row_rel_err(g["out"][rows], r["out"]) <= ACT_TOL
    N = T * D.k
    for i, t in enumerate(rows):
        for j in range(D.k):
            p_g = g["inv"][t * D.k + j]
            p_r = r["inv"][i * D.k + j]
            assert row_rel_err(g["act"][p_g][None], r["act"][p_r][None]) <= ACT_TOL
            assert row_rel_err(g["expert_out"][p_g][None], r["expert_out"][p_r][None]) <= ACT_TOL
    # full-size grouping: a stable sort of the GPU's own routing ids
    keys = g["idx"].reshape(-1)
    assert np.array_equal(g["offsets"], np.concatenate([[0], np.cumsum(np.bincount(keys, minlength=D.E))]))
    assert np.array_equal(g["perm"], np.argsort(keys, kind="stable"))
    assert np.array_equal(g["perm"][g["inv"]], np.arange(N))


def test_zero_router_closed_form(layer):
    """Router weights zero: every logit is 0, so experts 0..5 are chosen with
    weight 1/64 each (six full segments of T rows); outputs match the oracle."""
    T = 64
    lw = dict(layer)
    lw["router_w"] = np.zeros_like(layer["router_w"])
    x = si.hidden_states(0, 5, T, D.H)
    g = run_moe(x, lw, add_residual=False)
    assert np.array_equal(g["idx"], np.tile(np.arange(6, dtype=np.int32), (T, 1)))
    assert np.allclose(g["g"], 1 / 64, rtol=1e-6)
    assert np.array_equal(g["offsets"][:7], np.arange(7) * T) and np.all(g["offsets"][7:] == 6 * T)
    r = oracle.moe_ffn(x, lw["router_w"], lw["expert_w"], lw["shared_w"], k=D.k, I=D.I, add_residual=False)
    assert row_rel_err(g["out"], r["out"]) <= ACT_TOL


def test_repeatable_and_batch_invariant(layer):
    """Two runs give identical bytes; a token's routing and output do not
    depend on the other tokens in the batch (T=1 alone vs inside T=128)."""
    x = si.hidden_states(0, 6, 128, D.H)
    a = run_moe(x, layer)
    b = run_moe(x, layer)
    for key in ("out", "idx", "g", "perm", "act", "expert_out"):
        assert np.array_equal(a[key], b[key]), key
    for t in (0, 77, 127):
        s = run_moe(x[t:t + 1], layer)
        assert np.array_equal(s["idx"][0], a["idx"][t])
        assert np.array_equal(s["out"][0], a["out"][t])


def test_t_zero_is_noop(layer):
    import greedy_speculative_verify_b200 as vgv

    out = torch.full((1, D.H), 3.0, dtype=torch.bfloat16, device="cuda")
    x = torch.zeros((1, D.H), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(vgv.vg_moe_workspace_bytes(vgv.MOE_DIMS, 1), dtype=torch.uint8, device="cuda")
    w = dev(layer["router_w"])
    vgv.vg_moe_ffn(vgv.MOE_DIMS, 0, x, w, None, w, w, 1, out, None, ws)
    torch.cuda.synchronize()
    assert torch.all(out == 3.0)
    assert_device_ok()
