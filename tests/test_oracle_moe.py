"""Pins for the oracle's expert math and MoE layer (CPU only)."""
import math

import numpy as np

import oracle
import synth_inputs as si


def _bits(a):
    return si.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def _expert_block(gate, up, down):
    return np.concatenate([_bits(gate).ravel(), _bits(up).ravel(), _bits(down).ravel()])


def test_swiglu_hand_values():
    """H=2, I=3 worked by hand: gate x = [1,2,3], up x = [3,2,2],
    y = [silu(1)*3, silu(2)*2 + silu(3)*2]. A transposed matrix or silu on the
    wrong branch changes the result."""
    gate = [[1, 0], [0, 1], [1, 1]]
    up = [[1, 1], [2, 0], [0, 1]]
    down = [[1, 0, 0], [0, 1, 1]]
    x = np.array([[1.0, 2.0]])
    s = lambda z: z / (1 + math.exp(-z))
    want = np.array([[s(1) * 3, s(2) * 2 + s(3) * 2]])
    got = oracle.swiglu_expert(x, _expert_block(gate, up, down), I=3, H=2)
    assert np.allclose(got, want, rtol=1e-15, atol=0)
    # a single number: x=2, gate=1, up=3, down=0.5 -> 0.5 * silu(2) * 6
    got1 = oracle.swiglu_expert(np.array([[2.0]]), _expert_block([[1]], [[3]], [[0.5]]), I=1, H=1)
    assert math.isclose(got1[0, 0], 3 * 2 / (1 + math.exp(-2)), rel_tol=1e-15)


def test_silu_special_values():
    z = np.array([0.0, -1e4, 1e4, 1.0])
    s = oracle.silu(z)
    assert s[0] == 0 and s[1] == 0 and s[2] == 1e4
    assert math.isclose(s[3], 1 / (1 + math.exp(-1)))


def _layer(d, seed=0, cfg=50, layer=0):
    return si.layer_weights(seed, cfg, layer, d)


def test_identical_experts_reduce_to_scaled_dense_ffn():
    """With every routed expert equal to W and the shared weights zero,
    y = (sum_j g_j) * SwiGLU_W(x); with shared weights present y gains
    sum_s Shared_s(x)."""
    d = si.Dims(H=32, I=16, E=8, S=2, k=3, V=16)
    lw = _layer(d)
    same = np.tile(lw["expert_w"][3:4], (d.E, 1))
    x = si.hidden_states(0, 50, 11, d.H)
    xf = oracle.widen(x)
    dense = oracle.swiglu_expert(xf, same[0], d.I, d.H)
    r0 = oracle.moe_ffn(x, lw["router_w"], same, np.zeros_like(lw["shared_w"]), k=d.k, I=d.I, add_residual=False)
    gsum = r0["g"].sum(axis=1, keepdims=True)
    assert np.all(gsum < 1)
    assert np.allclose(r0["out"], gsum * dense, rtol=1e-12, atol=1e-12)
    r1 = oracle.moe_ffn(x, lw["router_w"], same, lw["shared_w"], k=d.k, I=d.I, add_residual=False)
    sh = sum(oracle.swiglu_expert(xf, lw["shared_w"][s], d.I, d.H) for s in range(d.S))
    assert np.allclose(r1["out"], gsum * dense + sh, rtol=1e-12, atol=1e-12)


def test_two_shared_experts_equal_one_of_double_width():
    d = si.Dims(H=24, I=8, E=4, S=2, k=2, V=16)
    lw = _layer(d, cfg=51)
    I, H = d.I, d.H
    sw = lw["shared_w"]
    g0, u0, d0 = sw[0][:I * H].reshape(I, H), sw[0][I * H:2 * I * H].reshape(I, H), sw[0][2 * I * H:].reshape(H, I)
    g1, u1, d1 = sw[1][:I * H].reshape(I, H), sw[1][I * H:2 * I * H].reshape(I, H), sw[1][2 * I * H:].reshape(H, I)
    wide = np.concatenate([np.concatenate([g0, g1]).ravel(), np.concatenate([u0, u1]).ravel(), np.concatenate([d0, d1], axis=1).ravel()])
    x = si.hidden_states(0, 51, 9, H)
    r = oracle.moe_ffn(x, lw["router_w"], lw["expert_w"], sw, k=d.k, I=I, add_residual=False)
    one = oracle.swiglu_expert(oracle.widen(x), wide, 2 * I, H)
    assert np.allclose(r["shared_out"].sum(axis=0), one, rtol=1e-12, atol=1e-12)


def test_residual_and_intermediates_consistent():
    d = si.Dims(H=32, I=16, E=8, S=1, k=2, V=16)
    lw = _layer(d, cfg=52)
    x = si.hidden_states(0, 52, 13, d.H)
    r = oracle.moe_ffn(x, lw["router_w"], lw["expert_w"], lw["shared_w"], k=d.k, I=d.I, add_residual=True)
    y = oracle.moe_ffn(x, lw["router_w"], lw["expert_w"], lw["shared_w"], k=d.k, I=d.I, add_residual=False)["out"]
    assert np.allclose(r["out"], oracle.widen(x) + y, rtol=1e-14, atol=1e-14)
    # every routed row of expert_out is its expert applied to its token
    xf = oracle.widen(x)
    for p in range(d.k * 13):
        a = r["perm"][p]
        t, j = a // d.k, a % d.k
        e = r["idx"][t, j]
        assert np.allclose(r["expert_out"][p], oracle.swiglu_expert(xf[t:t + 1], lw["expert_w"][e], d.I, d.H)[0], rtol=1e-12, atol=1e-13)
    # y recomposes from its parts
    rec = sum(r["g"][:, j:j + 1] * r["expert_out"][r["inv"].reshape(13, d.k)[:, j]] for j in range(d.k)) + r["shared_out"].sum(axis=0)
    assert np.allclose(rec, y, rtol=1e-12, atol=1e-13)


def test_stack_rounds_to_bf16_between_layers():
    d = si.Dims(H=32, I=16, E=8, S=1, k=2, V=16)
    layers = [si.layer_weights(0, 53, l, d) for l in range(3)]
    x = si.hidden_states(0, 53, 6, d.H)
    out, res = oracle.moe_stack(x, layers, k=d.k, I=d.I)
    cur = x
    for l in range(3):
        r = oracle.moe_ffn(cur, **{kk: layers[l][kk] for kk in ("router_w", "expert_w", "shared_w")}, k=d.k, I=d.I)
        cur = oracle.round_bf16_bits(r["out"])
    assert np.array_equal(out, cur)
