"""GPU parity of the single-launch verify step for a handful of rows
(vg_verify_step_small: the MoE layers, the LM-head argmax and the accept in one
kernel) against the CPU oracle, stage by stage on the kernel's own states:
every layer's routed experts bit-exact and its output x + MoE(x) within
ACT_TOL of the oracle on the same layer input; the argmax equal to the
oracle's on the final states (certified near-ties excepted); accepted lengths
and committed tokens equal to the prefix accept of that argmax."""
import numpy as np
import pytest
import torch

import greedy_speculative_verify_b200 as vgv
import oracle
import synth_inputs as si
from gpu_common import ACT_TOL, D, Guarded, assert_device_ok, check_argmax, dev, ensure_lib, f32, row_rel_err

pytestmark = pytest.mark.gpu

L = 12


@pytest.fixture(scope="module")
def stack():
    ensure_lib()
    layers_dev = [si.torch_layer_weights(0, 2, l, D) for l in range(L)]
    layers = [{k: si.torch_to_bits(v) for k, v in lw.items()} for lw in layers_dev]
    lm_bits = si.lm_head(0, 2, D.V, D.H)
    return layers_dev, layers, lm_bits, dev(lm_bits)


def _run(layers_dev, n_layers, B, K, x_bits, lm_t, V, drafts, bias=None):
    T = B * (K + 1)
    cuda = torch.device("cuda")
    gd = Guarded()
    am = gd.empty((T,), torch.int32, fill=-7)
    acc = gd.empty((B,), torch.int32, fill=-7)
    ot = gd.empty((B, K + 1), torch.int32, fill=-7)
    states = gd.empty((n_layers + 1, T, D.H), torch.bfloat16)
    idx = gd.empty((n_layers, T, D.k), torch.int32, fill=-1)
    ws = gd.empty((vgv.vg_verify_step_small_workspace_bytes(),), torch.uint8)
    d = torch.from_numpy(np.ascontiguousarray(drafts, dtype=np.int32)).to(cuda) if K > 0 else None
    rb = None if bias is None else [bias] * n_layers
    vgv.vg_verify_step_small(vgv.MOE_DIMS, n_layers, B, K, dev(x_bits), [l["router_w"] for l in layers_dev[:n_layers]],
                             rb, [l["expert_w"] for l in layers_dev[:n_layers]],
                             [l["shared_w"] for l in layers_dev[:n_layers]], lm_t, V, d, am, acc, ot, ws,
                             states_out=states, topk_idx_out=idx)
    torch.cuda.synchronize()
    assert_device_ok()
    gd.check()
    return (am.cpu().numpy(), acc.cpu().numpy(), ot.cpu().numpy(), si.torch_to_bits(states), idx.cpu().numpy())


def _check_stages(layers, n_layers, x_bits, states, idx, bias=None):
    assert np.array_equal(states[0], x_bits)
    for l in range(n_layers):
        r = oracle.moe_ffn(states[l], layers[l]["router_w"], layers[l]["expert_w"], layers[l]["shared_w"], k=D.k,
                           I=D.I, bias=bias, add_residual=False)
        assert np.array_equal(idx[l], r["idx"]), l
        assert row_rel_err(f32(states[l + 1]), f32(states[l]) + r["out"]) <= ACT_TOL, l


@pytest.mark.parametrize("B,K", [(1, 3), (1, 1), (4, 3), (2, 2), (3, 0)])
def test_small_step_matches_oracle(stack, B, K):
    """(1,3) and (1,1): the batch-1 verify at K = 3 and K = 1; (4,3): 16 rows,
    the largest size; (2,2): 6 ragged rows; (3,0): plain greedy."""
    layers_dev, layers, lm_bits, lm_t = stack
    T = B * (K + 1)
    x = si.hidden_states(0, 2, T, D.H, tensor_id=400 + T)
    # drafts from the oracle's argmax of a reference pass, p = 0.576
    ref_h, _ = oracle.moe_stack(x, layers, k=D.k, I=D.I)
    ref_arg, _ = oracle.lm_head_argmax(ref_h, lm_bits)
    drafts = si.drafts_from_argmax(ref_arg, B, K, 0.576, D.V, seed=0, cfg=2) if K > 0 else None
    am, acc, ot, states, idx = _run(layers_dev, L, B, K, x, lm_t, D.V, drafts)
    _check_stages(layers, L, x, states, idx)
    own_arg, _ = oracle.lm_head_argmax(states[L], lm_bits)
    check_argmax(am, own_arg, states[L], lm_bits)
    a2, o2 = oracle.prefix_accept(am, drafts if K > 0 else np.zeros((B, 0), np.int32), B, K)
    assert np.array_equal(acc, a2) and np.array_equal(ot, o2)


def test_small_step_repeatable_and_equal_to_layer_calls_routing(stack):
    """Two calls give identical bytes (the split-K pieces are summed in k
    order whatever their timing), and each layer's routing equals that of the
    multi-kernel stack path on the same layer input."""
    layers_dev, layers, lm_bits, lm_t = stack
    B, K = 1, 3
    x = si.hidden_states(0, 2, 4, D.H, tensor_id=450)
    drafts = np.zeros((B, K), np.int32)
    r1 = _run(layers_dev, L, B, K, x, lm_t, D.V, drafts)
    r2 = _run(layers_dev, L, B, K, x, lm_t, D.V, drafts)
    for a_, b_ in zip(r1, r2):
        assert np.array_equal(a_, b_)
    states, idx = r1[3], r1[4]
    cuda = torch.device("cuda")
    for l in range(L):
        tidx = torch.full((4, D.k), -1, dtype=torch.int32, device=cuda)
        out = torch.empty(4, D.H, dtype=torch.bfloat16, device=cuda)
        ws = torch.empty(vgv.vg_moe_workspace_bytes(vgv.MOE_DIMS, 4), dtype=torch.uint8, device=cuda)
        lw = layers_dev[l]
        vgv.vg_moe_ffn(vgv.MOE_DIMS, 4, dev(states[l]), lw["router_w"], None, lw["expert_w"], lw["shared_w"], 1, out,
                       vgv.make_taps(topk_idx=tidx), ws)
        torch.cuda.synchronize()
        assert np.array_equal(tidx.cpu().numpy(), idx[l]), l


def test_small_step_router_bias_and_small_vocabulary(stack):
    """Two layers with the per-expert bias 2 ln(1/(e+1)) (few experts touched),
    a 1,000-token vocabulary (not a multiple of the 128-row units)."""
    layers_dev, layers, lm_bits, _ = stack
    B, K, V = 2, 3, 1000
    T = B * (K + 1)
    bias_np = si.zipf_router_bias(D.E)
    bias = torch.from_numpy(bias_np).to("cuda")
    lm_small = lm_bits[:V].copy()
    x = si.hidden_states(0, 2, T, D.H, tensor_id=460)
    drafts = np.random.default_rng(7).integers(0, V, (B, K)).astype(np.int32)
    am, acc, ot, states, idx = _run(layers_dev, 2, B, K, x, dev(lm_small), V, drafts, bias=bias)
    _check_stages(layers, 2, x, states, idx, bias=bias_np)
    own_arg, _ = oracle.lm_head_argmax(states[2], lm_small)
    check_argmax(am, own_arg, states[2], lm_small)
    assert np.all((am >= 0) & (am < V))
    a2, o2 = oracle.prefix_accept(am, drafts, B, K)
    assert np.array_equal(acc, a2) and np.array_equal(ot, o2)
