"""The recursive draft block on the GPU against the oracle (oracle/mtp.py),
stage by stage on the GPU's own inputs, and inside the device decode loop,
where any drafter must leave the committed tokens equal to greedy decoding."""
import numpy as np
import pytest
import torch

import greedy_speculative_verify_b200 as vgv
import oracle
import synth_inputs as si

from gpu_common import ACT_TOL, D, check_argmax, dev, ensure_lib, row_rel_err
from test_gpu_decode import Decoder, V, _starts

pytestmark = pytest.mark.gpu


def _gammas(seed):
    g = np.random.default_rng(seed)
    return [(1.0 + 0.1 * g.standard_normal(D.H)).astype(np.float32) for _ in range(3)]


@pytest.fixture(scope="module")
def block():
    """Draft-block weights as bf16 bits (oracle) and device tensors (GPU)."""
    ensure_lib()
    cfg = 13
    proj = si.normal_bf16(si.rng(0, cfg, si.TID_EMB, 1), (D.H, 2 * D.H), 0.02)
    ffn = si.normal_bf16(si.rng(0, cfg, si.TID_EXPERTS, 1), (3 * D.I * D.H,), 0.02)
    emb = si.hidden_states(0, cfg, V, D.H, tensor_id=si.TID_EMB)
    lm = si.lm_head(0, cfg, V, D.H)
    gh, ge, gf = _gammas(7)
    bits = {"proj": proj, "ffn": ffn, "emb": emb, "lm": lm, "gamma_h": gh, "gamma_e": ge, "gamma_f": gf}
    t = {k: (dev(v) if v.dtype == np.uint16 else torch.from_numpy(v).cuda()) for k, v in bits.items()}
    w = vgv.make_mtp_weights(t["proj"], t["ffn"], t["gamma_h"], t["gamma_e"], t["gamma_f"], t["emb"], t["lm"])
    return bits, t, w


@pytest.mark.parametrize("B,K", [(5, 3), (32, 3), (2, 1), (130, 2)])
def test_draft_steps_match_oracle(block, B, K):
    bits, t, w = block
    R = K + 1
    h_bits = si.hidden_states(1, 13, B * R, D.H, tensor_id=si.TID_HID)
    rng = np.random.default_rng(B * 10 + K)
    acc = rng.integers(0, R, B).astype(np.int32)
    y0 = rng.integers(0, V, B).astype(np.int32)
    drafts = torch.empty(B, K, dtype=torch.int32, device="cuda")
    hid = torch.empty(K, B, D.H, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(vgv.vg_mtp_workspace_bytes(B, V), dtype=torch.uint8, device="cuda")
    vgv.vg_mtp_draft(B, K, w, dev(h_bits), R, torch.from_numpy(acc).cuda(), torch.from_numpy(y0).cuda(), drafts,
                     ws, hidden_out=hid)
    torch.cuda.synchronize()
    st, info = vgv.vg_get_device_status()
    assert st == 0, (st, info)
    gpu_y = drafts.cpu().numpy()
    gpu_g = si.torch_to_bits(hid)
    g_prev = h_bits[np.arange(B) * R + acc]
    y_prev = y0
    for i in range(K):
        g_ref, _, _ = oracle.mtp_step(g_prev, y_prev, bits, I=D.I)
        assert row_rel_err(oracle.widen(gpu_g[i]), oracle.widen(g_ref)) <= ACT_TOL, i
        # the draft is the argmax of the LM head at the GPU's own hidden state
        ref_y, _ = oracle.lm_head_argmax(gpu_g[i], bits["lm"])
        check_argmax(gpu_y[:, i], ref_y, gpu_g[i], bits["lm"])
        g_prev, y_prev = gpu_g[i], gpu_y[:, i]


def test_draft_block_in_the_decode_loop_is_lossless(block):
    """Greedy decoding vs speculative decoding whose drafts come from the draft
    block fed with each verify step's hidden state of the bonus row."""
    _, _, w = block
    decoder = Decoder(n_layers=2)
    B, K, N = 8, 3, 20
    starts = _starts(B, seed=8)
    greedy, _, _ = decoder.run(starts, 0, N + K + 1)
    spec, _, _ = decoder.run(starts, K, N, mtp=w)
    assert torch.equal(spec, greedy[:, :N])
