"""Multi-step speculative decoding on the GPU, through the library's calls only:
a synthetic Markov decoder (embedding row of the last token -> MoE layer stack
-> LM head -> argmax) decoded step by step on the device.

The pages' claim that greedy verification is lossless ("jina-ocr-v1:
Schnellere Dokumentenanalyse auf kostengünstigen GPUs", "Modell und
Training") is checked at GPU level: the speculative loop commits exactly the
tokens of plain greedy decoding (the same loop at K = 0), for any draft source.
The greedy loop itself is checked against the oracle's decoder."""
import numpy as np
import pytest
import torch

import greedy_speculative_verify_b200 as vgv
import oracle
import synth_inputs as si

from gpu_common import D, dev, ensure_lib

pytestmark = pytest.mark.gpu

V = 4096  # vocabulary of the synthetic decoder


class Decoder:
    """Device tensors of a synthetic decoder and the step of a decode loop."""

    def __init__(self, n_layers, cfg=11):
        self.layers = [si.torch_layer_weights(0, cfg, l, D) for l in range(n_layers)]
        self.emb = si.torch_normal_bf16((V, D.H), 1.0, 0, cfg, si.TID_EMB)
        self.lm = si.torch_normal_bf16((V, D.H), 0.02, 0, cfg, si.TID_LM_HEAD)

    def run(self, starts, K, n_tokens, ref=None, p=0.0, seed=1, graph=False, mtp=None):
        """Decodes until every sequence has n_tokens committed; returns
        (committed [B, n_tokens], accepted lengths per step [steps, B]). With
        mtp (draft-block weights), the drafts of every step after the first come
        from the draft block fed the previous verify step's hidden states."""
        B = starts.numel()
        T = B * (K + 1)
        i32 = dict(dtype=torch.int32, device="cuda")
        last, pos, step = starts.clone(), torch.zeros(B, **i32), torch.zeros(1, **i32)
        committed = torch.full((B, n_tokens + K + 1), -1, **i32)
        tokens, drafts = torch.empty(B, K + 1, **i32), torch.empty(B, max(K, 1), **i32)
        x, hid = torch.empty(T, D.H, dtype=torch.bfloat16, device="cuda"), torch.empty(T, D.H, dtype=torch.bfloat16,
                                                                                         device="cuda")
        argmax, accepted, out = torch.empty(T, **i32), torch.empty(B, **i32), torch.empty(B, K + 1, **i32)
        ws_s = torch.empty(vgv.vg_moe_stack_workspace_bytes(vgv.MOE_DIMS, T), dtype=torch.uint8, device="cuda")
        ws_v = torch.zeros(vgv.vg_verify_workspace_bytes(B, K, D.H, V), dtype=torch.uint8, device="cuda")
        assert ref is None or ref.is_contiguous()  # read as [B, ref_len] rows
        st = vgv.make_spec_state(B, K, V, last, pos, committed, ref, p, seed, step, tokens, drafts if K else None)
        rw = [l["router_w"] for l in self.layers]
        ew = [l["expert_w"] for l in self.layers]
        sw = [l["shared_w"] for l in self.layers]

        ws_m = torch.empty(vgv.vg_mtp_workspace_bytes(B, V), dtype=torch.uint8, device="cuda") if mtp else None
        first = [True]

        def one_step():
            if mtp is None or first[0]:
                vgv.vg_spec_rows(st)
            else:
                vgv.vg_spec_rows_given(st)
            first[0] = False
            vgv.vg_embed_rows(tokens.view(-1), self.emb, x)
            vgv.vg_moe_ffn_stack(vgv.MOE_DIMS, len(self.layers), T, x, rw, None, ew, sw, hid, ws_s)
            vgv.vg_verify_greedy(B, K, D.H, V, hid, self.lm, drafts if K else None, argmax, accepted, out, ws_v)
            vgv.vg_spec_commit(st, accepted, out)
            if mtp is not None:
                vgv.vg_mtp_draft(B, K, mtp, hid, K + 1, accepted, last, drafts, ws_m)

        g = None
        if graph:
            one_step()  # set-up outside the capture, then the step is replayed
            torch.cuda.synchronize()
            log = [accepted.clone()]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                one_step()
        else:
            log = []
        while int(pos.min()) < n_tokens:
            g.replay() if g is not None else one_step()
            log.append(accepted.clone())
        torch.cuda.synchronize()
        st_code, info = vgv.vg_get_device_status()
        assert st_code == 0, (st_code, info)
        return committed[:, :n_tokens].contiguous(), torch.stack(log), int(step)


@pytest.fixture(scope="module")
def decoder():
    ensure_lib()
    return Decoder(n_layers=2)


def _starts(B, seed=5):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return torch.randint(0, V, (B,), generator=g, device="cuda", dtype=torch.int32)


@pytest.mark.parametrize("K,p", [(3, 0.576), (3, 0.0), (3, 1.0), (1, 0.751), (4, 0.5)])
def test_speculative_equals_greedy(decoder, K, p):
    B, N = 8, 24
    starts = _starts(B)
    greedy, acc_g, steps_g = decoder.run(starts, 0, N + K + 1)
    assert steps_g == N + K + 1 and bool((acc_g == 0).all())  # K = 0: one token per step
    spec, acc, steps = decoder.run(starts, K, N, ref=greedy, p=p)
    assert torch.equal(spec, greedy[:, :N])  # lossless, token for token
    assert acc.shape[0] == steps and bool(((acc >= 0) & (acc <= K)).all())
    if p == 0.0:
        assert steps == N  # uniform drafts: only the bonus token per step
    if p == 1.0:
        assert bool((acc == K).all()) and steps == -(-N // (K + 1))  # perfect drafts: K + 1 tokens per step


def test_graph_replayed_loop_equals_greedy(decoder):
    """The whole step (rows, embedding, 2 layers, verify, commit) captured once in
    a CUDA graph and replayed: the device state carries the loop."""
    B, K, N = 8, 3, 20
    starts = _starts(B, seed=6)
    greedy, _, _ = decoder.run(starts, 0, N + K + 1)
    spec, acc, steps = decoder.run(starts, K, N, ref=greedy, p=0.6, graph=True)
    assert torch.equal(spec, greedy[:, :N])
    assert steps < N  # speculation committed more than one token per step on average


def test_greedy_loop_matches_oracle_decoder():
    """GPU greedy decoding of a one-layer decoder against the oracle's decoder
    (same bf16 bytes), token for token."""
    ensure_lib()
    cfg, n = 12, 6
    lw = si.layer_weights(0, cfg, 0, D)
    emb_bits = si.hidden_states(0, cfg, V, D.H, tensor_id=si.TID_EMB)
    lm_bits = si.lm_head(0, cfg, V, D.H)
    dec = oracle.MarkovDecoder(emb=emb_bits, layers=[lw], lm=lm_bits, k=D.k, I=D.I)
    start = 17
    ref = oracle.greedy_decode(dec, start, n)
    gpu = Decoder.__new__(Decoder)
    gpu.layers = [{k: dev(v) for k, v in lw.items()}]
    gpu.emb, gpu.lm = dev(emb_bits), dev(lm_bits)
    got, _, _ = gpu.run(torch.tensor([start], dtype=torch.int32, device="cuda"), 0, n)
    assert got[0].tolist() == ref
