#!/usr/bin/env python
"""Benchmark of the verifier hot path: verified tokens/s of one decode verify
step at concurrency 32 — 32 sequences x (K+1 = 4) rows = 128 tokens through 12
MoE feed-forward layers (64 routed + 2 shared SwiGLU experts, top-6, hidden
1280, width 896), then the LM-head argmax over 129,280 tokens and the
longest-prefix accept with the bonus token.

One rank per GPU (torchrun for N > 1); every rank verifies its own batch of 32
sequences with its own copy of the weights (data-parallel replicas, weak
scaling, no collective on the data path). Rank 0 prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl vgv|reference]

Inputs are seeded synthetic tensors drawn on the device (weights N(0, 0.02),
hidden states N(0, 1), bf16). Drafts follow the draft model of the workload:
each drafted token equals the verifier's argmax with probability 0.576, else a
uniform token; the argmax is taken from an untimed pass of the same step.
The 5.78 GB of weights streamed per step exceed the 126 MB L2, so no flush is
needed between steps.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

B, K, T, LAYERS = 32, 3, 128, 12
H, I, E, S, TOPK, V = 1280, 896, 64, 2, 6, 129280
P_DRAFT = 0.576
SEED = 0
CFG = 1
METRIC = "verified tokens/s, MoE verify step B=32 K=3"
UNIT = "tokens/s"
WORKLOAD = {
    "workload": "decode verify step: B=32 seqs x (K+1)=4 rows = 128 tokens, 12 MoE FFN layers "
                "(64 routed + 2 shared SwiGLU experts, top-6, H=1280, I=896) + LM-head argmax over "
                "129,280 + prefix accept",
    "B": B, "K": K, "tokens": T, "layers": LAYERS, "vocab": V, "draft_p": P_DRAFT,
    "l2": "inputs larger than L2: 5.78 GB of weights per step vs 126 MB L2, no flush",
}
EXPERT_W_BYTES = 3 * I * H * 2  # gate + up + down of one expert, bf16 (6,881,280 B)
ROUTER_W_BYTES = E * H * 2      # 163,840 B per layer
LM_HEAD_BYTES = V * H * 2       # 330,956,800 B
NOMINAL_HBM_GBS = 8000.0        # "about 8 TB/s", the nominal figure the decode target is stated on
# DRAM bytes (read + write) of one expert-GEMM launch at 128 tokens from one ncu
# capture, with the SHA-256 (first 16 hex digits) of the kernel source it was
# taken on; the bench reports it only while the source is unchanged.
EXPERT_TRAFFIC = {"bytes": 465.68e6, "source": "greedy_speculative_verify_b200/csrc/gemm_moe.cuh",
                  "source_sha16": "75dda351e238651c", "profile": "profiles/moe_expert_gemms_t128.md"}


def _traffic(rec):
    import hashlib

    try:
        with open(os.path.join(ROOT, rec["source"]), "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()[:16]
    except OSError:
        return None
    return rec["bytes"] if sha == rec["source_sha16"] else None


def step_weight_bytes(n_touched):
    """Algorithmic bytes of one decode verify step: per layer the router, the two
    shared experts and every touched routed expert, once; then the LM head.
    Activations are not counted (reported separately)."""
    return sum(ROUTER_W_BYTES + (n + S) * EXPERT_W_BYTES for n in n_touched) + LM_HEAD_BYTES


def _env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def _bf16_peak():
    """Dense bf16 TFLOP/s for a kernel timed alone (the burst figure)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


PREFILL_T = 32 * 1156  # 32 pages x 1,156 visual tokens
# FLOP of one prefill MoE layer: routed SwiGLU experts (gate, up, down) on 6T
# rows, the two shared experts on T rows each, the router
PREFILL_FLOP = 2 * TOPK * PREFILL_T * 3 * I * H + 2 * S * PREFILL_T * 3 * I * H + 2 * PREFILL_T * E * H


def measure_prefill(vgv, si, dev, reps=10):
    """One MoE layer at the prefill shape (T = 36,992, near-uniform routing), timed
    with CUDA events: the whole layer and, through the timing hook, the expert
    GEMM launch (the tensor-bound kernel)."""
    import torch

    d = si.FULL
    lw = si.torch_layer_weights(SEED, 3, 0, d, device=dev)
    x = si.torch_normal_bf16((PREFILL_T, H), 1.0, SEED, 3, si.TID_X, device=dev)
    out = torch.empty_like(x)
    ws = torch.empty(vgv.vg_moe_workspace_bytes(vgv.MOE_DIMS, PREFILL_T), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def layer():
        vgv.vg_moe_ffn(vgv.MOE_DIMS, PREFILL_T, x, lw["router_w"], None, lw["expert_w"], lw["shared_w"], 1, out, None, ws)

    for _ in range(3):
        layer()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        layer()
    e1.record(stream)
    e1.synchronize()
    layer_ms = e0.elapsed_time(e1) / reps
    kinds = {vgv.VG_KERNEL_ROUTER: "router", vgv.VG_KERNEL_GROUPING: "grouping", vgv.VG_KERNEL_EXPERTS: "expert_gemms",
             vgv.VG_KERNEL_COMBINE: "combine"}
    evs = {k: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for k in kinds}
    for e0_, e1_ in evs.values():
        e0_.record(stream)
        e1_.record(stream)
    torch.cuda.synchronize()
    for k, (e0_, e1_) in evs.items():
        vgv.vg_profile_set_events(k, [e0_], [e1_])
    parts = {n: [] for n in kinds.values()}
    for _ in range(3):
        layer()
        torch.cuda.synchronize()
        for k, (e0_, e1_) in evs.items():
            parts[kinds[k]].append(e0_.elapsed_time(e1_))
    for k in kinds:
        vgv.vg_profile_set_events(k, [], [])
    gemm = parts["expert_gemms"]
    gemm_ms = min(gemm)
    peak, kind = _bf16_peak()
    gemm_flop = PREFILL_FLOP - 2 * PREFILL_T * E * H
    del ws
    return {"workload": f"one MoE layer, T={PREFILL_T} (32 pages x 1,156 tokens), near-uniform routing",
            "layer_ms": layer_ms, "layer_tflops": PREFILL_FLOP / (layer_ms / 1e3) / 1e12,
            "expert_gemms_ms": gemm_ms, "expert_gemms_tflops": gemm_flop / (gemm_ms / 1e3) / 1e12,
            "peak_tflops": peak, "peak_source": f"{kind} bf16_tflops (burst)",
            "frac_layer": PREFILL_FLOP / (layer_ms / 1e3) / 1e12 / peak,
            "frac_expert_gemms": gemm_flop / (gemm_ms / 1e3) / 1e12 / peak,
            "breakdown_ms": {n: min(v) for n, v in parts.items()}}


SKEW_T = 4096
SKEW_FLOP = 2 * TOPK * SKEW_T * 3 * I * H + 2 * S * SKEW_T * 3 * I * H + 2 * SKEW_T * E * H
SKEW_B, SKEW_K = 2048, 1
SKEW_LM_FLOP = 2 * SKEW_B * (SKEW_K + 1) * V * H


def _hook_times(vgv, kinds, run, reps=3):
    """Per-kind launch durations (ms, minimum over reps) of one call of `run`,
    from CUDA events the library records around each launch on its stream."""
    import torch

    stream = torch.cuda.current_stream()
    evs = {k: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for k in kinds}
    for e0_, e1_ in evs.values():
        e0_.record(stream)
        e1_.record(stream)
    torch.cuda.synchronize()
    for k, (e0_, e1_) in evs.items():
        vgv.vg_profile_set_events(k, [e0_], [e1_])
    parts = {n: [] for n in kinds.values()}
    try:
        for _ in range(reps):
            run()
            torch.cuda.synchronize()
            for k, (e0_, e1_) in evs.items():
                parts[kinds[k]].append(e0_.elapsed_time(e1_))
    finally:
        for k in kinds:
            vgv.vg_profile_set_events(k, [], [])
    return {n: (min(v) if v else None) for n, v in parts.items()}


def _event_ms(run, reps):
    import torch

    stream = torch.cuda.current_stream()
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        run()
    e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / reps


def measure_skewed(vgv, si, lm, dev, reps=10):
    """The skewed-routing workload: one MoE layer over T = 4,096 tokens with the
    per-expert logit bias 2 ln(1/(e+1)) (hot experts take most tokens, many take
    none), then a K = 1 verify of 2,048 sequences x 2 rows of h = x + MoE(x) with
    the full LM head. Reports the tensor fraction of both (CUDA events) and the
    verified tokens/s."""
    import torch

    d = si.FULL
    lw = si.torch_layer_weights(SEED, 4, 0, d, device=dev)
    bias = torch.from_numpy(si.zipf_router_bias(E)).to(dev)
    x = si.torch_normal_bf16((SKEW_T, H), 1.0, SEED, 4, si.TID_X, device=dev)
    h = torch.empty_like(x)
    ws = torch.empty(vgv.vg_moe_workspace_bytes(vgv.MOE_DIMS, SKEW_T), dtype=torch.uint8, device=dev)
    off = torch.empty(E + 1, dtype=torch.int32, device=dev)
    taps = vgv.make_taps(expert_offsets=off)

    def layer():
        vgv.vg_moe_ffn(vgv.MOE_DIMS, SKEW_T, x, lw["router_w"], bias, lw["expert_w"], lw["shared_w"], 1, h, taps, ws)

    layer_ms = _event_ms(layer, reps)
    parts = _hook_times(vgv, {vgv.VG_KERNEL_ROUTER: "router", vgv.VG_KERNEL_GROUPING: "grouping",
                              vgv.VG_KERNEL_EXPERTS: "expert_gemms", vgv.VG_KERNEL_COMBINE: "combine"}, layer)
    cnt = (off[1:] - off[:-1]).cpu()
    peak, kind = _bf16_peak()
    gemm_flop = SKEW_FLOP - 2 * SKEW_T * E * H
    R = SKEW_B * (SKEW_K + 1)
    am = torch.empty(R, dtype=torch.int32, device=dev)
    acc = torch.empty(SKEW_B, dtype=torch.int32, device=dev)
    tok = torch.empty(SKEW_B, SKEW_K + 1, dtype=torch.int32, device=dev)
    drafts = torch.zeros(SKEW_B, SKEW_K, dtype=torch.int32, device=dev)
    wsv = torch.zeros(vgv.vg_verify_workspace_bytes(SKEW_B, SKEW_K, H, V), dtype=torch.uint8, device=dev)

    def verify():
        vgv.vg_verify_greedy(SKEW_B, SKEW_K, H, V, h, lm, drafts, am, acc, tok, wsv)

    verify()
    torch.cuda.synchronize()
    g = torch.Generator(device=dev)
    g.manual_seed(SEED + 41)
    a = am.view(SKEW_B, SKEW_K + 1)[:, :SKEW_K]
    u = torch.rand(SKEW_B, SKEW_K, generator=g, device=dev)
    noise = torch.randint(0, V, (SKEW_B, SKEW_K), generator=g, device=dev, dtype=torch.int32)
    drafts.copy_(torch.where(u < P_DRAFT, a, noise))
    ver_ms = _event_ms(verify, reps)
    vparts = _hook_times(vgv, {vgv.VG_KERNEL_LM_HEAD: "lm_head_argmax_accept"}, verify)
    tokens = int((acc.to(torch.int64) + 1).sum().item())
    del ws, wsv
    return {"workload": f"one MoE layer, T={SKEW_T}, router bias 2 ln(1/(e+1)); then K=1 verify of "
                        f"{SKEW_B} seqs x 2 rows with the full {V}-row LM head",
            "expert_counts_max": int(cnt.max()), "experts_untouched": int((cnt == 0).sum()),
            "layer_ms": layer_ms, "layer_tflops": SKEW_FLOP / (layer_ms / 1e3) / 1e12,
            "expert_gemms_ms": parts["expert_gemms"],
            "expert_gemms_tflops": gemm_flop / (parts["expert_gemms"] / 1e3) / 1e12,
            "frac_layer": SKEW_FLOP / (layer_ms / 1e3) / 1e12 / peak,
            "frac_expert_gemms": gemm_flop / (parts["expert_gemms"] / 1e3) / 1e12 / peak,
            "breakdown_ms": parts,
            "verify_ms": ver_ms, "verified_tokens": tokens, "verified_tokens_per_s": tokens / (ver_ms / 1e3),
            "tau": tokens / SKEW_B, "lm_head_ms": vparts["lm_head_argmax_accept"],
            "lm_head_tflops": SKEW_LM_FLOP / (vparts["lm_head_argmax_accept"] / 1e3) / 1e12,
            "frac_lm_head": SKEW_LM_FLOP / (vparts["lm_head_argmax_accept"] / 1e3) / 1e12 / peak,
            "peak_tflops": peak, "peak_source": f"{kind} bf16_tflops (burst)"}


def measure_spec_loop(vgv, si, rw, ew, sw, lm, dev, n_steps=20, p=P_DRAFT):
    """Multi-step speculative decoding of B=32 sequences at K=3 on the device,
    on a synthetic Markov decoder (embedding of the last token -> the 12 MoE
    layers -> LM head -> argmax): one step = draft rows, embedding gather,
    layer stack, verify, commit, replayed from a CUDA graph. Drafts are the
    decoder's own token (from a plain greedy run of the same loop) with
    probability p, else uniform. Reports committed tokens/s, tau, and whether
    the committed tokens equal the greedy run's."""
    import torch

    i32 = dict(dtype=torch.int32, device=dev)
    emb = si.torch_normal_bf16((V, H), 1.0, SEED, CFG, si.TID_EMB, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(SEED + 23)
    starts = torch.randint(0, V, (B,), generator=g, device=dev, dtype=torch.int32)
    stream = torch.cuda.current_stream()

    # draft-block weights (synthetic: the drafts are rarely accepted, the cost is real)
    mtp_t = {
        "proj": si.torch_normal_bf16((H, 2 * H), 0.02, SEED, CFG, si.TID_EMB, 1, device=dev),
        "ffn": si.torch_normal_bf16((3 * I * H,), 0.02, SEED, CFG, si.TID_EMB, 2, device=dev),
        "g": [torch.ones(H, dtype=torch.float32, device=dev) for _ in range(3)],
    }
    mtp_w = vgv.make_mtp_weights(mtp_t["proj"], mtp_t["ffn"], *mtp_t["g"], emb, lm)

    def loop(K, n_tokens, ref=None, steps=None, mtp=False):
        T_ = B * (K + 1)
        last, pos, step = starts.clone(), torch.zeros(B, **i32), torch.zeros(1, **i32)
        cap = n_tokens + (K + 1) * ((steps or 0) + 5) + K + 1  # every step of the run fits
        committed = torch.full((B, cap), -1, **i32)
        tokens, drafts = torch.empty(B, K + 1, **i32), torch.empty(B, max(K, 1), **i32)
        x = torch.empty(T_, H, dtype=torch.bfloat16, device=dev)
        hid = torch.empty_like(x)
        am, acc, out = torch.empty(T_, **i32), torch.empty(B, **i32), torch.empty(B, K + 1, **i32)
        ws_s = torch.empty(vgv.vg_moe_stack_workspace_bytes(vgv.MOE_DIMS, T_), dtype=torch.uint8, device=dev)
        ws_v = torch.zeros(vgv.vg_verify_workspace_bytes(B, K, H, V), dtype=torch.uint8, device=dev)
        st = vgv.make_spec_state(B, K, V, last, pos, committed, ref, p, SEED + 29, step, tokens, drafts if K else None)

        ws_m = torch.empty(vgv.vg_mtp_workspace_bytes(B, V), dtype=torch.uint8, device=dev) if mtp else None

        def one(rows=True):
            if rows:
                vgv.vg_spec_rows(st) if not mtp else vgv.vg_spec_rows_given(st)
            vgv.vg_embed_rows(tokens.view(-1), emb, x)
            vgv.vg_moe_ffn_stack(vgv.MOE_DIMS, LAYERS, T_, x, rw, None, ew, sw, hid, ws_s)
            vgv.vg_verify_greedy(B, K, H, V, hid, lm, drafts if K else None, am, acc, out, ws_v)
            vgv.vg_spec_commit(st, acc, out)
            if mtp:  # the next step's drafts from the draft block at this step's hidden states
                vgv.vg_mtp_draft(B, K, mtp_w, hid, K + 1, acc, last, drafts, ws_m)

        if mtp:  # first rows: uniform drafts
            vgv.vg_spec_rows(st)
            one(rows=False)
        else:
            one()
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            one()
        if steps is None:  # run until every sequence has n_tokens
            while int(pos.min()) < n_tokens:
                gr.replay()
            torch.cuda.synchronize()
            return committed, None, None
        for _ in range(3):
            gr.replay()
        torch.cuda.synchronize()
        p0 = int(pos.sum())
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            gr.replay()
        e1.record(stream)
        e1.synchronize()
        return committed, int(pos.sum()) - p0, e0.elapsed_time(e1) / steps

    ref_len = (n_steps + 5) * (K + 1) + K + 1
    greedy, _, _ = loop(0, ref_len)
    greedy = greedy[:, :ref_len].contiguous()
    spec, tokens_timed, ms = loop(K, 0, ref=greedy, steps=n_steps)
    n_cmp = min(int((spec >= 0).sum(1).min()), ref_len)
    lossless = bool(torch.equal(spec[:, :n_cmp], greedy[:, :n_cmp]))
    spec_m, tok_m, ms_m = loop(K, 0, steps=n_steps, mtp=True)
    n_cmp_m = min(int((spec_m >= 0).sum(1).min()), ref_len)
    lossless_m = bool(torch.equal(spec_m[:, :n_cmp_m], greedy[:, :n_cmp_m]))
    return {"workload": f"B={B} sequences, K={K}, {LAYERS} layers, V={V}: device loop of draft rows, embedding, "
                        f"MoE stack, verify, commit (CUDA graph), {n_steps} timed steps",
            "tokens_per_s": tokens_timed / (ms * n_steps / 1e3), "ms_per_step": ms,
            "tau": tokens_timed / (B * n_steps), "draft_p": p,
            "lossless_vs_greedy": lossless, "tokens_compared": n_cmp * B,
            "draft_block": {"ms_per_step": ms_m, "tau": tok_m / (B * n_steps),
                            "lossless_vs_greedy": lossless_m, "tokens_compared": n_cmp_m * B,
                            "note": "drafts from the recursive draft block (synthetic weights) at each verify "
                                    "step's hidden states; ms_per_step includes its K draft steps"}}


def measure_latency(vgv, x, rw, ew, sw, lm, dev, reps=20):
    """Batch-1 verify step latency (1 sequence, K = 3 and K = 1): 12 MoE layers,
    LM-head argmax and accept, replayed from a CUDA graph, two ways: the
    multi-kernel path (layer stack + verify) and the single launch
    (vg_verify_step_small). Bytes of a step: every layer's router, the experts
    its rows touch (from the single launch's routing) and the two shared ones,
    then the LM head."""
    import torch

    res = {}
    stream = torch.cuda.current_stream()
    peak, _ = _peaks()

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        e1.synchronize()
        del g
        return e0.elapsed_time(e1) / reps

    ws_small = torch.empty(vgv.vg_verify_step_small_workspace_bytes(), dtype=torch.uint8, device=dev)
    for k in (3, 1):
        t = k + 1
        xk = x[:t].contiguous()
        hid = torch.empty(t, H, dtype=torch.bfloat16, device=dev)
        dr = torch.zeros(1, k, dtype=torch.int32, device=dev)
        am = torch.empty(t, dtype=torch.int32, device=dev)
        ac = torch.empty(1, dtype=torch.int32, device=dev)
        tk = torch.empty(1, k + 1, dtype=torch.int32, device=dev)
        ws_s = torch.empty(vgv.vg_moe_stack_workspace_bytes(vgv.MOE_DIMS, t), dtype=torch.uint8, device=dev)
        ws_v = torch.zeros(vgv.vg_verify_workspace_bytes(1, k, H, V), dtype=torch.uint8, device=dev)
        idx = torch.empty(LAYERS, t, TOPK, dtype=torch.int32, device=dev)

        def step():
            vgv.vg_moe_ffn_stack(vgv.MOE_DIMS, LAYERS, t, xk, rw, None, ew, sw, hid, ws_s)
            vgv.vg_verify_greedy(1, k, H, V, hid, lm, dr, am, ac, tk, ws_v)

        def one_launch(taps=False):
            vgv.vg_verify_step_small(vgv.MOE_DIMS, LAYERS, 1, k, xk, rw, None, ew, sw, lm, V, dr, am, ac, tk,
                                     ws_small, topk_idx_out=idx if taps else None)

        res[f"K{k}_ms_per_step"] = timed(step)
        one_launch(taps=True)
        torch.cuda.synchronize()
        st, info = vgv.vg_get_device_status()
        if st != 0:
            raise RuntimeError(f"single-launch step: device status {st} at site {info}")
        touched = [len(set(idx[l].flatten().tolist())) for l in range(LAYERS)]
        nbytes = step_weight_bytes(touched)
        ms1 = timed(one_launch)
        res[f"K{k}_one_launch"] = {"ms_per_step": ms1, "algorithmic_bytes": nbytes,
                                   "touched_experts_per_layer": touched,
                                   "achieved_gbs": nbytes / (ms1 / 1e3) / 1e9,
                                   "frac_of_measured_hbm": nbytes / (ms1 / 1e3) / 1e9 / peak,
                                   "frac_of_nominal_8tbs": nbytes / (ms1 / 1e3) / 1e9 / NOMINAL_HBM_GBS}
        res[f"K{k}_multi_kernel_frac_of_measured_hbm"] = nbytes / (res[f"K{k}_ms_per_step"] / 1e3) / 1e9 / peak
    res["workload"] = ("B=1 verify step (K=3: 4 tokens, K=1: 2 tokens), 12 layers + LM head + accept, CUDA graph; "
                       "multi-kernel path and single launch")
    return res


ATTN_CONTEXTS = (2048, 8192)  # cached positions per sequence


def attention_bytes(L: int) -> int:
    """Algorithmic bytes of one verifier attention layer at B = 32, K = 3 over
    caches of L positions: the projections' weights (3H x H and H x H), the
    keys and values of every visible position read once, the new rows' keys and
    values written, the layer's input read and output written (bf16)."""
    R = B * (K + 1)
    return (4 * H * H + B * (L + K + 1) * 2 * H + B * (K + 1) * 2 * H + 2 * R * H) * 2


def attention_chunk_bytes(L: int) -> int:
    """Algorithmic bytes of one attn_chunk launch at B = 32, K = 3: every visible
    key and value read once (bf16), the rotated queries read, the fp32 chunk
    partials (max, exp-sum, 128 values per row) written."""
    K1, n_chunks = K + 1, -(-(L + K + 1) // 256)
    return B * (L + K1) * 2 * H * 2 + B * K1 * H * 2 + B * 10 * n_chunks * K1 * (2 + 128) * 4


def measure_attention(vgv, si, dev, reps=20, contexts=ATTN_CONTEXTS):
    """One verifier attention layer (q/k/v projection, rotary append, chunked
    attention, merge, output projection, residual) at B = 32, K = 3 over caches
    of L positions, replayed from a CUDA graph and timed with CUDA events. Every
    call rewrites the new rows' cache positions with the same values, so the
    replays are identical; the caches exceed the 126 MB L2."""
    import torch

    res = {}
    stream = torch.cuda.current_stream()
    R = B * (K + 1)
    x = si.torch_normal_bf16((R, H), 1.0, SEED, 5, si.TID_X, device=dev)
    wqkv = si.torch_normal_bf16((3 * H, H), 0.02, SEED, 5, si.TID_ATTN_QKV, device=dev)
    wo = si.torch_normal_bf16((H, H), 0.02, SEED, 5, si.TID_ATTN_O, device=dev)
    out = torch.empty_like(x)
    peak, _ = _peaks()
    for L in contexts:
        L_max = L + K + 1
        cache = si.torch_normal_bf16((B, 2, L_max, H), 0.7, SEED, 5, si.TID_KV, layer=L, device=dev)
        lens = torch.full((B,), L, dtype=torch.int32, device=dev)
        ws = torch.empty(vgv.vg_attn_workspace_bytes(B, K, L_max), dtype=torch.uint8, device=dev)

        def layer():
            vgv.vg_attn_verify(B, K, x, wqkv, wo, cache, lens, out, ws)

        layer()
        torch.cuda.synchronize()
        st, info = vgv.vg_get_device_status()
        if st != 0:
            raise RuntimeError(f"attention layer: device status {st} {info}")
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            layer()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        e1.synchronize()
        ms = e0.elapsed_time(e1) / reps
        nbytes = attention_bytes(L)
        # the chunk kernel's own launch time, through the library's timing hook
        h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        h0.record(stream)
        h1.record(stream)  # torch creates the CUDA events at their first record
        torch.cuda.synchronize()
        vgv.vg_profile_set_events(vgv.VG_KERNEL_ATTENTION, [h0], [h1])
        pg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(pg):
            layer()
        vgv.vg_profile_set_events(vgv.VG_KERNEL_ATTENTION, [], [])
        durs = []
        for _ in range(reps):
            pg.replay()
            torch.cuda.synchronize()
            durs.append(h0.elapsed_time(h1))
        chunk_ms, chunk_bytes = sum(durs) / len(durs), attention_chunk_bytes(L)
        res[f"L{L}"] = {"ms_per_layer": ms, "algorithmic_bytes": nbytes, "achieved_gbs": nbytes / (ms / 1e3) / 1e9,
                        "frac_of_measured_hbm": nbytes / (ms / 1e3) / 1e9 / peak,
                        "attn_chunk": {"avg_launch_ms": chunk_ms, "algorithmic_bytes": chunk_bytes,
                                       "achieved_gbs": chunk_bytes / (chunk_ms / 1e3) / 1e9,
                                       "frac_of_measured_hbm": chunk_bytes / (chunk_ms / 1e3) / 1e9 / peak}}
        del g, pg, cache, ws
    res["workload"] = ("one attention layer of a B=32, K=3 verify step: 128 rows, 10 heads x 128, rotary positions, "
                       "causal over L cached + 4 new positions, CUDA graph")
    return res


def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


# ------------------------------------------------------------------ oracle leg

def _oracle_threads():
    """Threads the oracle's BLAS calls use (numpy's thread pool)."""
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return _cores()


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_step(layers, lm, x, drafts, Bq=B, Kq=K):
    """One verify step of the CPU oracle, timed: the 12 MoE layers over the
    B(K+1) rows, then the LM-head argmax and the prefix accept. Inputs are bf16
    bits (uint16 arrays). Returns (seconds, verified tokens, argmax)."""
    import numpy as np

    import oracle

    t0 = time.perf_counter()
    h, _ = oracle.moe_stack(x, layers, k=TOPK, I=I)
    arg, _ = oracle.lm_head_argmax(h, lm)
    acc, _ = oracle.prefix_accept(arg, drafts, Bq, Kq)
    return time.perf_counter() - t0, int(np.sum(acc + 1)), arg


def oracle_one_thread(layers, lm, x, drafts):
    """1-thread wall clock of the oracle on the tiny verify (1 layer, B=4, K=3,
    16 rows) and on the batch-1 step (12 layers, B=1, K=3, 4 rows)."""
    from threadpoolctl import threadpool_limits

    with threadpool_limits(limits=1):
        s0, _, _ = oracle_step(layers[:1], lm, x[:16], drafts[:4], 4, K)
        s2, _, _ = oracle_step(layers, lm, x[:4], drafts[:1], 1, K)
    return {"tiny_verify_B4_K3_1_layer_s": s0, "batch1_K3_12_layers_s": s2}


def _host_inputs(dev):
    """The decode step's inputs as bf16 bits on the host: drawn by the seeded
    torch generator (on the GPU when there is one, else on the CPU)."""
    import synth_inputs as si

    d = si.FULL
    layers = []
    for l in range(LAYERS):
        lw = si.torch_layer_weights(SEED, CFG, l, d, device=dev)
        layers.append({k: si.torch_to_bits(v) for k, v in lw.items()})
        del lw
    lm = si.torch_to_bits(si.torch_normal_bf16((V, H), 0.02, SEED, CFG, si.TID_LM_HEAD, device=dev))
    x = si.torch_to_bits(si.torch_normal_bf16((T, H), 1.0, SEED, CFG, si.TID_X, device=dev))
    return layers, lm, x


def run_reference(args, rank, world):
    """The oracle as it stands, on the host cores: every step (warm-up and timed)
    is one whole verify step of the workload, 12 layers + LM head + accept over
    the 128 rows; the first warm-up step's argmax gives the drafts (p = 0.576)."""
    if rank != 0:
        return 0
    import numpy as np

    import synth_inputs as si

    try:
        import torch

        gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
    except Exception:
        gen_dev = "cpu"
    layers, lm, x = _host_inputs(gen_dev)
    drafts = np.zeros((B, K), dtype=np.int32)
    for i in range(args.warmup):
        _, _, arg = oracle_step(layers, lm, x, drafts)
        if i == 0:
            drafts = si.drafts_from_argmax(arg, B, K, P_DRAFT, V, SEED, CFG)
    times, toks = [], 0
    for _ in range(args.steps):
        s_, toks, _ = oracle_step(layers, lm, x, drafts)
        times.append(s_)
    step_s = statistics.mean(times)
    value = toks / step_s
    sample = (f"one whole verify step per step: {LAYERS} MoE layers over {T} tokens + LM-head argmax/accept "
              f"over {T} rows; numpy fp64 on {_cpu_model()}")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": dict(WORKLOAD, parallelism="host cores"),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": _oracle_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU leg

def aggregate_over_ranks(ms, e2e_ms, tokens_rank, world, device):
    """The job's step times are its slowest rank's (max over ranks); its
    committed tokens are all ranks' (sum). Every rank calls this once, in the
    same order, with the process group already initialised when world > 1."""
    if world == 1:
        return ms, e2e_ms, tokens_rank
    import torch
    import torch.distributed as dist

    t = torch.tensor([ms, e2e_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    n = torch.tensor([tokens_rank], dtype=torch.int64, device=device)
    dist.all_reduce(n)
    return float(t[0]), float(t[1]), int(n.item())


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.f = None

    def start(self):
        try:
            self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.gpu)], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
                for nm, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(nm)
            except (ValueError, IndexError):
                continue
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def measure_box_copy(dev, nbytes=2 << 30):
    """This GPU's device-to-device copy rate now (read + write bytes of a 2 GiB
    copy, best of 5): context for the spread between boxes of the pool. The
    roofline's peak stays the measured peak of MEASURED_PEAKS.json."""
    import torch

    src = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    dst = torch.empty_like(src)
    src.fill_(1)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    best = float("inf")
    for _ in range(5):
        torch.cuda.synchronize()
        e0.record()
        dst.copy_(src)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    del src, dst
    torch.cuda.empty_cache()
    return {"gbs": 2 * nbytes / (best / 1e3) / 1e9, "bytes_copied": nbytes,
            "rule": "read + write bytes of one 2 GiB device-to-device copy (torch), best of 5, after the step"}


def run_gpu(args, rank, world, local):
    import torch
    import torch.distributed as dist

    import greedy_speculative_verify_b200 as vgv
    import synth_inputs as si
    from greedy_speculative_verify_b200 import build as vbuild

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    if rank == 0 and not vbuild.up_to_date():
        vbuild.build()
    if world > 1:
        dist.barrier()
    vgv.load()
    d = si.FULL

    def barrier():
        if world > 1:
            dist.barrier()

    # ---- inputs (weights identical on every rank, the batch differs per rank)
    layers = [si.torch_layer_weights(SEED, CFG, l, d, device=dev) for l in range(LAYERS)]
    rw = [l["router_w"] for l in layers]
    ew = [l["expert_w"] for l in layers]
    sw = [l["shared_w"] for l in layers]
    lm = si.torch_normal_bf16((V, H), 0.02, SEED, CFG, si.TID_LM_HEAD, device=dev)
    x = si.torch_normal_bf16((T, H), 1.0, SEED + 1000 * rank, CFG, si.TID_X, device=dev)
    hid = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    drafts = torch.zeros(B, K, dtype=torch.int32, device=dev)
    argmax = torch.empty(T, dtype=torch.int32, device=dev)
    accepted = torch.empty(B, dtype=torch.int32, device=dev)
    toks = torch.empty(B, K + 1, dtype=torch.int32, device=dev)
    ws_stack = torch.empty(vgv.vg_moe_stack_workspace_bytes(vgv.MOE_DIMS, T), dtype=torch.uint8, device=dev)
    ws_ver = torch.zeros(vgv.vg_verify_workspace_bytes(B, K, H, V), dtype=torch.uint8, device=dev)

    def step(x_in, d_in):
        vgv.vg_moe_ffn_stack(vgv.MOE_DIMS, LAYERS, T, x_in, rw, None, ew, sw, hid, ws_stack)
        vgv.vg_verify_greedy(B, K, H, V, hid, lm, d_in, argmax, accepted, toks, ws_ver)

    # ---- drafts: the verifier's own argmax with probability p, else uniform
    step(x, drafts)
    torch.cuda.synchronize()
    g = torch.Generator(device=dev)
    g.manual_seed(SEED + 17 + rank)
    a = argmax.view(B, K + 1)[:, :K]
    u = torch.rand(B, K, generator=g, device=dev)
    noise = torch.randint(0, V, (B, K), generator=g, device=dev, dtype=torch.int32)
    drafts.copy_(torch.where(u < P_DRAFT, a, noise))

    # ---- expert-GEMM launch bytes per layer, from each layer's routing (untimed)
    n_touched = []
    off = torch.empty(E + 1, dtype=torch.int32, device=dev)
    ws_one = torch.empty(vgv.vg_moe_workspace_bytes(vgv.MOE_DIMS, T), dtype=torch.uint8, device=dev)
    cur, nxt = x.clone(), torch.empty_like(x)
    for l in range(LAYERS):
        vgv.vg_moe_ffn(vgv.MOE_DIMS, T, cur, rw[l], None, ew[l], sw[l], 1, nxt, vgv.make_taps(expert_offsets=off), ws_one)
        n_touched.append(int((off[1:] - off[:-1] > 0).sum().item()))
        cur, nxt = nxt, cur
    del ws_one
    N = T * TOPK
    # algorithmic bytes of an expert-GEMM launch: the weights of every touched
    # expert and the two shared ones, once; activations (token rows read, SwiGLU
    # rows written and read back, expert outputs written) are reported apart
    act_bytes = N * H * 2 + T * H * 2 + 2 * (N + S * T) * I * 2 + (N + S * T) * H * 2
    expert_bytes = [(n + S) * EXPERT_W_BYTES for n in n_touched]

    # ---- device-timed region: the whole step replayed from a CUDA graph
    step(x, drafts)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(x, drafts)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    # keep the GPU under load for about a second so the clock samples see it
    t_end = time.time() + 1.0
    while time.time() < t_end:
        graph.replay()
        torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        graph.replay()
    ev1.record(stream)
    ev1.synchronize()
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms = ev0.elapsed_time(ev1) / args.steps
    tokens_rank = int((accepted.to(torch.int64) + 1).sum().item())
    st, info = vgv.vg_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {vgv.STATUS_NAMES.get(st, st)} at site {info}")

    # ---- end to end through the public calls: pinned host inputs in, results out
    x_host = x.cpu().pin_memory()
    d_host = drafts.cpu().pin_memory()
    acc_host = torch.empty(B, dtype=torch.int32).pin_memory()
    tok_host = torch.empty(B, K + 1, dtype=torch.int32).pin_memory()
    x_in = torch.empty_like(x)
    d_in = torch.empty_like(drafts)

    def e2e_step():
        x_in.copy_(x_host, non_blocking=True)
        d_in.copy_(d_host, non_blocking=True)
        step(x_in, d_in)
        acc_host.copy_(accepted, non_blocking=True)
        tok_host.copy_(toks, non_blocking=True)

    for _ in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    ev0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    ev1.record(stream)
    ev1.synchronize()
    barrier()
    e2e_ms = ev0.elapsed_time(ev1) / args.steps
    assert int((acc_host.to(torch.int64) + 1).sum()) == tokens_rank
    h2d = x_host.numel() * x_host.element_size() + d_host.numel() * d_host.element_size()
    d2h = acc_host.numel() * acc_host.element_size() + tok_host.numel() * tok_host.element_size()

    # ---- kernel timing: CUDA events around every launch, on the launch stream.
    # One step is captured with the library's timing hook set, so every launch
    # is bracketed by event-record nodes; each replay is read before the next.
    kr = max(1, min(args.steps, 10))
    kinds = {vgv.VG_KERNEL_ROUTER: "layer_entry", vgv.VG_KERNEL_GROUPING: "grouping", vgv.VG_KERNEL_EXPERTS: "experts",
             vgv.VG_KERNEL_COMBINE: "combine", vgv.VG_KERNEL_LM_HEAD: "lm_head_argmax_accept"}
    cap = LAYERS + 1  # no kind launches more often than this in one step
    evs = {k: ([torch.cuda.Event(enable_timing=True) for _ in range(cap)],
               [torch.cuda.Event(enable_timing=True) for _ in range(cap)]) for k in kinds}
    for a0, a1 in evs.values():
        for e in a0 + a1:
            e.record(stream)  # torch creates the CUDA event at its first record
    torch.cuda.synchronize()
    for k, (a0, a1) in evs.items():
        vgv.vg_profile_set_events(k, a0, a1)
    pgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(pgraph):
        step(x, drafts)
    counts = {k: vgv.vg_profile_count(k) for k in kinds}  # launches of each kind in one step
    for k in kinds:
        vgv.vg_profile_set_events(k, [], [])
    dur = {k: [] for k in kinds}
    for _ in range(kr):
        pgraph.replay()
        torch.cuda.synchronize()
        for k, (a0, a1) in evs.items():
            dur[k].extend(s.elapsed_time(e) for s, e in zip(a0[:counts[k]], a1[:counts[k]]))
    del pgraph
    breakdown = {kinds[k]: sum(dur[k]) / kr for k in kinds if dur[k]}
    gu = dur[vgv.VG_KERNEL_EXPERTS]
    gu_bytes = sum(expert_bytes[i % LAYERS] for i in range(len(gu)))
    achieved = gu_bytes / (sum(gu) / 1e3) / 1e9
    launches_per_step = sum(counts.values())

    # ---- the other shapes of the workload, measured on their own (untimed by the step)
    prefill = measure_prefill(vgv, si, dev) if not args.no_extra else None
    skewed = measure_skewed(vgv, si, lm, dev) if not args.no_extra else None
    latency = measure_latency(vgv, x, rw, ew, sw, lm, dev) if not args.no_extra else None
    spec_loop = measure_spec_loop(vgv, si, rw, ew, sw, lm, dev) if not args.no_extra else None
    attention = measure_attention(vgv, si, dev) if not args.no_extra else None

    # ---- aggregate over ranks (max time, summed tokens)
    ms, e2e_ms, tokens_all = aggregate_over_ranks(ms, e2e_ms, tokens_rank, world, dev)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the oracle on the very same bytes: the step's inputs copied to the host
        h_layers = [{k: si.torch_to_bits(v) for k, v in lw.items()} for lw in layers]
        h_lm, h_x, h_d = si.torch_to_bits(lm), si.torch_to_bits(x), drafts.cpu().numpy()
        s_step, s_tok, _ = oracle_step(h_layers, h_lm, h_x, h_d)
        one = oracle_one_thread(h_layers, h_lm, h_x, h_d)
        cpu = {"value": s_tok / s_step, "unit": UNIT, "cores": _oracle_threads(), "kind": "oracle",
               "sample": f"one whole verify step on the bench's inputs: {LAYERS} MoE layers over {T} tokens + "
                         f"LM-head argmax/accept over {T} rows (numpy fp64)",
               "step_s": s_step, "cpu_model": _cpu_model(), "one_thread_s": one}
        del h_layers

    peak, peak_kind = _peaks()
    step_bytes = step_weight_bytes(n_touched)
    box_copy = measure_box_copy(dev)
    line = {
        "metric": METRIC, "value": tokens_all / (ms / 1e3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": dict(WORKLOAD, parallelism=f"replicas x{world}", cuda_graph=True),
        "tokens_per_step": tokens_all, "tau": tokens_rank / B,
        "e2e": {"value": tokens_all / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "roofline": {"bound": "hbm", "kernel": "moe_expert_gemms (gate/up + SwiGLU + down, routed + shared)",
                     "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": f"{peak_kind} hbm_gbs", "traffic": _traffic(EXPERT_TRAFFIC),
                     "traffic_profile": EXPERT_TRAFFIC["profile"],
                     "algorithmic_bytes_per_launch": gu_bytes / max(1, len(gu)),
                     "bytes_rule": "(touched routed experts + 2 shared) x 6,881,280 B of weights",
                     "activation_bytes_per_launch": act_bytes,
                     "n_touched_per_layer": n_touched,
                     "avg_launch_ms": sum(gu) / max(1, len(gu))},
        "step_roofline": {"bound": "hbm", "algorithmic_bytes": step_bytes, "ms_per_step": ms,
                          "achieved_gbs": step_bytes / (ms / 1e3) / 1e9,
                          "frac_of_measured": step_bytes / (ms / 1e3) / 1e9 / peak,
                          "frac_of_nominal_8tbs": step_bytes / (ms / 1e3) / 1e9 / NOMINAL_HBM_GBS,
                          "measured_peak_gbs": peak, "peak_source": f"{peak_kind} hbm_gbs",
                          "frac_of_this_box_copy": step_bytes / (ms / 1e3) / 1e9 / box_copy["gbs"],
                          "bytes_rule": "sum over layers of router + (touched + 2 shared) experts' weights, "
                                        "+ the LM head; activations excluded"},
        "box_copy": box_copy,
        "breakdown_ms_per_step": breakdown,
        "clocks": clk,
        "cpu_baseline": cpu,
        "prefill": prefill,
        "skewed_routing": skewed,
        "batch1_latency": latency,
        "spec_decode_loop": spec_loop,
        "attention_layer": attention,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_attention_only(L: int) -> int:
    import torch

    import greedy_speculative_verify_b200 as vgv
    import synth_inputs as si
    from greedy_speculative_verify_b200 import build as vbuild

    if not vbuild.up_to_date():
        vbuild.build()
    vgv.load()
    res = measure_attention(vgv, si, torch.device("cuda", 0), contexts=(L,))
    print(json.dumps({"attention_layer": res}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["vgv", "reference"], default="vgv")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the prefill and batch-1 measurements")
    ap.add_argument("--attention-only", type=int, default=0, metavar="L",
                    help="time only the attention layer over caches of L positions (one GPU) and print its figures")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    rank, world, local = _env()
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.attention_only:
        return run_attention_only(args.attention_only)
    return run_gpu(args, rank, world, local)


if __name__ == "__main__":
    sys.exit(main())
