"""Recursive draft block (FastMTP) — TEST INFRASTRUCTURE ONLY.

What the pages fix: the drafter is one dense block reused for every one of the
K prediction steps, so its parameters do not grow with the depth ("Jina AI's
3.4B OCR model targets faster page parsing", section "FastMTP cuts decoding
work"; "jina-ocr-v1: Schnellere Dokumentenanalyse auf kostengünstigen GPUs",
section "Modell und Training"), and it was trained with recursive hidden-state
feedback (same page, section "Erste Schritte": registered as "eagle", not
re-primed on the target each step). The block itself is not described; the
reading used here (each point a reading, listed in the design notes):

* step i (i = 1..K) takes the hidden state g_{i-1} and the token y_{i-1}
  (g_0 = the verifier's final hidden state of the row that produced the last
  committed token, y_0 = that token);
* u = [rmsnorm(g_{i-1}; gamma_h) ; rmsnorm(E[y_{i-1}]; gamma_e)], 2H wide, hidden
  half first; rmsnorm(x; gamma) = x / sqrt(mean(x^2) + 1e-6) * gamma;
* z = W_p u (W_p [H, 2H]);
* g_i = z + FFN(rmsnorm(z; gamma_f)), FFN a SwiGLU of width I laid out like one
  expert (gate | up | down);
* y_i = argmax of the shared LM head's logits at g_i (no further norm, as the
  verify step applies the LM head to its hidden states directly), decided in
  fp32 like the verifier's (lowest index among equal maxima);
* the drafts are y_1 .. y_K.

Arithmetic: fp64, with bf16 rounding where the block's tensors cross a
boundary of the library (u, z, rmsnorm(z), FFN output, g), the embedding and
weights as bf16 inputs.
"""
import numpy as np

from .bf16 import round_bf16_bits, widen
from .experts import swiglu_expert
from .verify import lm_head_argmax

RMS_EPS = 1e-6


def rmsnorm(x: np.ndarray, gamma: np.ndarray) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * gamma over the last axis, fp64."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + RMS_EPS) * np.asarray(gamma, dtype=np.float64)


def mtp_step(g_bits, y, w: dict, *, I: int):
    """One application of the draft block to rows (g [n,H] bf16 bits, y [n]).

    w: proj [H, 2H], ffn (one expert block), gamma_h, gamma_e, gamma_f [H] (fp32
    or fp64 values), emb [V, H], lm [V, H] (bf16 bits).
    Returns (g' bf16 bits [n,H], y' [n], intermediates dict).
    """
    g = widen(np.asarray(g_bits, dtype=np.uint16))
    H = g.shape[1]
    e = widen(np.asarray(w["emb"], dtype=np.uint16)[np.asarray(y, dtype=np.int64)])
    u_bits = np.concatenate([round_bf16_bits(rmsnorm(g, w["gamma_h"])),
                             round_bf16_bits(rmsnorm(e, w["gamma_e"]))], axis=1)
    z_bits = round_bf16_bits(widen(u_bits) @ widen(np.asarray(w["proj"], dtype=np.uint16)).reshape(H, 2 * H).T)
    zn_bits = round_bf16_bits(rmsnorm(widen(z_bits), w["gamma_f"]))
    o_bits = round_bf16_bits(swiglu_expert(widen(zn_bits), w["ffn"], I, H))
    g_next = round_bf16_bits(widen(z_bits) + widen(o_bits))
    y_next, _ = lm_head_argmax(g_next, w["lm"])
    return g_next, y_next, {"u": u_bits, "z": z_bits, "zn": zn_bits, "o": o_bits}


def mtp_draft(g0_bits, y0, K: int, w: dict, *, I: int):
    """K recursive steps from (g_0, y_0); returns (drafts [n, K], hidden states
    [K, n, H] bf16 bits)."""
    g, y = np.asarray(g0_bits, dtype=np.uint16), np.asarray(y0, dtype=np.int64)
    drafts, hs = [], []
    for _ in range(K):
        g, y, _ = mtp_step(g, y, w, I=I)
        drafts.append(np.asarray(y, dtype=np.int64))
        hs.append(g)
    if K == 0:
        return np.zeros((len(y), 0), dtype=np.int64), np.zeros((0,) + g.shape, dtype=np.uint16)
    return np.stack(drafts, axis=1), np.stack(hs)
