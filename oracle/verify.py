"""Greedy verification epilogue (test infrastructure only).

The verifier checks every drafted token greedily and commits the longest prefix
on which draft and verifier agree, so the committed sequence is the verifier's
own greedy sequence ("jina-ocr-v1: Schnellere Dokumentenanalyse auf
kostengünstigen GPUs", jina.ai/de, section "Modell und Training"). The mean
number of tokens committed per speculative step, tau, includes the bonus token
(same page, section "Spekulatives Decoding auf einer L4"). The vocabulary has
129,280 tokens (jina-ocr-v1 model card, architecture paragraph).

Layout: sequence b's K+1 verify rows are rows b*(K+1) .. b*(K+1)+K; row
b*(K+1)+i holds position i, and its argmax is the verifier's prediction for
position i+1. drafts[b, i] is the draft for position i+1.
"""
import numpy as np

from .bf16 import widen


def lm_head_argmax(hid_bits: np.ndarray, lm_bits: np.ndarray, chunk: int = 8192):
    """arg[r] = the smallest v with z32[r, v] = max_v z32[r, v], where
    z32[r, v] = fp32(sum_h hid[r, h] * LM[v, h]) is the fp64 dot product rounded
    once to fp32 (the decision is taken in fp32, the kernel's precision; the
    fp64 sum of 1280 bf16 products is exact to ~1e-13 relative).

    Returns (arg int32 [R], max fp32 [R]).
    """
    h = widen(hid_bits)
    R = h.shape[0]
    V = lm_bits.shape[0]
    best = np.full(R, -np.inf, dtype=np.float32)
    arg = np.zeros(R, dtype=np.int64)
    for v0 in range(0, V, chunk):
        v1 = min(V, v0 + chunk)
        z32 = (h @ widen(lm_bits[v0:v1]).T).astype(np.float32)
        loc = np.argmax(z32, axis=1)  # first index of the maximum
        val = z32[np.arange(R), loc]
        better = val > best  # strict: an earlier chunk keeps equal maxima
        best = np.where(better, val, best)
        arg = np.where(better, v0 + loc, arg)
    return arg.astype(np.int32), best


def logit_fp64(hid_bits: np.ndarray, lm_bits: np.ndarray, rows, vocab):
    """For pairs (rows[i], vocab[i]): (z64 = sum_h hid*LM in fp64,
    a = sum_h |hid*LM|, the magnitude that bounds any summation-order error)."""
    h = widen(hid_bits[np.asarray(rows)])
    w = widen(lm_bits[np.asarray(vocab)])
    prod = h * w
    return prod.sum(axis=1), np.abs(prod).sum(axis=1)


def prefix_accept(arg: np.ndarray, drafts: np.ndarray, B: int, K: int):
    """accepted[b] = the largest a <= K with drafts[b, i] == arg[b*(K+1)+i] for
    every i < a; out_tokens[b] = drafts[b, :a], then the bonus token
    arg[b*(K+1)+a], then -1 padding to K+1 entries.
    """
    arg = np.asarray(arg).reshape(B, K + 1)
    drafts = np.asarray(drafts).reshape(B, K)
    accepted = np.zeros(B, dtype=np.int32)
    out = np.full((B, K + 1), -1, dtype=np.int32)
    for b in range(B):
        a = 0
        while a < K and drafts[b, a] == arg[b, a]:
            a += 1
        accepted[b] = a
        out[b, :a] = drafts[b, :a]
        out[b, a] = arg[b, a]
    return accepted, out


def tau(accepted: np.ndarray) -> float:
    """Mean committed tokens per speculative step, bonus token included."""
    return float(np.mean(np.asarray(accepted) + 1))


def acceptance_rate(accepted: np.ndarray, K: int) -> float:
    """Fraction of drafted tokens that were committed: mean(a) / K = (tau - 1) / K."""
    return float(np.mean(accepted)) / K
