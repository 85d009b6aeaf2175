"""Router of the MoE layer: logits, top-k selection and gate weights.

Test infrastructure only. The pages state that top-6 routing picks six of the 64
routed experts for every token ("Jina AI's 3.4B OCR model targets faster page
parsing", section "A compressed visual front end"; jina-ocr-v1 model card,
architecture paragraph). They give no formula; the readings below are the
plainest ones consistent with the rest of the pages.
"""
import numpy as np

from .bf16 import widen


def segment_bounds(H: int, parts: int = 4):
    """h ranges of the partial chains: [floor(q*H/parts), floor((q+1)*H/parts))."""
    return [(q * H // parts, (q + 1) * H // parts) for q in range(parts)]


def router_logits(x_bits: np.ndarray, w_bits: np.ndarray, bias: np.ndarray | None = None) -> np.ndarray:
    """l[t, e] = sum_h x[t, h] * w[e, h] in fp32, in this order: four partial
    sums over the contiguous quarters of h (see segment_bounds), each an fp32
    fused-multiply-add chain in increasing h starting from +0; then
    (q0 + q1) + (q2 + q3) in fp32; then + bias[e] in one fp32 addition.

    Reading: the routing decision is integer output taken in fp32, so the order
    of the sum is part of its definition; the pages give none. Four contiguous
    chains combined pairwise are a plain blocked sum whose longest dependency
    chain is a quarter of the sequential one.

    Emulation of fp32 fma in fp64: the product of two bf16 numbers (8-bit
    significands) is exact in fp64, and so is its sum with an fp32 accumulator
    unless their exponents lie more than 29 binades apart. In that case the
    smaller term is below 2^-28 of the larger one's unit and cannot carry the
    fp64 result across an fp32 rounding boundary, so one rounding of the fp64
    sum to fp32 equals the single rounding of fma.
    """
    x = widen(x_bits)
    w = widen(w_bits)
    T, H = x.shape
    E = w.shape[0]
    part = []
    for h0, h1 in segment_bounds(H):
        acc = np.zeros((T, E), dtype=np.float32)
        for h in range(h0, h1):
            acc = (acc.astype(np.float64) + np.outer(x[:, h], w[:, h])).astype(np.float32)
        part.append(acc)
    logits = (part[0] + part[1]) + (part[2] + part[3])  # fp32 + fp32 -> fp32
    if bias is not None:
        logits = logits + np.asarray(bias, dtype=np.float32)[None, :]
    return logits.astype(np.float32)


def softmax_gates(logits: np.ndarray) -> np.ndarray:
    """p[t, e] = exp(l_e - max l) / sum_e' exp(l_e' - max l), in fp64 over all E."""
    l = np.asarray(logits, dtype=np.float64)
    z = np.exp(l - l.max(axis=1, keepdims=True))
    return z / z.sum(axis=1, keepdims=True)


def route(logits: np.ndarray, k: int):
    """Top-k experts per token and their gate weights.

    idx[t, :] = the k experts with the largest logits, in descending logit
    order, equal logits ordered by the lower expert index (a stable sort on the
    negated logits). Softmax is strictly increasing, so this is the same set
    and order as selecting on the softmax probabilities, without ties created
    by rounding exp. g[t, j] = p[t, idx[t, j]], the softmax over all E logits,
    not renormalised over the k selected (reading).
    """
    l = np.asarray(logits, dtype=np.float32)
    order = np.argsort(-l.astype(np.float64), axis=1, kind="stable")
    idx = order[:, :k].astype(np.int32)
    p = softmax_gates(l)
    g = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    return idx, g
