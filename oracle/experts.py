"""MoE feed-forward layer and the layer stack (test infrastructure only).

Structure from the pages: 64 routed experts, of which top-6 routing picks six per
token, plus two shared experts that every token visits ("Jina AI's 3.4B OCR model
targets faster page parsing", section "A compressed visual front end"); 12
decoder layers, hidden 1280 (jina-ocr-v1 model card, architecture paragraph).
The expert form (SwiGLU), the width I = 896, unweighted shared experts and the
residual add are readings of the pages, not facts they state.

Each expert's bf16 weights are one contiguous block gate [I,H] | up [I,H] |
down [H,I], row-major.
"""
import numpy as np

from .bf16 import widen, round_bf16_bits
from .permute import expert_permutation
from .router import route, router_logits


def silu(z: np.ndarray) -> np.ndarray:
    """silu(z) = z / (1 + exp(-z)), fp64."""
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def split_expert(w_bits: np.ndarray, I: int, H: int):
    """One expert's block -> (gate [I,H], up [I,H], down [H,I]) in fp64."""
    w = widen(np.asarray(w_bits).reshape(-1))
    assert w.size == 3 * I * H
    return (w[: I * H].reshape(I, H), w[I * H: 2 * I * H].reshape(I, H), w[2 * I * H:].reshape(H, I))


def swiglu_act(x: np.ndarray, w_bits: np.ndarray, I: int, H: int) -> np.ndarray:
    """act = silu(gate x) * (up x) for each row of x [n,H] -> [n,I], fp64."""
    gate, up, _ = split_expert(w_bits, I, H)
    return silu(x @ gate.T) * (x @ up.T)


def swiglu_expert(x: np.ndarray, w_bits: np.ndarray, I: int, H: int) -> np.ndarray:
    """down(silu(gate x) * up x) for each row of x [n,H] -> [n,H], fp64."""
    _, _, down = split_expert(w_bits, I, H)
    return swiglu_act(x, w_bits, I, H) @ down.T


def moe_ffn(x_bits, router_w, expert_w, shared_w, *, k: int, I: int, bias=None, add_residual: bool = True):
    """One MoE layer on tokens x [T,H] (bf16 bits).

    y[t] = sum_j g[t,j] * Expert_{idx[t,j]}(x[t]) + sum_s Shared_s(x[t]);
    out = x + y if add_residual else y. Everything after the router is fp64.

    Returns a dict with ``out`` (fp64 [T,H]) and the intermediates the library
    can expose: logits, idx, g, counts, offsets, perm, inv, act (routed rows in
    permutation order, fp64 [T*k, I]), expert_out (routed rows in permutation
    order, unweighted, fp64 [T*k, H]), shared_act [S,T,I], shared_out [S,T,H].
    """
    x_bits = np.asarray(x_bits, dtype=np.uint16)
    T, H = x_bits.shape
    E = router_w.shape[0]
    S = 0 if shared_w is None else shared_w.shape[0]
    x = widen(x_bits)

    logits = router_logits(x_bits, router_w, bias)
    idx, g = route(logits, k)
    counts, offsets, perm, inv = expert_permutation(idx, E)

    act = np.zeros((T * k, I))
    eout = np.zeros((T * k, H))
    for e in range(E):
        p0, p1 = int(offsets[e]), int(offsets[e + 1])
        if p0 == p1:
            continue
        toks = perm[p0:p1] // k
        _, _, down = split_expert(expert_w[e], I, H)
        a = swiglu_act(x[toks], expert_w[e], I, H)
        act[p0:p1] = a
        eout[p0:p1] = a @ down.T

    y = np.zeros((T, H))
    for j in range(k):
        rows = inv.reshape(T, k)[:, j]
        y += g[:, j: j + 1] * eout[rows]

    shared_act = np.zeros((S, T, I))
    shared_out = np.zeros((S, T, H))
    for s in range(S):
        _, _, down = split_expert(shared_w[s], I, H)
        shared_act[s] = swiglu_act(x, shared_w[s], I, H)
        shared_out[s] = shared_act[s] @ down.T
        y += shared_out[s]

    out = x + y if add_residual else y
    return {
        "out": out, "logits": logits, "idx": idx, "g": g, "counts": counts, "offsets": offsets,
        "perm": perm, "inv": inv, "act": act, "expert_out": eout,
        "shared_act": shared_act, "shared_out": shared_out,
    }


def moe_stack(x_bits, layers, *, k: int, I: int, bias=None):
    """x_{l+1} = bf16(x_l + MoE_l(x_l)) for the given list of layer weight dicts
    (keys router_w, expert_w, shared_w). The residual stream is a bf16 tensor at
    every layer boundary, as it is at the library's interface.

    Returns (final bf16 bits [T,H], list of per-layer moe_ffn results).
    """
    cur = np.asarray(x_bits, dtype=np.uint16)
    results = []
    for lw in layers:
        r = moe_ffn(cur, lw["router_w"], lw["expert_w"], lw["shared_w"], k=k, I=I, bias=bias, add_residual=True)
        results.append(r)
        cur = round_bf16_bits(r["out"])
    return cur, results
