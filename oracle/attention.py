"""Verifier attention over a KV cache — TEST INFRASTRUCTURE ONLY.

The pages describe the decoder only as DeepSeek-OCR's 3B mixture-of-experts
decoder with a 32,768-position limit (jina-ocr-v1 model card, architecture
paragraph) and say nothing about its attention. The reading used here, for
one layer of a verify step that scores K+1 new rows per sequence (the last
committed token and K drafts) against that sequence's cache of L positions:

* multi-head attention with n_heads = 10 heads of 128 (hidden 1280), no bias;
  q, k, v = x W_qkv^T (W_qkv [3H, H]: the q rows, then k, then v);
* rotary position embedding (RoFormer) on q and k: the pair (2j, 2j+1) of a
  head at position p turned by the angle p * 10000^(-2j/128); row i of a
  sequence sits at position L + i;
* the new k, v rows are written into the cache at positions L .. L+K (a later
  step overwrites the positions of rejected drafts);
* row i attends to cache positions 0 .. L+i (causal), scores q.k / sqrt(128),
  softmax over them; the heads' outputs are concatenated;
* out = x + (W_o o) (W_o [H, H]).

Arithmetic: fp64, with bf16 rounding where a tensor crosses a library
boundary: q/k/v after the projection, the rotated q and k, the cache, the
attention output o, W_o o and the result.
"""
import numpy as np

from .bf16 import round_bf16_bits, widen

N_HEADS, HEAD_DIM, ROPE_BASE = 10, 128, 10000.0


def rope(x: np.ndarray, pos: np.ndarray) -> np.ndarray:
    """Rotary embedding of rows x [n, heads*dim] at positions pos [n], fp64."""
    n, width = x.shape
    d = HEAD_DIM
    xr = x.reshape(n, width // d, d // 2, 2)
    j = np.arange(d // 2, dtype=np.float64)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * ROPE_BASE ** (-2.0 * j / d)  # [n, d/2]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    out = np.empty_like(xr)
    out[..., 0] = xr[..., 0] * c - xr[..., 1] * s
    out[..., 1] = xr[..., 0] * s + xr[..., 1] * c
    return out.reshape(n, width)


def attn_verify(x_bits, w_qkv_bits, w_o_bits, cache_bits, lens, K: int):
    """One attention layer of a verify step.

    x_bits [B*(K+1), H]; w_qkv [3H, H]; w_o [H, H]; cache [B, 2, L_max, H] (k, v),
    bf16 bits; lens [B]. Returns (out bits [B*(K+1), H], new cache bits, dict of
    intermediates: q, k (rotated), o, proj).
    """
    x = widen(np.asarray(x_bits, dtype=np.uint16))
    R, H = x.shape
    B = R // (K + 1)
    assert B * (K + 1) == R
    qkv = round_bf16_bits(x @ widen(w_qkv_bits).reshape(3 * H, H).T)
    q_raw, k_raw, v = qkv[:, :H], qkv[:, H: 2 * H], qkv[:, 2 * H:]
    lens = np.asarray(lens, dtype=np.int64)
    pos = (lens[:, None] + np.arange(K + 1)[None, :]).reshape(-1)
    q = round_bf16_bits(rope(widen(q_raw), pos))
    k = round_bf16_bits(rope(widen(k_raw), pos))
    cache = np.array(cache_bits, dtype=np.uint16, copy=True)
    for b in range(B):
        for i in range(K + 1):
            cache[b, 0, lens[b] + i] = k[b * (K + 1) + i]
            cache[b, 1, lens[b] + i] = v[b * (K + 1) + i]
    o = np.zeros((R, H))
    scale = 1.0 / np.sqrt(HEAD_DIM)
    for b in range(B):
        for i in range(K + 1):
            r = b * (K + 1) + i
            n = lens[b] + i + 1
            kc = widen(cache[b, 0, :n]).reshape(n, N_HEADS, HEAD_DIM)
            vc = widen(cache[b, 1, :n]).reshape(n, N_HEADS, HEAD_DIM)
            qr = widen(q[r]).reshape(N_HEADS, HEAD_DIM)
            s = np.einsum("hd,nhd->hn", qr, kc) * scale
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            o[r] = np.einsum("hn,nhd->hd", p, vc).reshape(H)
    o_bits = round_bf16_bits(o)
    proj_bits = round_bf16_bits(widen(o_bits) @ widen(w_o_bits).reshape(H, H).T)
    out = round_bf16_bits(x + widen(proj_bits))
    return out, cache, {"q": q, "k": k, "o": o_bits, "proj": proj_bits}
