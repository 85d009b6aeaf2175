"""Seeded synthetic inputs for the verifier hot path.

This module is the one piece of code that both the CUDA path's callers (tests,
bench) and the CPU oracle use. It holds no arithmetic of the method itself: it
only draws random tensors, rounds them to bf16 and mixes drafted tokens from a
given argmax vector with uniform noise. Everything the method computes lives
either in ``oracle/`` (the CPU restatement) or in the CUDA library.

Shapes follow the decoder described in the jina-ocr-v1 model card (jina.ai/ko,
architecture paragraph): 12 layers, hidden 1280, 64 routed + 2 shared experts,
top-6 routing, a 129,280-token vocabulary. The expert width 896 and the SwiGLU
form are chosen sizes (the pages give neither).

Two back ends draw the same *distributions*:

* ``numpy``: ``Generator(PCG64(SeedSequence([seed, cfg, tensor_id, layer])))``,
  standard normals in fp32 times the std, rounded to bf16 with
  round-to-nearest-even. Used for every CPU-checked size.
* ``torch`` (device): a ``torch.Generator`` seeded from the same four numbers,
  used only for the multi-GB weight sets (12 layers of experts) where numpy
  would take about a minute. Its bits differ from the numpy stream; whoever uses
  it hands the very same bytes to both sides.

bf16 tensors are carried as ``uint16`` arrays of raw bf16 bits on the numpy
side, and as ``torch.bfloat16`` on the torch side.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

# tensor ids inside the seed sequence
TID_X = 0
TID_ROUTER = 1
TID_EXPERTS = 2
TID_SHARED = 3
TID_LM_HEAD = 4
TID_DRAFTS = 5
TID_HID = 6
TID_EMB = 7  # token embedding of the synthetic decoder
TID_ATTN_QKV = 8  # attention q/k/v projection
TID_ATTN_O = 9  # attention output projection
TID_KV = 10  # KV cache contents


@dataclasses.dataclass(frozen=True)
class Dims:
    """Decoder dimensions: hidden H, expert width I, routed experts E,
    shared experts S, routed experts per token k, vocabulary V."""

    H: int = 1280
    I: int = 896
    E: int = 64
    S: int = 2
    k: int = 6
    V: int = 129280

    @property
    def expert_elems(self) -> int:
        """bf16 elements of one expert: gate [I,H] | up [I,H] | down [H,I]."""
        return 3 * self.I * self.H


FULL = Dims()


def rng(seed: int, cfg: int, tensor_id: int, layer: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, cfg, tensor_id, layer])))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(g: np.random.Generator, shape, std: float) -> np.ndarray:
    a = g.standard_normal(int(np.prod(shape)), dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return f32_to_bf16_bits(a).reshape(shape)


# ---------------------------------------------------------------- numpy back end

def hidden_states(seed: int, cfg: int, T: int, H: int, std: float = 1.0, tensor_id: int = TID_X) -> np.ndarray:
    """x ~ N(0, std^2) as bf16 bits, shape [T, H]."""
    return normal_bf16(rng(seed, cfg, tensor_id), (T, H), std)


def layer_weights(seed: int, cfg: int, layer: int, d: Dims, std: float = 0.02) -> dict:
    """One MoE layer: router [E,H], routed experts [E, 3*I*H], shared [S, 3*I*H]
    (each expert = gate [I,H] | up [I,H] | down [H,I], row-major), all bf16 bits."""
    return {
        "router_w": normal_bf16(rng(seed, cfg, TID_ROUTER, layer), (d.E, d.H), std),
        "expert_w": normal_bf16(rng(seed, cfg, TID_EXPERTS, layer), (d.E, d.expert_elems), std),
        "shared_w": normal_bf16(rng(seed, cfg, TID_SHARED, layer), (d.S, d.expert_elems), std),
    }


def lm_head(seed: int, cfg: int, V: int, H: int, std: float = 0.02) -> np.ndarray:
    return normal_bf16(rng(seed, cfg, TID_LM_HEAD), (V, H), std)


def zipf_router_bias(E: int) -> np.ndarray:
    """Per-expert logit bias b_e = 2*ln(1/(e+1)) of the skewed-routing workload, fp32."""
    return np.array([2.0 * math.log(1.0 / (e + 1)) for e in range(E)], dtype=np.float32)


def drafts_from_argmax(arg: np.ndarray, B: int, K: int, p: float, V: int, seed: int, cfg: int) -> np.ndarray:
    """Synthetic draft model: the draft for position i (1..K) of sequence b equals
    ``arg[b*(K+1) + i - 1]`` with probability p, else a uniform token in [0, V).
    Independent per position. ``arg`` is the verifier argmax the caller computed."""
    arg = np.asarray(arg, dtype=np.int64).reshape(B, K + 1)
    g = rng(seed, cfg, TID_DRAFTS)
    u = g.random((B, K))
    noise = g.integers(0, V, size=(B, K))
    d = np.where(u < p, arg[:, :K], noise)
    return d.astype(np.int32)


# ---------------------------------------------------------------- torch back end

def _torch_seed(seed: int, cfg: int, tensor_id: int, layer: int) -> int:
    return int(np.random.SeedSequence([seed, cfg, tensor_id, layer]).generate_state(1, np.uint64)[0] & ((1 << 63) - 1))


def torch_normal_bf16(shape, std: float, seed: int, cfg: int, tensor_id: int, layer: int = 0, device="cuda"):
    """bf16 tensor of N(0, std^2) drawn on ``device`` by a seeded torch.Generator
    (fp32 normals times std, rounded to bf16 by torch's round-to-nearest-even)."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(_torch_seed(seed, cfg, tensor_id, layer))
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def torch_layer_weights(seed: int, cfg: int, layer: int, d: Dims, std: float = 0.02, device="cuda") -> dict:
    return {
        "router_w": torch_normal_bf16((d.E, d.H), std, seed, cfg, TID_ROUTER, layer, device),
        "expert_w": torch_normal_bf16((d.E, d.expert_elems), std, seed, cfg, TID_EXPERTS, layer, device),
        "shared_w": torch_normal_bf16((d.S, d.expert_elems), std, seed, cfg, TID_SHARED, layer, device),
    }


def bits_to_torch(b: np.ndarray, device="cpu"):
    """uint16 bf16 bits -> torch.bfloat16 tensor with the same bytes."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16)
    return t.to(device) if device != "cpu" else t


def torch_to_bits(t) -> np.ndarray:
    """torch.bfloat16 tensor (any device) -> uint16 bf16 bits on the host."""
    import torch

    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
