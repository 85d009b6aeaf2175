"""CPU oracle for the verifier hot path — TEST INFRASTRUCTURE ONLY.

A plain, slow restatement of what the verifier pass computes, used to check the
CUDA library. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import it; the library and its Python binding never do,
and nothing here imports them. The only code shared with the GPU side is the
seeded input generator module ``synth_inputs`` (random tensors, no arithmetic of
the method).

What the pages fix, and where each piece comes from:

* the decoder shape — 12 layers, hidden 1280, 64 routed + 2 shared experts,
  top-6 routing, 129,280-token vocabulary: jina-ocr-v1 model card (jina.ai/ko),
  architecture paragraph; "Jina OCR v1: Быстрый парсинг документов на GPU с
  24 ГБ VRAM" (aikraft.ru), section "01 Архитектура и эффективность";
* six routed experts per token plus two always-on shared experts: "Jina AI's
  3.4B OCR model targets faster page parsing" (alphasignal.ai), section
  "A compressed visual front end";
* greedy verification that commits the longest prefix on which draft and
  verifier agree, so that the committed text equals plain greedy decoding:
  "jina-ocr-v1: Schnellere Dokumentenanalyse auf kostengünstigen GPUs"
  (jina.ai/de), section "Modell und Training"; the same page, section
  "Spekulatives Decoding auf einer L4", counts the bonus token in tau.

Readings where the pages are silent (each one a choice of this oracle, stated here):

* router logits are four fp32 fused-multiply-add chains over the contiguous
  quarters of h (each from +0, increasing h), combined as (q0+q1)+(q2+q3) in
  fp32, then + b_e in fp32; selection is on the logits (descending, ties to the
  lower expert index); gate weights are the softmax over all E logits with no
  renormalisation over the selected six;
* expert FFN = SwiGLU: down(silu(gate x) * up x), silu(z) = z / (1 + e^-z);
  shared experts are unweighted;
* LM-head logits are decided in fp32 (the kernel's precision): the exact fp64
  dot product rounded once to fp32, argmax = lowest index among equal maxima;
* every other quantity is computed in fp64 from the bf16 inputs, with no
  intermediate rounding, except the layer-to-layer residual stream, which is a
  bf16 tensor at every layer boundary of the library's interface.

Every function is dimension-generic so the self-tests can run on tiny shapes.
"""
from .bf16 import widen, round_bf16_bits
from .router import router_logits, route, softmax_gates, segment_bounds
from .permute import expert_permutation
from .experts import silu, swiglu_expert, moe_ffn, moe_stack
from .verify import lm_head_argmax, logit_fp64, prefix_accept, tau, acceptance_rate
from .decode import MarkovDecoder, greedy_decode, speculative_decode
from .mtp import rmsnorm, mtp_step, mtp_draft
from .attention import rope, attn_verify

__all__ = [
    "widen", "round_bf16_bits", "router_logits", "route", "softmax_gates", "segment_bounds",
    "expert_permutation", "silu", "swiglu_expert", "moe_ffn", "moe_stack",
    "lm_head_argmax", "logit_fp64", "prefix_accept", "tau", "acceptance_rate",
    "MarkovDecoder", "greedy_decode", "speculative_decode", "rmsnorm", "mtp_step", "mtp_draft",
    "rope", "attn_verify",
]
