"""Plain greedy decoding versus draft-and-verify decoding on a synthetic decoder
(test infrastructure only).

The pages claim that greedy verification is lossless: the committed output is
identical with speculation on or off ("Jina AI's 3.4B OCR model targets faster
page parsing", section "FastMTP cuts decoding work"; "jina-ocr-v1: Schnellere
Dokumentenanalyse auf kostengünstigen GPUs", section "Modell und Training";
jina-ocr-v1 model card, decoding paragraph). Byte identity needs a tokenizer,
which is not available, so it is checked as token identity.

The synthetic decoder is a Markov chain on the last token: embedding row of the
token -> MoE layer stack -> LM head -> argmax. Attention is not part of the
hot path, so there is no longer context; the draft-and-verify control flow is
the same as for a full decoder.
"""
import dataclasses

import numpy as np

from .experts import moe_stack
from .verify import lm_head_argmax, prefix_accept


@dataclasses.dataclass
class MarkovDecoder:
    emb: np.ndarray      # bf16 bits [V, H]
    layers: list         # moe layer weight dicts
    lm: np.ndarray       # bf16 bits [V, H]
    k: int
    I: int

    @property
    def V(self) -> int:
        return self.lm.shape[0]

    def next_tokens(self, tokens) -> np.ndarray:
        """Greedy next token after each input token (rows are independent)."""
        h, _ = moe_stack(self.emb[np.asarray(tokens, dtype=np.int64)], self.layers, k=self.k, I=self.I)
        arg, _ = lm_head_argmax(h, self.lm)
        return arg


def greedy_decode(dec: MarkovDecoder, start: int, n: int) -> list:
    out, last = [], start
    while len(out) < n:
        last = int(dec.next_tokens([last])[0])
        out.append(last)
    return out


def speculative_decode(dec: MarkovDecoder, start: int, n: int, K: int, p: float, seed: int):
    """Draft K tokens, verify K+1 rows, commit the accepted prefix and the bonus
    token; repeat until n tokens. The draft model proposes the decoder's own
    next token with probability p and a uniform token otherwise, each step
    continuing from its own previous proposal.

    Returns (committed tokens [n], list of accepted lengths per step).
    """
    g = np.random.default_rng(seed)
    committed, steps, last = [], [], start
    while len(committed) < n:
        drafts, prev = [], last
        for _ in range(K):
            true_next = int(dec.next_tokens([prev])[0])
            d = true_next if g.random() < p else int(g.integers(dec.V))
            drafts.append(d)
            prev = d
        arg = dec.next_tokens([last] + drafts)
        accepted, out = prefix_accept(arg, np.array(drafts, dtype=np.int64).reshape(1, K), 1, K)
        new = [int(t) for t in out[0, : accepted[0] + 1]]
        committed.extend(new)
        steps.append(int(accepted[0]))
        last = new[-1]
    return committed[:n], steps
