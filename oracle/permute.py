"""Token-to-expert grouping (test infrastructure only).

The pages imply it (each token visits six experts, "Jina AI's 3.4B OCR model
targets faster page parsing", section "A compressed visual front end") without
describing it. Definition used: assignment a = t*k + j (token t, slot j) has key
idx[t, j]; the permutation is the stable sort of the assignments by key.
"""
import numpy as np


def expert_permutation(idx: np.ndarray, E: int):
    """Returns (counts [E], offsets [E+1], perm [T*k], inv [T*k]) as int32.

    counts[e] = number of assignments to expert e; offsets = exclusive prefix
    sum with offsets[E] = T*k; perm[p] = the assignment id at sorted position p
    (stable: ids increase within an expert's segment); inv[a] = the position of
    assignment a, so perm[inv[a]] = a.
    """
    keys = np.asarray(idx, dtype=np.int64).reshape(-1)
    counts = np.bincount(keys, minlength=E)[:E]
    offsets = np.concatenate([[0], np.cumsum(counts)])
    perm = np.argsort(keys, kind="stable")
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size)
    return (counts.astype(np.int32), offsets.astype(np.int32), perm.astype(np.int32), inv.astype(np.int32))
