"""Pins of the draft-block oracle (oracle/mtp.py) against closed forms and
constructions whose answer is known without running the block's formula."""
import numpy as np

import oracle
from oracle.mtp import mtp_draft, mtp_step, rmsnorm
import synth_inputs as si

H, I, V = 16, 8, 12


def _bits(a):
    return oracle.round_bf16_bits(np.asarray(a, dtype=np.float64))


def _weights(proj, ffn, emb, lm, gh=None, ge=None, gf=None):
    one = np.ones(H)
    return {"proj": _bits(proj), "ffn": _bits(ffn), "emb": _bits(emb), "lm": _bits(lm),
            "gamma_h": one if gh is None else gh, "gamma_e": one if ge is None else ge,
            "gamma_f": one if gf is None else gf}


def test_rmsnorm_by_hand():
    x = np.array([3.0, 4.0])  # mean square 12.5
    got = rmsnorm(x, np.array([1.0, 2.0]))
    d = np.sqrt(12.5 + 1e-6)
    assert np.allclose(got, [3.0 / d, 8.0 / d], rtol=0, atol=1e-15)
    # scale invariance (up to eps) and the unit mean square it produces
    y = rmsnorm(np.array([1.0, -2.0, 2.0, 0.5]) * 1e3, np.ones(4))
    assert abs(np.mean(y * y) - 1.0) < 1e-9


def test_zero_projection_gives_token_zero():
    """W_p = 0: z = 0, rmsnorm(0) = 0, FFN(0) = 0 (silu(0) = 0), g = 0; all logits
    are 0 and the lowest index wins at every step."""
    rng = np.random.default_rng(1)
    w = _weights(np.zeros((H, 2 * H)), rng.normal(0, 0.3, 3 * I * H), rng.normal(0, 1, (V, H)),
                 rng.normal(0, 1, (V, H)))
    g0 = _bits(rng.normal(0, 1, (3, H)))
    drafts, hs = mtp_draft(g0, [5, 7, 11], 3, w, I=I)
    assert np.array_equal(drafts, np.zeros((3, 3)))
    assert not np.any(oracle.widen(hs))


def test_hidden_half_first_and_residual():
    """W_p = [Id, 0] and a zero down projection: z = rmsnorm(g) (the hidden half,
    which comes first), the FFN adds nothing, so g_1 = bf16(rmsnorm(g_0))."""
    rng = np.random.default_rng(2)
    ffn = rng.normal(0, 0.3, 3 * I * H)
    ffn[2 * I * H:] = 0.0  # down = 0
    proj = np.concatenate([np.eye(H), np.zeros((H, H))], axis=1)
    gh = rng.uniform(0.5, 1.5, H)
    w = _weights(proj, ffn, rng.normal(0, 1, (V, H)), rng.normal(0, 1, (V, H)), gh=gh)
    g0 = _bits(rng.normal(0, 2, (4, H)))
    g1, _, mid = mtp_step(g0, [0, 1, 2, 3], w, I=I)
    want = _bits(oracle.widen(_bits(rmsnorm(oracle.widen(g0), gh))))
    assert np.array_equal(g1, want)
    assert np.array_equal(mid["u"][:, :H], _bits(rmsnorm(oracle.widen(g0), gh)))


def test_token_feedback_follows_a_permutation():
    """W_p = [0, Id], zero down projection, LM head rows = embedding rows permuted
    (LM[v] = E[pi^-1(v)]): g_i = rmsnorm(E[y_{i-1}]) and the largest logit is at
    v = pi(y_{i-1}) (a |E|^2-sized dot product against ones of independent random
    vectors), so the drafts walk pi: y_i = pi^i(y_0). Pins the embedding half
    (second) and that each step feeds back its own token."""
    rng = np.random.default_rng(3)
    emb = rng.normal(0, 1, (V, H)) * 4
    pi = rng.permutation(V)
    lm = np.empty_like(emb)
    lm[pi] = emb  # LM[pi[y]] = E[y]
    ffn = rng.normal(0, 0.3, 3 * I * H)
    ffn[2 * I * H:] = 0.0
    proj = np.concatenate([np.zeros((H, H)), np.eye(H)], axis=1)
    w = _weights(proj, ffn, emb, lm)
    starts = np.array([3, 9, 0, 11])
    g0 = _bits(rng.normal(0, 1, (4, H)))
    drafts, _ = mtp_draft(g0, starts, 3, w, I=I)
    want = np.stack([pi[starts], pi[pi[starts]], pi[pi[pi[starts]]]], axis=1)
    assert np.array_equal(drafts, want)


def test_ffn_is_the_expert_swiglu_on_the_normed_input():
    """With W_p = [Id, 0], gamma = 1 and a one-hot down row, the FFN output's
    first element is silu(gate_0 . zn) * (up_0 . zn) with zn = rmsnorm(z):
    computed here by hand for a 2-wide expert block."""
    rng = np.random.default_rng(4)
    ffn = np.zeros(3 * I * H)
    gate, up = rng.normal(0, 0.3, H), rng.normal(0, 0.3, H)
    ffn[0:H] = gate                 # gate row 0
    ffn[I * H: I * H + H] = up      # up row 0
    ffn[2 * I * H + 0] = 1.0        # down[0, 0] = 1: out[0] = act[0]
    proj = np.concatenate([np.eye(H), np.zeros((H, H))], axis=1)
    # gamma_h = 3: z = rmsnorm(g) has mean square 9, so the FFN's own rmsnorm matters
    w = _weights(proj, ffn, rng.normal(0, 1, (V, H)), rng.normal(0, 1, (V, H)), gh=np.full(H, 3.0))
    g0 = _bits(rng.normal(0, 1, (1, H)))
    _, _, mid = mtp_step(g0, [0], w, I=I)
    assert abs(np.mean(oracle.widen(mid["z"]) ** 2) - 9.0) < 0.1
    assert abs(np.mean(oracle.widen(mid["zn"]) ** 2) - 1.0) < 0.02  # the FFN sees the normalised z
    zn = oracle.widen(mid["zn"])[0]
    g_w, u_w = oracle.widen(_bits(gate)), oracle.widen(_bits(up))
    a = zn @ g_w
    want = a / (1 + np.exp(-a)) * (zn @ u_w)
    assert abs(oracle.widen(mid["o"])[0, 0] - want) <= 2 ** -8 * abs(want) + 1e-12
    assert not np.any(oracle.widen(mid["o"])[0, 1:])


def test_k_zero_has_no_drafts():
    rng = np.random.default_rng(5)
    w = _weights(np.zeros((H, 2 * H)), np.zeros(3 * I * H), rng.normal(0, 1, (V, H)), rng.normal(0, 1, (V, H)))
    d, hs = mtp_draft(_bits(np.zeros((2, H))), [1, 2], 0, w, I=I)
    assert d.shape == (2, 0) and hs.shape[0] == 0


def test_draft_reads_the_block_output():
    """The LM head is applied to g = z + FFN(...): with W_p = [Id, 0], an FFN whose
    only path puts silu(zn_j) * zn_j times 100 on coordinate k (zn_j > 1 picked),
    g's coordinate k dominates and LM row 0 = 10 e_k wins; z_k itself is negative,
    so on z or rmsnorm(z) alone row 0 would lose to the small random rows."""
    rng = np.random.default_rng(6)
    g0 = _bits(rng.normal(0, 1, (1, H)))
    z = rmsnorm(oracle.widen(g0), np.ones(H))[0]
    j, k = int(np.argmax(z)), int(np.argmin(z))  # z_k < 0: row 0 loses unless the FFN term is there
    assert z[j] > 1.0 and z[k] < -0.5
    ffn = np.zeros(3 * I * H)
    ffn[j] = 1.0                # gate[0, j]
    ffn[I * H + j] = 1.0        # up[0, j]
    ffn[2 * I * H + k * I] = 100.0  # down[k, 0]
    lm = rng.normal(0, 0.05, (V, H))
    lm[0] = 0.0
    lm[0, k] = 10.0
    lm[1:, k] = 0.0             # no other row sees coordinate k
    proj = np.concatenate([np.eye(H), np.zeros((H, H))], axis=1)
    w = _weights(proj, ffn, rng.normal(0, 1, (V, H)), lm)
    g1, y1, mid = mtp_step(g0, [4], w, I=I)
    assert int(y1[0]) == 0
    # the FFN's input is the normalised z: unit mean square
    assert abs(np.mean(oracle.widen(mid["zn"]) ** 2) - 1.0) < 0.02
