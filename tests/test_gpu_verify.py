"""GPU parity of the greedy-verify epilogue (vg_verify_greedy) against the CPU
oracle: argmax bit-exact up to certified near-ties, accepted lengths and
committed tokens bit-exact."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
from gpu_common import D, check_argmax, dev, ensure_lib, run_verify

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lm():
    ensure_lib()
    bits = si.lm_head(0, 0, D.V, D.H)
    return bits, dev(bits)


@pytest.mark.parametrize("B,K,cfg", [(4, 3, 0), (32, 3, 1), (1, 3, 2), (1, 1, 2), (7, 2, 7), (5, 0, 8)])
def test_verify_parity(lm, B, K, cfg):
    """(4,3): the tiny verify; (32,3): the decode step at concurrency 32;
    (1,3), (1,1): batch 1; (7,2): ragged rows; (5,0): plain greedy."""
    lm_bits, lm_t = lm
    R = B * (K + 1)
    h = si.hidden_states(0, cfg, R, D.H, tensor_id=si.TID_HID)
    ref_arg, _ = oracle.lm_head_argmax(h, lm_bits)
    drafts = si.drafts_from_argmax(ref_arg, B, K, 0.576, D.V, seed=0, cfg=cfg)
    ref_acc, ref_out = oracle.prefix_accept(ref_arg, drafts, B, K)
    arg, acc, out = run_verify(dev(h), lm_t, drafts, B, K)
    ties = check_argmax(arg, ref_arg, h, lm_bits)
    if ties == 0:
        assert np.array_equal(acc, ref_acc)
        assert np.array_equal(out, ref_out)
    # in every case the accept step is exact given the argmax it saw
    a2, o2 = oracle.prefix_accept(arg, drafts, B, K)
    assert np.array_equal(acc, a2) and np.array_equal(out, o2)


def test_verify_skewed_shape_sampled(lm):
    """K=1 verify over 2,048 sequences x 2 rows (4,096 rows, 32 row tiles); the
    oracle computes the argmax of 256 sampled sequences."""
    lm_bits, lm_t = lm
    B, K = 2048, 1
    R = B * 2
    h = si.hidden_states(0, 4, R, D.H, tensor_id=si.TID_HID)
    rng = np.random.default_rng(4)
    seqs = np.sort(rng.choice(B, 256, replace=False))
    rows = (seqs[:, None] * 2 + np.arange(2)).ravel()
    ref_s, _ = oracle.lm_head_argmax(h[rows], lm_bits)
    ref_arg = np.full(R, -1, dtype=np.int64)
    ref_arg[rows] = ref_s
    # drafts of the sampled sequences follow the oracle; the rest are uniform
    drafts = si.drafts_from_argmax(np.where(ref_arg < 0, 0, ref_arg), B, K, 0.576, D.V, seed=0, cfg=4)
    other = np.setdiff1d(np.arange(B), seqs)
    drafts[other] = np.random.default_rng(5).integers(0, D.V, (len(other), K))
    arg, acc, out = run_verify(dev(h), lm_t, drafts, B, K)
    check_argmax(arg, ref_arg, h, lm_bits, rows=rows)
    a2, o2 = oracle.prefix_accept(arg, drafts, B, K)
    assert np.array_equal(acc, a2) and np.array_equal(out, o2)
    # the accepted-length distribution of the sampled sequences: E[tau] = 1 + p
    tau = oracle.tau(acc[seqs])
    assert abs(tau - 1.576) < 4 * np.sqrt(0.576 * 0.424 / len(seqs))


@pytest.mark.parametrize("V", [1, 175, 176, 177, 1000, 5000])
def test_verify_ragged_vocab(lm, V):
    """Vocabulary sizes around the 176-row tile: the padded columns of the last
    tile must never win."""
    lm_bits, _ = lm
    B, K = 6, 3
    lm_v = np.ascontiguousarray(lm_bits[:V])
    h = si.hidden_states(0, 9, B * (K + 1), D.H, tensor_id=si.TID_HID)
    ref_arg, _ = oracle.lm_head_argmax(h, lm_v)
    drafts = si.drafts_from_argmax(ref_arg, B, K, 0.7, V, seed=1, cfg=9)
    arg, acc, out = run_verify(dev(h), dev(lm_v), drafts, B, K, V=V)
    assert np.all((arg >= 0) & (arg < V))
    check_argmax(arg, ref_arg, h, lm_v)
    a2, o2 = oracle.prefix_accept(arg, drafts, B, K)
    assert np.array_equal(acc, a2) and np.array_equal(out, o2)


def test_verify_exact_ties_lowest_index(lm):
    """Duplicated vocabulary rows give equal logits: the lower index wins, in the
    same tile and across tiles."""
    lm_bits, _ = lm
    V = 2000
    lmv = np.ascontiguousarray(lm_bits[:V]).copy()
    h = si.hidden_states(0, 10, 8, D.H, tensor_id=si.TID_HID)
    ref0, _ = oracle.lm_head_argmax(h, lmv)
    # make the current winner of each row appear again at a lower and a higher index
    for r, a in enumerate(ref0):
        lmv[(a + 1) % V] = lmv[a]          # right after (often the same tile)
        lmv[(a + 900) % V] = lmv[a]        # another tile
    ref_arg, _ = oracle.lm_head_argmax(h, lmv)
    arg, _, _ = run_verify(dev(h), dev(lmv), np.zeros((8, 0), np.int32), 8, 0, V=V)
    assert np.array_equal(arg, ref_arg)


def test_verify_closed_forms(lm):
    """All drafts correct -> K accepted and K+1 tokens; first draft wrong ->
    only the verifier's token; drafts out of range never match."""
    lm_bits, lm_t = lm
    B, K = 4, 3
    h = si.hidden_states(0, 11, B * (K + 1), D.H, tensor_id=si.TID_HID)
    ref_arg, _ = oracle.lm_head_argmax(h, lm_bits)
    a = ref_arg.reshape(B, K + 1)
    drafts = np.array([a[0, :3], [-1, a[1, 1], a[1, 2]], [a[2, 0], D.V, a[2, 2]], [a[3, 0], a[3, 1], 2 ** 31 - 1]],
                      dtype=np.int32)
    arg, acc, out = run_verify(dev(h), lm_t, drafts, B, K)
    if np.array_equal(arg, ref_arg):
        assert acc.tolist() == [3, 0, 1, 2]
        assert out[0].tolist() == a[0].tolist()
        assert out[1].tolist() == [a[1, 0], -1, -1, -1]
        assert out[2].tolist() == [a[2, 0], a[2, 1], -1, -1]
        assert out[3].tolist() == [a[3, 0], a[3, 1], a[3, 2], -1]


def test_verify_b_zero_writes_nothing(lm):
    import greedy_speculative_verify_b200 as vgv

    _, lm_t = lm
    am = torch.full((4,), -7, dtype=torch.int32, device="cuda")
    h = torch.zeros((4, D.H), dtype=torch.bfloat16, device="cuda")
    vgv.vg_verify_greedy(0, 3, D.H, D.V, h, lm_t, am, am, am, am, None)
    torch.cuda.synchronize()
    assert torch.all(am == -7)


def test_verify_leaves_workspace_zero_and_reports_a_dirty_counter(lm):
    """The workspace (each row's running key, then the CTA counter) is left
    zero-filled by every call. A counter that is not zero at entry is reported
    as VG_ERR_DEVICE_BOUNDS (site 125) instead of being trusted; after clearing
    it the next call is correct again."""
    import greedy_speculative_verify_b200 as vgv

    lm_bits, lm_t = lm
    B, K = 8, 3
    R = B * (K + 1)
    h = si.hidden_states(0, 11, R, D.H, tensor_id=si.TID_HID)
    ref_arg, _ = oracle.lm_head_argmax(h, lm_bits)
    drafts = si.drafts_from_argmax(ref_arg, B, K, 0.576, D.V, seed=0, cfg=11)
    cuda = torch.device("cuda")
    ht, d = dev(h), torch.from_numpy(drafts).to(cuda)
    am = torch.empty(R, dtype=torch.int32, device=cuda)
    acc = torch.empty(B, dtype=torch.int32, device=cuda)
    ot = torch.empty(B, K + 1, dtype=torch.int32, device=cuda)
    nbytes = vgv.vg_verify_workspace_bytes(B, K, D.H, D.V)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=cuda)
    for _ in range(2):
        vgv.vg_verify_greedy(B, K, D.H, D.V, ht, lm_t, d, am, acc, ot, ws)
        torch.cuda.synchronize()
        assert vgv.vg_get_device_status() == (0, 0)
        assert int(ws.count_nonzero()) == 0
        check_argmax(am.cpu().numpy(), ref_arg, h, lm_bits)
    counter = ws[(R * 8 + 255) // 256 * 256:].view(torch.int32)
    counter[0] = 1000  # more than the grid has CTAs
    vgv.vg_verify_greedy(B, K, D.H, D.V, ht, lm_t, d, am, acc, ot, ws)
    torch.cuda.synchronize()
    assert vgv.vg_get_device_status() == (6, 125)
    ws.zero_()
    am.fill_(-1)
    vgv.vg_verify_greedy(B, K, D.H, D.V, ht, lm_t, d, am, acc, ot, ws)
    torch.cuda.synchronize()
    assert vgv.vg_get_device_status() == (0, 0)
    check_argmax(am.cpu().numpy(), ref_arg, h, lm_bits)
    a2, o2 = oracle.prefix_accept(am.cpu().numpy(), drafts, B, K)
    assert np.array_equal(acc.cpu().numpy(), a2) and np.array_equal(ot.cpu().numpy(), o2)

