"""The argmax comparison rule of the GPU parity tests, on the CPU: a differing
argmax passes only as a certified near-tie (fp64 logit margin within
2^-14 x the sum of |h_i LM_vi| of the two rows), and any real margin fails."""
import numpy as np
import pytest

import oracle
from gpu_common import check_argmax


def _case():
    g = np.random.default_rng(5)
    hid = oracle.round_bf16_bits(g.normal(0, 1, (2, 1280)))
    lm = oracle.round_bf16_bits(g.normal(0, 0.02, (4, 1280)))
    # rows 0 and 1 equal and aligned with both hidden rows: they tie exactly and
    # hold the largest logit of both rows (the oracle takes the lower index, 0)
    aligned = oracle.widen(hid).sum(axis=0)
    lm[0] = lm[1] = oracle.round_bf16_bits(0.05 * aligned / np.abs(aligned).max())
    ref, _ = oracle.lm_head_argmax(hid, lm)
    assert np.array_equal(ref, [0, 0])
    return hid, lm, ref


def test_equal_answers_need_no_certificate():
    hid, lm, ref = _case()
    assert check_argmax(ref, ref, hid, lm) == 0


def test_exact_tie_is_certified():
    hid, lm, ref = _case()
    for r in range(2):  # index 1 is an equally good answer on either row
        other = ref.copy()
        other[r] = 1
        assert check_argmax(other, ref, hid, lm) == 1
    assert check_argmax(np.array([1, 1]), ref, hid, lm) == 2


def test_real_margin_fails():
    hid, lm, ref = _case()
    z = oracle.widen(hid) @ oracle.widen(lm).T
    for r in range(2):
        worst = int(np.argmin(z[r]))
        if worst != ref[r]:
            other = ref.copy()
            other[r] = worst
            with pytest.raises(AssertionError):
                check_argmax(other, ref, hid, lm)
            return
    pytest.fail("no row with a distinct worst logit")


def test_out_of_range_answer_fails():
    hid, lm, ref = _case()
    other = ref.copy()
    other[0] = lm.shape[0]
    with pytest.raises(AssertionError):
        check_argmax(other, ref, hid, lm)
