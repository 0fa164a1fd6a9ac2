"""The row-by-row selection checker accepts the oracle's own selection and
rejects planted mistakes (on the CPU): a kept block swapped for one far below
the boundary, a count outside the rounding range, and an empty block kept."""
import numpy as np
import pytest

from oracle import prism_oracle as O
from tests.selection_check import check_head_selection


def _pooled(seed, nb=96, d=16):
    rng = np.random.default_rng(seed)
    return rng.normal(size=(nb, d)), rng.normal(size=(nb, d))


@pytest.mark.parametrize("k,tau", [(1, 0.05), (4, 0.2), (8, 0.5), (2, 1.0)])
def test_checker_accepts_the_oracle(k, tau):
    qp, kp = _pooled(k)
    ref = O.block_select(qp[None], kp[None], 0.7, k, tau)
    st = check_head_selection(ref["mask"][0], ref["kept"][0], qp, kp, 0.7, k, tau)
    assert st["exact"] == st["rows"] == 96


def test_checker_rejects_a_swap_far_from_the_boundary():
    qp, kp = _pooled(11)
    ref = O.block_select(qp[None], kp[None], 0.7, 4, 0.2)
    got, kept = ref["mask"][0].copy(), ref["kept"][0].copy()
    s = O.block_logits(qp[None], kp[None], 0.7)[0, 5]
    top, low = int(np.argmax(s)), int(np.argmin(s))
    got[5, top], got[5, low] = False, True  # the best block dropped for the worst: popcount unchanged
    with pytest.raises(AssertionError):
        check_head_selection(got, kept, qp, kp, 0.7, 4, 0.2)


def test_checker_rejects_a_count_outside_the_rounding_range():
    qp, kp = _pooled(12)
    ref = O.block_select(qp[None], kp[None], 0.7, 1, 0.3)
    got, kept = ref["mask"][0].copy(), ref["kept"][0].copy()
    s = O.block_logits(qp[None], kp[None], 0.7)[0, 7]
    order = np.lexsort((np.arange(s.size), -s))
    m = int(kept[7])
    got[7, order[m:m + 3]] = True  # three more blocks of the ranking: a larger prefix, far past tau
    kept[7] = m + 3
    with pytest.raises(AssertionError):
        check_head_selection(got, kept, qp, kp, 0.7, 1, 0.3)


def test_checker_rejects_a_kept_empty_block():
    qp, kp = _pooled(13)
    kp[9] = np.nan  # an empty key block
    ref = O.block_select(qp[None], kp[None], 0.7, 2, 0.2)
    got, kept = ref["mask"][0].copy(), ref["kept"][0].copy()
    assert not got[:, 9].any()
    got[3, 9] = True
    kept[3] += 1
    with pytest.raises(AssertionError):
        check_head_selection(got, kept, qp, kp, 0.7, 2, 0.2)
