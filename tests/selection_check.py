"""Row-by-row check of a GPU block selection against the oracle's.

Several selections can be correct on a row whose answer sits within rounding of
a decision (hybrid rule, walkthrough section "三者如何协同": top-k, then extend
along the cumulative score mass until cdf_threshold). The check accepts exactly
those:

* the kept count m of the GPU lies in [m(tau - delta), m(tau + delta)], both
  taken from the oracle's fp64 cumulative mass (delta = the stated error of the
  GPU's mass sums);
* the kept set equals the oracle's top-m prefix (m the GPU's count) except for
  blocks whose oracle logits lie within ``logit_band`` of the logit at rank m;
* rows whose oracle margins are safe (boundary logit gap > LOGIT_GAP and mass
  margin > CDF_MARGIN) are bit-exact.

The reference selection, logits and m bounds all come from ``oracle/``.
"""
import numpy as np

from oracle import prism_oracle as O
from tests.gpu_util import CDF_MARGIN, LOGIT_GAP


def check_head_selection(got, kept, qpr_h, kpr_h, scale, top_k, tau, key_bias=None, logit_band=LOGIT_GAP,
                         cdf_delta=CDF_MARGIN):
    """got: bool [nb, nb] GPU kept sets of one head; kept: int [nb] GPU counts;
    qpr_h, kpr_h: the oracle's own fp64 pooled features [nb, d] of that head.
    Asserts the rules above and returns the row counts (exact, qualified,
    accepted through the m range, accepted through boundary swaps)."""
    nb = got.shape[0]
    ref = O.block_select(qpr_h[None], kpr_h[None], scale, top_k, tau, key_bias=key_bias)
    rmask, rkept = ref["mask"][0], ref["kept"][0]
    qual = (ref["gap"][0] > LOGIT_GAP) & (ref["margin"][0] > CDF_MARGIN)
    exact = np.all(got == rmask, axis=1) & (kept == rkept)
    assert exact[qual].all(), f"{int((~exact[qual]).sum())} qualified rows differ"
    assert np.array_equal(got.sum(axis=1), kept), "popcount differs from kept"
    present = ~np.isnan(kpr_h).any(axis=1)
    assert not (got & ~present[None, :]).any(), "an empty block was kept"
    valid = np.nonzero(present)[0]
    bias = np.zeros(nb) if key_bias is None else np.asarray(key_bias, np.float64)
    n_mrange = n_swap = 0
    for i in np.nonzero(~exact)[0]:
        assert not np.isnan(qpr_h[i]).any(), f"row {i}: an empty query row differs"
        s = scale * (kpr_h[valid] @ qpr_h[i]) + bias[valid]
        m_lo = O.select_row(s, top_k, max(tau - cdf_delta, 0.0))[1]
        m_hi = O.select_row(s, top_k, tau + cdf_delta)[1]
        m = int(kept[i])
        assert m_lo <= m <= m_hi, f"row {i}: kept {m} outside [{m_lo}, {m_hi}] (oracle {rkept[i]})"
        n_mrange += m != rkept[i]
        order = np.lexsort((np.arange(valid.size), -s))
        prefix = np.zeros(nb, dtype=bool)
        prefix[valid[order[:m]]] = True
        diff = got[i] ^ prefix
        if diff.any():
            boundary = s[order[m - 1]]
            sd = np.full(nb, np.nan)
            sd[valid] = s
            assert np.all(np.abs(sd[diff] - boundary) <= logit_band), (
                f"row {i}: blocks {np.nonzero(diff)[0][:8].tolist()} differ outside the boundary band")
            n_swap += 1
    return {"rows": nb, "exact": int(exact.sum()), "qualified": int(qual.sum()), "m_range": n_mrange,
            "swaps": n_swap}
