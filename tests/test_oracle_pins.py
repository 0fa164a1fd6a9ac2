"""Pins for the CPU oracle, independent of the oracle's own code paths.

Each test fixes a value from something other than the oracle itself: closed
forms, library routines (torch SDPA in fp64, scipy logsumexp), brute force over
subsets, finite differences, and invariants that follow from the Prism pages'
statements (finer blocks along axes of rapid variation; (4,4,4) is the
isotropic shape; (8,2,4) for vertical detail; (2,4,8) for fast motion; hybrid
top-k then CDF selection with default threshold 0.20).
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

from oracle import prism_oracle as O
from dynamic_block_sparse_shape_b200.synth import DEFAULT_CANDIDATES

CAND = list(DEFAULT_CANDIDATES)
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = line.split("=", 1)
                out[k.strip()] = v.strip()
    return out


# ----------------------------------------------------------------- tiling
def test_zone_tokens_are_a_partition():
    grid, zone = (8, 16, 24), (4, 8, 8)
    nz = np.prod(O.zone_counts(grid, zone))
    seen = np.concatenate([O.zone_token_ids(grid, zone, z).ravel() for z in range(nz)])
    assert np.array_equal(np.sort(seen), np.arange(np.prod(grid)))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_blocks_are_64_token_boxes_partitioning_the_grid(seed):
    grid, zone = (8, 16, 16), (8, 8, 8)
    rng = np.random.default_rng(seed)
    nz = np.prod(O.zone_counts(grid, zone))
    shape_idx = rng.integers(0, len(CAND), nz)
    blocks = O.block_tokens(grid, zone, CAND, shape_idx)
    T, H, W = grid
    assert np.array_equal(np.sort(blocks.ravel()), np.arange(T * H * W))
    for b, toks in enumerate(blocks):
        t, r = np.divmod(toks, H * W)
        h, w = np.divmod(r, W)
        ext = (t.max() - t.min() + 1, h.max() - h.min() + 1, w.max() - w.min() + 1)
        assert ext == CAND[shape_idx[b // 8]]
        # raster (t, h, w) order inside the block
        assert np.all(np.diff(toks) > 0)


def test_block_ids_explicit_444():
    # zone 8x8x8 on an 8x8x8 grid with (4,4,4): block 1 is the box w in 4..7.
    blocks = O.block_tokens((8, 8, 8), (8, 8, 8), [(4, 4, 4)], [0])
    assert blocks[0][:5].tolist() == [0, 1, 2, 3, 8]
    assert blocks[1][0] == 4 and blocks[2][0] == 32 and blocks[4][0] == 256
    assert blocks[7][-1] == 511


# ----------------------------------------------------------------- statistics
def test_line_variance_closed_forms():
    t = np.arange(8)[:, None, None, None] * np.ones((8, 8, 8, 1))
    # alternating sign along t: population variance 1 along t, 0 elsewhere
    V = O.line_variance((-1.0) ** t)
    assert np.allclose(V, [1.0, 0.0, 0.0], atol=1e-15)
    # linear ramp 0..7 along h: variance (8^2-1)/12
    h = np.arange(8)[None, :, None, None] * np.ones((8, 8, 8, 2))
    assert np.allclose(O.line_variance(h), [0.0, 63.0 / 12.0, 0.0], atol=1e-12)
    # two full periods of a quarter-wave along w: variance 1/2 for any phase
    w = np.arange(8)[None, None, :, None]
    X = np.sin(np.pi / 2 * w + np.array([0.3, 1.1, 2.9])[None, None, None, :]) * np.ones((8, 8, 8, 3))
    assert np.allclose(O.line_variance(X), [0.0, 0.0, 0.5], atol=1e-12)


def test_token_norms_closed_form():
    R = np.array([[3.0, 4.0, 0.0], [0.0, 0.0, 0.0], [1.0, 1.0, 1.0]])
    assert np.allclose(O.token_norms(R), [5.0, 0.0, math.sqrt(3.0)])


# ----------------------------------------------------------------- shape rule
def _choice(V, A=(0, 0, 0), m=0.0, mbar=1.0, cand=CAND):
    c = O.shape_cost(np.array(V, float), np.array(A, float), m, mbar, cand)
    return cand[int(np.argmin(c))]


def test_isotropic_zone_takes_444():
    g = _golden("pages_constants.txt")
    assert tuple(int(x) for x in g["isotropic_shape"].split(",")) == (4, 4, 4)
    assert _choice([1.0, 1.0, 1.0]) == (4, 4, 4)
    assert _choice([0.0, 0.0, 0.0]) == (4, 4, 4)


def test_named_shapes_of_the_walkthrough():
    g = _golden("pages_constants.txt")
    vertical = tuple(int(x) for x in g["vertical_detail_shape"].split(","))
    motion = tuple(int(x) for x in g["fast_motion_shape"].split(","))
    # h varies most, then w, then t: the vertical-detail shape
    assert _choice([0.5, 1.5, 1.0]) == vertical
    # t varies most, then h, then w: the fast-motion shape
    assert _choice([1.5, 1.0, 0.5]) == motion
    assert vertical in CAND and motion in CAND


def test_variation_along_one_axis_gives_finest_extent_there():
    for a in range(3):
        V = [0.0, 0.0, 0.0]
        V[a] = 1.0
        s = _choice(V)
        assert s[a] == min(c[a] for c in CAND)


def test_shape_rule_permutes_with_axes():
    rng = np.random.default_rng(5)
    for _ in range(200):
        V = rng.random(3)
        A = rng.random(3)
        base = _choice(V, A, m=2.5, mbar=1.0)
        for perm in itertools.permutations(range(3)):
            got = _choice(V[list(perm)], A[list(perm)], m=2.5, mbar=1.0)
            # candidate costs are distinct for random stats, so the argmin moves with the axes
            assert got == tuple(base[p] for p in perm)


def test_shape_rule_scale_invariant():
    rng = np.random.default_rng(6)
    for _ in range(100):
        V, A = rng.random(3), rng.random(3)
        m, mbar = 3.0 * rng.random(), 1.0
        ref = _choice(V, A, m, mbar)
        assert _choice(7.5 * V, A, m, mbar) == ref
        assert _choice(V, 0.01 * A, m, mbar) == ref
        assert _choice(V, 4.0 * A, 9.0 * m, 9.0 * mbar) == ref  # scaling R scales m and mbar alike


def test_audio_gate_only_acts_above_the_mean_norm():
    V = [1.0, 1.0, 1.0]
    A = [0.0, 1.0, 0.0]
    assert _choice(V, A, m=0.9, mbar=1.0) == (4, 4, 4)  # quieter than average: no audio term
    s = _choice(V, A, m=3.0, mbar=1.0)  # sounding zone with norm varying along h
    assert s[1] < 4  # finer along h


def test_finer_with_more_variation_monotone():
    rng = np.random.default_rng(7)
    for _ in range(200):
        V = rng.random(3)
        a = rng.integers(3)
        before = _choice(V)[a]
        V2 = V.copy()
        V2[a] *= 1.0 + 3.0 * rng.random()
        assert _choice(V2)[a] <= before


def test_zone_statistics_end_to_end_on_planted_zones():
    # two zones on a 8x8x16 grid: zone 0 oscillates along t, zone 1 along w.
    grid, zone = (8, 8, 16), (8, 8, 8)
    T, H, W = grid
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    F = np.where(w < 8, (-1.0) ** t, (-1.0) ** w).reshape(-1, 1) * np.ones((1, 4))
    idx, margin, st = O.zone_shapes(grid, zone, CAND, F=F)
    assert CAND[idx[0]] == (1, 8, 8) and CAND[idx[1]] == (8, 8, 1)
    assert np.allclose(st["V"][0], [1, 0, 0]) and np.allclose(st["V"][1], [0, 0, 1])
    assert np.all(margin > 0.1)
    # no signal at all: candidate 0 everywhere
    idx0, _, _ = O.zone_shapes(grid, zone, CAND)
    assert np.all(idx0 == 0)


# ----------------------------------------------------------------- shape rule, by value
# Cost vectors worked out by hand from the documented reading of the rule
# (README "Overview": finer partitioning along axes of rapid visual change and
# strong audio-visual coupling; walkthrough section "桥接残差反哺稀疏注意力":
# the a2v residual's per-token norm marks sounding regions, which get finer
# blocks). The reading: V^_a = 3 V_a / sum V, A^_a = 3 A_a / sum A, gate
# g = clip(m / mbar - 1, 0, 4), S = V^ + 1 * g * A^ renormalised to sum 3,
# cost(c) = sum_a S_a log2(ext_a) + 0.25 sum_a (log2(ext_a) - 2)^2.
# Every extent is a power of two, so each cost is an exact fraction; the
# derivations are written beside each case, and no value is computed by code.
# For the ten default candidates, in order, e = log2(ext) is
#   (2,2,2) (3,1,2) (3,2,1) (2,3,1) (1,3,2) (1,2,3) (2,1,3) (0,3,3) (3,0,3) (3,3,0)
# and the isotropy penalty 0.25 * sum (e-2)^2 is
#   0       0.5     0.5     0.5     0.5     0.5     0.5     1.5     1.5     1.5
SHAPE_COST_CASES = [
    # (a) features only, anisotropic: V = (1, 2, 5), sum 8 -> S = (3/8, 6/8, 15/8) (already sum 3).
    #     e.g. (8,8,1): 3*3/8 + 3*6/8 + 0 = 27/8, + 1.5 = 4.875; (8,4,2): 9/8 + 12/8 + 15/8 = 36/8, + 0.5 = 5.0
    dict(V=(1, 2, 5), A=(0, 0, 0), m=0.0, mbar=0.0, use_audio=False,
         cost=(6.0, 6.125, 5.0, 5.375, 6.875, 8.0, 7.625, 9.375, 8.25, 4.875), best=9, margin=0.125),
    # (b) isotropic features, sounding zone below the gate cap: V = (1,1,1) -> (1,1,1);
    #     A = (0, 3, 1) -> A^ = (0, 9/4, 3/4); m/mbar = 2 -> g = 1;
    #     S = (1, 13/4, 7/4), sum 6 -> renormalised (1/2, 13/8, 7/8).
    #     e.g. (8,2,4): 3/2 + 13/8 + 14/8 = 39/8, + 0.5 = 5.375; (8,1,8): 3/2 + 0 + 21/8 = 33/8, + 1.5 = 5.625
    dict(V=(1, 1, 1), A=(0, 3, 1), m=2.0, mbar=1.0, use_audio=True,
         cost=(6.0, 5.375, 6.125, 7.25, 7.625, 6.875, 5.75, 9.0, 5.625, 7.875), best=1, margin=0.25),
    # (c) as (b) but m/mbar = 7: m/mbar - 1 = 6 is capped at 4 -> S = (1, 1 + 9, 1 + 3) = (1, 10, 4),
    #     sum 15 -> renormalised (1/5, 2, 4/5).
    #     e.g. (8,1,8): 3/5 + 0 + 12/5 = 3, + 1.5 = 4.5; (8,2,4): 3/5 + 2 + 8/5 = 4.2, + 0.5 = 4.7
    dict(V=(1, 1, 1), A=(0, 3, 1), m=7.0, mbar=1.0, use_audio=True,
         cost=(6.0, 4.7, 5.9, 7.7, 8.3, 7.1, 5.3, 9.9, 4.5, 8.1), best=8, margin=0.2),
    # (d) anisotropic features and audio: V^ = (3/8, 6/8, 15/8); A = (2, 1, 1) -> A^ = (3/2, 3/4, 3/4);
    #     m/mbar = 3 -> g = 2; S = (27/8, 18/8, 27/8), sum 9 -> renormalised (9/8, 6/8, 9/8).
    #     The isotropic candidate wins: (4,4,4) 6.0 against (4,8,2) and (2,8,4) at 45/8 + 0.5 = 6.125
    dict(V=(1, 2, 5), A=(2, 1, 1), m=3.0, mbar=1.0, use_audio=True,
         cost=(6.0, 6.875, 6.5, 6.125, 6.125, 6.5, 6.875, 7.125, 8.25, 7.125), best=0, margin=0.125),
]


def _shape_cost_mismatches(cost_fn):
    """Differences between cost_fn and the hand-worked costs, argmins and margins."""
    bad = []
    for i, c in enumerate(SHAPE_COST_CASES):
        got = np.asarray(cost_fn(np.array(c["V"], float), np.array(c["A"], float), c["m"], c["mbar"], CAND,
                                 use_audio=c["use_audio"]), dtype=np.float64)
        if got.shape != (len(CAND),) or not np.allclose(got, c["cost"], rtol=0, atol=1e-9):
            bad.append((i, "cost", got.tolist()))
            continue
        if int(np.argmin(got)) != c["best"]:
            bad.append((i, "argmin", int(np.argmin(got))))
        if abs(float(np.sort(got)[1] - got.min()) - c["margin"]) > 1e-9:
            bad.append((i, "margin", float(np.sort(got)[1] - got.min())))
    return bad


def test_shape_cost_equals_hand_worked_values():
    assert _shape_cost_mismatches(O.shape_cost) == []


def test_choose_shapes_margin_equals_hand_worked_values():
    for c in SHAPE_COST_CASES:
        st = {"V": np.array([c["V"]], float), "A": np.array([c["A"]], float), "m": np.array([c["m"]]),
              "mbar": c["mbar"]}
        idx, margin = O.choose_shapes(st, CAND, have_features=True, have_residual=c["use_audio"])
        assert int(idx[0]) == c["best"] and abs(margin[0] - c["margin"]) < 1e-9


# Plausible slips in the cost: each must change at least one hand-worked value.
SHAPE_COST_MUTANTS = {
    "natural log for log2": ("np.log2(", "np.log("),
    "|e - 2| for (e - 2)^2": ("((e - 2.0) ** 2)", "np.abs(e - 2.0)"),
    "audio gate without its cap": ("min(max(m / mbar - 1.0, 0.0), gate_max)", "max(m / mbar - 1.0, 0.0)"),
    "no renormalisation to sum 3": ("S = 3.0 * S / tot if tot > 0 else np.ones(3)", "S = S"),
    "gate without the -1": ("m / mbar - 1.0", "m / mbar"),
    "gamma 1 for 0.25": ("gamma * ((e - 2.0)", "1.0 * ((e - 2.0)"),
    "audio term unweighted by the gate": ("S = Vh + w_audio * g * Ah", "S = Vh + w_audio * Ah"),
    "unnormalised feature variances": ("Vh = 3.0 * V / (V.sum() + EPS)", "Vh = V"),
}


@pytest.mark.parametrize("name", sorted(SHAPE_COST_MUTANTS))
def test_shape_cost_pins_catch_planted_mistakes(name):
    """Plants one slip into a copy of the oracle's cost (on the CPU) and checks
    that the hand-worked values reject it."""
    import inspect
    import textwrap
    src = textwrap.dedent(inspect.getsource(O.shape_cost))
    old, new = SHAPE_COST_MUTANTS[name]
    assert src.count(old) >= 1, f"mutation site not found: {old}"
    ns = dict(vars(O))
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)
    assert _shape_cost_mismatches(ns["shape_cost"]) != [], name


# ----------------------------------------------------------------- pooling
def test_pooling_of_a_linear_field_is_its_value_at_the_block_centre():
    grid, zone = (8, 8, 16), (8, 8, 8)
    T, H, W = grid
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    coef = np.array([[0.5, -1.0, 2.0, 0.25], [1.5, 0.0, -0.5, 3.0]])  # (a_t, a_h, a_w, c) per channel
    X = np.stack([coef[c, 0] * t + coef[c, 1] * h + coef[c, 2] * w + coef[c, 3] for c in range(2)], -1)
    X = X.reshape(-1, 1, 2)
    shape_idx = [1, 5]
    blocks = O.block_tokens(grid, zone, CAND, shape_idx)
    pooled = O.block_pool(X, blocks)  # [1, nb, 2]
    for b, toks in enumerate(blocks):
        tt, r = np.divmod(toks, H * W)
        hh, ww = np.divmod(r, W)
        centre = np.array([(tt.min() + tt.max()) / 2, (hh.min() + hh.max()) / 2, (ww.min() + ww.max()) / 2])
        expect = coef[:, :3] @ centre + coef[:, 3]
        assert np.allclose(pooled[0, b], expect, atol=1e-12)


# ----------------------------------------------------------------- grids that are not whole zones
PARTIAL_GRID, PARTIAL_ZONE = (10, 13, 9), (8, 8, 8)


def test_partial_grid_blocks_from_coordinates():
    """Every token of a 10x13x9 grid (zones 8x8x8, clipped at the far edges),
    placed by direct coordinate arithmetic, sits at its raster slot of its
    block's box; every token appears once and nothing else is a member."""
    T, H, W = PARTIAL_GRID
    nt, nh, nw = O.zone_counts(PARTIAL_GRID, PARTIAL_ZONE)
    assert (nt, nh, nw) == (2, 2, 2)
    rng = np.random.default_rng(4)
    idx = rng.integers(0, len(CAND), nt * nh * nw)
    blocks = O.block_tokens(PARTIAL_GRID, PARTIAL_ZONE, CAND, idx)
    assert blocks.shape == (8 * 8, 64)
    for t in range(T):
        for h in range(H):
            for w in range(W):
                z = ((t // 8) * nh + h // 8) * nw + w // 8
                bt, bh, bw = CAND[idx[z]]
                lt, lh, lw = (t % 8) // bt, (h % 8) // bh, (w % 8) // bw
                b = z * 8 + (lt * (8 // bh) + lh) * (8 // bw) + lw
                r = (((t % 8) % bt) * bh + (h % 8) % bh) * bw + (w % 8) % bw
                assert blocks[b, r] == (t * H + h) * W + w
    assert (blocks >= 0).sum() == T * H * W
    assert np.array_equal(np.sort(blocks[blocks >= 0]), np.arange(T * H * W))


def test_clipped_zone_line_variance_closed_forms():
    """Grid 8x8x11: the second zone along w holds columns 8..10. A feature
    equal to w gives V_w = (L^2 - 1)/12 with L the clipped line length (63/12
    in the full zone, 8/12 in the clipped one) and V_t = V_h = 0."""
    grid = (8, 8, 11)
    N = 8 * 8 * 11
    w = np.arange(N) % 11
    F = np.stack([w, 2.0 * w], axis=1).astype(np.float64)
    st = O.zone_statistics(grid, (8, 8, 8), F=F)
    assert st["V"].shape == (2, 3)
    assert np.allclose(st["V"][0], [0, 0, 2.5 * 63 / 12], atol=1e-12)  # channel mean of 1 and 4
    assert np.allclose(st["V"][1], [0, 0, 2.5 * 8 / 12], atol=1e-12)
    # zone mean of the residual norm over the member tokens only
    r = np.where(w >= 8, 3.0, 1.0)
    st = O.zone_statistics(grid, (8, 8, 8), r=r)
    assert np.allclose(st["m"], [1.0, 3.0]) and np.isclose(st["mbar"], (8 * 1 + 3 * 3) / 11)


def test_partial_block_pooling_is_the_field_at_the_member_centroid():
    T, H, W = PARTIAL_GRID
    tt, hh, ww = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    coef = np.array([[0.5, -1.0, 0.25, 2.0], [1.5, 0.5, -0.75, 0.0]])
    X = (coef[:, 0] * tt.reshape(-1, 1) + coef[:, 1] * hh.reshape(-1, 1) + coef[:, 2] * ww.reshape(-1, 1)
         + coef[:, 3])[:, None, :]  # [N, 1 head, 2 channels]
    idx = np.random.default_rng(8).integers(0, len(CAND), 8)
    blocks = O.block_tokens(PARTIAL_GRID, PARTIAL_ZONE, CAND, idx)
    pooled = O.block_pool(X, blocks)
    n_empty = 0
    for b in range(blocks.shape[0]):
        m = blocks[b][blocks[b] >= 0]
        if not m.size:
            assert np.isnan(pooled[0, b]).all()
            n_empty += 1
            continue
        t, h, w = m // (H * W), (m // W) % H, m % W
        c = np.array([t.mean(), h.mean(), w.mean()])
        assert np.allclose(pooled[0, b], coef[:, :3] @ c + coef[:, 3], atol=1e-12)
    assert n_empty > 0  # the draw leaves some boxes wholly outside the grid


def test_selection_skips_empty_blocks():
    """Grid 8x8x10, zones 8x8x8; the second zone takes (8,8,1), whose boxes at
    w >= 10 are empty: they are never kept and their rows are empty; on the
    other blocks the rule equals subset brute force."""
    grid, zone = (8, 8, 10), (8, 8, 8)
    cand = [(4, 4, 4), (8, 8, 1)]
    blocks = O.block_tokens(grid, zone, cand, [0, 1])
    empty = (blocks < 0).all(axis=1)
    assert empty.sum() == 6
    rng = np.random.default_rng(6)
    X = rng.normal(size=(8 * 8 * 10, 2, 6))
    Y = rng.normal(size=(8 * 8 * 10, 2, 6))
    qp, kp = O.block_pool(X, blocks), O.block_pool(Y, blocks)
    sc = 0.9
    for k, tau in ((1, 0.3), (3, 0.05), (20, 0.2), (2, 1.0)):
        r = O.block_select(qp, kp, sc, k, tau)
        assert not r["mask"][:, :, empty].any()
        assert (r["kept"][:, empty] == 0).all() and not r["mask"][:, empty].any()
        valid = np.nonzero(~empty)[0]
        for h in range(2):
            for i in valid:
                s = sc * kp[h, valid] @ qp[h, i]
                p = np.exp(s - s.max())
                p /= p.sum()
                want = {int(valid[j]) for j in _brute_force_selection_fast(p, k, tau)}
                assert set(np.nonzero(r["mask"][h, i])[0].tolist()) == want
        if tau >= 1.0:
            assert (r["kept"][:, valid] == valid.size).all()


def _brute_force_selection_fast(p, k, tau):
    """The subset rule on many blocks: the best subset of each size is the top
    of the sorted masses (ties to the lower index), so only prefixes are tried."""
    n = len(p)
    if k >= n or tau >= 1.0:
        return set(range(n))
    order = sorted(range(n), key=lambda j: (-p[j], j))
    c, m_min = 0.0, n
    for m in range(1, n + 1):
        c += p[order[m - 1]]
        if c >= tau:
            m_min = m
            break
    return set(order[:max(k, m_min)])


def test_partial_grid_dense_selection_is_full_attention():
    """Keeping every non-empty block of a 6x8x10 grid (zones 4x8x8, clipped)
    gives full softmax attention over all tokens (torch SDPA, fp64), through
    both the masked form and the row-gathered form."""
    grid, zone = (6, 8, 10), (4, 8, 8)
    cand = [(4, 4, 4), (2, 4, 8), (4, 8, 2), (1, 8, 8)]
    nz = int(np.prod(O.zone_counts(grid, zone)))
    idx = np.random.default_rng(2).integers(0, len(cand), nz)
    blocks = O.block_tokens(grid, zone, cand, idx)
    N, H, d = 6 * 8 * 10, 2, 8
    rng = np.random.default_rng(3)
    Q, K, V, dO = (rng.normal(size=(N, H, d)) for _ in range(4))
    qp, kp = O.block_pool(Q, blocks), O.block_pool(K, blocks)
    sc = 1 / math.sqrt(d)
    sel = O.block_select(qp, kp, sc, 1, 1.0)
    allowed = O.token_mask(sel["mask"], blocks, N)
    assert allowed.all()
    Oo, lse = O.masked_attention_fwd(Q, K, V, allowed, sc)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(Q).permute(1, 0, 2), torch.tensor(K).permute(1, 0, 2), torch.tensor(V).permute(1, 0, 2),
        scale=sc).permute(1, 0, 2).numpy()
    assert np.allclose(Oo, ref, atol=1e-12)
    dQ, dK, dV = O.masked_attention_bwd(Q, K, V, Oo, lse, dO, allowed, sc)
    nonempty = np.nonzero((blocks >= 0).any(axis=1))[0]
    cache = {}
    for b in nonempty[:: max(1, len(nonempty) // 6)]:
        m = O.block_members(blocks, b)
        rr = O.attention_block_rows(Q, K, V, blocks, np.nonzero(sel["mask"][1, b])[0], 1, b, sc, dO=dO)
        assert np.array_equal(rr["tokens"], m)
        assert np.allclose(rr["O"], Oo[m, 1], atol=1e-12) and np.allclose(rr["dQ"], dQ[m, 1], atol=1e-12)
        gk, gv = O.attention_kv_block_grads(Q, K, V, dO, blocks, sel["mask"][1], 1, b, sc, row_cache=cache)
        assert np.allclose(gk, dK[m, 1], atol=1e-12) and np.allclose(gv, dV[m, 1], atol=1e-12)


def test_partial_grid_audio_bias_uses_member_tokens():
    grid, zone = (8, 8, 10), (8, 8, 8)
    blocks = O.block_tokens(grid, zone, [(4, 4, 4), (8, 8, 1)], [0, 1])
    N = 640
    w = np.arange(N) % 10
    R = np.zeros((N, 3))
    R[:, 2] = np.where(w >= 8, 4.0, 1.0)  # the two clipped columns are loud
    b = O.block_key_bias(R, blocks, 1.0)
    mbar = (8 * 1 + 2 * 4) / 10
    assert np.allclose(b[:8], 1.0 / mbar)
    assert np.allclose(b[8:10], 4.0 / mbar) and (b[10:] == 0).all()


# ----------------------------------------------------------------- selection
def _brute_force_selection(p, k, tau):
    """Smallest m such that SOME subset of size m carries mass >= tau (the
    top-m subset carries the most), floored at k; the kept set is the size-m
    subset of largest mass. Enumerates all subsets."""
    n = len(p)
    if k >= n or tau >= 1.0:
        return set(range(n))
    best = {}
    for m in range(1, n + 1):
        best[m] = max(itertools.combinations(range(n), m), key=lambda S: sum(p[i] for i in S))
    m_min = next((m for m in range(1, n + 1) if sum(p[i] for i in best[m]) >= tau), n)
    return set(best[max(k, m_min)])


@pytest.mark.parametrize("seed", range(12))
def test_selection_matches_subset_brute_force(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(3, 10))
    s = rng.normal(0, 1.5, n)
    p = np.exp(s - s.max())
    p /= p.sum()
    for k in (1, 2, 3):
        for tau in (0.05, 0.2, 0.5, 0.9, 1.0):
            kept, m, m_star, gap, margin = O.select_row(s, k, tau)
            assert set(kept.tolist()) == _brute_force_selection(p, k, tau)
            assert m >= min(k, n)


def test_selection_invariants_and_special_cases():
    rng = np.random.default_rng(3)
    H, nb, d = 2, 16, 8
    qp, kp = rng.normal(size=(H, nb, d)), rng.normal(size=(H, nb, d))
    sc = 1 / math.sqrt(d)
    s = O.block_logits(qp, kp, sc)
    # tau = 1 or k = nb: dense
    assert O.block_select(qp, kp, sc, 1, 1.0)["mask"].all()
    assert O.block_select(qp, kp, sc, nb, 0.2)["mask"].all()
    # tau -> 0: exactly the k largest logits
    r = O.block_select(qp, kp, sc, 3, 1e-12)
    for h in range(H):
        for i in range(nb):
            top = set(np.argsort(-s[h, i], kind="stable")[:3].tolist())
            assert set(np.nonzero(r["mask"][h, i])[0].tolist()) == top
    # minimal prefix: C_{m*-1} < tau <= C_{m*}; kept >= k
    r = O.block_select(qp, kp, sc, 2, 0.3)
    for h in range(H):
        for i in range(nb):
            row = s[h, i]
            p = np.exp(row - row.max())
            p /= p.sum()
            kept = np.nonzero(r["mask"][h, i])[0]
            assert len(kept) >= 2
            order = np.argsort(-row, kind="stable")
            C = np.cumsum(p[order])
            m_star = int(np.searchsorted(C, 0.3)) + 1
            assert C[m_star - 1] >= 0.3 and (m_star == 1 or C[m_star - 2] < 0.3)
            assert len(kept) == max(2, m_star)


def test_default_cdf_threshold_from_the_pages():
    g = _golden("pages_constants.txt")
    assert float(g["cdf_threshold_default"]) == 0.20


def test_topk_from_sparsity_is_the_smallest_count_keeping_the_fraction():
    """k = the least count >= 1 whose share of the blocks is at least 1 - rho,
    checked in exact rational arithmetic on the float32 value of rho."""
    from fractions import Fraction
    rng = np.random.default_rng(5)
    cases = [(0.0, 10), (0.5, 10), (0.9, 4608), (0.75, 4608), (0.999, 10), (0.1, 10), (0.3, 10)]
    cases += [(float(rng.uniform(0, 1)), int(rng.integers(1, 6000))) for _ in range(200)]
    for rho, nb in cases:
        r32 = Fraction(float(np.float32(rho)))
        want = next(k for k in range(1, nb + 1) if Fraction(k, nb) >= 1 - r32)
        assert O.topk_from_sparsity(rho, nb) == want, (rho, nb)
    assert O.topk_from_sparsity(0.9, 4608) == 461
    assert O.topk_from_sparsity(0.0, 7) == 7
    for bad in (-0.1, 1.0, float("nan")):
        with pytest.raises(ValueError):
            O.topk_from_sparsity(bad, 10)


@pytest.mark.parametrize("seed", range(4))
def test_per_head_selection_matches_subset_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    H, nb, d = 3, 8, 4
    qp, kp = rng.normal(size=(H, nb, d)), rng.normal(0, 1.5, size=(H, nb, d))
    ks, taus = [1, 3, 2], [0.6, 0.05, 0.35]
    bias = rng.normal(0, 1.0, nb)
    for kb in (None, bias):
        r = O.block_select(qp, kp, 0.5, ks, taus, key_bias=kb)
        for h in range(H):
            for i in range(nb):
                s = 0.5 * np.array([qp[h, i] @ kp[h, j] for j in range(nb)])
                if kb is not None:
                    s = s + kb
                p = np.exp(s - s.max())
                p /= p.sum()
                want = _brute_force_selection(p, ks[h], taus[h])
                assert set(np.nonzero(r["mask"][h, i])[0].tolist()) == want


def test_key_bias_closed_form_on_two_blocks():
    """Grid 4x4x8 in one zone, shape (4,4,4): block 0 holds w < 4, block 1
    w >= 4. Residual rows c_n e_0 with |c| = 1 in block 0 and 3 in block 1
    (signs mixed): block means 1 and 3, grid mean 2."""
    grid, zone = (4, 4, 8), (4, 4, 8)
    blocks = O.block_tokens(grid, zone, [(4, 4, 4)], [0])
    N = 128
    R = np.zeros((N, 5))
    for n in range(N):
        w = n % 8
        R[n, 0] = (1.0 if w < 4 else 3.0) * (-1.0 if n % 3 == 0 else 1.0)
    b = O.block_key_bias(R, blocks, beta=2.0)
    assert np.allclose(b, [2.0 * 1 / 2, 2.0 * 3 / 2], rtol=0, atol=1e-15)
    # norms, not values: spreading the same norm over other channels leaves b unchanged
    R2 = np.zeros((N, 5))
    R2[:, 1] = R[:, 0] * 0.6
    R2[:, 3] = R[:, 0] * 0.8
    assert np.allclose(O.block_key_bias(R2, blocks, 2.0), b, atol=1e-14)
    # scale invariance and the zero residual
    assert np.allclose(O.block_key_bias(7.5 * R, blocks, 2.0), b, atol=1e-14)
    assert (O.block_key_bias(np.zeros((N, 5)), blocks, 2.0) == 0).all()


def test_key_bias_invariants_in_selection():
    rng = np.random.default_rng(11)
    H, nb, d = 2, 12, 8
    qp, kp = rng.normal(size=(H, nb, d)), rng.normal(size=(H, nb, d))
    sc = 1 / math.sqrt(d)
    base = O.block_select(qp, kp, sc, 2, 0.3)
    # a constant bias shifts every logit of a row equally: selection unchanged
    same = O.block_select(qp, kp, sc, 2, 0.3, key_bias=np.full(nb, 0.8))
    assert (same["mask"] == base["mask"]).all()
    # beta = 0: unchanged
    zero = O.block_select(qp, kp, sc, 2, 0.3, key_bias=np.zeros(nb))
    assert (zero["mask"] == base["mask"]).all()
    # one loud block with a large bias is kept by every row
    kb = np.zeros(nb)
    kb[5] = 40.0
    loud = O.block_select(qp, kp, sc, 1, 0.2, key_bias=kb)
    assert loud["mask"][:, :, 5].all()
    assert (loud["kept"] == 1).all()


# ----------------------------------------------------------------- attention
def _tiny_problem(seed=0, N=128, H=2, d=16, nblocks=None):
    rng = np.random.default_rng(seed)
    Q, K, V, dO = (rng.normal(size=(N, H, d)) for _ in range(4))
    return Q, K, V, dO


def _sdpa(Q, K, V, allowed, scale):
    q = torch.tensor(Q).permute(1, 0, 2)
    k = torch.tensor(K).permute(1, 0, 2)
    v = torch.tensor(V).permute(1, 0, 2)
    out = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=torch.tensor(allowed), scale=scale)
    return out.permute(1, 0, 2).numpy()


def test_dense_selection_equals_full_attention():
    Q, K, V, _ = _tiny_problem()
    N, H, d = Q.shape
    allowed = np.ones((H, N, N), bool)
    Oo, lse = O.masked_attention_fwd(Q, K, V, allowed, 1 / math.sqrt(d))
    assert np.allclose(Oo, _sdpa(Q, K, V, allowed, 1 / math.sqrt(d)), atol=1e-12)
    S = np.einsum("ihd,jhd->hij", Q, K) / math.sqrt(d)
    assert np.allclose(lse, logsumexp(S, axis=-1), atol=1e-12)


def test_masked_attention_matches_library_with_block_mask():
    grid, zone = (4, 8, 8), (4, 8, 8)
    rng = np.random.default_rng(1)
    N, H, d = 256, 2, 16
    Q, K, V = (rng.normal(size=(N, H, d)) for _ in range(3))
    blocks = O.block_tokens(grid, zone, [(4, 4, 4)], [0])
    bm = rng.random((H, 4, 4)) < 0.5
    bm[:, np.arange(4), rng.integers(0, 4, 4)] = True  # every row keeps a block
    allowed = O.token_mask(bm, blocks, N)
    sc = 1 / math.sqrt(d)
    Oo, lse = O.masked_attention_fwd(Q, K, V, allowed, sc)
    assert np.allclose(Oo, _sdpa(Q, K, V, allowed, sc), atol=1e-12)
    S = np.where(allowed, np.einsum("ihd,jhd->hij", Q, K) * sc, -np.inf)
    assert np.allclose(lse, logsumexp(S, axis=-1), atol=1e-12)


def test_masked_attention_backward_matches_autograd_and_finite_differences():
    rng = np.random.default_rng(2)
    N, H, d = 64, 1, 8
    Q, K, V, dO = (rng.normal(size=(N, H, d)) for _ in range(4))
    allowed = rng.random((H, N, N)) < 0.4
    allowed[:, np.arange(N), np.arange(N)] = True
    sc = 1 / math.sqrt(d)
    Oo, lse = O.masked_attention_fwd(Q, K, V, allowed, sc)
    dQ, dK, dV = O.masked_attention_bwd(Q, K, V, Oo, lse, dO, allowed, sc)
    # library autograd in fp64
    q, k, v = (torch.tensor(x).permute(1, 0, 2).requires_grad_(True) for x in (Q, K, V))
    out = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=torch.tensor(allowed), scale=sc)
    (out * torch.tensor(dO).permute(1, 0, 2)).sum().backward()
    assert np.allclose(dQ, q.grad.permute(1, 0, 2).numpy(), atol=1e-10)
    assert np.allclose(dK, k.grad.permute(1, 0, 2).numpy(), atol=1e-10)
    assert np.allclose(dV, v.grad.permute(1, 0, 2).numpy(), atol=1e-10)
    # central finite differences on a few coordinates
    def loss(Qx, Kx, Vx):
        return float((O.masked_attention_fwd(Qx, Kx, Vx, allowed, sc)[0] * dO).sum())
    h = 1e-6
    for (arr_i, grad) in ((0, dQ), (1, dK), (2, dV)):
        for _ in range(5):
            i, j = rng.integers(N), rng.integers(d)
            args = [Q.copy(), K.copy(), V.copy()]
            args[arr_i][i, 0, j] += h
            lp = loss(*args)
            args[arr_i][i, 0, j] -= 2 * h
            lm = loss(*args)
            assert abs((lp - lm) / (2 * h) - grad[i, 0, j]) < 1e-6


def test_sampled_rows_equal_masked_dense_form():
    grid, zone = (4, 8, 16), (4, 8, 8)
    rng = np.random.default_rng(4)
    N, H, d = 512, 2, 16
    Q, K, V, dO = (rng.normal(size=(N, H, d)) for _ in range(4))
    blocks = O.block_tokens(grid, zone, [(4, 4, 4)], [0, 0])
    nb = blocks.shape[0]
    bm = rng.random((H, nb, nb)) < 0.5
    bm[:, np.arange(nb), np.arange(nb)] = True
    sc = 1 / math.sqrt(d)
    allowed = O.token_mask(bm, blocks, N)
    Oo, lse = O.masked_attention_fwd(Q, K, V, allowed, sc)
    dQ, dK, dV = O.masked_attention_bwd(Q, K, V, Oo, lse, dO, allowed, sc)
    cache = {}
    for h in range(H):
        for I in range(nb):
            rr = O.attention_block_rows(Q, K, V, blocks, np.nonzero(bm[h, I])[0], h, I, sc, dO=dO)
            assert np.allclose(rr["O"], Oo[blocks[I], h], atol=1e-12)
            assert np.allclose(rr["lse"], lse[h, blocks[I]], atol=1e-12)
            assert np.allclose(rr["dQ"], dQ[blocks[I], h], atol=1e-12)
        for J in range(nb):
            gk, gv = O.attention_kv_block_grads(Q, K, V, dO, blocks, bm[h], h, J, sc, row_cache=cache)
            assert np.allclose(gk, dK[blocks[J], h], atol=1e-12)
            assert np.allclose(gv, dV[blocks[J], h], atol=1e-12)


def test_empty_selection_row_is_zero_with_no_gradient():
    rng = np.random.default_rng(8)
    N, H, d = 32, 1, 4
    Q, K, V, dO = (rng.normal(size=(N, H, d)) for _ in range(4))
    allowed = rng.random((H, N, N)) < 0.5
    allowed[0, 5, :] = False
    Oo, lse = O.masked_attention_fwd(Q, K, V, allowed, 0.5)
    assert np.all(Oo[5] == 0.0) and lse[0, 5] == -np.inf
    dQ, dK, dV = O.masked_attention_bwd(Q, K, V, Oo, lse, dO, allowed, 0.5)
    assert np.all(np.isfinite(dK)) and np.all(np.isfinite(dV)) and np.all(dQ[5] == 0.0)
    # removing the empty query changes no key gradient
    keep = np.arange(N) != 5
    O2, l2 = O.masked_attention_fwd(Q[keep], K, V, allowed[:, keep], 0.5)
    _, dK2, dV2 = O.masked_attention_bwd(Q[keep], K, V, O2, l2, dO[keep], allowed[:, keep], 0.5)
    assert np.allclose(dK, dK2) and np.allclose(dV, dV2)


def test_bf16_rounding_bound_covers_emulated_rounding():
    """The oracle's bf16 rounding bound holds for an explicit emulation of the
    roundings (P and dS rounded to bf16 as product operands, O / dQ / dK / dV
    rounded when stored) on peaked softmax rows, and it is tight enough that
    dropping one key block of a row breaks it."""
    import torch

    def bf16(x):
        return torch.tensor(x, dtype=torch.float64).to(torch.bfloat16).to(torch.float64).numpy()

    rng = np.random.default_rng(23)
    grid, zone, cand = (4, 8, 8), (4, 8, 8), ((4, 4, 4),)
    blocks = O.block_tokens(grid, zone, cand, np.zeros(1, dtype=np.int32))
    nb, N, H, d = blocks.shape[0], 256, 1, 64
    q = bf16(4.0 * rng.standard_normal((N, H, d)))
    k = bf16(4.0 * rng.standard_normal((N, H, d)))
    v = bf16(rng.standard_normal((N, H, d)))
    do = bf16(rng.standard_normal((N, H, d)))
    sc = 1.0 / np.sqrt(d)
    mask = np.ones((nb, nb), dtype=bool)
    I = 1
    rr = O.attention_block_rows(q, k, v, blocks, np.arange(nb), 0, I, sc, dO=do, bf16_bound=True)
    # emulation of the roundings, everything else exact
    qi, kj = blocks[I], blocks.reshape(-1)
    S = sc * q[qi, 0] @ k[kj, 0].T
    P = np.exp(S - S.max(axis=1, keepdims=True))
    l = P.sum(axis=1, keepdims=True)
    O_fp = (bf16(P) / l) @ v[kj, 0]  # O with P rounded for the product, before its storage rounding
    O_em = bf16(O_fp)
    dP = do[qi, 0] @ v[kj, 0].T
    D_em = (do[qi, 0] * O_fp).sum(axis=1)  # D from the computed O (stored with its rounding residual)
    dS = (P / l) * (dP - D_em[:, None])
    dQ_em = bf16(sc * bf16(dS) @ k[kj, 0])
    assert (P / l).max(axis=1).mean() > 0.5  # peaked rows
    for name, em, ref, bound in (("O", O_em, rr["O"], rr["O_bound"]), ("dQ", dQ_em, rr["dQ"], rr["dQ_bound"])):
        err = np.abs(em - ref)
        assert np.all(err <= 1.001 * bound + 1e-12), name
        assert bound.max() < 0.05 * np.abs(ref).max(), name  # not vacuous
    # a planted error: the same row with its last key block dropped
    bad = O.attention_block_rows(q, k, v, blocks, np.arange(nb - 1), 0, I, sc, dO=do)
    assert np.any(np.abs(bad["dQ"] - rr["dQ"]) > rr["dQ_bound"])
    # dK, dV of one key block over all query blocks
    J = 2
    dK, dV, bK, bV = O.attention_kv_block_grads(q, k, v, do, blocks, mask, 0, J, sc, bf16_bound=True)
    kb = blocks[J]
    dK_em = np.zeros_like(dK)
    dV_em = np.zeros_like(dV)
    for Iq in range(nb):
        r2 = O.attention_block_rows(q, k, v, blocks, np.arange(nb), 0, Iq, sc, dO=do)
        qq, dd = q[blocks[Iq], 0], do[blocks[Iq], 0]
        Sq = sc * qq @ k[kj, 0].T
        Pr = np.exp(Sq - Sq.max(axis=1, keepdims=True))
        D_q = (dd * ((bf16(Pr) / Pr.sum(axis=1, keepdims=True)) @ v[kj, 0])).sum(axis=1)
        Pq = np.exp(sc * qq @ k[kb, 0].T - r2["lse"][:, None])
        dSq = Pq * (dd @ v[kb, 0].T - D_q[:, None])
        dV_em += bf16(Pq).T @ dd
        dK_em += sc * bf16(dSq).T @ qq
    for name, em, ref, bound in (("dK", bf16(dK_em), dK, bK), ("dV", bf16(dV_em), dV, bV)):
        assert np.all(np.abs(em - ref) <= 1.001 * bound + 1e-12), name
