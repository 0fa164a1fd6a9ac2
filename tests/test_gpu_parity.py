"""GPU parity: every C-ABI entry point against the fp64 CPU oracle.

Inputs come from the seeded generators in dynamic_block_sparse_shape_b200.synth
(or plain seeded torch draws) and are shared by both sides; expected values are
computed by ``oracle/`` only. Integer outputs (zone shapes, block masks, CSR)
are compared bit-exactly where the oracle's margins say the answer is robust
to rounding; floating outputs within max-abs 2e-2 / mean-abs 2e-3.
"""
import math

import numpy as np
import pytest
import torch

import dynamic_block_sparse_shape_b200 as P
from dynamic_block_sparse_shape_b200 import synth
from oracle import prism_oracle as O
from tests.gpu_util import (CDF_MARGIN, LOGIT_GAP, assert_close, csr_from_mask, f64, mask_bits_to_bool,
                            require_gpu, scale_for)
from tests.selection_check import check_head_selection

pytestmark = pytest.mark.gpu

CAND = tuple(synth.DEFAULT_CANDIDATES)


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _oracle_attention(q, k, v, do, blocks, mask, scale):
    N = q.shape[0]
    allowed = O.token_mask(mask, blocks, N)
    Oo, lse = O.masked_attention_fwd(q, k, v, allowed, scale)
    dq, dk, dv = O.masked_attention_bwd(q, k, v, Oo, lse, do, allowed, scale)
    return Oo, lse, dq, dk, dv


# The forward's two plans: "dense" (block images, long rows in the main kernel, the hint
# nnz unknown) and "sparse" (every row in the short-row kernel, K / V gathered through
# tensor maps; a hint of 0 kept pairs asks for it whatever the rows hold)
FWD_NNZ = {"dense": None, "sparse": 0}


def _check_attention(geo, zone_shape_np, q, k, v, do, mask, with_bwd=True, plan="dense"):
    """Run bsa_fwd / bsa_bwd on the CSR of `mask` and compare with the oracle."""
    dev = q.device
    H, d = q.shape[1], q.shape[2]
    sc = scale_for(d)
    blocks = O.block_tokens(geo.grid, geo.zone, geo.cand, zone_shape_np)
    zs = torch.tensor(zone_shape_np, dtype=torch.int32, device=dev)
    row_ptr, col_idx, nnz = csr_from_mask(mask, dev)
    ws = P.Workspace(dev)
    o_lo = torch.empty_like(q) if q.dtype == torch.bfloat16 else None
    o, lse = P.bsa_fwd(geo, zs, q, k, v, sc, row_ptr, col_idx, ws=ws, o_lo=o_lo, nnz=FWD_NNZ[plan])
    qd, kd, vd, dod = (f64(t) for t in (q, k, v, do))
    Or, lser, dqr, dkr, dvr = _oracle_attention(qd, kd, vd, dod, blocks, mask, sc)
    res = {"O": assert_close("O", f64(o), Or)}
    if o_lo is not None:
        # the rounding residual: below half a bf16 ulp of o (bf16-rounded itself), and o + o_lo
        # closer to the fp64 result than o alone
        ob, ol = f64(o), f64(o_lo)
        assert np.all(np.abs(ol) <= np.abs(ob) * 2.0 ** -8 * 1.01 + 1e-30)
        assert np.mean(np.abs(ob + ol - Or)) <= np.mean(np.abs(ob - Or)) + 1e-7
    lse_g = f64(lse)
    fin = np.isfinite(lser)
    assert np.array_equal(np.isfinite(lse_g), fin)
    res["lse"] = assert_close("LSE", lse_g[fin], lser[fin])
    if with_bwd:
        dq, dk, dv = P.bsa_bwd(geo, zs, q, k, v, o, lse, do, sc, row_ptr, col_idx, nnz, ws=ws, o_lo=o_lo)
        res["dQ"] = assert_close("dQ", f64(dq), dqr)
        res["dK"] = assert_close("dK", f64(dk), dkr)
        res["dV"] = assert_close("dV", f64(dv), dvr)
    P.check_device_status(ws)
    return res


# --------------------------------------------------------------------------- tiny
def test_tiny_end_to_end():
    """The fixed-shape fp32 workload: grid 4x8x8, one zone, (4,4,4), k=1, tau=0.2."""
    wl = synth.WORKLOADS["tiny"]
    x = synth.qkv(wl)  # CPU generator, fp32
    dev = torch.device("cuda")
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    geo = P.Geometry(wl.grid, wl.zone, tuple(synth.candidates_for(wl)))
    ws = P.Workspace(dev)
    zs, margin = P.zone_shapes(geo, ws=ws)
    idx_r, _, _ = O.zone_shapes(wl.grid, wl.zone, geo.cand)
    assert np.array_equal(zs.cpu().numpy(), idx_r)
    qp, kp = P.block_pool(geo, zs, q, k, ws=ws)
    blocks = O.block_tokens(wl.grid, wl.zone, geo.cand, idx_r)
    qpr, kpr = O.block_pool(f64(q), blocks), O.block_pool(f64(k), blocks)
    assert np.abs(f64(qp) - qpr).max() < 1e-5 and np.abs(f64(kp) - kpr).max() < 1e-5
    sc = scale_for(wl.head_dim)
    sel = P.block_select(qp, kp, sc, wl.top_k, wl.cdf_threshold, ws=ws)
    ref = O.block_select(qpr, kpr, sc, wl.top_k, wl.cdf_threshold)
    got = mask_bits_to_bool(sel["mask"], blocks.shape[0])
    assert np.array_equal(got, ref["mask"])
    assert np.array_equal(sel["kept"].cpu().numpy(), ref["kept"])
    # the GPU CSR lists the oracle's kept blocks in ascending order
    rp = sel["row_ptr"].cpu().numpy()
    ci = sel["col_idx"].cpu().numpy()
    H, nb = ref["kept"].shape
    for r in range(H * nb):
        assert ci[rp[r]:rp[r + 1]].tolist() == np.nonzero(ref["mask"].reshape(H * nb, nb)[r])[0].tolist()
    _check_attention(geo, idx_r, q, k, v, do, ref["mask"])
    _check_attention(geo, idx_r, q, k, v, do, ref["mask"], with_bwd=False, plan="sparse")


# --------------------------------------------------------------------------- attention
@pytest.mark.parametrize("plan", ["dense", "sparse"])
@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("density", [0.12, 0.5, 1.0])
def test_attention_random_masks_all_shapes(d, density, plan):
    """Every candidate shape in use, ragged rows (odd counts, one empty row)."""
    grid, zone = (8, 16, 24), (8, 8, 8)
    geo = P.Geometry(grid, zone, CAND)
    nz, nb = geo.counts()
    rng = np.random.default_rng(int(1000 * density) + d)
    zone_shape = np.arange(nz) % len(CAND)
    rng.shuffle(zone_shape)
    H = 2
    mask = rng.random((H, nb, nb)) < density
    mask[:, np.arange(nb), rng.integers(0, nb, nb)] = True
    mask[0, 3, :] = False  # an empty row
    mask[1, 5, :] = False
    mask[1, 5, 7] = True  # a single-block row
    gen = torch.Generator().manual_seed(7 + d)
    N = geo.n_tokens
    dev = torch.device("cuda")
    q, k, v, do = (torch.randn((N, H, d), generator=gen).to(torch.bfloat16).to(dev) for _ in range(4))
    _check_attention(geo, zone_shape, q, k, v, do, mask, plan=plan)


@pytest.mark.parametrize("plan", ["dense", "sparse"])
@pytest.mark.parametrize("d", [128, 64])
def test_attention_row_lengths_across_the_short_row_kernel(d, plan):
    """Rows of every length from 0 to 12 key blocks: in the dense plan the forward
    sends rows of at most eight blocks (four steps) to its short-row kernel and
    longer ones to the main kernel, so both run on the same data; the lengths
    cross the boundary, and odd lengths leave a half step. In the sparse plan the
    short-row kernel pipelines every row, empty ones in between."""
    grid, zone = (8, 16, 24), (8, 8, 8)
    geo = P.Geometry(grid, zone, CAND)
    nz, nb = geo.counts()
    rng = np.random.default_rng(40 + d)
    zone_shape = rng.integers(0, len(CAND), nz)
    H = 2
    mask = np.zeros((H, nb, nb), dtype=bool)
    for h in range(H):
        for i in range(nb):
            n = (i + 5 * h) % 13  # 0 .. 12 blocks
            mask[h, i, rng.choice(nb, size=n, replace=False)] = True
    gen = torch.Generator().manual_seed(70 + d)
    N = geo.n_tokens
    dev = torch.device("cuda")
    q, k, v, do = (torch.randn((N, H, d), generator=gen).to(torch.bfloat16).to(dev) for _ in range(4))
    _check_attention(geo, zone_shape, q, k, v, do, mask, plan=plan)


def test_attention_fp32_short_rows():
    """fp32 inputs and outputs (rounded to bf16 operands inside) with rows of 0 to
    12 key blocks at d = 128: the sparse plan's short-row forward and dQ kernels
    and the gathering dK/dV pass on their fp32 output paths."""
    grid, zone = (8, 16, 24), (8, 8, 8)
    geo = P.Geometry(grid, zone, CAND)
    nz, nb = geo.counts()
    rng = np.random.default_rng(57)
    zone_shape = rng.integers(0, len(CAND), nz)
    H, d = 2, 128
    mask = np.zeros((H, nb, nb), dtype=bool)
    for h in range(H):
        for i in range(nb):
            mask[h, i, rng.choice(nb, size=(3 * i + h) % 13, replace=False)] = True
    gen = torch.Generator().manual_seed(59)
    dev = torch.device("cuda")
    q, k, v, do = (torch.randn((geo.n_tokens, H, d), generator=gen).to(dev) for _ in range(4))
    _check_attention(geo, zone_shape, q, k, v, do, mask, plan="sparse")


@pytest.mark.parametrize("plan", ["dense", "sparse"])
def test_attention_strided_tokens(plan):
    """Q/K/V/O as views with a token stride larger than heads*head_dim."""
    grid, zone = (8, 8, 16), (8, 8, 8)
    geo = P.Geometry(grid, zone, CAND)
    nz, nb = geo.counts()
    H, d = 2, 128
    N = geo.n_tokens
    rng = np.random.default_rng(3)
    zone_shape = np.array([1, 5])
    mask = rng.random((H, nb, nb)) < 0.4
    mask[:, np.arange(nb), np.arange(nb)] = True
    dev = torch.device("cuda")
    gen = torch.Generator().manual_seed(11)
    base = torch.randn((N, 4, H, d), generator=gen).to(torch.bfloat16).to(dev)  # packed q|k|v|do
    q, k, v, do = base[:, 0], base[:, 1], base[:, 2], base[:, 3]
    blocks = O.block_tokens(grid, zone, CAND, zone_shape)
    zs = torch.tensor(zone_shape, dtype=torch.int32, device=dev)
    row_ptr, col_idx, nnz = csr_from_mask(mask, dev)
    sc = scale_for(d)
    o = torch.empty((N, 4, H, d), dtype=torch.bfloat16, device=dev)[:, 1]
    o, lse = P.bsa_fwd(geo, zs, q, k, v, sc, row_ptr, col_idx, out=o, nnz=FWD_NNZ[plan])
    Or, lser, _, _, _ = _oracle_attention(f64(q), f64(k), f64(v), f64(do), blocks, mask, sc)
    assert_close("O strided", f64(o), Or)


def test_attention_peaked_softmax():
    """Nearly one-hot softmax rows (Q, K scaled by 4; gradients of order 1-10):
    dS = P (dP - D) cancels, so D must come from O and its rounding residual,
    not from bf16 O alone. Compared row by row with the oracle, each element
    within max(2e-2, its bf16 rounding bound), mean-abs within 2e-3."""
    grid, zone = (8, 16, 16), (8, 8, 8)
    geo = P.Geometry(grid, zone, CAND)
    nz, nb = geo.counts()
    rng = np.random.default_rng(17)
    zone_shape = np.arange(nz) % len(CAND)
    H, d = 2, 128
    mask = rng.random((H, nb, nb)) < 0.3
    mask[:, np.arange(nb), np.arange(nb)] = True
    gen = torch.Generator().manual_seed(19)
    dev = torch.device("cuda")
    N = geo.n_tokens
    q = (4.0 * torch.randn((N, H, d), generator=gen)).to(torch.bfloat16).to(dev)
    k = (4.0 * torch.randn((N, H, d), generator=gen)).to(torch.bfloat16).to(dev)
    v, do = (torch.randn((N, H, d), generator=gen).to(torch.bfloat16).to(dev) for _ in range(2))
    sc = scale_for(d)
    blocks = O.block_tokens(grid, zone, CAND, zone_shape)
    zs = torch.tensor(zone_shape, dtype=torch.int32, device=dev)
    row_ptr, col_idx, nnz = csr_from_mask(mask, dev)
    ws = P.Workspace(dev)
    o_lo = torch.empty_like(q)
    o, lse = P.bsa_fwd(geo, zs, q, k, v, sc, row_ptr, col_idx, ws=ws, o_lo=o_lo)
    dq, dk, dv = P.bsa_bwd(geo, zs, q, k, v, o, lse, do, sc, row_ptr, col_idx, nnz, ws=ws, o_lo=o_lo)
    torch.cuda.synchronize()
    P.check_device_status(ws)
    qd, kd, vd, dod = (f64(t) for t in (q, k, v, do))
    parts = {n: ([], [], []) for n in ("O", "dQ", "dK", "dV")}
    for h in range(H):
        cache = {}
        for I in range(nb):
            rr = O.attention_block_rows(qd, kd, vd, blocks, np.nonzero(mask[h, I])[0], h, I, sc, dO=dod,
                                        bf16_bound=True)
            cache[(h, I)] = rr
            tk = torch.as_tensor(blocks[I], device=dev)
            for n, got, key in (("O", o, "O"), ("dQ", dq, "dQ")):
                parts[n][0].append(f64(got[tk, h]))
                parts[n][1].append(rr[key])
                parts[n][2].append(rr[key + "_bound"])
        for J in range(nb):
            gk, gv, bk, bv = O.attention_kv_block_grads(qd, kd, vd, dod, blocks, mask[h], h, J, sc, row_cache=cache,
                                                        bf16_bound=True)
            tk = torch.as_tensor(blocks[J], device=dev)
            for n, got, r, b in (("dK", dk, gk, bk), ("dV", dv, gv, bv)):
                parts[n][0].append(f64(got[tk, h]))
                parts[n][1].append(r)
                parts[n][2].append(b)
    for n, (g, r, b) in parts.items():
        assert_close(n, np.concatenate(g), np.concatenate(r), bound=np.concatenate(b))


# --------------------------------------------------------------------------- pooling
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_block_pool_all_shapes(dtype):
    grid, zone = (16, 16, 24), (8, 8, 8)
    geo = P.Geometry(grid, zone, CAND)
    nz, nb = geo.counts()
    zone_shape = np.arange(nz) % len(CAND)
    H, d = 24, 128
    gen = torch.Generator().manual_seed(5)
    dev = torch.device("cuda")
    q = torch.randn((geo.n_tokens, H, d), generator=gen).to(dtype).to(dev)
    k = torch.randn((geo.n_tokens, H, d), generator=gen).to(dtype).to(dev)
    zs = torch.tensor(zone_shape, dtype=torch.int32, device=dev)
    qp, kp = P.block_pool(geo, zs, q, k)
    blocks = O.block_tokens(grid, zone, CAND, zone_shape)
    assert np.abs(f64(qp) - O.block_pool(f64(q), blocks)).max() < 2e-6
    assert np.abs(f64(kp) - O.block_pool(f64(k), blocks)).max() < 2e-6


# --------------------------------------------------------------------------- selection
def _selection_parity(qp, kp, sc, top_k, tau, qpr, kpr, key_bias=None, key_bias_r=None):
    """GPU selection on (qp, kp[, key_bias]) against the oracle's selection on
    its own fp64 inputs (qpr, kpr[, key_bias_r]). top_k / tau are scalars (the
    plain entry point) or per-head lists (the _ex entry point)."""
    H, nb, _ = qp.shape
    per_head = not np.isscalar(top_k) or not np.isscalar(tau)
    if per_head or key_bias is not None:
        sel = P.block_select_ex(qp, kp, sc, top_k, tau, key_bias=key_bias)
    else:
        sel = P.block_select(qp, kp, sc, top_k, tau)
    ref = O.block_select(qpr, kpr, sc, top_k, tau, key_bias=key_bias_r)
    got = mask_bits_to_bool(sel["mask"], nb)
    kept = sel["kept"].cpu().numpy()
    qual = (ref["gap"] > LOGIT_GAP) & (ref["margin"] > CDF_MARGIN)
    assert np.array_equal(got[qual], ref["mask"][qual])
    assert np.array_equal(kept[qual], ref["kept"][qual])
    # every row: kept >= its head's k, popcount == kept;
    # empty blocks (NaN pooled features, grids clipped at an edge) take no part
    present = ~np.isnan(kpr).any(axis=2)
    empty_row = np.isnan(qpr).any(axis=2)
    ks = np.broadcast_to(np.asarray(top_k), (H,))
    floor = np.where(empty_row, 0, np.minimum(ks, present.sum(axis=1))[:, None])
    assert np.all(kept >= floor) and np.all(kept[empty_row] == 0)
    assert not (got & ~present[:, None, :]).any()
    assert np.array_equal(got.sum(axis=2), kept)
    # every row: one of the selections the rule admits within the stated rounding
    taus = np.broadcast_to(np.asarray(tau, dtype=np.float64), (H,))
    for h in range(H):
        check_head_selection(got[h], kept[h], qpr[h], kpr[h], sc, int(ks[h]), float(taus[h]),
                             key_bias=key_bias_r)
    # CSR matches the mask
    rp = sel["row_ptr"].cpu().numpy()
    assert rp[-1] == kept.sum() and sel["total"] == kept.sum()
    ci = sel["col_idx"].cpu().numpy()
    for r in range(0, H * nb, max(1, H * nb // 64)):
        assert ci[rp[r]:rp[r + 1]].tolist() == np.nonzero(got.reshape(H * nb, nb)[r])[0].tolist()
    return int(qual.sum()), qual.size


def _pooled_720p(heads=2, seed=None):
    """720p grid, Q/K from the workload's generator. The zone shapes are the
    oracle's rule applied to Q viewed as the feature input (as the 720p workload
    does), or with ``seed`` a seeded draw over all candidates; either way they
    are an input to both sides. Returns the GPU pooled features and the oracle's
    own fp64 pooling of the same Q/K."""
    import dataclasses
    wl = dataclasses.replace(synth.WORKLOADS["720p"], heads=heads)
    x = synth.qkv(wl)
    geo = P.Geometry(wl.grid, wl.zone, CAND)
    nz, _ = geo.counts()
    if seed is None:
        zone_shape, _, _ = O.zone_shapes(wl.grid, wl.zone, CAND, F=f64(x["q"].reshape(wl.n_tokens, -1)))
    else:
        zone_shape = np.random.default_rng(seed).integers(0, len(CAND), nz)
    dev = torch.device("cuda")
    q, k = x["q"].to(dev), x["k"].to(dev)
    zs = torch.tensor(zone_shape, dtype=torch.int32, device=dev)
    qp, kp = P.block_pool(geo, zs, q, k)
    blocks = O.block_tokens(wl.grid, wl.zone, CAND, zone_shape)
    return wl, geo, zs, zone_shape, blocks, qp, kp, O.block_pool(f64(x["q"]), blocks), O.block_pool(f64(x["k"]), blocks)


@pytest.fixture(scope="module")
def pooled_720p():
    return _pooled_720p()


@pytest.mark.parametrize("top_k,tau", [(1, 0.05), (4, 0.2), (16, 0.5), (4, 1.0), (4, 0.0), (2000, 0.2)])
def test_block_select_synthetic_720p_heads(top_k, tau, pooled_720p):
    wl, _, _, _, _, qp, kp, qpr, kpr = pooled_720p
    n_q, n = _selection_parity(qp, kp, scale_for(wl.head_dim), top_k, tau, qpr, kpr)
    assert n_q > 0.2 * n


def test_block_select_random_zone_shapes():
    """Pooled features over a seeded mix of all candidate shapes."""
    wl, _, _, _, _, qp, kp, qpr, kpr = _pooled_720p(heads=2, seed=21)
    _selection_parity(qp, kp, scale_for(wl.head_dim), 4, 0.2, qpr, kpr)
    _selection_parity(qp, kp, scale_for(wl.head_dim), [2, 8], [0.5, 0.1], qpr, kpr)


def test_block_select_ragged_block_count():
    """n_blocks not a multiple of 8 or 32 (tail rows and words)."""
    gen = torch.Generator().manual_seed(9)
    dev = torch.device("cuda")
    for nb in (37, 1, 65, 200):
        qp = torch.randn((3, nb, 64), generator=gen)
        kp = torch.randn((3, nb, 64), generator=gen)
        _selection_parity(qp.to(dev), kp.to(dev), 0.125, 3, 0.3, f64(qp), f64(kp))


@pytest.mark.slow
@pytest.mark.parametrize("nb,top_k,tau,amp", [(6000, 4, 0.2, 1.0), (7200, 16, 0.05, 3.0), (10240, 1, 0.5, 2.0)])
def test_block_select_large_block_counts(nb, top_k, tau, amp):
    """Block counts of the largest grids (7,200 blocks on the 2K latent grid),
    where each selection thread holds 48, 64 or 80 logits of its row; the last
    case also has empty blocks (NaN pooled features) spread over the row."""
    gen = torch.Generator().manual_seed(nb)
    dev = torch.device("cuda")
    qp = amp * torch.randn((1, nb, 128), generator=gen)
    kp = torch.randn((1, nb, 128), generator=gen)
    if nb == 10240:
        empty = torch.randperm(nb, generator=gen)[:97]
        qp[0, empty[:40]] = float("nan")
        kp[0, empty] = float("nan")
    _selection_parity(qp.to(dev), kp.to(dev), 1.0 / math.sqrt(128), top_k, tau, f64(qp), f64(kp))


def test_block_select_per_head_k_and_tau():
    """Per-head floors and thresholds (the ratio form gives the floors of two heads)."""
    wl, _, _, _, _, qp, kp, qpr, kpr = _pooled_720p(heads=4)
    nb = qp.shape[1]
    ks = [1, P.topk_from_sparsity(0.99, nb), P.topk_from_sparsity(0.9, nb), 4]
    assert ks[1:3] == [O.topk_from_sparsity(0.99, nb), O.topk_from_sparsity(0.9, nb)]
    taus = [0.05, 0.2, 0.5, 1.0]
    n_q, n = _selection_parity(qp, kp, scale_for(wl.head_dim), ks, taus, qpr, kpr)
    assert n_q > 0.2 * n
    # per-head arrays equal to the scalars reproduce the plain entry point bit for bit
    a = P.block_select(qp, kp, scale_for(wl.head_dim), 4, 0.2)
    b = P.block_select_ex(qp, kp, scale_for(wl.head_dim), [4] * 4, [0.2] * 4)
    assert torch.equal(a["mask"], b["mask"]) and torch.equal(a["col_idx"], b["col_idx"])


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_block_audio_bias_matches_oracle(dtype):
    import dataclasses
    wl = dataclasses.replace(synth.WORKLOADS["1080p"], grid=(16, 32, 48))
    dev = torch.device("cuda")
    R, _ = synth.a2v_residual(wl, device=dev)
    R = R.to(dtype)
    geo = P.Geometry(wl.grid, wl.zone, CAND)
    nz, nb = geo.counts()
    zone_shape = np.random.default_rng(23).integers(0, len(CAND), nz)
    zs = torch.tensor(zone_shape, dtype=torch.int32, device=dev)
    ws = P.Workspace(dev)
    blocks = O.block_tokens(wl.grid, wl.zone, CAND, zone_shape)
    for beta in (0.0, 2.0, -0.5):
        b = P.block_audio_bias(geo, zs, R, beta, ws=ws)
        ref = O.block_key_bias(f64(R), blocks, beta)
        assert np.allclose(f64(b), ref, rtol=1e-5, atol=1e-6), np.abs(f64(b) - ref).max()
    # strided residual rows (row stride 3072 + 64) and the zero residual
    Rs = torch.zeros((geo.n_tokens, 3136), dtype=dtype, device=dev)
    Rs[:, :3072] = R
    b = P.block_audio_bias(geo, zs, Rs[:, :3072], 2.0, ws=ws)
    assert np.allclose(f64(b), O.block_key_bias(f64(R), blocks, 2.0), rtol=1e-5, atol=1e-6)
    assert (P.block_audio_bias(geo, zs, torch.zeros_like(R), 2.0, ws=ws) == 0).all()
    P.check_device_status(ws)


def test_block_select_with_audio_bias_end_to_end():
    """720p Q/K with a synthetic a2v residual: bias from the residual norms on
    both sides, then the biased hybrid selection; the bias raises the loud
    blocks' share of the kept sets."""
    wl, geo, zs, zone_shape, blocks, qp, kp, qpr, kpr = _pooled_720p(heads=2)
    dev = torch.device("cuda")
    R, _ = synth.a2v_residual(wl, channels=768, device=dev)
    sc = scale_for(wl.head_dim)
    beta = 3.0
    b = P.block_audio_bias(geo, zs, R, beta)
    br = O.block_key_bias(f64(R), blocks, beta)
    n_q, n = _selection_parity(qp, kp, sc, 4, 0.2, qpr, kpr, key_bias=b, key_bias_r=br)
    assert n_q > 0.2 * n
    plain = mask_bits_to_bool(P.block_select(qp, kp, sc, 4, 0.2)["mask"], qp.shape[1])
    biased = mask_bits_to_bool(P.block_select_ex(qp, kp, sc, 4, 0.2, key_bias=b)["mask"], qp.shape[1])
    loud = br > np.quantile(br, 0.9)
    # the loud blocks' share of what the rows keep rises (the rows also keep
    # fewer blocks: the softmax mass concentrates on them)
    share = lambda m: m[:, :, loud].sum() / m.sum()
    assert share(biased) > share(plain) and biased.sum() <= plain.sum()


# --------------------------------------------------------------------------- grids that are not whole zones
PARTIAL_GRID, PARTIAL_ZONE = (10, 13, 9), (8, 8, 8)  # every zone axis clipped


def _partial_geometry(seed):
    geo = P.Geometry(PARTIAL_GRID, PARTIAL_ZONE, CAND)
    nz, nb = geo.counts()
    zone_shape = np.random.default_rng(seed).integers(0, len(CAND), nz)
    blocks = O.block_tokens(PARTIAL_GRID, PARTIAL_ZONE, CAND, zone_shape)
    return geo, nz, nb, zone_shape, blocks


@pytest.mark.parametrize("plan", ["dense", "sparse"])
@pytest.mark.parametrize("d", [128, 64])
def test_attention_partial_grid(d, plan):
    """Blocks clipped by the grid's edge (fewer than 64 member tokens) as queries
    and keys, empty blocks inside the selected sets, a row whose only selected
    block is empty (no keys: O = 0, LSE = -inf), forward and backward."""
    geo, nz, nb, zone_shape, blocks = _partial_geometry(31 + d)
    members = (blocks >= 0).sum(axis=1)
    assert (members == 0).any() and ((members > 0) & (members < 64)).any()
    rng = np.random.default_rng(d)
    H = 2
    mask = rng.random((H, nb, nb)) < 0.3
    mask[:, np.arange(nb), np.arange(nb)] = True
    e = int(np.nonzero(members == 0)[0][0])
    r = int(np.nonzero(members > 0)[0][1])
    mask[0, r, :] = False
    mask[0, r, e] = True  # only an empty block
    gen = torch.Generator().manual_seed(41 + d)
    N = geo.n_tokens
    dev = torch.device("cuda")
    q, k, v, do = (torch.randn((N, H, d), generator=gen).to(torch.bfloat16).to(dev) for _ in range(4))
    _check_attention(geo, zone_shape, q, k, v, do, mask, plan=plan)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_block_pool_partial_grid(dtype):
    geo, nz, nb, zone_shape, blocks = _partial_geometry(5)
    H, d = 4, 128
    gen = torch.Generator().manual_seed(6)
    dev = torch.device("cuda")
    q = torch.randn((geo.n_tokens, H, d), generator=gen).to(dtype)
    k = torch.randn((geo.n_tokens, H, d), generator=gen).to(dtype)
    zs = torch.tensor(zone_shape, dtype=torch.int32, device=dev)
    qp, kp = P.block_pool(geo, zs, q.to(dev), k.to(dev))
    for got, x in ((qp, q), (kp, k)):
        ref = O.block_pool(f64(x), blocks)
        g = f64(got)
        assert np.array_equal(np.isnan(g), np.isnan(ref))
        fin = ~np.isnan(ref)
        assert np.abs(g[fin] - ref[fin]).max() < 2e-6


def test_block_select_partial_grid():
    """Empty blocks are never kept and their rows are empty; clipped blocks
    take part like whole ones; per-head settings and the bias as well."""
    geo, nz, nb, zone_shape, blocks = _partial_geometry(7)
    H, d = 3, 64
    gen = torch.Generator().manual_seed(8)
    dev = torch.device("cuda")
    q = torch.randn((geo.n_tokens, H, d), generator=gen) + 1.5 * torch.randn((1, H, d), generator=gen)
    k = torch.randn((geo.n_tokens, H, d), generator=gen)
    zs = torch.tensor(zone_shape, dtype=torch.int32, device=dev)
    qp, kp = P.block_pool(geo, zs, q.to(dev), k.to(dev))
    qpr, kpr = O.block_pool(f64(q), blocks), O.block_pool(f64(k), blocks)
    sc = scale_for(d)
    for top_k, tau in ((1, 0.2), (3, 0.5), (100, 0.2), (2, 1.0)):
        _selection_parity(qp, kp, sc, top_k, tau, qpr, kpr)
    _selection_parity(qp, kp, sc, [1, 4, 2], [0.1, 0.3, 1.0], qpr, kpr)
    R = torch.randn((geo.n_tokens, 64), generator=gen) * torch.rand((geo.n_tokens, 1), generator=gen)
    b = P.block_audio_bias(geo, zs, R.to(dev), 2.0)
    br = O.block_key_bias(f64(R), blocks, 2.0)
    assert np.allclose(f64(b), br, rtol=1e-5, atol=1e-6)
    _selection_parity(qp, kp, sc, 2, 0.2, qpr, kpr, key_bias=b, key_bias_r=br)


def test_zone_shapes_partial_grid():
    """The real 720p latent rows (45 = 5 zones + 5) and a clipped t axis."""
    import dataclasses
    wl = dataclasses.replace(synth.WORKLOADS["720p-latent"], grid=(12, 45, 32))
    dev = torch.device("cuda")
    F = synth.video_features(wl, device=dev)
    R, _ = synth.a2v_residual(wl, device=dev)
    geo = P.Geometry(wl.grid, wl.zone, CAND)
    nz, _ = geo.counts()
    assert nz == 2 * 6 * 4
    for feat, res in ((F, R), (F, None), (None, R)):
        zs, margin = P.zone_shapes(geo, feat=feat, res=res)
        idx_r, margin_r, st = O.zone_shapes(wl.grid, wl.zone, CAND, F=None if feat is None else f64(feat),
                                            R=None if res is None else f64(res))
        got = zs.cpu().numpy()
        qual = margin_r > 1e-3
        assert qual.mean() > 0.5
        assert np.array_equal(got[qual], idx_r[qual])
        assert np.allclose(margin.cpu().numpy()[qual], margin_r[qual], rtol=1e-3, atol=1e-4)


# --------------------------------------------------------------------------- zone shapes
def test_zone_shapes_features_and_residual():
    import dataclasses
    wl = dataclasses.replace(synth.WORKLOADS["1080p"], grid=(16, 32, 48))
    dev = torch.device("cuda")
    F = synth.video_features(wl, device=dev)
    R, _ = synth.a2v_residual(wl, device=dev)
    geo = P.Geometry(wl.grid, wl.zone, CAND)
    for feat, res in ((F, R), (F, None), (None, R)):
        zs, margin = P.zone_shapes(geo, feat=feat, res=res)
        idx_r, margin_r, st = O.zone_shapes(wl.grid, wl.zone, CAND, F=None if feat is None else f64(feat),
                                            R=None if res is None else f64(res))
        got = zs.cpu().numpy()
        qual = margin_r > 1e-3
        assert qual.mean() > 0.5
        assert np.array_equal(got[qual], idx_r[qual])
        assert np.allclose(margin.cpu().numpy()[qual], margin_r[qual], rtol=1e-3, atol=1e-4)


def test_zone_shapes_fp32_features_match_bf16():
    dev = torch.device("cuda")
    import dataclasses
    wl = dataclasses.replace(synth.WORKLOADS["1080p"], grid=(8, 16, 32))
    F = synth.video_features(wl, device=dev)
    geo = P.Geometry(wl.grid, wl.zone, CAND)
    a, ma = P.zone_shapes(geo, feat=F)
    b, mb = P.zone_shapes(geo, feat=F.float())
    assert torch.equal(a, b)
