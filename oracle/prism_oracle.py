"""CPU oracle for the Prism dynamic block-sparse attention hot path (fp64).

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it. It shares no code with the
CUDA library; inputs come from ``dynamic_block_sparse_shape_b200.synth`` or
from the tests.

Sources (the method is described in prose only; no formula is printed):

* [README] "Tencent-Hunyuan/Prism" README, section "Overview": the token
  sequence is organised into spatiotemporal macro-zones; each zone's local
  structure is estimated from the video features' variance along the channel
  and from the norms of the audio-to-video cross-attention output; a tailored
  block shape is assigned per zone, finer along axes of fast visual change and
  strong audio-visual coupling; block-level features represent the blocks; a
  hybrid block selection fixes each query's sparsity.
* [WT-bridge] Prism architecture walkthrough (wmrh.cn/news/72296), section
  "桥接残差反哺稀疏注意力" (the bridge residual feeds sparse attention): the
  unscaled a2v residual's per-token L2 norm is the proxy of audio influence;
  sounding regions (large norm) get finer blocks.
* [WT-step] same walkthrough, section "三者如何协同" (how the three parts work in
  one denoising step): a candidate list of block shapes such as (4,4,4)
  isotropic, (8,2,4) for vertical detail (mouth/face), (2,4,8) for fast
  motion; one shape per zone from content variance and audio coupling; the
  gating step takes the k highest-scoring blocks, then extends along the CDF
  until ``cdf_threshold`` (default 0.20) is reached.
* [Sol-Attn] abstract on the "Prism: Dynamic Sparse Attention ..." paper page
  (thelatestinai.com/papers/2610.05416): dynamic sparse attention computes
  only selected key/value blocks, ranked by a block proxy score.

Where the pages leave a step open, the readings taken here are (R1..R21 in the
design notes):

* zones tile the grid in raster (zt, zh, zw) order; a shape is (bt, bh, bw);
  a grid that is not a whole number of zones is tiled as if rounded up, and
  zones and block boxes are clipped to it: statistics, pooling and attention
  use the member tokens only, and a box with no member is an empty block that
  takes no part in the selection (R16);
* V_a = mean over channels and over the lines parallel to axis a of the
  population variance of the feature channel along the line (R3);
* r(n) = ||R[n, :]||_2; A_a = mean over lines parallel to a of the population
  variance of r; audio gate g_z = clip(mean_z r / mean_grid r - 1, 0, G) (R4);
* S_a = 3 V_a/(sum V + eps) + w * g_z * 3 A_a/(sum A + eps), renormalised to
  sum 3; cost(c) = sum_a S_a log2(ext_a) + gamma sum_a (log2(ext_a) - 2)^2;
  the shape is the argmin, ties to the lower candidate index (R4, R12);
* blocks are raster over the zone's sub-grid, tokens raster inside a block;
  block id = zone id * blocks_per_zone + local id;
* pooled features are arithmetic means (R6); logits s = qbar . kbar / sqrt(d)
  (R7); blocks are ranked by (s descending, block index ascending), which is
  the softmax-probability order with ties to the lower index (R8, R12);
* m = max(k, min{m : C_m >= tau}), C_m the cumulative softmax mass of the top
  m; k >= n_blocks or tau >= 1 keeps every block (R8, R9);
* attention is exact softmax attention restricted to the selected blocks,
  scale 1/sqrt(d); gradients hold the selection fixed;
* optional scoring bias b_J = beta * mean_J r / mean_grid r added to every
  logit of key block J (R20); per-head k and tau, and a top-k sparsity ratio
  rho giving k = max(1, n_b - floor(rho n_b)) (R21).

Parity of the shape rule and of the candidate set with Prism's own code is
unpinned (the pages print neither); what is pinned is this documented rule.
"""
from __future__ import annotations

import math

import numpy as np

EPS = 1e-12
DEFAULT_W_AUDIO = 1.0
DEFAULT_GAMMA = 0.25
DEFAULT_GATE_MAX = 4.0


# --------------------------------------------------------------------------
# a1: macro-zone tiling  [README "Overview"]
# --------------------------------------------------------------------------
def zone_counts(grid, zone):
    """Number of zones along (t, h, w). Zones tile the grid rounded up to whole
    zones; where an extent is not a multiple of the zone, the last zone along that
    axis is clipped to the grid (reading R16)."""
    T, H, W = grid
    Zt, Zh, Zw = zone
    return -(-T // Zt), -(-H // Zh), -(-W // Zw)


def zone_token_ids(grid, zone, z):
    """Token ids of zone z as a [zt', zh', zw'] array (raster token order
    n = (t*H+h)*W+w); the extents are the zone's, clipped to the grid."""
    T, H, W = grid
    Zt, Zh, Zw = zone
    nt, nh, nw = zone_counts(grid, zone)
    zt, rem = divmod(z, nh * nw)
    zh, zw = divmod(rem, nw)
    t = np.arange(zt * Zt, min(T, zt * Zt + Zt))
    h = np.arange(zh * Zh, min(H, zh * Zh + Zh))
    w = np.arange(zw * Zw, min(W, zw * Zw + Zw))
    return (t[:, None, None] * H + h[None, :, None]) * W + w[None, None, :]


# --------------------------------------------------------------------------
# a2: zone statistics and shape choice  [README "Overview"; WT-bridge; WT-step]
# --------------------------------------------------------------------------
def line_variance(X):
    """For a zone array X [Zt, Zh, Zw, C]: for each axis a, the mean over channels
    and over all lines parallel to a of the population variance along the line."""
    X = np.asarray(X, dtype=np.float64)
    return np.array([X.var(axis=a).mean() for a in range(3)])


def token_norms(R):
    """r(n) = ||R[n, :]||_2 in fp64."""
    R = np.asarray(R, dtype=np.float64)
    return np.sqrt((R * R).sum(axis=1))


def zone_statistics(grid, zone, F=None, R=None, zones=None, r=None):
    """Per-zone statistics.

    Returns dict with V [nz, 3] (feature line variance per axis), A [nz, 3]
    (line variance of the residual norm per axis), m [nz] (zone mean of r) and
    mbar (grid mean of r). ``zones`` restricts the work to a subset (rows of
    the outputs follow that subset); ``r`` may pass precomputed token norms.
    """
    nt, nh, nw = zone_counts(grid, zone)
    nz = nt * nh * nw
    zl = list(range(nz)) if zones is None else list(zones)
    V = np.zeros((len(zl), 3))
    A = np.zeros((len(zl), 3))
    m = np.zeros(len(zl))
    mbar = 0.0
    if R is not None and r is None:
        r = token_norms(R)
    if r is not None:
        mbar = float(np.mean(r))
    for i, z in enumerate(zl):
        ids = zone_token_ids(grid, zone, z)
        if F is not None:
            V[i] = line_variance(np.asarray(F[ids.reshape(-1)], dtype=np.float64).reshape(ids.shape + (-1,)))
        if r is not None:
            rz = r[ids]
            A[i] = line_variance(rz[..., None])
            m[i] = rz.mean()
    return {"V": V, "A": A, "m": m, "mbar": mbar}


def shape_cost(V, A, m, mbar, cand, w_audio=DEFAULT_W_AUDIO, gamma=DEFAULT_GAMMA, gate_max=DEFAULT_GATE_MAX,
               use_audio=True):
    """Cost of every candidate for one zone (lower is better)."""
    V = np.asarray(V, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    Vh = 3.0 * V / (V.sum() + EPS)
    if use_audio and mbar > 0:
        Ah = 3.0 * A / (A.sum() + EPS)
        g = min(max(m / mbar - 1.0, 0.0), gate_max)
    else:
        Ah = np.zeros(3)
        g = 0.0
    S = Vh + w_audio * g * Ah
    tot = S.sum()
    S = 3.0 * S / tot if tot > 0 else np.ones(3)
    e = np.log2(np.asarray(cand, dtype=np.float64))  # [n_cand, 3]
    return e @ S + gamma * ((e - 2.0) ** 2).sum(axis=1)


def choose_shapes(stats, cand, have_features=True, have_residual=True, **params):
    """Shape index per zone (argmin of the cost, ties to the lower index) and
    the margin (second-best cost minus best). With neither features nor a
    residual every zone takes candidate 0."""
    nz = stats["V"].shape[0]
    idx = np.zeros(nz, dtype=np.int32)
    margin = np.full(nz, np.inf)
    if not have_features and not have_residual:
        return idx, margin
    for z in range(nz):
        c = shape_cost(stats["V"][z], stats["A"][z], stats["m"][z], stats["mbar"], cand,
                       use_audio=have_residual, **params)
        b = int(np.argmin(c))
        idx[z] = b
        if len(c) > 1:
            margin[z] = float(np.sort(c)[1] - c[b])
    return idx, margin


def zone_shapes(grid, zone, cand, F=None, R=None, zones=None, r=None, **params):
    """a2 end to end: statistics then choice. Returns (shape_idx, margin, stats)."""
    st = zone_statistics(grid, zone, F=F, R=R, zones=zones, r=r)
    idx, margin = choose_shapes(st, cand, have_features=F is not None,
                                have_residual=(R is not None or r is not None), **params)
    return idx, margin, st


# --------------------------------------------------------------------------
# a3: block partition and mean pooling  [README "Overview": block-level features]
# --------------------------------------------------------------------------
def blocks_per_zone(zone):
    vol = zone[0] * zone[1] * zone[2]
    if vol % 64:
        raise ValueError("zone volume is not a multiple of 64")
    return vol // 64


def block_tokens(grid, zone, cand, shape_idx):
    """Token ids [n_blocks, 64] of every block (tokens raster (t,h,w) inside the
    block's box). Blocks tile the zones of the rounded-up grid; a box position
    outside the grid holds -1, so an edge block has fewer than 64 members and a
    box wholly outside the grid is an empty block (reading R16)."""
    T, H, W = grid
    nt, nh, nw = zone_counts(grid, zone)
    nz = nt * nh * nw
    bpz = blocks_per_zone(zone)
    out = np.full((nz * bpz, 64), -1, dtype=np.int64)
    for z in range(nz):
        zt, rem = divmod(z, nh * nw)
        zh, zw = divmod(rem, nw)
        bt, bh, bw = cand[int(shape_idx[z])]
        if bt * bh * bw != 64 or zone[0] % bt or zone[1] % bh or zone[2] % bw:
            raise ValueError("candidate does not tile the zone with 64-token blocks")
        gt, gh, gw = zone[0] // bt, zone[1] // bh, zone[2] // bw
        for lt in range(gt):
            for lh in range(gh):
                for lw in range(gw):
                    local = (lt * gh + lh) * gw + lw
                    t = zt * zone[0] + lt * bt + np.arange(bt)
                    h = zh * zone[1] + lh * bh + np.arange(bh)
                    w = zw * zone[2] + lw * bw + np.arange(bw)
                    tt, hh, ww = np.meshgrid(t, h, w, indexing="ij")
                    ids = (tt * H + hh) * W + ww
                    ids[(tt >= T) | (hh >= H) | (ww >= W)] = -1
                    out[z * bpz + local] = ids.reshape(-1)
    return out


def block_members(blocks, b):
    """Token ids of block b that lie in the grid (raster order kept)."""
    row = np.asarray(blocks[b])
    return row[row >= 0]


def block_pool(X, blocks):
    """Mean of the member token rows of every block: X [N, heads, d] ->
    [heads, n_blocks, d]. An empty block has no feature: NaN (R16)."""
    X = np.asarray(X, dtype=np.float64)
    blocks = np.asarray(blocks)
    out = np.full((X.shape[1], blocks.shape[0], X.shape[2]), np.nan)
    for b in range(blocks.shape[0]):
        m = block_members(blocks, b)
        if m.size:
            out[:, b] = X[m].mean(axis=0)
    return out


# --------------------------------------------------------------------------
# a4 + a5: block scoring and hybrid top-k / CDF selection  [WT-step; Sol-Attn]
# --------------------------------------------------------------------------
def block_logits(qp, kp, scale):
    """s[h, I, J] = scale * qbar[h, I] . kbar[h, J]."""
    return scale * np.einsum("hid,hjd->hij", np.asarray(qp, np.float64), np.asarray(kp, np.float64))


def select_row(s, top_k, tau):
    """Hybrid selection for one query block.

    s: logits over all key blocks. Returns (kept indices ascending, m, m_star,
    logit_gap, cdf_margin) where the gap is s_(m) - s_(m+1) in the ranked
    order. The margin says how far the cumulative mass is from changing m:
    min(|C_{m*} - tau|, |C_{m*-1} - tau|) when the crossing decides m
    (m* >= k), else C_k - tau.
    """
    s = np.asarray(s, dtype=np.float64)
    n = s.shape[0]
    order = np.lexsort((np.arange(n), -s))  # s descending, index ascending
    p = np.exp(s - s.max())
    p = p / p.sum()
    C = np.cumsum(p[order])
    if top_k >= n or tau >= 1.0:
        return np.arange(n), n, n, math.inf, math.inf
    reach = np.nonzero(C >= tau)[0]
    m_star = int(reach[0]) + 1 if reach.size else n
    m = max(int(top_k), m_star)
    kept = np.sort(order[:m])
    gap = float(s[order[m - 1]] - s[order[m]]) if m < n else math.inf
    if m_star < top_k:
        # the floor k decides m; it stays decided while C_k stays above tau
        margin = float(C[int(top_k) - 1] - tau)
    else:
        c_hi = C[m_star - 1]
        c_lo = C[m_star - 2] if m_star >= 2 else 0.0
        margin = float(min(abs(c_hi - tau), abs(c_lo - tau)))
    return kept, m, m_star, gap, margin


def block_select(qp, kp, scale, top_k, tau, rows=None, key_bias=None):
    """Selection for every (head, query block) or for ``rows`` = list of (h, I).

    ``top_k`` and ``tau`` are scalars or per-head sequences of length heads
    (R21: each head keeps its own floor and mass threshold). ``key_bias`` is
    None or [nb]: b_J added to every head's logit of key block J before the
    ranking and the softmax (R20, the audio-norm scoring bias).

    A block whose pooled feature is NaN (an empty block, R16) takes no part: as
    a key it is never kept and carries no mass; as a query its row is empty
    (kept 0). The rule then runs over the other key blocks, so "k >= n_blocks"
    and "tau >= 1" keep every non-empty block.

    Returns dict: mask bool [heads, nb, nb] (only selected rows filled when
    ``rows`` is given), kept [heads, nb] (-1 where not computed), gap and
    margin arrays (nan where not computed).
    """
    qp = np.asarray(qp, np.float64)
    kp = np.asarray(kp, np.float64)
    H, nb, _ = qp.shape
    ks = np.broadcast_to(np.asarray(top_k, dtype=np.int64), (H,))
    taus = np.broadcast_to(np.asarray(tau, dtype=np.float64), (H,))
    bias = np.zeros(nb) if key_bias is None else np.asarray(key_bias, np.float64).reshape(nb)
    mask = np.zeros((H, nb, nb), dtype=bool)
    kept = np.full((H, nb), -1, dtype=np.int64)
    gap = np.full((H, nb), np.nan)
    margin = np.full((H, nb), np.nan)
    if rows is None:
        rows = [(h, i) for h in range(H) for i in range(nb)]
    present = {}  # per head: the key blocks that take part, and their pooled features and biases
    for h, i in rows:
        if np.isnan(qp[h, i]).any():
            kept[h, i] = 0
            gap[h, i] = margin[h, i] = math.inf
            continue
        if h not in present:
            v = np.nonzero(~np.isnan(kp[h]).any(axis=1))[0]
            present[h] = (v, kp[h, v], bias[v])
        valid, kv, bv = present[h]
        s = scale * (kv @ qp[h, i]) + bv
        idx, m, _, g, mg = select_row(s, int(ks[h]), float(taus[h]))
        idx = valid[idx]
        mask[h, i, idx] = True
        kept[h, i] = m
        gap[h, i] = g
        margin[h, i] = mg
    return {"mask": mask, "kept": kept, "gap": gap, "margin": margin}


def topk_from_sparsity(rho, n_blocks):
    """Top-k floor from a top-k sparsity ratio [WT-step, section "实际案例与上手参考":
    ``BSA_SPARSITY`` switches the block-sparse attention on and sets its top-k
    sparsity ratio].

    Reading R21: the ratio is the fraction of key blocks the top-k part drops,
    so k = n_blocks - floor(rho * n_blocks), at least 1. rho is taken as a
    float32 (the precision the library's argument has) and the product is
    formed in fp64. 0 <= rho < 1.
    """
    rho = float(np.float32(rho))
    if not (0.0 <= rho < 1.0):
        raise ValueError("sparsity ratio must lie in [0, 1)")
    return max(1, int(n_blocks) - int(math.floor(rho * int(n_blocks))))


def block_key_bias(R, blocks, beta):
    """Audio-norm bias of every key block [WT-bridge: the per-token L2 norm of
    the unscaled a2v residual is the proxy of audio influence, and the walkthrough
    says it is taken "during BSA scoring"; sounding regions keep more attention].

    Reading R20: b_J = beta * (mean over the 64 tokens n of block J of r(n)) /
    (mean over all tokens of r(n)), r(n) = ||R[n, :]||_2. The ratio makes the
    bias independent of the residual's scale; adding b_J to the logits raises
    the proxy probability of key blocks with a strong audio coupling. A zero
    residual gives b = 0.
    """
    r = token_norms(R)
    blocks = np.asarray(blocks)
    mean_grid = r.mean()
    out = np.zeros(blocks.shape[0])
    if mean_grid == 0.0:
        return out
    for b in range(blocks.shape[0]):
        m = block_members(blocks, b)
        if m.size:  # an empty block keeps 0 (it is never selected)
            out[b] = beta * r[m].mean() / mean_grid
    return out


# --------------------------------------------------------------------------
# a6 + a7: block-sparse attention, explicitly masked dense form  [Sol-Attn]
# --------------------------------------------------------------------------
def token_block_index(blocks, n_tokens):
    """Block id of every token."""
    b = np.full(n_tokens, -1, dtype=np.int64)
    for i, row in enumerate(blocks):
        row = np.asarray(row)
        b[row[row >= 0]] = i
    return b


def token_mask(block_mask, blocks, n_tokens):
    """allowed[h, i, j] = block_mask[h, block(i), block(j)]."""
    tb = token_block_index(blocks, n_tokens)
    return block_mask[:, tb][:, :, tb]


def masked_attention_fwd(Q, K, V, allowed, scale):
    """O [N, heads, d] and LSE [heads, N] of softmax attention with logits
    scale * q.k set to -inf where ``allowed`` is False. A query with no allowed
    key (an empty selection, which the hybrid rule never produces since
    k >= 1) gets O = 0 and LSE = -inf, and contributes no gradient."""
    Qh, Kh, Vh = (np.asarray(x, np.float64).transpose(1, 0, 2) for x in (Q, K, V))  # [heads, N, d]
    S = scale * (Qh @ Kh.transpose(0, 2, 1))
    S = np.where(allowed, S, -np.inf)
    empty = ~np.asarray(allowed).any(axis=-1, keepdims=True)  # a query with no selected key
    mx = np.where(empty, 0.0, S.max(axis=-1, keepdims=True))
    P = np.exp(S - mx)
    l = P.sum(axis=-1, keepdims=True)
    O = (np.where(empty, 0.0, P / np.where(empty, 1.0, l)) @ Vh).transpose(1, 0, 2)
    with np.errstate(divide="ignore"):
        lse = np.where(empty, -np.inf, mx + np.log(l))[..., 0]
    return O, lse


def masked_attention_bwd(Q, K, V, O, lse, dO, allowed, scale):
    """dQ, dK, dV of the masked attention with the mask held fixed."""
    Qh, Kh, Vh, Oh, dOh = (np.asarray(x, np.float64).transpose(1, 0, 2) for x in (Q, K, V, O, dO))
    S = scale * (Qh @ Kh.transpose(0, 2, 1))
    with np.errstate(over="ignore", invalid="ignore"):
        P = np.where(allowed, np.exp(S - np.asarray(lse, np.float64)[..., None]), 0.0)
    dV = P.transpose(0, 2, 1) @ dOh
    dP = dOh @ Vh.transpose(0, 2, 1)
    D = (dOh * Oh).sum(axis=-1)
    dS = P * (dP - D[..., None])
    dQ = scale * (dS @ Kh)
    dK = scale * (dS.transpose(0, 2, 1) @ Qh)
    return dQ.transpose(1, 0, 2), dK.transpose(1, 0, 2), dV.transpose(1, 0, 2)


# --------------------------------------------------------------------------
# Sampled rows for large grids: the same sums restricted to the unmasked
# columns (masked terms are exactly zero, so this equals the masked form).
# --------------------------------------------------------------------------
# Unit roundoff of bf16 (8 significant bits, round to nearest).
BF16_U = 2.0 ** -8


def attention_block_rows(Q, K, V, blocks, kept_blocks, h, I, scale, dO=None, bf16_bound=False):
    """O, LSE (and dQ, D when dO is given) for the 64 query tokens of block I of head h.

    With ``bf16_bound``, also the elementwise worst-case effect of the bf16
    roundings a bf16 tensor-core implementation performs on top of exact
    arithmetic: P rounded for the P V product and O rounded when stored
    (``O_bound``); D formed from that computed O (``D_bound``), which enters
    dS = P (dP - D); dS rounded for the dS K product and dQ rounded when
    stored (``dQ_bound``). First order in the unit roundoff; a tolerance
    model, not a reference value."""
    qi = block_members(blocks, I)
    kj = np.asarray(blocks)[np.asarray(kept_blocks, dtype=np.int64)].reshape(-1)
    kj = kj[kj >= 0]
    q = np.asarray(Q[qi, h], np.float64)
    k = np.asarray(K[kj, h], np.float64)
    v = np.asarray(V[kj, h], np.float64)
    S = scale * q @ k.T
    mx = S.max(axis=1, keepdims=True)
    P = np.exp(S - mx)
    l = P.sum(axis=1, keepdims=True)
    O = (P / l) @ v
    lse = (mx + np.log(l))[:, 0]
    out = {"O": O, "lse": lse, "tokens": qi}
    if bf16_bound:
        out["O_bound"] = BF16_U * ((P / l) @ np.abs(v) + np.abs(O))
    if dO is not None:
        do = np.asarray(dO[qi, h], np.float64)
        Pn = P / l
        D = (do * O).sum(axis=1)
        dP = do @ v.T
        dS = Pn * (dP - D[:, None])
        out["dQ"] = scale * dS @ k
        out["D"] = D
        if bf16_bound:
            bD = BF16_U * (np.abs(do) * (Pn @ np.abs(v))).sum(axis=1)
            out["D_bound"] = bD
            out["dQ_bound"] = (BF16_U * (scale * np.abs(dS) @ np.abs(k) + np.abs(out["dQ"])) +
                               scale * bD[:, None] * (Pn @ np.abs(k)))
    return out


def attention_kv_block_grads(Q, K, V, dO, blocks, sel_mask_h, h, J, scale, row_cache=None, bf16_bound=False):
    """dK, dV for the 64 key tokens of block J of head h.

    ``sel_mask_h`` [nb, nb] is the head's block mask; every query block I that
    selected J contributes, with its own LSE and D = rowsum(dO * O) computed
    from its full selected set. With ``bf16_bound`` the result is
    (dK, dV, dK_bound, dV_bound): the worst-case effect of rounding P^T and
    dS^T to bf16 for the products and dK, dV when stored (see
    attention_block_rows).
    """
    kj = block_members(blocks, J)
    k = np.asarray(K[kj, h], np.float64)
    v = np.asarray(V[kj, h], np.float64)
    dK = np.zeros_like(k)
    dV = np.zeros_like(v)
    bK = np.zeros_like(k)
    bV = np.zeros_like(v)
    bKD = np.zeros_like(k)  # through D formed from the computed O (already carries the unit roundoff)
    for I in np.nonzero(sel_mask_h[:, J])[0]:
        key = (h, int(I))
        if row_cache is not None and key in row_cache:
            rr = row_cache[key]
        else:
            rr = attention_block_rows(Q, K, V, blocks, np.nonzero(sel_mask_h[I])[0], h, int(I), scale, dO=dO)
            if row_cache is not None:
                row_cache[key] = rr
        qi = block_members(blocks, I)
        q = np.asarray(Q[qi, h], np.float64)
        do = np.asarray(dO[qi, h], np.float64)
        S = scale * q @ k.T
        P = np.exp(S - rr["lse"][:, None])
        dV += P.T @ do
        dP = do @ v.T
        dS = P * (dP - rr["D"][:, None])
        dK += scale * dS.T @ q
        if bf16_bound:
            if "D_bound" in rr:
                bD = rr["D_bound"]
            else:
                ks_ = np.asarray(blocks)[np.nonzero(sel_mask_h[I])[0]].reshape(-1)
                ks_ = ks_[ks_ >= 0]
                Pn_ = np.exp(scale * q @ np.asarray(K[ks_, h], np.float64).T - rr["lse"][:, None])
                bD = BF16_U * (np.abs(do) * (Pn_ @ np.abs(np.asarray(V[ks_, h], np.float64)))).sum(axis=1)
            bV += P.T @ np.abs(do)
            bK += scale * np.abs(dS).T @ np.abs(q)
            bKD += scale * P.T @ (bD[:, None] * np.abs(q))
    if bf16_bound:
        return dK, dV, BF16_U * (bK + np.abs(dK)) + bKD, BF16_U * (bV + np.abs(dV))
    return dK, dV
