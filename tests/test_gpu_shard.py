"""The head-sharded layer through the CUDA library.

Every stage after the zone shapes reads one head only, so a layer shards by
heads with no exchange (the Prism walkthrough, section "实际案例与上手参考",
trains 1080p / 2K across several cards). Each rank owns a contiguous slice of
the heads (dynamic_block_sparse_shape_b200.shard.head_shard) as its own
contiguous tensors, and computes the zone shapes itself from the replicated
video features and a2v residual.

On a 2K-grid workload with four heads, split into the two slices of a
two-rank layer, this checks that:
* both "ranks" derive identical zone shapes;
* each slice's pooled features, selection (mask, counts, CSR), O, LSE, dQ, dK
  and dV are bit-identical to the full-head run's heads of that slice (every
  kernel reduces in a fixed order and reads only its own head);
* sampled rows of one slice match the fp64 oracle.
"""
import dataclasses
import math

import numpy as np
import pytest
import torch

import dynamic_block_sparse_shape_b200 as P
from dynamic_block_sparse_shape_b200 import synth
from dynamic_block_sparse_shape_b200.shard import head_shard
from oracle import prism_oracle as O
from tests.gpu_util import assert_close, f64, mask_bits_to_bool, require_gpu

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _layer(geo, x, feats, res, wl, sc):
    ws = P.Workspace(torch.device("cuda"))
    zs, _ = P.zone_shapes(geo, feat=feats, res=res, ws=ws)
    qp, kp = P.block_pool(geo, zs, x["q"], x["k"], ws=ws)
    sel = P.block_select(qp, kp, sc, wl.top_k, wl.cdf_threshold, ws=ws)
    o_lo = torch.empty_like(x["q"])
    o, lse = P.bsa_fwd(geo, zs, x["q"], x["k"], x["v"], sc, sel["row_ptr"], sel["col_idx"], ws=ws, o_lo=o_lo)
    dq, dk, dv = P.bsa_bwd(geo, zs, x["q"], x["k"], x["v"], o, lse, x["do"], sc, sel["row_ptr"], sel["col_idx"],
                           sel["total"], ws=ws, o_lo=o_lo)
    torch.cuda.synchronize()
    P.check_device_status(ws)
    return {"zs": zs, "qp": qp, "kp": kp, "sel": sel, "o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv}


def test_head_slices_reassemble_the_full_layer():
    require_gpu()
    dev = torch.device("cuda")
    wl = dataclasses.replace(synth.WORKLOADS["2k"], heads=4)
    cand = tuple(synth.candidates_for(wl))
    geo = P.Geometry(wl.grid, wl.zone, cand)
    nz, nb = geo.counts()
    sc = 1.0 / math.sqrt(wl.head_dim)
    x = synth.qkv(wl, device=dev)
    feats = synth.video_features(wl, device=dev)
    res = synth.a2v_residual(wl, device=dev)[0]
    full = _layer(geo, x, feats, res, wl, sc)
    world = 2
    for r in range(world):
        h0, h1 = head_shard(wl.heads, world, r)
        xs = {k: v[:, h0:h1].contiguous() for k, v in x.items()}  # the rank's own heads
        part = _layer(geo, xs, feats, res, dataclasses.replace(wl, heads=h1 - h0), sc)
        assert torch.equal(part["zs"], full["zs"]), "the ranks derive different zone shapes"
        for name in ("qp", "kp"):
            assert torch.equal(part[name], full[name][h0:h1]), name
        ps, fs = part["sel"], full["sel"]
        assert torch.equal(ps["mask"], fs["mask"][h0:h1]) and torch.equal(ps["kept"], fs["kept"][h0:h1])
        rp_full = fs["row_ptr"][h0 * nb:h1 * nb + 1]
        assert torch.equal(ps["row_ptr"], rp_full - rp_full[0])
        assert torch.equal(ps["col_idx"][:ps["total"]], fs["col_idx"][int(rp_full[0]):int(rp_full[-1])])
        assert torch.equal(part["lse"], full["lse"][h0:h1])
        for name in ("o", "dq", "dk", "dv"):
            assert torch.equal(part[name], full[name][:, h0:h1]), name
    # sampled rows of the last slice's first head against the oracle, where the
    # GPU selection of the row equals the oracle's
    h0, _ = head_shard(wl.heads, world, world - 1)
    zs = full["zs"].cpu().numpy()
    blocks = O.block_tokens(wl.grid, wl.zone, cand, zs)
    qh = x["q"][:, h0].to("cpu", torch.float64).numpy()[:, None, :]
    kh = x["k"][:, h0].to("cpu", torch.float64).numpy()[:, None, :]
    vh = x["v"][:, h0].to("cpu", torch.float64).numpy()[:, None, :]
    doh = x["do"][:, h0].to("cpu", torch.float64).numpy()[:, None, :]
    got = mask_bits_to_bool(full["sel"]["mask"][h0:h0 + 1], nb)[0]
    rng = np.random.default_rng(1)
    rows = rng.choice(nb, size=24, replace=False)
    ref = O.block_select(O.block_pool(qh, blocks), O.block_pool(kh, blocks), sc, wl.top_k, wl.cdf_threshold,
                         rows=[(0, int(I)) for I in rows])
    checked = 0
    for I in rows:
        if not np.array_equal(got[I], ref["mask"][0][I]) or checked == 4:
            continue
        rr = O.attention_block_rows(qh, kh, vh, blocks, np.nonzero(got[I])[0], 0, int(I), sc, dO=doh)
        tk = torch.as_tensor(O.block_members(blocks, int(I)), device=dev)
        assert_close("O", f64(full["o"][tk, h0]), rr["O"])
        assert_close("LSE", f64(full["lse"][h0, tk]), rr["lse"])
        assert_close("dQ", f64(full["dq"][tk, h0]), rr["dQ"])
        checked += 1
    assert checked == 4
