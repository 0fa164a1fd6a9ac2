"""prism_zone_shapes_static: the zone-shape entry point that allocates nothing.

It exists for callers that may not allocate device memory while they run:
code hosted by a framework that owns every device allocation (a serving
runtime's fixed pool, a plugin interface that passes no scratch buffer), or
code that must not call cudaMalloc mid-work because it synchronises the
device. Its scratch is a static device array inside the library. This test
calls it through the C ABI three times in a row, with different inputs (a
smaller grid with a residual last, after a larger one), and checks each result
against the workspace entry point prism_zone_shapes, which runs the same
kernels: shapes and margins bit-identical. It sits in a file of its own,
collected last.
"""
import ctypes
import dataclasses

import numpy as np
import pytest
import torch

import dynamic_block_sparse_shape_b200 as P
from dynamic_block_sparse_shape_b200 import synth
from tests.gpu_util import require_gpu

pytestmark = pytest.mark.gpu


def _static_call(geo, feat, res):
    nz, _ = geo.counts()
    dev = torch.device("cuda")
    shape = torch.full((nz,), -1, dtype=torch.int32, device=dev)
    margin = torch.full((nz,), float("nan"), dtype=torch.float32, device=dev)
    g = geo.c()
    st = P.lib().prism_zone_shapes_static(
        ctypes.byref(g), P._ptr(feat), feat.stride(0) if feat is not None else 0,
        feat.shape[1] if feat is not None else 0, P.BF16, P._ptr(res), res.stride(0) if res is not None else 0,
        res.shape[1] if res is not None else 0, P.BF16, None, P._ptr(shape), P._ptr(margin), P._stream())
    assert st == 0, P.STATUS.get(st, st)
    torch.cuda.synchronize()
    return shape, margin


def test_static_scratch_matches_workspace_entry_point_twice():
    require_gpu()
    dev = torch.device("cuda")
    cand = tuple(synth.DEFAULT_CANDIDATES)
    # call 1: features + residual on a 1080p-like grid slice
    wl1 = dataclasses.replace(synth.WORKLOADS["1080p"], grid=(16, 32, 48))
    F1 = synth.video_features(wl1, device=dev)
    R1, _ = synth.a2v_residual(wl1, device=dev)
    geo1 = P.Geometry(wl1.grid, wl1.zone, cand)
    # call 2: another grid and seed, features only (the static scratch keeps
    # the first call's contents; the result must not depend on them)
    wl2 = dataclasses.replace(synth.WORKLOADS["1080p"], grid=(8, 24, 32), seed=9)
    F2 = synth.video_features(wl2, device=dev)
    geo2 = P.Geometry(wl2.grid, wl2.zone, cand)
    # call 3: a smaller grid with a residual after the larger one, so the first
    # call's residual norms and zone statistics are still in the array
    wl3 = dataclasses.replace(synth.WORKLOADS["1080p"], grid=(8, 16, 24), seed=11)
    F3 = synth.video_features(wl3, device=dev)
    R3, _ = synth.a2v_residual(wl3, device=dev)
    geo3 = P.Geometry(wl3.grid, wl3.zone, cand)
    for geo, F, R in ((geo1, F1, R1), (geo2, F2, None), (geo3, F3, R3)):
        got_shape, got_margin = _static_call(geo, F, R)
        ref_shape, ref_margin = P.zone_shapes(geo, feat=F, res=R)
        torch.cuda.synchronize()
        # the same kernels on the same inputs: identical shapes and margins
        assert torch.equal(got_shape, ref_shape)
        assert torch.equal(got_margin, ref_margin)


def test_static_scratch_rejects_grids_beyond_its_size():
    require_gpu()
    dev = torch.device("cuda")
    # 64x128x128 tokens: the residual norms alone need 4 MiB, beyond the
    # static scratch. The residual buffer has the full size the geometry
    # declares (8 channels, 16 MB), so nothing could read out of bounds even
    # if the size check were missing.
    geo = P.Geometry((64, 128, 128), (8, 8, 8), tuple(synth.DEFAULT_CANDIDATES))
    nz, _ = geo.counts()
    res = torch.zeros((geo.n_tokens, 8), dtype=torch.bfloat16, device=dev)
    shape = torch.empty(nz, dtype=torch.int32, device=dev)
    g = geo.c()
    st = P.lib().prism_zone_shapes_static(ctypes.byref(g), None, 0, 0, P.BF16, P._ptr(res), 8, 8, P.BF16, None,
                                          P._ptr(shape), None, P._stream())
    assert P.STATUS[st] == "PRISM_ERR_UNSUPPORTED"
    torch.cuda.synchronize()
