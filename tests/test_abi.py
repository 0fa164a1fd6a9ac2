"""The C-ABI library loads without a GPU, exports every declared entry point,
and its host-side validation returns the documented status codes (no CUDA
call is reached in these cases)."""
import ctypes
import os
import re

import numpy as np
import pytest

import dynamic_block_sparse_shape_b200 as P
from dynamic_block_sparse_shape_b200 import build as pbuild
from dynamic_block_sparse_shape_b200.synth import DEFAULT_CANDIDATES

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "prism.h")


@pytest.fixture(scope="module")
def lib():
    pbuild.build()
    return P.lib()


def declared_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^PRISM_API\s+[^(]*?\b(prism_\w+)\s*\(", txt, flags=re.M)))


def test_every_declared_symbol_is_exported(lib):
    syms = declared_symbols()
    assert len(syms) >= 10
    for s in syms:
        assert hasattr(lib, s), s
    # and the binding declares a signature for each of them
    assert set(syms) == set(P._SIGNATURES), set(syms) ^ set(P._SIGNATURES)


def test_status_strings_and_version(lib):
    for code in P.STATUS:
        assert lib.prism_status_string(code)
    assert lib.prism_status_string(12345) == b"unknown status"
    assert lib.prism_version() >= 100


def _geo(grid=(32, 72, 128), zone=(8, 8, 8), cand=DEFAULT_CANDIDATES):
    return P.Geometry(grid, zone, tuple(cand))


def test_geometry_counts_and_errors(lib):
    assert _geo().counts() == (576, 4608)
    assert _geo((4, 8, 8), (4, 8, 8), [(4, 4, 4)]).counts() == (1, 4)
    # grids that are not whole zones: zones tile the grid rounded up
    from oracle import prism_oracle as O
    for grid in ((32, 72, 127), (16, 45, 80), (32, 90, 160), (1, 1, 1), (9, 17, 8)):
        nz = int(np.prod(O.zone_counts(grid, (8, 8, 8))))
        assert _geo(grid, (8, 8, 8), DEFAULT_CANDIDATES).counts() == (nz, 8 * nz), grid
    bad = [
        ((32, 72, 128), (8, 8, 8), [(4, 4, 2)], 2),  # candidate volume != 64
        ((32, 72, 128), (8, 8, 8), [(16, 2, 2)], 2),  # candidate does not divide the zone
        ((32, 64, 128), (16, 16, 16), [(4, 4, 4)], 9),  # zone larger than 512 tokens
        ((8, 8, 8), (4, 4, 2), [(4, 4, 2)], 2),  # zone volume not a multiple of 64
    ]
    for grid, zone, cand, code in bad:
        with pytest.raises(P.PrismError) as e:
            _geo(grid, zone, cand).counts()
        assert e.value.status == code, (grid, zone, cand)


def test_workspace_sizes(lib):
    g = _geo()
    # the status word, the tf32 halves of the pooled q and k (4 x heads x n_blocks x head_dim floats), and the
    # logits of one round of heads: as many heads as fit in 1 GiB (n_blocks x n_blocks rounded up to 4 floats
    # each), at least one
    def sel_bytes(heads, nb, d):
        up = lambda x: (x + 255) // 256 * 256
        nbp = (nb + 3) // 4 * 4
        per_head = nb * nbp * 4
        rounds = max(1, min(heads, (1024 << 20) // per_head))
        return 256 + 4 * up(heads * nb * d * 4) + up(rounds * nb * nbp * 4)
    assert P.workspace_size("block_select", g) == sel_bytes(1, 4608, 128)
    assert P.workspace_size("block_select", g, heads=24, head_dim=128) == P.select_workspace_size(24, 4608, 128)
    assert P.select_workspace_size(24, 4608, 128) == sel_bytes(24, 4608, 128)  # 12 heads per round at 2K
    assert P.select_workspace_size(24, 960, 128) == sel_bytes(24, 960, 128)  # every head in one round at 720p
    assert P.select_workspace_size(3, 37, 64) == sel_bytes(3, 37, 64)
    z = P.workspace_size("zone_shapes", g, feat_c=3072, res_c=3072)
    assert z >= 576 * 48 * 8 * 4 + 294912 * 4
    b = P.workspace_size("bsa_bwd", g, heads=24, head_dim=128, nnz=1000)
    b2 = P.workspace_size("bsa_bwd", g, heads=24, head_dim=128, nnz=2000)
    assert b2 - b == 4096 or b2 - b == 3840 or b2 > b
    f32 = P.workspace_size("bsa_fwd", g, heads=24, head_dim=128, dtype=__import__("torch").float32)
    assert f32 >= 3 * 294912 * 24 * 128 * 2
    # bf16 forward: the status word and the block images of K and V, one d x 128-byte tile per
    # (head, block) each
    image = 24 * 4608 * 128 * 128
    assert P.workspace_size("bsa_fwd", g, heads=24, head_dim=128) == 256 + 2 * image
    assert P.workspace_size("bsa_fwd", g, heads=2, head_dim=64) == 256 + 2 * (2 * 4608 * 64 * 128)
    assert f32 == 256 + 3 * 294912 * 24 * 128 * 2 + 2 * image
    # backward: two image buffers (K and V, then Q and dO) on top of the block-order LSE / D and the CSC
    assert b > 2 * image and b - 2 * image < 2 ** 28


def test_host_validation_codes(lib):
    g = _geo().c()
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    ws = ctypes.c_void_p(1 << 24)
    # block_select: top_k < 1, bad tau, unsupported d, too many blocks, missing workspace
    sel = lib.prism_block_select
    assert sel(fake, fake, 24, 4608, 128, 0.088, 0, 0.2, fake, fake, fake, None, 0, None, ws, 256, None) == 1
    assert sel(fake, fake, 24, 4608, 128, 0.088, 4, -0.1, fake, fake, fake, None, 0, None, ws, 256, None) == 1
    assert sel(fake, fake, 24, 4608, 96, 0.088, 4, 0.2, fake, fake, fake, None, 0, None, ws, 256, None) == 9
    assert sel(fake, fake, 24, 10241, 128, 0.088, 4, 0.2, fake, fake, fake, None, 0, None, ws, 256, None) == 9
    assert sel(fake, fake, 24, 4608, 128, 0.088, 4, 0.2, fake, fake, fake, None, 0, None, None, 256, None) == 4
    assert sel(None, fake, 24, 4608, 128, 0.088, 4, 0.2, fake, fake, fake, None, 0, None, ws, 256, None) == 1
    # block_pool: dtype, head_dim, token stride
    pool = lib.prism_block_pool
    assert pool(ctypes.byref(g), fake, fake, fake, 7, 24, 128, 3072, fake, fake, ws, 256, None) == 3
    assert pool(ctypes.byref(g), fake, fake, fake, 0, 24, 96, 3072, fake, fake, ws, 256, None) == 9
    assert pool(ctypes.byref(g), fake, fake, fake, 0, 24, 128, 3000, fake, fake, ws, 256, None) == 1
    # attention: null pointers, bad scale, small workspace
    fwd = lib.prism_bsa_fwd
    assert fwd(ctypes.byref(g), fake, None, fake, fake, 0, 24, 128, 3072, 0.088, fake, fake, -1, fake, fake, None, ws,
               256, None) == 1
    assert fwd(ctypes.byref(g), fake, fake, fake, fake, 0, 24, 128, 3072, -1.0, fake, fake, -1, fake, fake, None, ws,
               256, None) == 1
    assert fwd(ctypes.byref(g), fake, fake, fake, fake, 1, 24, 128, 3072, 0.088, fake, fake, -1, fake, fake, None, ws,
               256, None) == 4  # fp32 inputs need staging space
    # the optional output residual must be 16-byte aligned like o
    assert fwd(ctypes.byref(g), fake, fake, fake, fake, 0, 24, 128, 3072, 0.088, fake, fake, -1, fake, fake,
               ctypes.c_void_p((1 << 20) + 2), ws, 1 << 40, None) == 1
    # nnz below -1
    assert fwd(ctypes.byref(g), fake, fake, fake, fake, 0, 24, 128, 3072, 0.088, fake, fake, -2, fake, fake, None,
               ws, 1 << 40, None) == 1
    bwd = lib.prism_bsa_bwd
    assert bwd(ctypes.byref(g), fake, fake, fake, fake, fake, None, fake, fake, 0, 24, 128, 3072, 0.088, fake, fake,
               1000, fake, fake, fake, ws, 256, None) == 4
    assert bwd(ctypes.byref(g), fake, fake, fake, fake, fake, None, fake, fake, 0, 24, 128, 3072, 0.088, fake, fake,
               -5, fake, fake, fake, ws, 1 << 40, None) == 1
    assert bwd(ctypes.byref(g), fake, fake, fake, fake, fake, ctypes.c_void_p((1 << 20) + 2), fake, fake, 0, 24, 128,
               3072, 0.088, fake, fake, 1000, fake, fake, fake, ws, 1 << 40, None) == 1
    # zone shapes: channels not a multiple of 64, misaligned workspace
    zs = lib.prism_zone_shapes
    assert zs(ctypes.byref(g), fake, 3072, 3000, 0, None, 0, 0, 0, None, fake, None, ws, 1 << 30, None) == 1
    assert zs(ctypes.byref(g), None, 0, 0, 0, None, 0, 0, 0, None, fake, None, ctypes.c_void_p((1 << 24) + 8),
              1 << 30, None) == 4
    # mask_to_csr
    assert lib.prism_mask_to_csr(fake, fake, 0, 10, fake, 10, ws, 256, None) == 1


def test_select_ex_and_audio_bias_validation(lib):
    g = _geo().c()
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    ws = ctypes.c_void_p(1 << 24)
    SP = P._SelectParams
    sel = lib.prism_block_select_ex

    def call(params, heads=24, nb=4608, d=128, w=ws):
        return sel(fake, fake, heads, nb, d, 0.088, params, fake, fake, fake, None, 0, None, w, 256, None)

    assert call(None) == 1
    assert call(ctypes.byref(SP(0, 0.2))) == 1                       # k < 1
    assert call(ctypes.byref(SP(4, float("nan")))) == 1              # tau NaN
    ks = (ctypes.c_int32 * 24)(*([4] * 23 + [0]))                    # one head with k = 0
    assert call(ctypes.byref(SP(4, 0.2, ctypes.cast(ks, ctypes.POINTER(ctypes.c_int32))))) == 1
    taus = (ctypes.c_float * 24)(*([0.2] * 23 + [-1.0]))             # one head with tau < 0
    assert call(ctypes.byref(SP(4, 0.2, None, ctypes.cast(taus, ctypes.POINTER(ctypes.c_float))))) == 1
    many = (ctypes.c_int32 * 129)(*([4] * 129))                      # per-head arrays need heads <= 128
    assert call(ctypes.byref(SP(4, 0.2, ctypes.cast(many, ctypes.POINTER(ctypes.c_int32)))), heads=129, nb=64) == 9
    good = SP(4, 0.2, ctypes.cast(ks, ctypes.POINTER(ctypes.c_int32)))
    ks[23] = 4
    assert call(ctypes.byref(good), d=96) == 9
    assert call(ctypes.byref(good), w=None) == 4
    assert call(ctypes.byref(SP(4, 0.2, None, None, (1 << 20) + 2))) == 1  # misaligned key_bias
    bias = lib.prism_block_audio_bias
    assert bias(ctypes.byref(g), fake, None, 3072, 3072, 0, 1.0, fake, ws, 256, None) == 1
    assert bias(ctypes.byref(g), fake, fake, 3072, 3072, 5, 1.0, fake, ws, 256, None) == 3
    assert bias(ctypes.byref(g), fake, fake, 3072, 3070, 0, 1.0, fake, ws, 256, None) == 1
    assert bias(ctypes.byref(g), fake, fake, 3000, 3072, 0, 1.0, fake, ws, 256, None) == 1
    assert bias(ctypes.byref(g), fake, fake, 3072, 3072, 0, float("inf"), fake, ws, 256, None) == 1
    assert bias(ctypes.byref(g), fake, fake, 3072, 3072, 0, 1.0, fake, None, 256, None) == 4


def test_topk_from_sparsity_matches_oracle(lib):
    """Host logic of the ratio form of top-k, against the oracle's rule."""
    from oracle import prism_oracle as O
    rng = np.random.default_rng(7)
    cases = [(0.0, 1), (0.0, 4608), (0.9, 4608), (0.75, 4608), (0.5, 10), (0.3, 10), (0.999, 3)]
    cases += [(float(rng.uniform(0, 1)), int(rng.integers(1, 6000))) for _ in range(500)]
    k = ctypes.c_int32()
    for rho, nb in cases:
        assert lib.prism_topk_from_sparsity(rho, nb, ctypes.byref(k)) == 0
        assert k.value == O.topk_from_sparsity(rho, nb), (rho, nb)
    for rho, nb in ((-0.1, 10), (1.0, 10), (float("nan"), 10), (0.5, 0)):
        assert lib.prism_topk_from_sparsity(rho, nb, ctypes.byref(k)) == 1
    assert lib.prism_topk_from_sparsity(0.5, 10, None) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(P, "_LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(P, "_lib", None)
    with pytest.raises(P.PrismError):
        P.lib()


def test_bench_restates_the_plan_threshold():
    """bench.py counts its kernel launches per plan from a restated copy of the
    library's sparse-plan threshold (kept blocks per row on average); the
    library's constant and the header's documentation must say the same."""
    import bench
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    csrc = os.path.join(root, "dynamic_block_sparse_shape_b200", "csrc")
    txt = open(os.path.join(csrc, "bsa_common.cuh")).read()
    m = re.search(r"constexpr int kSparseBlocksPerRow = (\d+);", txt)
    assert m and int(m.group(1)) == bench.SPARSE_BLOCKS_PER_ROW
    hdr = open(HEADER).read()
    assert hdr.count(f"at most {bench.SPARSE_BLOCKS_PER_ROW} selected key blocks per row") == 2


def test_bench_launch_count_per_plan():
    """The bench's claimed kernel launches per step, for the 2K layer (two
    selection rounds of 12 heads): 28 in the dense plan (the launch list of one
    step: 4 zone-shape, 1 pooling, 8 selection, 4 forward, 11 backward kernels),
    21 in the sparse plan (no block images, no main forward kernel), 15 / 12
    for a forward-only layer without the bridge residual."""
    import types
    import bench
    from dynamic_block_sparse_shape_b200 import synth
    wl = synth.WORKLOADS["2k"]
    geo = P.Geometry(wl.grid, wl.zone, tuple(synth.candidates_for(wl)))
    rows = wl.heads * geo.counts()[1]

    def count(nnz, backward=True, res=True):
        fake = types.SimpleNamespace(wl=wl, geo=geo, nnz=nnz, backward=backward, feats=object(),
                                     res=object() if res else None, LAUNCHES=bench.Pipeline.LAUNCHES)
        fake.select_rounds = lambda: bench.Pipeline.select_rounds(fake)
        return bench.Pipeline.launches_per_step(fake)

    assert count(60958374) == 28
    assert count(4 * rows) == 21
    assert count(60958374, backward=False, res=False) == 28 - 11 - 2
    assert count(4 * rows, backward=False, res=False) == 28 - 11 - 2 - 3
