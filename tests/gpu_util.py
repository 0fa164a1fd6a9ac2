"""Helpers shared by the GPU parity tests (no method arithmetic here)."""
import math

import numpy as np
import pytest
import torch

import dynamic_block_sparse_shape_b200 as P
from dynamic_block_sparse_shape_b200 import build as _build

ATOL_MAX = 2e-2  # max-abs tolerance on O / dQ / dK / dV (bf16 against the fp64 oracle)
ATOL_MEAN = 2e-3  # mean-abs tolerance
LOGIT_GAP = 1e-3  # selections compared bit-exactly where the boundary logit gap exceeds this
CDF_MARGIN = 1e-5  # ... and the cumulative mass is this far from the threshold


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    _build.build()
    P.lib()


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def mask_bits_to_bool(mask_words: torch.Tensor, nb: int) -> np.ndarray:
    """[H, nb, words] int32 bit words -> bool [H, nb, nb]."""
    w = mask_words.cpu().numpy().astype(np.uint32)
    bits = ((w[..., :, None] >> np.arange(32, dtype=np.uint32)) & 1).astype(bool)
    return bits.reshape(w.shape[0], w.shape[1], -1)[..., :nb]


def csr_from_mask(mask: np.ndarray, device):
    """bool [H, nb, nb] -> (row_ptr, col_idx) int32 device tensors, rows in (h, I) order."""
    H, nb, _ = mask.shape
    counts = mask.reshape(H * nb, nb).sum(axis=1)
    row_ptr = np.zeros(H * nb + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(counts)
    col = np.nonzero(mask.reshape(H * nb, nb))[1]
    return (torch.tensor(row_ptr, dtype=torch.int32, device=device),
            torch.tensor(col if col.size else np.zeros(1), dtype=torch.int32, device=device), int(row_ptr[-1]))


def assert_close(name, got, ref, atol_max=ATOL_MAX, atol_mean=ATOL_MEAN, bound=None):
    """Max-abs and mean-abs error against the fp64 oracle. With ``bound`` (the
    oracle's elementwise worst-case effect of the bf16 roundings a bf16
    tensor-core implementation performs), an element may exceed atol_max up to
    its bound: at unit data scale the bound stays below atol_max, at larger
    scales (gradients of order 1-10) bf16 rounding alone can exceed it."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin), f"{name}: finiteness differs"
    err = np.abs(got[fin] - ref[fin])
    if bound is not None and err.size:
        allowed = np.maximum(atol_max, np.asarray(bound, dtype=np.float64)[fin])
        worst = float((err / allowed).max())
        mean = float(err.mean())
        n_over = int((err > atol_max).sum())  # elements admitted by the bound alone
        assert worst <= 1.0 and mean <= atol_mean, (
            f"{name}: error / max({atol_max}, bf16 bound) {worst:.3f}, mean-abs {mean:.3e}, max-abs {err.max():.3e}")
        if n_over:
            print(f"{name}: {n_over} of {err.size} elements above {atol_max} (within the bf16 bound)")
        return float(err.max()), mean
    mx = float(err.max()) if err.size else 0.0
    mean = float(err.mean()) if err.size else 0.0
    ref_max = float(np.abs(ref[fin]).max()) if err.size else 0.0
    ref_rms = float(np.sqrt(np.mean(ref[fin] ** 2))) if err.size else 0.0
    assert mx <= atol_max and mean <= atol_mean, (
        f"{name}: max-abs {mx:.3e} mean-abs {mean:.3e} (reference max-abs {ref_max:.3e}, rms {ref_rms:.3e})")
    return mx, mean


def scale_for(d):
    return 1.0 / math.sqrt(d)
