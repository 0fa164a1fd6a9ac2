"""Python binding of libprism.so, the C ABI of the Prism block-sparse attention
hot path on B200 (see include/prism.h).

Argument marshalling only: every step runs in the CUDA library. PyTorch
provides device memory and streams. Importing this module does not need a GPU;
calling an entry point without the built library raises ``PrismError``.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

__all__ = [
    "PrismError", "Geometry", "ShapeParams", "lib", "library_path", "workspace_size", "Workspace", "zone_shapes",
    "block_pool", "block_select", "block_select_ex", "select_workspace_size", "topk_from_sparsity",
    "block_audio_bias", "mask_to_csr",
    "bsa_fwd", "bsa_bwd", "check_device_status", "STATUS", "OP", "DEFAULT_CDF_THRESHOLD",
]

DEFAULT_CDF_THRESHOLD = 0.20

_HERE = os.path.dirname(os.path.abspath(__file__))
# PRISM_LIBRARY names another build of the library (a test variant) to load instead
_LIB_PATH = os.environ.get("PRISM_LIBRARY") or os.path.join(_HERE, "libprism.so")

STATUS = {
    0: "PRISM_OK", 1: "PRISM_ERR_ARG", 2: "PRISM_ERR_SHAPE", 3: "PRISM_ERR_DTYPE", 4: "PRISM_ERR_WORKSPACE",
    5: "PRISM_ERR_CAPACITY", 6: "PRISM_ERR_CUDA", 7: "PRISM_ERR_TIMEOUT", 8: "PRISM_ERR_DEVICE",
    9: "PRISM_ERR_UNSUPPORTED",
}
OP = {"zone_shapes": 0, "block_select": 1, "bsa_fwd": 2, "bsa_bwd": 3}
BF16, FP32 = 0, 1


class PrismError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        self.name = STATUS.get(status, str(status))
        msg = _lib.prism_status_string(status).decode() if _lib is not None else self.name
        super().__init__(f"{what}: {self.name} ({msg})")


class _Dim3(ctypes.Structure):
    _fields_ = [("t", ctypes.c_int32), ("h", ctypes.c_int32), ("w", ctypes.c_int32)]


class _Geometry(ctypes.Structure):
    _fields_ = [("grid", _Dim3), ("zone", _Dim3), ("cand", ctypes.POINTER(_Dim3)), ("n_cand", ctypes.c_int32)]


class _ShapeParams(ctypes.Structure):
    _fields_ = [("w_audio", ctypes.c_float), ("gamma", ctypes.c_float), ("gate_max", ctypes.c_float)]


class _SelectParams(ctypes.Structure):
    _fields_ = [("top_k", ctypes.c_int32), ("cdf_threshold", ctypes.c_float),
                ("head_top_k", ctypes.POINTER(ctypes.c_int32)), ("head_cdf_threshold", ctypes.POINTER(ctypes.c_float)),
                ("key_bias", ctypes.c_void_p)]


_P = ctypes.c_void_p
_I32, _I64, _F32, _SZ = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
_GEO = ctypes.POINTER(_Geometry)

_SIGNATURES = {
    "prism_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "prism_version": (_I32, []),
    "prism_geometry_counts": (ctypes.c_int, [_GEO, ctypes.POINTER(_I32), ctypes.POINTER(_I32)]),
    "prism_workspace_size": (ctypes.c_int, [ctypes.c_int, _GEO, _I32, _I32, _I32, _I32, ctypes.c_int, _I64,
                                            ctypes.POINTER(_SZ)]),
    "prism_check_device_status": (ctypes.c_int, [_P, _P]),
    "prism_zone_shapes": (ctypes.c_int, [_GEO, _P, _I64, _I32, ctypes.c_int, _P, _I64, _I32, ctypes.c_int,
                                         ctypes.POINTER(_ShapeParams), _P, _P, _P, _SZ, _P]),
    "prism_zone_shapes_static": (ctypes.c_int, [_GEO, _P, _I64, _I32, ctypes.c_int, _P, _I64, _I32, ctypes.c_int,
                                                ctypes.POINTER(_ShapeParams), _P, _P, _P]),
    "prism_block_pool": (ctypes.c_int, [_GEO, _P, _P, _P, ctypes.c_int, _I32, _I32, _I64, _P, _P, _P, _SZ, _P]),
    "prism_block_select": (ctypes.c_int, [_P, _P, _I32, _I32, _I32, _F32, _I32, _F32, _P, _P, _P, _P, _I64,
                                          ctypes.POINTER(_I64), _P, _SZ, _P]),
    "prism_block_select_ex": (ctypes.c_int, [_P, _P, _I32, _I32, _I32, _F32, ctypes.POINTER(_SelectParams), _P, _P,
                                             _P, _P, _I64, ctypes.POINTER(_I64), _P, _SZ, _P]),
    "prism_topk_from_sparsity": (ctypes.c_int, [_F32, _I32, ctypes.POINTER(_I32)]),
    "prism_block_select_workspace_size": (ctypes.c_int, [_I32, _I32, _I32, ctypes.POINTER(_SZ)]),
    "prism_block_audio_bias": (ctypes.c_int, [_GEO, _P, _P, _I64, _I32, ctypes.c_int, _F32, _P, _P, _SZ, _P]),
    "prism_mask_to_csr": (ctypes.c_int, [_P, _P, _I32, _I32, _P, _I64, _P, _SZ, _P]),
    "prism_bsa_fwd": (ctypes.c_int, [_GEO, _P, _P, _P, _P, ctypes.c_int, _I32, _I32, _I64, _F32, _P, _P, _I64, _P,
                                     _P, _P, _P, _SZ, _P]),
    "prism_bsa_bwd": (ctypes.c_int, [_GEO, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_int, _I32, _I32, _I64, _F32,
                                     _P, _P, _I64, _P, _P, _P, _P, _SZ, _P]),
}


def _load():
    if not os.path.exists(_LIB_PATH):
        return None
    lib = ctypes.CDLL(_LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = None  # loaded on first use, so that building the library needs no library


def lib():
    """The loaded ctypes library; raises if libprism.so was not built."""
    global _lib
    if _lib is None:
        _lib = _load()
    if _lib is None:
        raise PrismError(6, f"libprism.so not found at {_LIB_PATH}; run dynamic_block_sparse_shape_b200.build")
    return _lib


def library_path() -> str:
    return _LIB_PATH


def _check(status: int, what: str):
    if status != 0:
        raise PrismError(status, what)


@dataclass(frozen=True)
class Geometry:
    """Token grid (T, H, W), macro-zone extents and candidate block shapes."""
    grid: tuple
    zone: tuple
    cand: tuple

    def c(self):
        arr = (_Dim3 * len(self.cand))(*[_Dim3(*c) for c in self.cand])
        g = _Geometry(_Dim3(*self.grid), _Dim3(*self.zone), arr, len(self.cand))
        g._keep = arr  # keep the candidate array alive with the struct
        return g

    @property
    def n_tokens(self):
        return self.grid[0] * self.grid[1] * self.grid[2]

    def counts(self):
        nz, nb = _I32(), _I32()
        g = self.c()
        _check(lib().prism_geometry_counts(ctypes.byref(g), ctypes.byref(nz), ctypes.byref(nb)), "geometry")
        return nz.value, nb.value


@dataclass(frozen=True)
class ShapeParams:
    w_audio: float = 1.0
    gamma: float = 0.25
    gate_max: float = 4.0


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return FP32
    raise PrismError(3, f"dtype {t.dtype}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def workspace_size(op: str, geo: Geometry, heads=1, head_dim=128, feat_c=0, res_c=0, dtype=torch.bfloat16,
                   nnz=0) -> int:
    out = _SZ()
    g = geo.c()
    code = FP32 if dtype == torch.float32 else BF16
    _check(lib().prism_workspace_size(OP[op], ctypes.byref(g), heads, head_dim, feat_c, res_c, code, nnz,
                                      ctypes.byref(out)), f"workspace_size({op})")
    return out.value


class Workspace:
    """A caller-owned device scratch buffer (torch allocation, 256-byte aligned)
    that grows on demand. The library itself never allocates."""

    def __init__(self, device="cuda", nbytes=1 << 20):
        self.device = torch.device(device)
        self.buf = None
        self.ensure(nbytes)

    def ensure(self, nbytes: int):
        nbytes = max(int(nbytes), 256)
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.zeros(nbytes + 256, dtype=torch.uint8, device=self.device)
        return self

    @property
    def ptr(self):
        p = self.buf.data_ptr()
        return ctypes.c_void_p((p + 255) // 256 * 256)

    @property
    def nbytes(self):
        p = self.buf.data_ptr()
        return self.buf.numel() - ((p + 255) // 256 * 256 - p)


def check_device_status(ws: Workspace, stream=None):
    _check(lib().prism_check_device_status(ws.ptr, _stream(stream)), "device status")


def zone_shapes(geo: Geometry, feat: Optional[torch.Tensor] = None, res: Optional[torch.Tensor] = None,
                params: Optional[ShapeParams] = None, ws: Optional[Workspace] = None, stream=None):
    """a1+a2: per-zone candidate index (int32 [n_zones]) and cost margin (fp32)."""
    nz, _ = geo.counts()
    device = (feat if feat is not None else res).device if (feat is not None or res is not None) else "cuda"
    feat_c = feat.shape[1] if feat is not None else 0
    res_c = res.shape[1] if res is not None else 0
    fdt = feat.dtype if feat is not None else torch.bfloat16
    need = workspace_size("zone_shapes", geo, feat_c=feat_c, res_c=res_c, dtype=fdt)
    ws = (ws or Workspace(device)).ensure(need)
    shape = torch.empty(nz, dtype=torch.int32, device=device)
    margin = torch.empty(nz, dtype=torch.float32, device=device)
    p = params or ShapeParams()
    cp = _ShapeParams(p.w_audio, p.gamma, p.gate_max)
    g = geo.c()
    if feat is not None:
        assert feat.stride(1) == 1
    if res is not None:
        assert res.stride(1) == 1
    _check(lib().prism_zone_shapes(
        ctypes.byref(g), _ptr(feat), feat.stride(0) if feat is not None else 0, feat_c,
        _dtype_code(feat) if feat is not None else BF16, _ptr(res), res.stride(0) if res is not None else 0, res_c,
        _dtype_code(res) if res is not None else BF16, ctypes.byref(cp), _ptr(shape), _ptr(margin), ws.ptr, ws.nbytes,
        _stream(stream)), "prism_zone_shapes")
    return shape, margin


def block_pool(geo: Geometry, zone_shape: torch.Tensor, q: torch.Tensor, k: torch.Tensor,
               ws: Optional[Workspace] = None, stream=None):
    """a3: mean-pooled block features, fp32 [heads, n_blocks, head_dim] each."""
    _, nb = geo.counts()
    N, H, d = q.shape
    assert q.stride(2) == 1 and q.stride(1) == d and k.stride() == q.stride()
    ws = (ws or Workspace(q.device)).ensure(256)
    qp = torch.empty((H, nb, d), dtype=torch.float32, device=q.device)
    kp = torch.empty_like(qp)
    g = geo.c()
    _check(lib().prism_block_pool(ctypes.byref(g), _ptr(zone_shape), _ptr(q), _ptr(k), _dtype_code(q), H, d,
                                  q.stride(0), _ptr(qp), _ptr(kp), ws.ptr, ws.nbytes, _stream(stream)),
           "prism_block_pool")
    return qp, kp


def select_workspace_size(heads: int, n_blocks: int, head_dim: int) -> int:
    """Workspace bytes of block_select / block_select_ex for these pooled shapes."""
    b = _SZ()
    _check(lib().prism_block_select_workspace_size(int(heads), int(n_blocks), int(head_dim), ctypes.byref(b)),
           "prism_block_select_workspace_size")
    return int(b.value)


def block_select(qp: torch.Tensor, kp: torch.Tensor, scale: float, top_k: int,
                 cdf_threshold: float = DEFAULT_CDF_THRESHOLD, ws: Optional[Workspace] = None, csr: bool = True,
                 stream=None):
    """a4+a5: hybrid top-k + CDF selection. Returns dict with mask (int32 view of
    the uint32 words [H, nb, ceil(nb/32)]), kept [H, nb], row_ptr [H*nb+1],
    col_idx [total] and total (int)."""
    H, nb, d = qp.shape
    words = (nb + 31) // 32
    dev = qp.device
    ws = (ws or Workspace(dev)).ensure(select_workspace_size(H, nb, d))
    mask = torch.empty((H, nb, words), dtype=torch.int32, device=dev)
    kept = torch.empty((H, nb), dtype=torch.int32, device=dev)
    row_ptr = torch.empty(H * nb + 1, dtype=torch.int32, device=dev)
    total = _I64()
    _check(lib().prism_block_select(_ptr(qp), _ptr(kp), H, nb, d, float(scale), int(top_k), float(cdf_threshold),
                                    _ptr(mask), _ptr(kept), _ptr(row_ptr), None, 0, ctypes.byref(total), ws.ptr,
                                    ws.nbytes, _stream(stream)), "prism_block_select")
    out = {"mask": mask, "kept": kept, "row_ptr": row_ptr, "total": int(total.value), "col_idx": None}
    if csr:
        col = torch.empty(max(1, total.value), dtype=torch.int32, device=dev)
        mask_to_csr(mask, row_ptr, nb, col, ws=ws, stream=stream)
        out["col_idx"] = col[:total.value]
    return out


def block_select_ex(qp: torch.Tensor, kp: torch.Tensor, scale: float, top_k,
                    cdf_threshold=DEFAULT_CDF_THRESHOLD, key_bias: Optional[torch.Tensor] = None,
                    ws: Optional[Workspace] = None, csr: bool = True, stream=None):
    """a4+a5 with per-head settings: ``top_k`` and ``cdf_threshold`` are scalars
    or sequences of one value per head; ``key_bias`` is None or a device fp32
    [n_blocks] added to every head's logit of each key block (for example from
    ``block_audio_bias``). Returns the same dict as ``block_select``."""
    H, nb, d = qp.shape
    words = (nb + 31) // 32
    dev = qp.device
    ws = (ws or Workspace(dev)).ensure(select_workspace_size(H, nb, d))
    cp = _SelectParams()
    keep = []
    if isinstance(top_k, (int,)) or (torch.is_tensor(top_k) and top_k.dim() == 0):
        cp.top_k = int(top_k)
    else:
        arr = (ctypes.c_int32 * H)(*[int(x) for x in top_k])
        keep.append(arr)
        cp.top_k = int(arr[0]) if H else 1
        cp.head_top_k = ctypes.cast(arr, ctypes.POINTER(ctypes.c_int32))
    if isinstance(cdf_threshold, (int, float)) or (torch.is_tensor(cdf_threshold) and cdf_threshold.dim() == 0):
        cp.cdf_threshold = float(cdf_threshold)
    else:
        arr = (ctypes.c_float * H)(*[float(x) for x in cdf_threshold])
        keep.append(arr)
        cp.cdf_threshold = float(arr[0]) if H else 0.0
        cp.head_cdf_threshold = ctypes.cast(arr, ctypes.POINTER(ctypes.c_float))
    if key_bias is not None:
        assert key_bias.dtype == torch.float32 and key_bias.numel() == nb and key_bias.is_contiguous()
        cp.key_bias = key_bias.data_ptr()
    mask = torch.empty((H, nb, words), dtype=torch.int32, device=dev)
    kept = torch.empty((H, nb), dtype=torch.int32, device=dev)
    row_ptr = torch.empty(H * nb + 1, dtype=torch.int32, device=dev)
    total = _I64()
    _check(lib().prism_block_select_ex(_ptr(qp), _ptr(kp), H, nb, d, float(scale), ctypes.byref(cp), _ptr(mask),
                                       _ptr(kept), _ptr(row_ptr), None, 0, ctypes.byref(total), ws.ptr, ws.nbytes,
                                       _stream(stream)), "prism_block_select_ex")
    out = {"mask": mask, "kept": kept, "row_ptr": row_ptr, "total": int(total.value), "col_idx": None}
    if csr:
        col = torch.empty(max(1, total.value), dtype=torch.int32, device=dev)
        mask_to_csr(mask, row_ptr, nb, col, ws=ws, stream=stream)
        out["col_idx"] = col[:total.value]
    return out


def topk_from_sparsity(sparsity: float, n_blocks: int) -> int:
    """Top-k floor for a top-k sparsity ratio: n_blocks - floor(sparsity * n_blocks), at least 1."""
    k = _I32()
    _check(lib().prism_topk_from_sparsity(float(sparsity), int(n_blocks), ctypes.byref(k)), "prism_topk_from_sparsity")
    return int(k.value)


def block_audio_bias(geo: Geometry, zone_shape: torch.Tensor, res: torch.Tensor, beta: float,
                     ws: Optional[Workspace] = None, stream=None) -> torch.Tensor:
    """Audio-norm bias of every key block, device fp32 [n_blocks]:
    beta * (block mean of ||res[n]||) / (grid mean of ||res[n]||)."""
    _, nb = geo.counts()
    assert res.dim() == 2 and res.stride(1) == 1
    ws = (ws or Workspace(res.device)).ensure(256)
    out = torch.empty(nb, dtype=torch.float32, device=res.device)
    g = geo.c()
    _check(lib().prism_block_audio_bias(ctypes.byref(g), _ptr(zone_shape), _ptr(res), res.stride(0), res.shape[1],
                                        _dtype_code(res), float(beta), _ptr(out), ws.ptr, ws.nbytes, _stream(stream)),
           "prism_block_audio_bias")
    return out


def mask_to_csr(mask: torch.Tensor, row_ptr: torch.Tensor, n_blocks: int, col_idx: torch.Tensor,
                ws: Optional[Workspace] = None, stream=None):
    """Expands selection bitmask rows into ascending CSR column lists."""
    rows = row_ptr.numel() - 1
    ws = (ws or Workspace(mask.device)).ensure(256)
    _check(lib().prism_mask_to_csr(_ptr(mask), _ptr(row_ptr), rows, n_blocks, _ptr(col_idx), col_idx.numel(), ws.ptr,
                                   ws.nbytes, _stream(stream)), "prism_mask_to_csr")
    return col_idx


def bsa_fwd(geo: Geometry, zone_shape, q, k, v, scale, row_ptr, col_idx, ws: Optional[Workspace] = None,
            out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, stream=None,
            o_lo: Optional[torch.Tensor] = None, nnz: Optional[int] = None):
    """a6: block-sparse attention forward. Returns (O like q, LSE fp32 [H, N]).

    o_lo (optional, bf16 like a bf16 q): receives the rounding residual of O,
    to be passed to bsa_bwd so that D = dO . O is formed from O to ~16 bits.
    nnz (optional): the selection's total kept pairs; it chooses the kernels'
    plan (rows short on average: no block images), not the result."""
    N, H, d = q.shape
    assert q.stride(2) == 1 and q.stride(1) == d and k.stride() == q.stride() and v.stride() == q.stride()
    need = workspace_size("bsa_fwd", geo, heads=H, head_dim=d, dtype=q.dtype)
    ws = (ws or Workspace(q.device)).ensure(need)
    o = out if out is not None else torch.empty_like(q)
    assert o.stride() == q.stride()
    lse_t = lse if lse is not None else torch.empty((H, N), dtype=torch.float32, device=q.device)
    if o_lo is not None:
        assert o_lo.dtype == torch.bfloat16 and o_lo.stride() == q.stride()
    g = geo.c()
    _check(lib().prism_bsa_fwd(ctypes.byref(g), _ptr(zone_shape), _ptr(q), _ptr(k), _ptr(v), _dtype_code(q), H, d,
                               q.stride(0), float(scale), _ptr(row_ptr), _ptr(col_idx),
                               -1 if nnz is None else int(nnz), _ptr(o), _ptr(lse_t),
                               _ptr(o_lo), ws.ptr, ws.nbytes, _stream(stream)), "prism_bsa_fwd")
    return o, lse_t


def bsa_bwd(geo: Geometry, zone_shape, q, k, v, o, lse, do, scale, row_ptr, col_idx, nnz: int,
            ws: Optional[Workspace] = None, grads: Optional[Sequence[torch.Tensor]] = None, stream=None,
            o_lo: Optional[torch.Tensor] = None):
    """a7: block-sparse attention backward. Returns (dQ, dK, dV) like q.

    o_lo: the forward's rounding residual of O (bsa_fwd's o_lo), or None."""
    N, H, d = q.shape
    for t in (k, v, o, do):
        assert t.stride() == q.stride()
    need = workspace_size("bsa_bwd", geo, heads=H, head_dim=d, dtype=q.dtype, nnz=nnz)
    ws = (ws or Workspace(q.device)).ensure(need)
    dq, dk, dv = grads if grads is not None else (torch.empty_like(q), torch.empty_like(q), torch.empty_like(q))
    g = geo.c()
    if o_lo is not None:
        assert o_lo.dtype == torch.bfloat16 and o_lo.stride() == q.stride()
    _check(lib().prism_bsa_bwd(ctypes.byref(g), _ptr(zone_shape), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(o_lo),
                               _ptr(lse), _ptr(do), _dtype_code(q), H, d, q.stride(0), float(scale), _ptr(row_ptr),
                               _ptr(col_idx), int(nnz), _ptr(dq), _ptr(dk), _ptr(dv), ws.ptr, ws.nbytes,
                               _stream(stream)), "prism_bsa_bwd")
    return dq, dk, dv


def default_scale(head_dim: int) -> float:
    return 1.0 / math.sqrt(head_dim)
