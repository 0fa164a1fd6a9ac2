"""Child process of tests/test_gpu_timeout.py: loads the fault-injection build
of the library (named by PRISM_LIBRARY), makes the forward's bounded wait run
out once, then runs the same forward normally, and prints a JSON report."""
import json
import math
import sys
import time

import numpy as np
import torch

import dynamic_block_sparse_shape_b200 as P
from dynamic_block_sparse_shape_b200 import synth
from oracle import prism_oracle as O


def main():
    dev = torch.device("cuda")
    cand = tuple(synth.DEFAULT_CANDIDATES)
    grid, zone = (8, 16, 24), (8, 8, 8)
    geo = P.Geometry(grid, zone, cand)
    nz, nb = geo.counts()
    H, d = 2, 128
    rng = np.random.default_rng(3)
    zone_shape = rng.integers(0, len(cand), nz)
    mask = rng.random((H, nb, nb)) < 0.25
    mask[:, np.arange(nb), np.arange(nb)] = True
    mask[0, 0, :16] = True  # query block 0 of head 0 takes eight steps or more (the long-row kernel)
    counts = mask.reshape(H * nb, nb).sum(axis=1)
    row_ptr = np.zeros(H * nb + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(counts)
    col = np.nonzero(mask.reshape(H * nb, nb))[1]
    rp = torch.tensor(row_ptr, dtype=torch.int32, device=dev)
    ci = torch.tensor(col, dtype=torch.int32, device=dev)
    gen = torch.Generator().manual_seed(11)
    q, k, v = (torch.randn((geo.n_tokens, H, d), generator=gen).to(torch.bfloat16).to(dev) for _ in range(3))
    zs = torch.tensor(zone_shape, dtype=torch.int32, device=dev)
    sc = 1.0 / math.sqrt(d)
    ws = P.Workspace(dev).ensure(P.workspace_size("bsa_fwd", geo, heads=H, head_dim=d))
    word = ws.buf[(ws.ptr.value - ws.buf.data_ptr()) + 4:(ws.ptr.value - ws.buf.data_ptr()) + 8].view(torch.int32)
    report = {"library": P.library_path()}
    # 0. a normal call first (loads the library's kernels)
    word.fill_(0)
    P.bsa_fwd(geo, zs, q, k, v, sc, rp, ci, ws=ws)
    torch.cuda.synchronize()
    P.check_device_status(ws)
    # 1. the injected fault: one step's copies are never issued
    word.fill_(1)
    torch.cuda.synchronize()
    t0 = time.time()
    P.bsa_fwd(geo, zs, q, k, v, sc, rp, ci, ws=ws)
    torch.cuda.synchronize()
    report["faulted_call_s"] = time.time() - t0
    try:
        P.check_device_status(ws)
        report["status"] = "PRISM_OK"
    except P.PrismError as e:
        report["status"] = P.STATUS.get(e.status, str(e.status))
    # 2. the same call without the fault, in the same process and context
    word.fill_(0)
    torch.cuda.synchronize()
    o, lse = P.bsa_fwd(geo, zs, q, k, v, sc, rp, ci, ws=ws)
    torch.cuda.synchronize()
    try:
        P.check_device_status(ws)
        report["status_after"] = "PRISM_OK"
    except P.PrismError as e:
        report["status_after"] = P.STATUS.get(e.status, str(e.status))
    blocks = O.block_tokens(grid, zone, cand, zone_shape)
    allowed = O.token_mask(mask, blocks, geo.n_tokens)
    f = lambda t: t.detach().to("cpu", torch.float64).numpy()
    Or, lser = O.masked_attention_fwd(f(q), f(k), f(v), allowed, sc)
    err = np.abs(f(o) - Or)
    report["o_max_abs"] = float(err.max())
    report["o_mean_abs"] = float(err.mean())
    report["lse_max_abs"] = float(np.abs(f(lse) - lser).max())
    print("REPORT " + json.dumps(report), flush=True)


if __name__ == "__main__":
    sys.exit(main())
