#!/usr/bin/env python
"""Benchmark of the Prism block-sparse attention hot path on B200.

One step = one layer of the 2K training workload through every stage:
zone shapes (video features + a2v residual) -> block pooling -> hybrid top-k +
CDF selection (+ CSR) -> block-sparse attention forward -> backward. Inputs are
resident in HBM before the timed region and every input tensor (1.8 GB) is
larger than L2, so no flush is needed between steps.

Prints one JSON line (rank 0). ``--impl reference`` times the CPU oracle on a
bounded sample of the same workload instead. Multi-GPU runs are independent
replicas by default (the path has no exchange step; ``value`` is whole-job ms
per layer, weak scaling). ``--shard heads`` splits one layer's heads across the
ranks instead (every stage after the zone shapes is per head; each rank
computes the zone shapes from the replicated features): ``value`` is the
slowest rank's time for its shard, i.e. ms per layer, strong scaling.
``--head-slice a:b`` times one such shard alone on one GPU (per-GPU timing).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "2K block-sparse attn fwd+bwd ms/layer; achieved TFLOP/s vs BF16 tensor peak"
UNIT = "ms/layer"
FWD_FLOP_PER_PAIR = 4 * 64 * 64 * 128  # QK^T and PV over one (query block, key block) pair, d = 128
# the attention takes its sparse plan (the forward's short-row kernel alone, no block images in the
# forward or the backward) up to this many kept key blocks per row on average (the library's
# threshold, restated for the launch count)
SPARSE_BLOCKS_PER_ROW = 32
BWD_FLOP_PER_PAIR = 2.5 * FWD_FLOP_PER_PAIR
# DRAM bytes (read + write) per selected (query block, key block) pair of the three attention
# kernels together (forward, dQ, dK/dV), from one ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum) of the 2-head 2K workload taken after the last change to each kernel:
# 92.42 GB over 4,445,106 pairs (forward 27.35, dQ 26.35, dK/dV 38.73 GB). Scaled by the selected
# pairs of the timed workload; the operand re-reads that miss L2 grow with the pairs. The
# block-image passes before each kernel (one read and one write of the streamed operands) are not
# included.
ATTN_DRAM_BYTES_PER_PAIR = 92.42e9 / 4445106
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def max_over_ranks(value: float, device="cpu") -> float:
    """The largest per-rank value (timings are reported as the slowest rank);
    a no-op without an initialised process group."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_ms_per_layer(ms_per_step_max: float, world: int, shard: str = "replicas") -> float:
    """Replicas: every rank runs one layer per step, so the job finishes
    `world` layers in the slowest rank's step time. Head shards: the ranks
    together run one layer per step, finished when the slowest rank is."""
    return ms_per_step_max / world if shard == "replicas" else ms_per_step_max


def workload_config(wl, parallelism):
    """The `config` object of the JSON line (the same for both arms)."""
    return {"workload": f"{wl.name}: grid {wl.grid[0]}x{wl.grid[1]}x{wl.grid[2]} ({wl.n_tokens} tokens), "
                        f"{wl.heads} heads x d{wl.head_dim}, zones {wl.zone}, top_k {wl.top_k}, "
                        f"cdf_threshold {wl.cdf_threshold}, {'fwd+bwd' if wl.backward else 'fwd only'}",
            "parallelism": parallelism,
            "l2": "inputs larger than L2 (each 1.8 GB), no flush"}


# ---------------------------------------------------------------------------- GPU arm
def build_inputs(wl, device):
    import torch
    from dynamic_block_sparse_shape_b200 import synth
    x = synth.qkv(wl, device=device)
    feats = None
    if wl.features == "synthetic":
        feats = synth.video_features(wl, device=device)
    elif wl.features == "q":
        feats = x["q"].view(wl.n_tokens, -1)
    res = synth.a2v_residual(wl, device=device)[0] if wl.residual else None
    torch.cuda.synchronize()
    return x, feats, res


class Pipeline:
    """One layer of the hot path through the public binding, with every
    buffer preallocated so a step launches kernels only (no host sync)."""

    def __init__(self, wl, x, feats, res):
        import torch
        import dynamic_block_sparse_shape_b200 as P
        from dynamic_block_sparse_shape_b200 import synth
        self.P, self.torch = P, torch
        self.wl = wl
        self.geo = P.Geometry(wl.grid, wl.zone, tuple(synth.candidates_for(wl)))
        self.nz, self.nb = self.geo.counts()
        self.x, self.feats, self.res = x, feats, res
        dev = x["q"].device
        H, d = wl.heads, wl.head_dim
        self.scale = 1.0 / math.sqrt(d)
        self.ws = P.Workspace(dev)
        self.qp = torch.empty((H, self.nb, d), dtype=torch.float32, device=dev)
        self.kp = torch.empty_like(self.qp)
        words = (self.nb + 31) // 32
        self.mask = torch.empty((H, self.nb, words), dtype=torch.int32, device=dev)
        self.kept = torch.empty((H, self.nb), dtype=torch.int32, device=dev)
        self.row_ptr = torch.empty(H * self.nb + 1, dtype=torch.int32, device=dev)
        self.o = torch.empty_like(x["q"])
        # rounding residual of the bf16 output, so that the backward's D = dO . O uses O to ~16 bits
        self.o_lo = torch.empty_like(x["q"]) if x["q"].dtype == torch.bfloat16 else None
        self.lse = torch.empty((H, wl.n_tokens), dtype=torch.float32, device=dev)
        # forward-only workloads (720p, 1080p) have no dO and no backward stage
        self.backward = "do" in x
        self.grads = tuple(torch.empty_like(x["q"]) for _ in range(3)) if self.backward else ()
        self.zone_shape = torch.empty(self.nz, dtype=torch.int32, device=dev)
        self.zone_margin = torch.empty(self.nz, dtype=torch.float32, device=dev)
        self.ws.ensure(P.workspace_size("zone_shapes", self.geo, feat_c=feats.shape[1] if feats is not None else 0,
                                        res_c=res.shape[1] if res is not None else 0))
        self.ws.ensure(P.workspace_size("block_select", self.geo, heads=H, head_dim=d))
        # size the CSR and the workspaces from one selection pass
        self.stage_zone()
        self.stage_pool()
        sel = P.block_select(self.qp, self.kp, self.scale, wl.top_k, wl.cdf_threshold, ws=self.ws, csr=False)
        self.nnz = sel["total"]
        self.col_idx = torch.empty(max(1, self.nnz), dtype=torch.int32, device=dev)
        need = max(P.workspace_size("zone_shapes", self.geo, feat_c=feats.shape[1] if feats is not None else 0,
                                    res_c=res.shape[1] if res is not None else 0),
                   P.workspace_size("block_select", self.geo, heads=H, head_dim=d),
                   P.workspace_size("bsa_fwd", self.geo, heads=H, head_dim=d),
                   P.workspace_size("bsa_bwd", self.geo, heads=H, head_dim=d, nnz=self.nnz))
        self.ws.ensure(need)
        self.events = {}

    def _lib(self):
        return self.P.lib()

    def stage_zone(self):
        import ctypes
        P, g = self.P, self.geo.c()
        f, r = self.feats, self.res
        P._check(P.lib().prism_zone_shapes(
            ctypes.byref(g), P._ptr(f), f.stride(0) if f is not None else 0, f.shape[1] if f is not None else 0,
            P.BF16, P._ptr(r), r.stride(0) if r is not None else 0, r.shape[1] if r is not None else 0, P.BF16,
            None, P._ptr(self.zone_shape), P._ptr(self.zone_margin), self.ws.ptr, self.ws.nbytes, P._stream()),
            "zone_shapes")

    def stage_pool(self):
        import ctypes
        P, g, q, k = self.P, self.geo.c(), self.x["q"], self.x["k"]
        P._check(P.lib().prism_block_pool(ctypes.byref(g), P._ptr(self.zone_shape), P._ptr(q), P._ptr(k), P.BF16,
                                          q.shape[1], q.shape[2], q.stride(0), P._ptr(self.qp), P._ptr(self.kp),
                                          self.ws.ptr, self.ws.nbytes, P._stream()), "block_pool")

    def stage_select(self):
        P = self.P
        H, nb, d = self.qp.shape
        P._check(P.lib().prism_block_select(P._ptr(self.qp), P._ptr(self.kp), H, nb, d, self.scale, self.wl.top_k,
                                            self.wl.cdf_threshold, P._ptr(self.mask), P._ptr(self.kept),
                                            P._ptr(self.row_ptr), P._ptr(self.col_idx), self.col_idx.numel(), None,
                                            self.ws.ptr, self.ws.nbytes, P._stream()), "block_select")

    def stage_fwd(self):
        x = self.x
        self.P.bsa_fwd(self.geo, self.zone_shape, x["q"], x["k"], x["v"], self.scale, self.row_ptr, self.col_idx,
                       ws=self.ws, out=self.o, lse=self.lse, o_lo=self.o_lo, nnz=self.nnz)

    def stage_bwd(self):
        x = self.x
        self.P.bsa_bwd(self.geo, self.zone_shape, x["q"], x["k"], x["v"], self.o, self.lse, x["do"], self.scale,
                       self.row_ptr, self.col_idx, self.nnz, ws=self.ws, grads=self.grads, o_lo=self.o_lo)

    STAGES = ("zone_shapes", "block_pool", "block_select", "bsa_fwd", "bsa_bwd")
    # kernels each stage launches (prism kernels only; memsets excluded)
    # (bsa_fwd: K and V block images + the short-row and main attention kernels, or the short-row kernel
    # alone when the rows hold at most 32 key blocks on average; bsa_bwd: prep, CSC (3), K/V images, dQ,
    # Q/dO images, dK/dV, without the images in that case)
    # (block_select: the tf32 split of q and k, then per round of heads whose logits fit in 1 GiB a score
    # GEMM and a selection launch, then the CSR scan and the list fill; the rounds are counted in
    # launches_per_step)
    LAUNCHES = {"zone_shapes": 4, "block_pool": 1, "block_select": 4, "bsa_fwd": 4, "bsa_bwd": 11}

    def step(self, record=None):
        fns = (self.stage_zone, self.stage_pool, self.stage_select, self.stage_fwd, self.stage_bwd)
        for name, fn in zip(self.STAGES, fns):
            if name == "bsa_bwd" and not self.backward:
                continue
            if record is not None:
                e0 = self.torch.cuda.Event(enable_timing=True)
                e1 = self.torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                record.setdefault(name, []).append((e0, e1))
            else:
                fn()

    def select_rounds(self):
        nb = self.geo.counts()[1]
        nbp = (nb + 3) // 4 * 4
        per_round = max(1, min(self.wl.heads, (1024 << 20) // (nb * nbp * 4)))
        return -(-self.wl.heads // per_round)

    def launches_per_step(self):
        n = sum(self.LAUNCHES.values()) + 2 * self.select_rounds()
        sparse = self.nnz <= SPARSE_BLOCKS_PER_ROW * self.wl.heads * self.geo.counts()[1]
        if sparse:
            n -= 3  # the forward's sparse plan: no K/V block images, no main forward kernel
        if not self.backward:
            n -= self.LAUNCHES["bsa_bwd"]
        elif sparse:
            n -= 4  # the backward's sparse plan: no block images of K, V, Q, dO
        if self.feats is None:
            n -= 1
        if self.res is None:
            n -= 2
        return n


def cpu_sample(wl, x, feats, res, q_blocks=4, kv_blocks=2, sel_rows=256, users_per_kv=8):
    """Times the fp64 oracle on a bounded sample of the workload and
    extrapolates each stage linearly to one layer (ms). Oracle only: the
    selection it uses is its own; no CUDA-path value enters."""
    import numpy as np
    import torch
    from oracle import prism_oracle as O
    from dynamic_block_sparse_shape_b200 import synth
    t_all = time.time()
    cand = synth.candidates_for(wl)
    N = wl.n_tokens
    nzt, nzh, nzw = O.zone_counts(wl.grid, wl.zone)
    nz = nzt * nzh * nzw
    nb = nz * O.blocks_per_zone(wl.zone)
    heads = wl.heads
    rng = np.random.default_rng(0)
    timings = {}
    # a2: token norms of 1/16 of the residual rows, statistics + choice on 4 zones
    zs_sample = sorted(rng.choice(nz, size=min(4, nz), replace=False).tolist())
    ids = np.concatenate([O.zone_token_ids(wl.grid, wl.zone, z).ravel() for z in zs_sample])
    fmap = {int(n): i for i, n in enumerate(ids)}

    class _Rows:  # the sampled zones' rows only, indexed by token id
        def __init__(self, sub):
            self.sub = sub

        def __getitem__(self, idx):
            return self.sub[[fmap[int(n)] for n in np.asarray(idx).ravel()]]
    t_norm = 0.0
    r = None
    if res is not None:
        chunk = N // 16
        t0 = time.time()
        O.token_norms(res[:chunk].to("cpu", torch.float64).numpy())
        t_norm = (time.time() - t0) * 16
        r = np.ones(N)  # norms outside the sample are not needed for the timing
        r[ids] = O.token_norms(res[torch.as_tensor(ids, device=res.device)].to("cpu", torch.float64).numpy())
    Fz = None
    if feats is not None:
        Fz = _Rows(feats[torch.as_tensor(ids, device=feats.device)].to("cpu", torch.float64).numpy())
    t0 = time.time()
    st = O.zone_statistics(wl.grid, wl.zone, F=Fz, zones=zs_sample, r=r)
    O.choose_shapes(st, cand, have_features=feats is not None, have_residual=r is not None)
    timings["zone_shapes"] = t_norm + (time.time() - t0) * nz / len(zs_sample)
    # a3: pooling of head 0 over all blocks (the selection needs every key block)
    blocks = O.block_tokens(wl.grid, wl.zone, cand, np.zeros(nz, dtype=np.int64))
    q0, k0, v0, do0 = (x[n][:, 0].to("cpu", torch.float64).numpy()[:, None, :] for n in ("q", "k", "v", "do"))
    t0 = time.time()
    qp = O.block_pool(q0, blocks)
    kp = O.block_pool(k0, blocks)
    timings["block_pool"] = (time.time() - t0) * heads
    # a4/a5: sel_rows query blocks of head 0
    sc = 1.0 / math.sqrt(wl.head_dim)
    srows = sorted(rng.choice(nb, size=min(sel_rows, nb), replace=False).tolist())
    t0 = time.time()
    sel = O.block_select(qp, kp, sc, wl.top_k, wl.cdf_threshold, rows=[(0, i) for i in srows])
    timings["block_select"] = (time.time() - t0) * heads * nb / len(srows)
    mask0 = sel["mask"][0]
    mean_kept = float(np.mean([sel["kept"][0, i] for i in srows]))
    # a6/a7 (q side): forward rows + dQ of q_blocks sampled query blocks
    t0 = time.time()
    cache = {}
    for I in srows[:q_blocks]:
        cache[(0, I)] = O.attention_block_rows(q0, k0, v0, blocks, np.nonzero(mask0[I])[0], 0, I, sc, dO=do0)
    t_q = (time.time() - t0) / q_blocks
    # a7 (kv side): dK/dV of kv_blocks key blocks, restricted to users_per_kv
    # users whose rows are cached; time per user, times the mean users per block
    users = srows[q_blocks:q_blocks + users_per_kv]
    for I in users:
        cache[(0, I)] = O.attention_block_rows(q0, k0, v0, blocks, np.nonzero(mask0[I])[0], 0, I, sc, dO=do0)
    t_user = 0.0
    n_user = 0
    for J in range(kv_blocks):
        sub = np.zeros_like(mask0)
        for I in users:
            sub[I] = mask0[I]
            sub[I, J] = True
        t0 = time.time()
        O.attention_kv_block_grads(q0, k0, v0, do0, blocks, sub, 0, J, sc, row_cache=cache)
        t_user += time.time() - t0
        n_user += len(users)
    t_kv = t_user / max(n_user, 1) * mean_kept  # users per key block = mean kept per query block
    timings["attention"] = (t_q + t_kv) * nb * heads
    total_ms = 1e3 * sum(timings.values())
    sample = (f"oracle (numpy fp64) on {wl.name}: zone statistics on {len(zs_sample)} of {nz} zones and residual "
              f"norms of 1/16 of the tokens; pooling of all {nb} blocks of head 0; selection of {len(srows)} query "
              f"blocks of head 0; attention forward + dQ rows of {q_blocks} query blocks; dK/dV per user row on "
              f"{kv_blocks} key blocks x {len(users)} users; each stage extrapolated linearly to {heads} heads x "
              f"{nb} blocks (mean kept {mean_kept:.1f})")
    return {"value": round(total_ms, 1), "unit": UNIT, "cores": int(os.cpu_count() or 1),
            "threads": int(torch.get_num_threads()), "kind": "oracle", "sample": sample,
            "wall_s": round(time.time() - t_all, 1), "stage_ms": {k: round(1e3 * v, 1) for k, v in timings.items()}}


def selection_path_roofline(wl, stage_ms, feats, res, peaks, peak_src, nb):
    """Rooflines of the selection path.

    zone_shapes and block_pool are HBM streams: the zone statistics read the
    features and the a2v residual once, the pooling reads Q and K once
    (algorithmic bytes). block_select is not bound by HBM: its dominant work is
    the block scoring, 2 * heads * nb^2 * d FLOP of dot products, executed on
    the tensor cores as three tf32 products (hi.hi + hi.lo + lo.hi); it is
    reported against the tf32 dense peak (the measured bf16 peak x 1/2, the
    nominal tf32 / bf16 ratio) over the whole stage time (scores, threshold
    search and bitmask), with its HBM bytes (pooled q and k read, bitmask and
    counts written) for completeness. "path" sums the algorithmic bytes of all
    three stages over their summed time against the HBM copy bandwidth."""
    hbm = float(peaks.get("hbm_gbs"))
    q_bytes = wl.n_tokens * wl.heads * wl.head_dim * 2
    stat_bytes = sum(t.numel() * t.element_size() for t in (feats, res) if t is not None)
    pooled_bytes = 2 * wl.heads * nb * wl.head_dim * 4
    sel_bytes = pooled_bytes + wl.heads * nb * ((nb + 31) // 32) * 4 + wl.heads * nb * 4 * 2
    out = {}
    for name, nbytes in (("zone_shapes", stat_bytes), ("block_pool", 2 * q_bytes + pooled_bytes)):
        ms = stage_ms.get(name)
        if not ms or not nbytes:
            continue
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[name] = {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                     "frac": round(gbs / hbm, 4), "algorithmic_bytes": nbytes,
                     "peak_source": f"{peak_src} copy bandwidth"}
    ms = stage_ms.get("block_select")
    if ms:
        flop = 2.0 * wl.heads * nb * nb * wl.head_dim
        tf32_peak = float(peaks.get("bf16_tflops")) / 2.0
        executed = 3.0 * flop / (ms * 1e-3) / 1e12
        out["block_select"] = {"bound": "tensor", "achieved": round(executed, 1), "peak": round(tf32_peak, 1),
                               "unit": "TFLOP/s", "frac": round(executed / tf32_peak, 4),
                               "scoring_flop": flop, "executed_tf32_flop": 3.0 * flop,
                               "peak_source": f"{peak_src} bf16 burst x 1/2 (nominal tf32/bf16)",
                               "hbm_gbs": round(sel_bytes / (ms * 1e-3) / 1e9, 1), "algorithmic_bytes": sel_bytes}
    names = [n for n in ("zone_shapes", "block_pool", "block_select") if stage_ms.get(n)]
    if names:
        tot_ms = sum(stage_ms[n] for n in names)
        tot_b = stat_bytes + 2 * q_bytes + pooled_bytes + sel_bytes
        gbs = tot_b / (tot_ms * 1e-3) / 1e9
        out["path"] = {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                       "frac": round(gbs / hbm, 4), "algorithmic_bytes": tot_b, "ms": round(tot_ms, 3),
                       "stages": names, "peak_source": f"{peak_src} copy bandwidth"}
    return out


def measure_selection_variants(pipe, res, peaks, peak_src, reps=5):
    """Per-call times of the selection variants outside the timed step (CUDA events,
    same stream, after the step's warm-up): the audio-norm key-block bias over the
    a2v residual (an HBM stream: algorithmic bytes = the residual read once), and
    the selection with per-head k / tau and that bias next to the plain selection."""
    import ctypes
    import torch
    P, wl = pipe.P, pipe.wl
    H, nb, d = pipe.qp.shape
    g = pipe.geo.c()
    bias = torch.empty(nb, dtype=torch.float32, device=pipe.qp.device)

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    out = {}
    if res is not None:
        def run_bias():
            P._check(P.lib().prism_block_audio_bias(ctypes.byref(g), P._ptr(pipe.zone_shape), P._ptr(res),
                                                    res.stride(0), res.shape[1], P.BF16, 1.0, P._ptr(bias),
                                                    pipe.ws.ptr, pipe.ws.nbytes, P._stream()), "audio_bias")
        ms = timed(run_bias)
        nbytes = res.numel() * res.element_size()
        hbm = float(peaks.get("hbm_gbs"))
        gbs = nbytes / (ms * 1e-3) / 1e9
        out["block_audio_bias"] = {"ms": round(ms, 4), "bound": "hbm", "achieved": round(gbs, 1), "peak": hbm,
                                   "unit": "GB/s", "frac": round(gbs / hbm, 4), "algorithmic_bytes": nbytes,
                                   "peak_source": f"{peak_src} copy bandwidth"}
    else:
        bias.zero_()
    ks = (ctypes.c_int32 * H)(*[max(1, wl.top_k >> (h % 3)) for h in range(H)])
    taus = (ctypes.c_float * H)(*[wl.cdf_threshold * (1 + (h % 2)) for h in range(H)])
    cp = P._SelectParams(wl.top_k, wl.cdf_threshold, ctypes.cast(ks, ctypes.POINTER(ctypes.c_int32)),
                         ctypes.cast(taus, ctypes.POINTER(ctypes.c_float)), bias.data_ptr())
    mask = torch.empty_like(pipe.mask)
    kept = torch.empty_like(pipe.kept)
    row_ptr = torch.empty_like(pipe.row_ptr)

    def run_ex():
        P._check(P.lib().prism_block_select_ex(P._ptr(pipe.qp), P._ptr(pipe.kp), H, nb, d, pipe.scale,
                                               ctypes.byref(cp), P._ptr(mask), P._ptr(kept), P._ptr(row_ptr), None,
                                               0, None, pipe.ws.ptr, pipe.ws.nbytes, P._stream()), "select_ex")
    out["block_select_ex"] = {"ms": round(timed(run_ex), 4),
                              "settings": "per-head k in {k, k/2, k/4}, tau in {tau, 2 tau}, audio-norm bias beta 1",
                              "plain_block_select_ms": round(timed(pipe.stage_select), 4)}
    P.check_device_status(pipe.ws)
    return out


def run_gpu(args):
    import torch
    import torch.distributed as dist
    from dynamic_block_sparse_shape_b200 import synth
    from dynamic_block_sparse_shape_b200 import build as pbuild
    world, rank, local = _dist()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=300))
    pbuild.build()
    wl = synth.WORKLOADS[args.config]
    dev = torch.device("cuda", local)
    x, feats, res = build_inputs(wl, dev)
    full_heads = wl.heads
    h0, h1 = 0, wl.heads
    if args.shard == "heads" or args.head_slice:
        import dataclasses
        from dynamic_block_sparse_shape_b200.shard import head_shard, parse_head_slice
        h0, h1 = parse_head_slice(args.head_slice, wl.heads) if args.head_slice else head_shard(wl.heads, world, rank)
        # this rank's heads of Q, K, V, dO; the features and the residual stay whole (zone shapes on every rank)
        x = {k: v[:, h0:h1].contiguous() for k, v in x.items()}
        torch.cuda.empty_cache()
        wl = dataclasses.replace(wl, heads=h1 - h0)
    shard = "heads" if (args.shard == "heads" or args.head_slice) else "replicas"
    pipe = Pipeline(wl, x, feats, res)
    for _ in range(args.warmup):
        pipe.step()
    torch.cuda.synchronize()
    pipe.P.check_device_status(pipe.ws)
    sampler = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    rec = {}
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        pipe.step(record=rec)
    e1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    ms_step = max_over_ranks(e0.elapsed_time(e1), device=dev) / args.steps
    stage_ms = {k: sum(a.elapsed_time(b) for a, b in v) / len(v) for k, v in rec.items()}
    pipe.P.check_device_status(pipe.ws)
    # end to end through the public API with host buffers
    e2e = None if args.no_e2e else run_e2e(pipe, wl, x, feats, res, steps=min(args.steps, args.e2e_steps))
    peaks, peak_src = _peaks()
    variants = measure_selection_variants(pipe, res, peaks, peak_src)
    nnz = pipe.nnz
    flop_per_pair = FWD_FLOP_PER_PAIR + (BWD_FLOP_PER_PAIR if pipe.backward else 0)
    attn_flop = nnz * flop_per_pair
    t_attn = (stage_ms["bsa_fwd"] + stage_ms.get("bsa_bwd", 0.0)) * 1e-3
    achieved = attn_flop / t_attn / 1e12
    peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    out = {
        "metric": METRIC, "value": round(whole_job_ms_per_layer(ms_step, world, shard), 4), "unit": UNIT,
        "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": False,
        "scaling": "strong" if shard == "heads" else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(wl, (f"one shard alone: heads {h0}:{h1} of {full_heads} (per-GPU timing)"
                                       if args.head_slice else
                                       f"heads sharded over {world} ranks (rank 0: {h0}:{h1})" if shard == "heads"
                                       else "replicas" if world > 1 else "single")),
        "tflops": round(achieved, 1),
        "selected_pairs": nnz, "density": round(nnz / (wl.heads * pipe.nb * pipe.nb), 4),
        "stage_ms": {k: round(v, 3) for k, v in stage_ms.items()},
        "roofline": {"bound": "tensor", "kernel": "bsa_fwd + bsa_bwd (dq, dkdv)" if pipe.backward else "bsa_fwd",
                     "achieved": round(achieved, 1),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": round(nnz * ATTN_DRAM_BYTES_PER_PAIR) if pipe.backward else None,
                     "traffic_source": "ncu dram bytes per selected pair (2-head 2K capture) x selected pairs",
                     "peak_source": f"{peak_src} bf16 sustained",
                     "peak_burst": float(peaks.get("bf16_tflops")),
                     "frac_burst": round(achieved / float(peaks.get("bf16_tflops")), 4),
                     "flop_per_pair": flop_per_pair},
        "roofline_selection_path": selection_path_roofline(wl, stage_ms, feats, res, peaks, peak_src, pipe.nb),
        "selection_variants": variants,
        "e2e": e2e,
        "gpu_launches": pipe.launches_per_step() * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_sample(wl, x, feats, res, q_blocks=160, kv_blocks=8, sel_rows=4608,
                                         users_per_kv=48)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_e2e(pipe, wl, x, feats, res, steps):
    """Same metric through the public API: every step copies its inputs (Q, K,
    V, dO, features, a2v residual) host -> device from pinned memory, runs the
    five stages and reads O, dQ, dK, dV back device -> host. Steps are streamed
    the way a training loop feeds layers: two sets of device buffers, the
    copies on their own streams, so step i+1's inputs and step i-1's results
    cross PCIe while step i computes. The timed region spans every step's
    copies and compute, from the first input copy to the last result read."""
    import torch
    def pinned_copy(t):
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t)
        return h
    host_in = {k: pinned_copy(v) for k, v in x.items()}
    host_f = pinned_copy(feats) if feats is not None else None
    host_r = pinned_copy(res) if res is not None else None
    # second buffer set: its own device inputs, outputs and workspace
    x2 = {k: torch.empty_like(v) for k, v in x.items()}
    f2 = torch.empty_like(feats) if feats is not None else None
    r2 = torch.empty_like(res) if res is not None else None
    for k2 in x2:
        x2[k2].copy_(x[k2])
    if f2 is not None:
        f2.copy_(feats)
    if r2 is not None:
        r2.copy_(res)
    sets = [(pipe, x, feats, res), (Pipeline(wl, x2, f2, r2), x2, f2, r2)]
    outs0 = (pipe.o, *pipe.grads)
    host_out = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs0]
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    h2d += sum(t.numel() * t.element_size() for t in (host_f, host_r) if t is not None)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    in_ready = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_read = [torch.cuda.Event() for _ in range(2)]

    def step(i):
        b = i % 2
        p, xb, fb, rb = sets[b]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(comp_done[b])  # this set's inputs are free once its last step computed
            for k2, v2 in host_in.items():
                xb[k2].copy_(v2, non_blocking=True)
            if host_f is not None:
                fb.copy_(host_f, non_blocking=True)
            if host_r is not None:
                rb.copy_(host_r, non_blocking=True)
            in_ready[b].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(in_ready[b])
            if i >= 2:
                s_comp.wait_event(out_read[b])  # this set's outputs are free once read back
            p.step()
            comp_done[b].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[b])
            for h, o in zip(host_out, (p.o, *p.grads)):
                h.copy_(o, non_blocking=True)
            out_read[b].record(s_out)

    for i in range(2):  # untimed: both buffer sets once
        step(i)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    s_comp.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(2, 2 + steps):
        step(i)
    e1.record(s_out)  # the last result read follows every earlier copy and step
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    return {"value": round(ms, 3), "unit": UNIT, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "steps": steps, "overlap": "two buffer sets; copies on their own streams overlap the neighbouring "
                                       "steps' compute"}


# ---------------------------------------------------------------------------- reference arm
def run_reference(args):
    import torch
    from dynamic_block_sparse_shape_b200 import synth
    world, rank, local = _dist()
    if rank != 0:
        return
    wl = synth.WORKLOADS[args.config]
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    x, feats, res = build_inputs(wl, dev) if dev.type == "cuda" else _cpu_inputs(wl)
    vals = []
    last = None
    for i in range(args.warmup + args.steps):
        last = cpu_sample(wl, x, feats, res)
        if i >= args.warmup:
            vals.append(last["value"])
    v = statistics.mean(vals)
    cpu = dict(last)
    cpu["value"] = round(v, 1)
    out = {"metric": METRIC, "value": round(v, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
           "dtype": "f64", "data": "synthetic", "impl": "reference",
           "config": workload_config(wl, "single"),
           "cpu_baseline": cpu,
           "e2e": {"value": round(v, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def run_sweep(args):
    """The selection/sparsity sweep on the 2K grid: for amplitude x top_k x
    cdf_threshold, kept-block statistics per row and fwd / bwd times."""
    import numpy as np
    import torch
    from dynamic_block_sparse_shape_b200 import synth
    from dynamic_block_sparse_shape_b200 import build as pbuild
    pbuild.build()
    dev = torch.device("cuda")
    points = synth.sweep_workloads()
    if args.sweep_filter:
        import re
        points = [w for w in points if re.search(args.sweep_filter, w.name)]
    by_amp = {}
    for wl in points:
        by_amp.setdefault(wl.amplitude, []).append(wl)
    for amp, wls in by_amp.items():
        x, feats, res = build_inputs(wls[0], dev)
        pipe = None
        for wl in wls:
            if pipe is None:
                pipe = Pipeline(wl, x, feats, res)
            pipe.wl = wl
            sel = pipe.P.block_select(pipe.qp, pipe.kp, pipe.scale, wl.top_k, wl.cdf_threshold, ws=pipe.ws,
                                      csr=False)
            pipe.nnz = sel["total"]
            pipe.col_idx = torch.empty(max(1, pipe.nnz), dtype=torch.int32, device=dev)
            pipe.ws.ensure(pipe.P.workspace_size("bsa_bwd", pipe.geo, heads=wl.heads, head_dim=wl.head_dim,
                                                 nnz=pipe.nnz))
            kept = sel["kept"].cpu().numpy().ravel()
            rec = {}
            for rep in range(2):  # one warm-up, one timed
                rec = {}
                pipe.step(record=rec)
                torch.cuda.synchronize()
            ms = {k: v[0][0].elapsed_time(v[0][1]) for k, v in rec.items()}
            t_attn = (ms["bsa_fwd"] + ms["bsa_bwd"]) * 1e-3
            pipe.P.check_device_status(pipe.ws)
            print(json.dumps({
                "point": wl.name, "amplitude": amp, "top_k": wl.top_k, "cdf_threshold": wl.cdf_threshold,
                "kept_mean": round(float(kept.mean()), 2), "kept_p50": float(np.percentile(kept, 50)),
                "kept_p99": float(np.percentile(kept, 99)), "kept_max": int(kept.max()),
                "density": round(pipe.nnz / (wl.heads * pipe.nb * pipe.nb), 5), "pairs": pipe.nnz,
                "stage_ms": {k: round(v, 3) for k, v in ms.items()},
                "tflops": round(pipe.nnz * (FWD_FLOP_PER_PAIR + BWD_FLOP_PER_PAIR) / t_attn / 1e12, 1)}),
                flush=True)
        del pipe, x, feats, res
        torch.cuda.empty_cache()


def _cpu_inputs(wl):
    from dynamic_block_sparse_shape_b200 import synth
    x = synth.qkv(wl)
    feats = synth.video_features(wl) if wl.features == "synthetic" else (
        x["q"].view(wl.n_tokens, -1) if wl.features == "q" else None)
    res = synth.a2v_residual(wl)[0] if wl.residual else None
    return x, feats, res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="prism", choices=["prism", "reference"])
    ap.add_argument("--config", default="2k")
    ap.add_argument("--e2e-steps", type=int, default=10,
                    help="steps streamed through the e2e measurement (the first step's input copy and the last "
                         "step's result copy are not overlapped with compute)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--sweep", action="store_true", help="run the 45-point selection/sparsity sweep instead")
    ap.add_argument("--sweep-filter", default="", help="with --sweep: only the points whose name matches this regex")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="multi-GPU layout: independent replicas, or one layer's heads split across ranks")
    ap.add_argument("--head-slice", default="", help="a:b, time heads a..b-1 of the layer alone (one shard)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.sweep:
        run_sweep(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
