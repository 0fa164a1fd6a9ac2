"""Head sharding of one attention layer across ranks (host-side plumbing).

Every stage after the zone shapes is independent per head: pooling, scoring,
selection and attention of head h read only head h of Q, K, V and dO. So a
layer shards by heads with no exchange on the hot path. Each rank owns a
contiguous, balanced slice of the heads; the zone shapes depend only on the
video features and the a2v residual, which every rank holds, and are computed
by kernels with fixed-order reductions, so every rank derives the same block
partition without a broadcast. (The Prism README and walkthrough train the
model with FSDP / DeepSpeed across GPUs; head-parallel attention is this
library's layout for one layer.)
"""
from __future__ import annotations


def head_shard(heads: int, world: int, rank: int) -> tuple[int, int]:
    """Half-open head range [h0, h1) of `rank` among `world` ranks: contiguous,
    sizes differing by at most one, the larger slices first."""
    if heads < 1 or world < 1 or not 0 <= rank < world:
        raise ValueError("need heads >= 1, world >= 1 and 0 <= rank < world")
    if world > heads:
        raise ValueError("more ranks than heads")
    base, extra = divmod(heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def parse_head_slice(spec: str, heads: int) -> tuple[int, int]:
    """'a:b' -> (a, b) with 0 <= a < b <= heads."""
    a, b = (int(x) for x in spec.split(":"))
    if not 0 <= a < b <= heads:
        raise ValueError(f"head slice {spec} outside 0..{heads}")
    return a, b
