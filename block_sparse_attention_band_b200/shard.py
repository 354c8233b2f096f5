"""Splitting one attention layer across GPUs with no exchange step.

Every step of the estimator works per head or per KV group: the block means,
the RMS energies and temperatures of a Q head use that head and its KV head
only, and the scores, Top-P and union are per (Q head, query-block row)
("Prism: Spectral-Aware Block-Sparse Attention", paper.rainbus.top review,
method paragraph, steps (1)-(7)); the block-sparse attention of a Q head reads
only its own KV head.  A layer therefore splits into independent units, one
per (batch element, KV group) -- a KV head and the hq / hkv Q heads that read
it -- and each rank takes a contiguous range of units.  For a fixed batch
element the heads of a range are contiguous in the [b, h, N, 128] layouts, so a
rank's share is a few runs of whole heads: plain pointer offsets into the
caller's tensors and one library call per run, whose outputs are bit-identical
to the same rows of a call on the whole layer.

This module is host-side bookkeeping only (which heads, which offsets); the
calls it prepares go through the C ABI like any other.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence


@dataclasses.dataclass(frozen=True)
class Run:
    """KV heads [kv0, kv1) of batch element ``batch`` (and their Q heads)."""

    batch: int
    kv0: int
    kv1: int

    def q_heads(self, group: int) -> range:
        return range(self.kv0 * group, self.kv1 * group)


def shard_runs(batch: int, hkv: int, world: int, rank: int) -> List[Run]:
    """The runs of rank ``rank`` of ``world``: units u = b * hkv + kv, rank r
    taking [floor(U r / world), floor(U (r + 1) / world)), cut at batch
    boundaries.  Ranks beyond the unit count get no runs."""
    if world <= 0 or not 0 <= rank < world or batch <= 0 or hkv <= 0:
        raise ValueError("need world > 0, 0 <= rank < world, batch > 0, hkv > 0")
    units = batch * hkv
    lo, hi = units * rank // world, units * (rank + 1) // world
    runs, u = [], lo
    while u < hi:
        b, kv0 = divmod(u, hkv)
        kv1 = min(hkv, kv0 + (hi - u))
        runs.append(Run(b, kv0, kv1))
        u += kv1 - kv0
    return runs


def run_offsets(run: Run, hq: int, hkv: int, seqlen: int, head_dim: int = 128, block: int = 128):
    """Element offsets of a run's first row in the q/o, k/v and mask tensors
    ([b, hq, N, D], [b, hkv, N, D], [b, hq, nb, W]) and its head counts."""
    g = hq // hkv
    nb = -(-seqlen // block)
    words = (nb + 31) // 32
    h0 = run.batch * hq + run.kv0 * g
    kvh0 = run.batch * hkv + run.kv0
    return {"q": h0 * seqlen * head_dim, "kv": kvh0 * seqlen * head_dim, "mask": h0 * nb * words,
            "hq": (run.kv1 - run.kv0) * g, "hkv": run.kv1 - run.kv0}


def run_views(run: Run, group: int, q, k, v, mask, o):
    """Contiguous sub-tensors of a run (torch views, no copies)."""
    b, h0, h1 = run.batch, run.kv0 * group, run.kv1 * group
    sl = slice(b, b + 1)
    return (q[sl, h0:h1], k[sl, run.kv0:run.kv1], None if v is None else v[sl, run.kv0:run.kv1],
            None if mask is None else mask[sl, h0:h1], None if o is None else o[sl, h0:h1])


def run_seqlens(run: Run, seqlens: Optional[Sequence[int]]):
    """Per-sequence lengths of a run's call (its one batch element), or None."""
    return None if seqlens is None else [int(seqlens[run.batch])]


__all__ = ["Run", "shard_runs", "run_offsets", "run_views", "run_seqlens"]
