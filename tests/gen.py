"""Seeded synthetic inputs for the Prism estimator and block-sparse prefill.

This module only draws random numbers and builds post-RoPE Q/K/V tensors; it
holds none of the estimator's or the attention's arithmetic.  Both the CPU
oracle tests and the CUDA parity tests / bench take their inputs from here, so
the two sides always see the same bf16 tensors.

Recipe (Prism: Spectral-Aware Block-Sparse Attention, gist.science Technical
Summary section 1: Prism consumes Q/K *after* RoPE):

* ``torch.Generator('cpu')`` seeded with the workload seed; all draws N(0, 1)
  fp32, in this order: a_q [Hq, D], a_k [Hkv, D], z [Hq, N, D], z' [Hkv, N, D],
  V [Hkv, N, D], then the workload's extras.
* pre-RoPE q_t = a_q + 0.5 z_t and k_t = a_k + 0.5 z'_t.
* half-split RoPE (pair j = dims (j, j + D/2), theta_j = base^(-2j/D)) in fp64
  at positions 0..N-1, then rounded to bf16 (round-to-nearest-even); a
  workload with ``interleaved`` set uses the interleaved layout (pair j =
  dims (2j, 2j + 1)) instead.
* extras: ``stripes`` -- 64 key positions per KV head (drawn without
  replacement) get pre-RoPE k = 3 * a_q of the group's first Q head;
  ``slash`` -- KV heads 0..Hkv/2-1 get pre-RoPE k_t = q_t(first Q head of the
  group) + 0.3 n_t (slash applied first, stripes after);
  ``segments`` -- Q heads Hq/4..Hq-1 resample a_q every ``segment`` tokens
  (fresh draws for every segment, segment 0 included), Q heads 0..Hq/4-1 keep
  a stationary a_q.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

HEAD_DIM = 128
BLOCK = 128


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic attention layer.  Sizes follow the named model shapes."""

    name: str
    batch: int
    hq: int
    hkv: int
    seqlen: int
    seed: int
    p: float = 0.95
    rope_base: float = 500000.0
    head_dim: int = HEAD_DIM
    block: int = BLOCK
    stripes: bool = False
    slash: bool = False
    segment: int = 0  # 0: stationary a_q for every head
    interleaved: bool = False  # RoPE pairs (2j, 2j+1) instead of (j, j + D/2)

    @property
    def nb(self) -> int:
        return -(-self.seqlen // self.block)  # the last block may be short


# The five workloads: a tiny single head, the Llama-3-8B-shaped layer at 32K
# and 128K, the Qwen3-8B-shaped layer with planted stripes + slash at 64K, and
# the long-context sweep (non-stationary segments) at 8K..256K.
WORKLOADS = {
    "tiny_2k": Workload("tiny_2k", 1, 1, 1, 2048, seed=0),
    "llama3_8b_32k": Workload("llama3_8b_32k", 1, 32, 8, 32768, seed=1),
    "llama3_8b_128k": Workload("llama3_8b_128k", 1, 32, 8, 131072, seed=2),
    "qwen3_8b_64k_planted": Workload("qwen3_8b_64k_planted", 1, 32, 8, 65536, seed=3,
                                     p=0.93, rope_base=1e6, stripes=True, slash=True),
}
for _n in (8192, 16384, 65536, 131072, 262144):
    WORKLOADS[f"sweep_{_n // 1024}k"] = Workload(f"sweep_{_n // 1024}k", 1, 32, 8, _n, seed=4,
                                                 segment=4096)


def rope_tables(seqlen: int, head_dim: int, base: float, start: int = 0, theta=None):
    """fp64 cos/sin tables [seqlen, head_dim/2], column j for pair j (either
    layout).  ``theta`` overrides the plain ladder base^(-2j/D) (e.g. with a
    YaRN-rescaled one)."""
    half = head_dim // 2
    j = torch.arange(half, dtype=torch.float64)
    theta = base ** (-2.0 * j / head_dim) if theta is None else torch.as_tensor(theta, dtype=torch.float64)
    t = torch.arange(start, start + seqlen, dtype=torch.float64)
    ang = t[:, None] * theta[None, :]
    return torch.cos(ang), torch.sin(ang)


def mrope_tables(pos_thw: torch.Tensor, head_dim: int, base: float, sections=(16, 24, 24)):
    """Multimodal RoPE (M-RoPE) cos/sin tables [N, head_dim/2]: every token has a
    (temporal, height, width) position and the frequency pairs are split into
    consecutive sections, pair j taking the position component of its section
    (the fastest ``sections[0]`` pairs the temporal one, then height, then
    width; 16 / 24 / 24 pairs at head_dim 128).  A text token has t = h = w =
    its index, which makes the tables those of plain RoPE."""
    half = head_dim // 2
    assert sum(sections) == half
    j = torch.arange(half, dtype=torch.float64)
    theta = base ** (-2.0 * j / head_dim)
    comp = torch.cat([torch.full((n,), c, dtype=torch.long) for c, n in enumerate(sections)])
    pos = torch.as_tensor(pos_thw, dtype=torch.float64)[:, comp]  # [N, half]: each pair's position
    ang = pos * theta[None, :]
    return torch.cos(ang), torch.sin(ang)


def video_positions(frames: int, height: int, width: int, t0: int = 0) -> torch.Tensor:
    """(t, h, w) positions of a video's patch tokens, frame by frame, row by row."""
    t = torch.arange(frames).repeat_interleave(height * width) + t0
    h = torch.arange(height).repeat_interleave(width).repeat(frames)
    w = torch.arange(width).repeat(frames * height)
    return torch.stack([t, h, w], dim=1)


def apply_rope(x: torch.Tensor, cos: torch.Tensor, sin: torch.Tensor, interleaved: bool = False) -> torch.Tensor:
    """RoPE on the last dim of fp64 ``x`` [..., N, D]: pair j = (j, j+D/2)
    (half-split) or (2j, 2j+1) (interleaved)."""
    if interleaved:
        a, b = x[..., 0::2], x[..., 1::2]
        out = torch.empty_like(x)
        out[..., 0::2] = a * cos - b * sin
        out[..., 1::2] = a * sin + b * cos
        return out
    half = x.shape[-1] // 2
    a, b = x[..., :half], x[..., half:]
    return torch.cat([a * cos - b * sin, a * sin + b * cos], dim=-1)


def make_inputs(w: Workload, seqlen: Optional[int] = None, with_v: bool = True):
    """Return bf16 CPU tensors q [b,Hq,N,D], k [b,Hkv,N,D], v [b,Hkv,N,D].

    ``seqlen`` overrides the workload length (used by the sweep); the draws are
    made per batch element in the documented order.
    """
    n = w.seqlen if seqlen is None else seqlen
    d, hq, hkv = w.head_dim, w.hq, w.hkv
    g = hq // hkv
    gen = torch.Generator("cpu")
    gen.manual_seed(w.seed)
    cos, sin = rope_tables(n, d, w.rope_base)
    qs, ks, vs = [], [], []
    for _ in range(w.batch):
        a_q = torch.randn(hq, d, generator=gen)
        a_k = torch.randn(hkv, d, generator=gen)
        z = torch.randn(hq, n, d, generator=gen)
        zk = torch.randn(hkv, n, d, generator=gen)
        v = torch.randn(hkv, n, d, generator=gen)
        stripe_pos = None
        slash_noise = None
        seg_aq = None
        if w.slash:
            slash_noise = torch.randn(hkv // 2, n, d, generator=gen)
        if w.stripes:
            stripe_pos = torch.stack([torch.randperm(n, generator=gen)[:64] for _ in range(hkv)])
        if w.segment:
            nseg = (n + w.segment - 1) // w.segment
            seg_aq = torch.randn(hq, nseg, d, generator=gen)

        q_out = torch.empty(hq, n, d, dtype=torch.bfloat16)
        k_out = torch.empty(hkv, n, d, dtype=torch.bfloat16)
        pre_q = {}
        for h in range(hq):
            if seg_aq is not None and h >= hq // 4:
                seg_idx = torch.arange(n) // w.segment
                base_vec = seg_aq[h][seg_idx].double()
            else:
                base_vec = a_q[h].double()[None, :]
            qh = base_vec + 0.5 * z[h].double()
            if w.slash and h % g == 0 and (h // g) < hkv // 2:
                pre_q[h] = qh
            q_out[h] = apply_rope(qh, cos, sin, w.interleaved).to(torch.bfloat16)
        for kv in range(hkv):
            kh = a_k[kv].double()[None, :] + 0.5 * zk[kv].double()
            if w.slash and kv < hkv // 2:
                kh = pre_q[kv * g] + 0.3 * slash_noise[kv].double()
            if w.stripes:
                kh[stripe_pos[kv]] = 3.0 * a_q[kv * g].double()
            k_out[kv] = apply_rope(kh, cos, sin, w.interleaved).to(torch.bfloat16)
        qs.append(q_out)
        ks.append(k_out)
        vs.append(v.to(torch.bfloat16))
    q = torch.stack(qs)
    k = torch.stack(ks)
    v = torch.stack(vs) if with_v else None
    return q, k, v


def small_workload(name: str, batch: int, hq: int, hkv: int, seqlen: int, seed: int,
                   p: float = 0.95, **kw) -> Workload:
    """A parity-test case built from the same recipe at a size the oracle runs in seconds."""
    return Workload(name, batch, hq, hkv, seqlen, seed=seed, p=p, **kw)


# Default band index sets in frequency-pair order for the half-split layout:
# high band = the fastest 32 pairs {0..31} u {64..95} (d_high = 64), low band =
# the slowest 48 pairs {16..63} u {80..127} (d_low = 96).
def default_bands(head_dim: int = HEAD_DIM):
    half = head_dim // 2
    hi_pairs = list(range(0, 32))
    lo_pairs = list(range(16, half))
    band_hi = sorted(hi_pairs + [j + half for j in hi_pairs])
    band_lo = sorted(lo_pairs + [j + half for j in lo_pairs])
    return band_hi, band_lo


def rope_theta(head_dim: int, base: float):
    half = head_dim // 2
    return [base ** (-2.0 * j / head_dim) for j in range(half)]


__all__ = ["Workload", "WORKLOADS", "make_inputs", "rope_tables", "apply_rope", "mrope_tables",
           "video_positions", "small_workload", "default_bands", "rope_theta", "HEAD_DIM", "BLOCK"]
