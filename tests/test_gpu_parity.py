"""CUDA path vs the fp64 oracle on small seeded workloads (all outputs compared).

Sizes span several 64-wide score tiles, several 32-bit mask words and a ragged
tail (nb = 1, 2, 3, 17, 33, 70), GQA 1:1 / 2:1 / 4:1, batch 2.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests import gen
from tests import parity as P

pytestmark = pytest.mark.gpu

import block_sparse_attention_band_b200 as pb  # noqa: E402


def _inputs(w, device):
    q, k, v = gen.make_inputs(w)
    return q, k, v, q.to(device), k.to(device), v.to(device)


CASES = [
    gen.WORKLOADS["tiny_2k"],
    gen.small_workload("gqa2_nb17", 1, 4, 2, 17 * 128, seed=21),
    gen.small_workload("gqa4_nb33", 1, 8, 2, 33 * 128, seed=22, p=0.9),
    gen.small_workload("batch2_nb3", 2, 2, 1, 3 * 128, seed=23),
    gen.small_workload("nb1", 1, 2, 2, 128, seed=24),
    gen.small_workload("nb2", 1, 2, 1, 256, seed=25),
    gen.small_workload("planted_nb70", 1, 4, 2, 70 * 128, seed=26, p=0.93, rope_base=1e6,
                       stripes=True, slash=True),
    gen.small_workload("segments_nb40", 1, 8, 2, 40 * 128, seed=27, segment=1024),
    gen.small_workload("gqa3_nb9", 1, 3, 1, 9 * 128, seed=28),
    gen.small_workload("mha_b2_nb5", 2, 3, 3, 5 * 128, seed=29),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_estimator_parity(w, cuda_device):
    q, k, v, qd, kd, vd = _inputs(w, cuda_device)
    cfg = P.make_cfg(w)
    ex = {}
    mask, sc, tau, _ = P.run_estimate(cfg, qd, kd, extras=ex)
    hi, lo = gen.default_bands()
    ref = oracle.estimate(q, k, hi, lo, w.p)
    P.check_pooled(ex["pooled"], q, k)
    P.check_tau(tau, ref)
    P.check_scores(sc, ref)
    n_diff, n_exempt = P.check_mask(mask, ref, w.p)
    # Top-P on the GPU's own weights, restated in fixed point: bit-exact
    P.check_topp_exact(mask, ex["weights"], w.p)
    # the oracle's fp64 Top-P on the GPU's own scores: exact except where the
    # fp32 weights' rounding can flip a decision right at p
    self_mask, self_cx = P.topp_on_scores(sc, w.p)
    diff = self_mask != mask
    near = (np.abs(self_cx[..., 0, :, :] - w.p) < P.SELF_WINDOW) | (np.abs(self_cx[..., 1, :, :] - w.p) < P.SELF_WINDOW)
    assert not np.any(diff & ~near), f"{np.sum(diff & ~near)} bits differ from Top-P on the GPU scores"
    print(f"{w.name}: density {P.density(mask):.3f} mismatches {n_diff} (exempt {n_exempt}); "
          f"oracle Top-P on GPU scores: {int(diff.sum())} bits in the {P.SELF_WINDOW} window")


@pytest.mark.parametrize("w", CASES[:4] + CASES[6:7] + CASES[8:], ids=lambda w: w.name)
def test_attention_parity_with_estimator_mask(w, cuda_device):
    q, k, v, qd, kd, vd = _inputs(w, cuda_device)
    cfg = P.make_cfg(w)
    mask, _, _, words = P.run_estimate(cfg, qd, kd, with_scores=False)
    o = P.run_attention(cfg, qd, kd, vd, torch.from_numpy(words.view(np.int32)).to(cuda_device))
    rows = [(b, h, i) for b in range(w.batch) for h in range(w.hq) for i in range(w.nb)]
    if len(rows) > 96:
        rng = np.random.default_rng(0)
        rows = [rows[x] for x in sorted(rng.choice(len(rows), 96, replace=False))]
    P.check_attention_rows(o, q, k, v, mask, rows, w.hq // w.hkv)


@pytest.mark.parametrize("w", [gen.small_workload("short_5x128p1", 1, 2, 1, 5 * 128 + 1, seed=51, p=0.9),
                               gen.small_workload("short_9x128p77", 1, 4, 2, 9 * 128 + 77, seed=52, p=0.9),
                               gen.small_workload("short_33x128p127", 2, 4, 1, 33 * 128 + 127, seed=53, p=0.9),
                               gen.small_workload("short_100", 1, 2, 2, 100, seed=54, p=0.9)],
                         ids=lambda w: w.name)
def test_short_last_block(w, cuda_device):
    """seqlen not a multiple of 128: the last block pools over its own tokens,
    and attention sees only real tokens; estimator and attention match the
    oracle on every row, the short last query block included."""
    q, k, v, qd, kd, vd = _inputs(w, cuda_device)
    hi, lo = gen.default_bands()
    cfg = P.make_cfg(w)
    ex = {}
    mask, sc, tau, words = P.run_estimate(cfg, qd, kd, extras=ex)
    ref = oracle.estimate(q, k, hi, lo, w.p)
    P.check_pooled(ex["pooled"], q, k)  # the short last block divides by its own token count
    P.check_tau(tau, ref)
    P.check_scores(sc, ref)
    P.check_mask(mask, ref, w.p)
    P.check_topp_exact(mask, ex["weights"], w.p)
    o = P.run_attention(cfg, qd, kd, vd, torch.from_numpy(words.view(np.int32)).to(cuda_device))
    rows = [(b, h, i) for b in range(w.batch) for h in range(w.hq) for i in range(w.nb)]
    P.check_attention_rows(o, q, k, v, mask, rows, w.hq // w.hkv)


@pytest.mark.parametrize("w", [gen.small_workload("dense_nb9", 1, 4, 2, 9 * 128, seed=31),
                               gen.small_workload("dense_b2", 2, 2, 2, 4 * 128, seed=32)],
                         ids=lambda w: w.name)
def test_p1_is_dense_causal(w, cuda_device):
    q, k, v, qd, kd, vd = _inputs(w, cuda_device)
    cfg = P.make_cfg(w, p=1.0)
    mask, _, _, words = P.run_estimate(cfg, qd, kd, with_scores=False)
    assert np.array_equal(mask, np.broadcast_to(np.tril(np.ones((w.nb, w.nb), dtype=bool)), mask.shape))
    o = P.run_attention(cfg, qd, kd, vd, torch.from_numpy(words.view(np.int32)).to(cuda_device))
    dense = oracle.dense_causal_attention(q, k, v, group=w.hq // w.hkv)
    err = np.abs(o.float().cpu().numpy() - dense)
    assert err.max() <= P.ATTN_MAX_ABS and err.mean() <= P.ATTN_MEAN_ABS, (err.max(), err.mean())


def test_attention_arbitrary_masks(cuda_device):
    """Random masks incl. empty rows, diagonal-only rows and bits above the
    diagonal (ignored), fed straight to prism_sparse_attn."""
    w = gen.small_workload("masks_nb37", 1, 4, 2, 37 * 128, seed=33)
    q, k, v, qd, kd, vd = _inputs(w, cuda_device)
    nb = w.nb
    rng = np.random.default_rng(5)
    m = rng.random((1, 4, nb, nb)) < 0.3
    m[0, 0, 5, :] = False          # empty row -> zeros
    m[0, 1, 7, :] = False
    m[0, 1, 7, 7] = True           # diagonal only
    m[0, 2, 9, :] = True           # bits above the diagonal too
    words = oracle.pack_mask(m)
    o = P.run_attention(P.make_cfg(w), qd, kd, vd, torch.from_numpy(words.view(np.int32)).to(cuda_device))
    causal_m = m & np.tril(np.ones((nb, nb), dtype=bool))
    rows = [(0, h, i) for h in range(4) for i in range(nb)]
    P.check_attention_rows(o, q, k, v, causal_m, rows, 2)
    assert torch.all(o[0, 0, 5 * 128:6 * 128] == 0)


def test_explicit_tau_and_custom_bands(cuda_device):
    w = gen.small_workload("custom_nb20", 1, 4, 4, 20 * 128, seed=34, p=0.8)
    q, k, v, qd, kd, vd = _inputs(w, cuda_device)
    bands = (list(range(0, 64)), list(range(32, 128)))  # the literal first-64 / last-96 reading
    cfg = P.make_cfg(w, bands=bands, tau_mode=pb.PRISM_TAU_EXPLICIT, tau_hi=0.5, tau_lo=1.5)
    mask, sc, tau, _ = P.run_estimate(cfg, qd, kd)
    ref = oracle.estimate(q, k, bands[0], bands[1], w.p, tau_mode="explicit", tau_explicit=(0.5, 1.5))
    np.testing.assert_allclose(tau, 0 * tau + np.array([0.5, 1.5]), rtol=0)
    P.check_scores(sc, ref)
    P.check_mask(mask, ref, w.p)


@pytest.mark.parametrize("force", [pb.PRISM_FORCE_SINK, pb.PRISM_FORCE_DIAG,
                                   pb.PRISM_FORCE_SINK | pb.PRISM_FORCE_DIAG])
def test_forced_blocks(force, cuda_device):
    """Optional sink / diagonal blocks are OR-ed into the mask; the attention
    with that mask matches the oracle."""
    w = gen.small_workload(f"force{force}_nb21", 1, 4, 2, 21 * 128, seed=37, p=0.5)
    q, k, v, qd, kd, vd = _inputs(w, cuda_device)
    hi, lo = gen.default_bands()
    cfg = P.make_cfg(w, force_blocks=force)
    ex = {}
    mask, _, _, words = P.run_estimate(cfg, qd, kd, extras=ex)
    ref = oracle.estimate(q, k, hi, lo, w.p, force_sink=bool(force & 1), force_diag=bool(force & 2))
    P.check_mask(mask, ref, w.p)
    P.check_topp_exact(mask, ex["weights"], w.p, force_sink=bool(force & 1), force_diag=bool(force & 2))
    nb = w.nb
    if force & 1:
        assert mask[..., 0].all()
    if force & 2:
        assert mask[..., np.arange(nb), np.arange(nb)].all()
    o = P.run_attention(cfg, qd, kd, vd, torch.from_numpy(words.view(np.int32)).to(cuda_device))
    rows = [(0, h, i) for h in range(w.hq) for i in range(nb)]
    P.check_attention_rows(o, q, k, v, mask, rows, w.hq // w.hkv)


def test_plain_pooling_baseline(cuda_device):
    """The single-band, temperature-free estimator (the coarse-grained baseline)
    matches the oracle run with the same settings, and its two bands coincide."""
    w = gen.small_workload("plain_nb24", 1, 4, 2, 24 * 128, seed=36, p=0.9)
    q, k, v, qd, kd, vd = _inputs(w, cuda_device)
    cfg = pb.plain_pooling_config(w.batch, w.hq, w.hkv, w.seqlen, w.p)
    mask, sc, tau, _ = P.run_estimate(cfg, qd, kd)
    dims = list(range(128))
    ref = oracle.estimate(q, k, dims, dims, w.p, tau_mode="explicit", tau_explicit=(1.0, 1.0))
    np.testing.assert_array_equal(ref["keep_hi"], ref["keep_lo"])
    P.check_scores(sc, ref)
    P.check_mask(mask, ref, w.p)


@pytest.mark.parametrize("seed,n_hi,n_lo", [(41, 17, 50), (42, 60, 90), (43, 5, 3), (44, 100, 100)])
def test_irregular_bands(seed, n_hi, n_lo, cuda_device):
    """Arbitrary band index sets (any sizes, overlaps, dims in neither band):
    exercises the zero-padded segment layout of the pooled rows."""
    w = gen.small_workload(f"bands_{seed}", 1, 4, 2, 19 * 128, seed=seed, p=0.9)
    q, k, v, qd, kd, vd = _inputs(w, cuda_device)
    rng = np.random.default_rng(seed)
    hi = sorted(rng.choice(128, n_hi, replace=False).tolist())
    lo = sorted(rng.choice(128, n_lo, replace=False).tolist())
    cfg = P.make_cfg(w, bands=(hi, lo))
    mask, sc, tau, _ = P.run_estimate(cfg, qd, kd)
    ref = oracle.estimate(q, k, hi, lo, w.p)
    P.check_tau(tau, ref)
    P.check_scores(sc, ref)
    P.check_mask(mask, ref, w.p)


def test_long_rows_in_parts_with_the_widest_layout(cuda_device):
    """Rows longer than one score part (512 key blocks) with band sets whose
    pooled layout is 192 columns wide (64-block column chunks): the parts'
    row maxima and counters combine to the oracle's scores and masks."""
    w = gen.small_workload("parts_dp192_nb600", 1, 1, 1, 600 * 128, seed=90, p=0.9)
    q, k, _ = gen.make_inputs(w, with_v=False)
    rng = np.random.default_rng(42)  # 60 / 90 dims: a 192-column pooled layout
    hi = sorted(rng.choice(128, 60, replace=False).tolist())
    lo = sorted(rng.choice(128, 90, replace=False).tolist())
    cfg = P.make_cfg(w, bands=(hi, lo))
    mask, sc, tau, _ = P.run_estimate(cfg, q.to(cuda_device), k.to(cuda_device))
    ref = oracle.estimate(q, k, hi, lo, w.p)
    P.check_tau(tau, ref)
    P.check_scores(sc, ref)
    P.check_mask(mask, ref, w.p)


@pytest.mark.parametrize("layout", ["interleaved", "half_split"])
def test_rope_layout_presets(layout, cuda_device):
    """Inputs rotated in either RoPE layout, bands from the matching preset:
    estimator and attention match the oracle."""
    w = gen.small_workload(f"rope_{layout}_nb21", 1, 4, 2, 21 * 128, seed=63, p=0.9,
                           interleaved=layout == "interleaved")
    q, k, v, qd, kd, vd = _inputs(w, cuda_device)
    hi, lo = pb.rope_band_sets(layout)
    cfg = P.make_cfg(w, bands=(hi, lo))
    mask, sc, tau, words = P.run_estimate(cfg, qd, kd)
    ref = oracle.estimate(q, k, hi, lo, w.p)
    P.check_tau(tau, ref)
    P.check_scores(sc, ref)
    P.check_mask(mask, ref, w.p)
    o = P.run_attention(cfg, qd, kd, vd, torch.from_numpy(words.view(np.int32)).to(cuda_device))
    rows = [(0, h, i) for h in range(w.hq) for i in range(0, w.nb, 2)]
    P.check_attention_rows(o, q, k, v, mask, rows, w.hq // w.hkv)


def _crowded_inputs(kind: str, nb: int, seed: int):
    """Q, K (bf16, [1, 2, N, 128] / [1, 1, N, 128]) whose pooled logits tie or
    crowd into one Top-P bin: every K token of block j is c + s * r_j, so the
    pooled K rows differ only by s * r_j (s = 0: exact ties in every row);
    "mixed" keeps random K tokens in the second half of the blocks."""
    g = torch.Generator("cpu")
    g.manual_seed(seed)
    n = nb * 128
    a_q = torch.randn(2, 1, 128, generator=g)
    q = (a_q + 0.5 * torch.randn(2, n, 128, generator=g)).to(torch.bfloat16)[None]
    c = torch.randn(1, 128, generator=g)
    r = torch.randn(nb, 128, generator=g)
    s = {"ties": 0.0, "crowded": 0.005, "mixed": 0.005}[kind]
    kb = c + s * r  # [nb, 128]
    k = kb.repeat_interleave(128, dim=0)[None]  # [1, N, 128]
    if kind == "mixed":
        k[:, n // 2:] = torch.randn(1, n - n // 2, 128, generator=g)
    return q, k.to(torch.bfloat16)[None]


@pytest.mark.parametrize("kind", ["ties", "crowded", "mixed"])
def test_topp_ties_and_crowded_bins(kind, cuda_device):
    """Rows whose blocks share (or nearly share) one logit: the crossing bin
    holds many members, so the exact Top-P refines on lower key bits and, for
    equal keys, cuts by block index -- the oracle's stable order."""
    nb, p = 40, 0.91
    q, k = _crowded_inputs(kind, nb, seed=71 + len(kind))
    w = gen.small_workload(f"crowd_{kind}", 1, 2, 1, nb * 128, seed=0, p=p)
    cfg = P.make_cfg(w)
    ex = {}
    mask, sc, tau, _ = P.run_estimate(cfg, q.to(cuda_device), k.to(cuda_device), extras=ex)
    hi, lo = gen.default_bands()
    ref = oracle.estimate(q, k, hi, lo, p)
    P.check_tau(tau, ref)
    P.check_scores(sc, ref)
    P.check_mask(mask, ref, p)
    P.check_topp_exact(mask, ex["weights"], p)  # the refinement and equal-key paths, bit-exact
    self_mask, self_cx = P.topp_on_scores(sc, p)
    near = (np.abs(self_cx[..., 0, :, :] - p) < P.SELF_WINDOW) | (np.abs(self_cx[..., 1, :, :] - p) < P.SELF_WINDOW)
    assert not np.any((self_mask != mask) & ~near)
    if kind == "ties":  # every row keeps exactly its first ceil(p (i + 1)) blocks
        for i in range(nb):
            keep = int(np.ceil(p * (i + 1) - 1e-9))
            assert mask[0, 0, i, :keep].all() and not mask[0, 0, i, keep:].any(), i


def test_variable_length_batch(cuda_device):
    """A padded batch of sequences of different lengths (seqlens): every
    sequence's mask rows and outputs equal those of the same sequence run
    alone (bit for bit) and match the oracle; rows past a sequence are empty
    mask rows and unwritten outputs."""
    lens = [9 * 128 + 77, 700, 129, 128]
    n_max, hq, hkv = max(lens), 4, 2
    singles = [gen.small_workload(f"varlen_{n}", 1, hq, hkv, n, seed=80 + x, p=0.9) for x, n in enumerate(lens)]
    b = len(lens)
    q = torch.zeros(b, hq, n_max, 128, dtype=torch.bfloat16)
    k = torch.zeros(b, hkv, n_max, 128, dtype=torch.bfloat16)
    v = torch.full((b, hkv, n_max, 128), 7.0, dtype=torch.bfloat16)  # finite padding, never used
    parts = []
    for x, w in enumerate(singles):
        qs, ks, vs = gen.make_inputs(w)
        q[x, :, :w.seqlen], k[x, :, :w.seqlen], v[x, :, :w.seqlen] = qs[0], ks[0], vs[0]
        parts.append((qs, ks, vs))
    hi, lo = gen.default_bands()
    cfg = pb.PrismConfig(b, hq, hkv, n_max, hi, lo, 0.9, seqlens=lens)
    nb, W = cfg.nb, cfg.words
    qd, kd, vd = q.to(cuda_device), k.to(cuda_device), v.to(cuda_device)
    ws = torch.empty(pb.prism_workspace_size(cfg), dtype=torch.uint8, device=cuda_device)
    mask = torch.full((b, hq, nb, W), 0x5A5A5A5A, dtype=torch.int32, device=cuda_device)
    o = torch.full_like(qd, 3.0)
    pb.prism_prefill(cfg, qd, kd, vd, mask, o, ws)
    torch.cuda.synchronize()
    assert pb.prism_get_last_device_error() == 0
    words = mask.cpu().numpy().view(np.uint32)
    ocpu = o.cpu()
    # the padded batch's pooled means: each sequence's blocks over its own tokens
    ex = {}
    P.run_estimate(cfg, qd, kd, with_scores=False, extras=ex)
    P.check_pooled(ex["pooled"], q, k, seq_tokens=lens)
    for x, w in enumerate(singles):
        qs, ks, vs = parts[x]
        nbx = w.nb
        assert not words[x, :, nbx:].any(), "mask rows past the sequence must be empty"
        assert torch.all(ocpu[x, :, w.seqlen:] == 3.0), "output rows past the sequence were written"
        # the same sequence alone
        cfg1 = P.make_cfg(w)
        m1, sc1, tau1, w1 = P.run_estimate(cfg1, qs.to(cuda_device), ks.to(cuda_device))
        assert np.array_equal(words[x, :, :nbx, :cfg1.words], w1[0])
        o1 = P.run_attention(cfg1, qs.to(cuda_device), ks.to(cuda_device), vs.to(cuda_device),
                             torch.from_numpy(w1.view(np.int32)).to(cuda_device))
        assert torch.equal(o[x, :, :w.seqlen].cpu(), o1[0].cpu())
        # and the oracle on it
        ref = oracle.estimate(qs, ks, hi, lo, w.p)
        P.check_tau(tau1, ref)
        P.check_mask(m1, ref, w.p)
        rows = [(0, h, i) for h in range(hq) for i in range(nbx)]
        P.check_attention_rows(o1, qs, ks, vs, m1, rows, hq // hkv)


def test_widest_gqa_group(cuda_device):
    """64 Q heads on one KV head (the largest group the temperature step
    takes): estimator and attention match the oracle."""
    w = gen.small_workload("gqa64_nb5", 1, 64, 1, 5 * 128 + 40, seed=91, p=0.9)
    q, k, v, qd, kd, vd = _inputs(w, cuda_device)
    hi, lo = gen.default_bands()
    cfg = P.make_cfg(w)
    mask, sc, tau, words = P.run_estimate(cfg, qd, kd)
    ref = oracle.estimate(q, k, hi, lo, w.p)
    P.check_tau(tau, ref)
    P.check_scores(sc, ref)
    P.check_mask(mask, ref, w.p)
    o = P.run_attention(cfg, qd, kd, vd, torch.from_numpy(words.view(np.int32)).to(cuda_device))
    rows = [(0, h, i) for h in (0, 1, 31, 62, 63) for i in range(w.nb)]
    P.check_attention_rows(o, q, k, v, mask, rows, 64)


@pytest.mark.parametrize("shape", [(1, 2, 1, 128, None), (1, 3, 1, 2 * 128, None), (2, 4, 2, 3 * 128 - 5, None),
                                   (1, 2, 2, 17 * 128, None), (3, 2, 1, 9 * 128 + 3, [9 * 128 + 3, 1, 300])],
                         ids=["nb1", "nb2", "nb3_short", "nb17", "varlen"])
def test_outputs_stay_inside_their_buffers(shape, cuda_device):
    """The caller's mask and output sit between guard regions filled with a
    pattern; a prefill over odd shapes (1, 2, 3, 17 blocks, a short last block,
    a padded batch) writes inside them only, and its mask matches a separate
    estimate."""
    b, hq, hkv, n, lens = shape
    w = gen.small_workload("guard", b, hq, hkv, n, seed=95, p=0.9)
    q, k, v, qd, kd, vd = _inputs(w, cuda_device)
    if lens is not None:  # padded batch: zero q, k past each sequence
        for x, nx in enumerate(lens):
            qd[x, :, nx:] = 0
            kd[x, :, nx:] = 0
    hi, lo = gen.default_bands()
    cfg = pb.PrismConfig(b, hq, hkv, n, hi, lo, w.p, seqlens=lens)
    nb, W = cfg.nb, cfg.words
    guard = 4096
    m_n, o_n = b * hq * nb * W, b * hq * n * 128
    m_full = torch.full((guard + m_n + guard,), 0x7E57C0DE, dtype=torch.int32, device=cuda_device)
    o_full = torch.full((guard + o_n + guard,), 1234.0, dtype=torch.bfloat16, device=cuda_device)
    mask = m_full[guard:guard + m_n].view(b, hq, nb, W)
    o = o_full[guard:guard + o_n].view(b, hq, n, 128)
    ws = torch.empty(pb.prism_workspace_size(cfg), dtype=torch.uint8, device=cuda_device)
    pb.prism_prefill(cfg, qd, kd, vd, mask, o, ws)
    torch.cuda.synchronize()
    assert pb.prism_get_last_device_error() == 0
    assert torch.all(m_full[:guard] == 0x7E57C0DE) and torch.all(m_full[guard + m_n:] == 0x7E57C0DE)
    assert torch.all(o_full[:guard] == 1234.0) and torch.all(o_full[guard + o_n:] == 1234.0)
    mask2 = torch.empty_like(mask)
    pb.prism_estimate(cfg, qd, kd, mask2, ws)
    torch.cuda.synchronize()
    assert torch.equal(mask, mask2)


def test_small_p_sparse_rows(cuda_device):
    w = gen.small_workload("sparse_nb48", 1, 2, 1, 48 * 128, seed=35, p=0.3)
    q, k, v, qd, kd, vd = _inputs(w, cuda_device)
    mask, sc, tau, words = P.run_estimate(P.make_cfg(w), qd, kd)
    hi, lo = gen.default_bands()
    ref = oracle.estimate(q, k, hi, lo, w.p)
    P.check_mask(mask, ref, w.p)
    assert P.density(mask) < 0.9
    o = P.run_attention(P.make_cfg(w), qd, kd, vd, torch.from_numpy(words.view(np.int32)).to(cuda_device))
    rows = [(0, h, i) for h in range(2) for i in range(w.nb)]
    P.check_attention_rows(o, q, k, v, mask, rows, 2)


def test_prefill_matches_separate_calls_and_is_deterministic(cuda_device):
    w = gen.small_workload("prefill_nb25", 1, 8, 2, 25 * 128, seed=36)
    q, k, v, qd, kd, vd = _inputs(w, cuda_device)
    cfg = P.make_cfg(w)
    ws = torch.empty(pb.prism_workspace_size(cfg), dtype=torch.uint8, device=cuda_device)
    outs, masks = [], []
    for _ in range(2):
        mask = torch.empty(1, 8, w.nb, cfg.words, dtype=torch.int32, device=cuda_device)
        o = torch.empty_like(qd)
        pb.prism_prefill(cfg, qd, kd, vd, mask, o, ws)
        outs.append(o)
        masks.append(mask)
    torch.cuda.synchronize()
    assert torch.equal(masks[0], masks[1]) and torch.equal(outs[0], outs[1])
    m2, _, _, words = P.run_estimate(cfg, qd, kd, with_scores=False)
    assert np.array_equal(masks[0].cpu().numpy().view(np.uint32), words)
    o2 = P.run_attention(cfg, qd, kd, vd, masks[0])
    assert torch.equal(o2, outs[0])
    # prefill with the mask kept in the workspace gives the same output
    o3 = torch.empty_like(qd)
    pb.prism_prefill(cfg, qd, kd, vd, None, o3, ws)
    torch.cuda.synchronize()
    assert torch.equal(o3, outs[0])
    assert pb.prism_get_last_device_error() == 0


def test_softmax_scale_argument(cuda_device):
    w = gen.small_workload("scale_nb6", 1, 2, 1, 6 * 128, seed=37)
    q, k, v, qd, kd, vd = _inputs(w, cuda_device)
    nb = w.nb
    m = np.tril(np.ones((1, 2, nb, nb), dtype=bool))
    words = oracle.pack_mask(m)
    cfg = P.make_cfg(w, softmax_scale=0.05)
    o = P.run_attention(cfg, qd, kd, vd, torch.from_numpy(words.view(np.int32)).to(cuda_device))
    rows = [(0, h, i) for h in range(2) for i in range(nb)]
    P.check_attention_rows(o, q, k, v, m, rows, 2, scale=0.05)


@pytest.mark.parametrize("base,nb", [(5e5, 6), (1e6, 5)])
def test_pooled_rope_attenuation_on_gpu(base, nb, cuda_device):
    """The pooling-attenuation closed form (paper.rainbus.top review, novelty
    paragraph: a RoPE pair pooled over B positions keeps the fraction
    lambda_j(B) ~ sinc(B theta_j / 2 pi) of its length) on the kernel's pooled
    means.  Input: one constant pre-RoPE vector per head, rotated at
    positions 0..N-1 and rounded to bf16.  Every block's pooled pair j has
    length |a_j| |sin(B theta_j / 2) / (B sin(theta_j / 2))| (the Dirichlet
    form; the block's start only rotates it).  bf16 rounding (an 8-bit
    significand: unit roundoff 2^-8) moves each coordinate by <= 2^-8 of the
    pair length, so the measured ratio is within sqrt(2) 2^-8 of the exact
    form; fp32 pooling adds < 2^-18.  The normalised sinc is within 6.2e-4 of
    the exact form (oracle pin)."""
    d, half, B = 128, 64, 128
    n = nb * B
    g = torch.Generator("cpu")
    g.manual_seed(int(base) % 1000 + nb)
    a = torch.randn(2, d, generator=g, dtype=torch.float64)  # one vector per head (Q head, KV head)
    cos, sin = gen.rope_tables(n, d, base)
    x = gen.apply_rope(a[:, None, :].expand(2, n, d), cos, sin).to(torch.bfloat16)
    q, k = x[0][None, None].contiguous(), x[1][None, None].contiguous()
    w = gen.small_workload("sinc_pin", 1, 1, 1, n, seed=0, p=0.9)
    ex = {}
    P.run_estimate(P.make_cfg(w), q.to(cuda_device), k.to(cuda_device), with_scores=False, extras=ex)
    pooled = ex["pooled"]  # [2, nb, 128]: the Q head, then the KV head
    P.check_pooled(pooled, q, k)
    theta = np.array(gen.rope_theta(d, base))
    exact = np.abs(np.sin(B * theta / 2) / (B * np.sin(theta / 2)))
    sinc = np.abs(np.sinc(B * theta / (2 * np.pi)))  # numpy's sinc is the normalised one
    bound = math.sqrt(2) * 2.0 ** -8 + 2.0 ** -17
    for r in range(2):
        a_len = np.hypot(a[r, :half].numpy(), a[r, half:].numpy())
        for blk in range(nb):
            pair_len = np.hypot(pooled[r, blk, :half], pooled[r, blk, half:])
            lam = pair_len / a_len
            assert np.all(np.abs(lam - exact) <= bound), (r, blk, np.abs(lam - exact).max())
            assert np.all(np.abs(lam - sinc) <= bound + 6.2e-4), (r, blk, np.abs(lam - sinc).max())
            # the dead zone (B theta_j >= 2 pi) stays under the first side-lobe
            # peak of |sinc| (0.2172...); the slow pairs pass almost unattenuated
            dead = B * theta >= 2 * np.pi
            assert np.all(lam[dead] < 0.2173 + 6.2e-4 + bound)
            assert np.all(lam[32:] > 0.99 - bound)
