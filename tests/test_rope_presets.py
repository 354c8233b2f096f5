"""Band presets for the two RoPE layouts (host logic + oracle invariants).

Prism's bands are chosen in frequency order (Prism: Spectral-Aware
Block-Sparse Attention, gist.science Technical Summary section 2, step (1):
high band = the first d_high dims, low band = the last d_low dims), and RoPE
turns pair j at theta_j = base^(-2j/D).  Which physical dims carry pair j is a
property of the checkpoint's RoPE layout; ``rope_band_sets`` maps the frequency
choice to dim index sets for either layout.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_band_b200 as pb
import oracle
from tests import gen


def test_half_split_preset_is_the_default_bands():
    assert pb.rope_band_sets("half_split") == gen.default_bands()


def test_interleaved_preset():
    hi, lo = pb.rope_band_sets("interleaved")
    # pair j sits at dims (2j, 2j+1): the 32 fastest pairs are dims 0..63,
    # the 48 slowest pairs are dims 32..127
    assert hi == list(range(64)) and lo == list(range(32, 128))


def test_preset_sizes_and_errors():
    hi, lo = pb.rope_band_sets("interleaved", d_high=32, d_low=16)
    assert hi == list(range(32)) and lo == list(range(112, 128))
    hi, lo = pb.rope_band_sets("half_split", d_high=128, d_low=128)
    assert hi == list(range(128)) and lo == list(range(128))
    for bad in (dict(layout="neox"), dict(d_high=63), dict(d_low=0), dict(d_high=130)):
        with pytest.raises(ValueError):
            pb.rope_band_sets(**bad)


def test_presets_are_accepted_by_the_config():
    for layout in ("half_split", "interleaved"):
        hi, lo = pb.rope_band_sets(layout)
        cfg = pb.PrismConfig(1, 4, 2, 1024, hi, lo, 0.95)
        assert cfg.c.n_hi == 64 and cfg.c.n_lo == 96


def _perm_interleaved_to_half_split(d=128):
    # half-split dim j <- interleaved dim 2j, half-split dim j + D/2 <- interleaved dim 2j + 1
    return np.array([2 * j for j in range(d // 2)] + [2 * j + 1 for j in range(d // 2)])


def test_interleaved_estimate_equals_permuted_half_split():
    """Reordering the head dims consistently in Q, K and the band sets leaves
    every estimator output unchanged (pooling is per dim, band sums are order
    free).  The interleaved preset on interleaved inputs is therefore the same
    estimator as the half-split preset on the same vectors in half-split order."""
    w = gen.small_workload("il", 1, 4, 2, 12 * 128, seed=61, interleaved=True)
    q, k, _ = gen.make_inputs(w, with_v=False)
    q, k = q.double().numpy(), k.double().numpy()
    perm = _perm_interleaved_to_half_split()
    r_il = oracle.estimate(q, k, *pb.rope_band_sets("interleaved"), 0.9)
    r_hs = oracle.estimate(q[..., perm], k[..., perm], *pb.rope_band_sets("half_split"), 0.9)
    np.testing.assert_allclose(r_il["tau"], r_hs["tau"], rtol=1e-12)
    f = np.isfinite(r_il["logits"])
    np.testing.assert_allclose(r_il["logits"][f], r_hs["logits"][f], rtol=1e-10, atol=1e-13)
    assert np.array_equal(r_il["mask"], r_hs["mask"])


def test_layout_mismatch_changes_the_estimate():
    """The half-split preset on interleaved inputs mixes fast and slow pairs in
    both bands: the high band's temperature no longer drops below the low
    band's, as it does with the matching preset."""
    w = gen.small_workload("il2", 1, 4, 2, 16 * 128, seed=62, interleaved=True)
    q, k, _ = gen.make_inputs(w, with_v=False)
    q, k = q.double().numpy(), k.double().numpy()
    good = oracle.estimate(q, k, *pb.rope_band_sets("interleaved"), 0.9)
    wrong = oracle.estimate(q, k, *pb.rope_band_sets("half_split"), 0.9)
    assert np.all(good["tau"][..., 0] < good["tau"][..., 1])
    assert not np.allclose(good["tau"], wrong["tau"])


def _yarn_theta(head_dim, base, scale, orig_len, alpha=1.0, beta=32.0):
    """YaRN's "NTK-by-parts" frequencies (Peng et al., YaRN, 2023): pair j with
    r_j = orig_len * theta_j / (2 pi) rotations over the original context keeps
    theta_j when r_j > beta, is interpolated to theta_j / scale when r_j < alpha,
    and blends linearly in between."""
    theta = np.array(gen.rope_theta(head_dim, base))
    r = orig_len * theta / (2 * np.pi)
    gamma = np.clip((r - alpha) / (beta - alpha), 0.0, 1.0)
    return (1.0 - gamma) * theta / scale + gamma * theta


def _dirichlet(theta, block):
    return np.abs(np.sin(block * theta / 2.0) / (block * np.sin(theta / 2.0)))


@pytest.mark.parametrize("layout", ["half_split", "interleaved"])
@pytest.mark.parametrize("ladder", ["plain", "yarn"])
def test_pooling_attenuation_by_layout_and_ladder(layout, ladder):
    """A constant pre-RoPE vector rotated over one block and mean pooled keeps
    the Dirichlet fraction of each pair's magnitude whatever the layout, and
    under YaRN's rescaled ladder too.  The ladder stays monotone (pair 0 the
    fastest), so the presets' high band still holds the most attenuated pairs."""
    B, D, base = 128, 128, 5e5
    theta = np.array(gen.rope_theta(D, base)) if ladder == "plain" else _yarn_theta(D, base, 4.0, 8192)
    assert np.all(np.diff(theta) < 0)
    rng = np.random.default_rng(11)
    c = torch.from_numpy(rng.standard_normal(D))
    cos, sin = gen.rope_tables(B, D, base, start=128 * 5, theta=theta)
    x = gen.apply_rope(c[None, :].expand(B, D).clone(), cos, sin, interleaved=layout == "interleaved").numpy()
    pooled = oracle.mean_pool(x, B)[0]
    hi, lo = pb.rope_band_sets(layout)
    if layout == "interleaved":
        pin, pout = np.hypot(c.numpy()[0::2], c.numpy()[1::2]), np.hypot(pooled[0::2], pooled[1::2])
    else:
        pin, pout = np.hypot(c.numpy()[:64], c.numpy()[64:]), np.hypot(pooled[:64], pooled[64:])
    lam = pout / pin
    np.testing.assert_allclose(lam, _dirichlet(theta, B), rtol=0, atol=1e-12)
    # energy kept per band: the high band loses most of it, the low band almost none
    e_in, e_out = c.numpy() ** 2, pooled ** 2
    kept_hi = e_out[hi].sum() / e_in[hi].sum()
    kept_lo = e_out[lo].sum() / e_in[lo].sum()
    assert kept_hi < 0.75 and kept_lo > 0.85 and kept_hi < kept_lo


def test_mrope_on_text_is_plain_rope():
    """Text tokens under M-RoPE (t = h = w = index) rotate exactly as under
    plain RoPE, so the presets, the pooling attenuation and the whole estimate
    are unchanged (gist.science Technical Summary, results: Prism carries over
    to M-RoPE)."""
    n, d, base = 1024, 128, 1e6
    idx = torch.arange(n)
    cos_m, sin_m = gen.mrope_tables(torch.stack([idx, idx, idx], dim=1), d, base)
    cos_r, sin_r = gen.rope_tables(n, d, base)
    assert torch.equal(cos_m, cos_r) and torch.equal(sin_m, sin_r)


@pytest.mark.parametrize("height,width", [(8, 16), (4, 32)])
def test_mrope_video_block_attenuation(height, width):
    """One frame of height x width = 128 patch tokens pooled as one block: the
    temporal pairs do not rotate inside it (no attenuation), the height pairs
    step once per row (Dirichlet kernel over `height` positions), the width
    pairs once per token within a row (Dirichlet kernel over `width`).  So on
    video the fastest pairs are not the most attenuated ones: the text-derived
    high band holds the unattenuated temporal section."""
    d, base = 128, 1e6
    sections = (16, 24, 24)
    pos = gen.video_positions(1, height, width, t0=3)
    assert pos.shape[0] == 128
    cos, sin = gen.mrope_tables(pos, d, base, sections)
    rng = np.random.default_rng(5)
    c = torch.from_numpy(rng.standard_normal(d))
    x = gen.apply_rope(c[None, :].expand(128, d).clone(), cos, sin).numpy()
    pooled = oracle.mean_pool(x, 128)[0]
    lam = np.hypot(pooled[:64], pooled[64:]) / np.hypot(c.numpy()[:64], c.numpy()[64:])
    theta = np.array(gen.rope_theta(d, base))
    expect = np.concatenate([np.ones(sections[0]),
                             _dirichlet(theta[16:40], height),
                             _dirichlet(theta[40:64], width)])
    np.testing.assert_allclose(lam, expect, rtol=0, atol=1e-12)
    hi, lo = pb.rope_band_sets("half_split")
    e_in, e_out = c.numpy() ** 2, pooled ** 2
    temporal_hi = [k for k in hi if k % 64 < 16]
    assert np.isclose(e_out[temporal_hi].sum(), e_in[temporal_hi].sum(), rtol=1e-12)
