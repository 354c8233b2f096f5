"""The seeded generator is deterministic and follows its stated recipe."""
import torch

from tests import gen


def test_generator_deterministic_and_shapes():
    w = gen.small_workload("g", 2, 4, 2, 512, seed=3)
    q1, k1, v1 = gen.make_inputs(w)
    q2, k2, v2 = gen.make_inputs(w)
    assert q1.shape == (2, 4, 512, 128) and k1.shape == (2, 2, 512, 128) and v1.shape == k1.shape
    assert q1.dtype == torch.bfloat16
    assert torch.equal(q1, q2) and torch.equal(k1, k2) and torch.equal(v1, v2)


def test_generator_position_zero_is_unrotated():
    # at t = 0 RoPE is the identity, so q_0 = bf16(a_q + 0.5 z_0)
    w = gen.small_workload("g0", 1, 1, 1, 256, seed=9)
    q, _, _ = gen.make_inputs(w)
    g = torch.Generator("cpu")
    g.manual_seed(9)
    a_q = torch.randn(1, 128, generator=g)
    torch.randn(1, 128, generator=g)
    z = torch.randn(1, 256, 128, generator=g)
    ref = (a_q[0].double() + 0.5 * z[0, 0].double()).to(torch.bfloat16)
    assert torch.equal(q[0, 0, 0], ref)


def test_planted_workload_small():
    w = gen.small_workload("planted", 1, 4, 2, 1024, seed=3, rope_base=1e6, stripes=True, slash=True)
    q, k, v = gen.make_inputs(w)
    assert torch.isfinite(q.float()).all() and torch.isfinite(k.float()).all()


def test_default_bands():
    hi, lo = gen.default_bands()
    assert len(hi) == 64 and len(lo) == 96
    assert hi[:32] == list(range(32)) and hi[32:] == list(range(64, 96))
    assert lo[:48] == list(range(16, 64)) and lo[48:] == list(range(80, 128))


def test_interleaved_rope_is_permuted_half_split():
    # interleaved pair j = dims (2j, 2j+1); moving dim 2j to j and 2j+1 to
    # j + D/2 turns it into the half-split layout with the same angles
    cos, sin = gen.rope_tables(64, 128, 10000.0)
    x = torch.randn(3, 64, 128, dtype=torch.float64, generator=torch.Generator().manual_seed(1))
    perm = [2 * j for j in range(64)] + [2 * j + 1 for j in range(64)]
    a = gen.apply_rope(x, cos, sin, interleaved=True)[..., perm]
    b = gen.apply_rope(x[..., perm], cos, sin)
    assert torch.allclose(a, b, rtol=0, atol=1e-15)
    # the rotation keeps every pair's norm
    n0 = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    n1 = gen.apply_rope(x, cos, sin, interleaved=True)
    assert torch.allclose(n1[..., 0::2] ** 2 + n1[..., 1::2] ** 2, n0, rtol=1e-12)
