"""One layer split by KV group (block_sparse_attention_band_b200.shard), run
as separate calls on one GPU: the slices' masks and outputs equal the rows
of the call on the whole layer, bit for bit.  This is what each rank of a
multi-GPU prefill computes (no exchange step: every step of the estimator and
the attention is per head or per KV group)."""
import numpy as np
import pytest
import torch

import block_sparse_attention_band_b200 as pb
from block_sparse_attention_band_b200 import shard
from tests import gen
from tests import parity as P

pytestmark = pytest.mark.gpu


def _prefill(cfg, q, k, v, mask, o):
    ws = torch.empty(pb.prism_workspace_size(cfg), dtype=torch.uint8, device=q.device)
    pb.prism_prefill(cfg, q, k, v, mask, o, ws)


@pytest.mark.parametrize("w,lens", [
    (gen.small_workload("shard_nb40", 1, 32, 8, 40 * 128, seed=61), None),
    (gen.small_workload("shard_b2_nb21", 2, 8, 4, 21 * 128 - 9, seed=62, p=0.9), None),
    (gen.small_workload("shard_varlen", 3, 4, 2, 17 * 128, seed=63, p=0.9), [17 * 128, 700, 129]),
], ids=["llama_shape_nb40", "batch2_short", "varlen"])
@pytest.mark.parametrize("world", [2, 4])
def test_kv_group_slices_reproduce_the_whole_layer(w, lens, world, cuda_device):
    q, k, v = gen.make_inputs(w)
    if lens is not None:
        for x, n in enumerate(lens):  # padding: zero q, k
            q[x, :, n:] = 0
            k[x, :, n:] = 0
    qd, kd, vd = q.to(cuda_device), k.to(cuda_device), v.to(cuda_device)
    hi, lo = gen.default_bands()
    cfg = pb.PrismConfig(w.batch, w.hq, w.hkv, w.seqlen, hi, lo, w.p, seqlens=lens)
    nb, W = cfg.nb, cfg.words
    mask = torch.full((w.batch, w.hq, nb, W), 0x11, dtype=torch.int32, device=cuda_device)
    o = torch.full_like(qd, 5.0)
    _prefill(cfg, qd, kd, vd, mask, o)
    mask_s = torch.full_like(mask, 0x22)
    o_s = torch.full_like(qd, 6.0)
    g = w.hq // w.hkv
    n_runs = 0
    for rank in range(world):
        for run in shard.shard_runs(w.batch, w.hkv, world, rank):
            qs, ks, vs, ms, os_ = shard.run_views(run, g, qd, kd, vd, mask_s, o_s)
            c = pb.PrismConfig(1, qs.shape[1], ks.shape[1], w.seqlen, hi, lo, w.p,
                               seqlens=shard.run_seqlens(run, lens))
            _prefill(c, qs, ks, vs, ms, os_)
            n_runs += 1
    torch.cuda.synchronize()
    assert pb.prism_get_last_device_error() == 0
    assert n_runs >= world
    assert torch.equal(mask_s, mask), f"{(mask_s != mask).sum().item()} mask words differ"
    if lens is None:
        assert torch.equal(o_s, o), "outputs differ"
    else:  # rows past a sequence are not written by either call
        for x, n in enumerate(lens):
            assert torch.equal(o_s[x, :, :n], o[x, :, :n])
    assert P.density(oracle_unpack(mask, nb)) < 1.0


def oracle_unpack(mask, nb):
    import oracle
    return oracle.unpack_mask(mask.cpu().numpy().view(np.uint32), nb)
