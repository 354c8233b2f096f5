"""The C-ABI library loads, exports every entry point include/prism.h declares,
and rejects bad arguments on the host before touching the GPU (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

import block_sparse_attention_band_b200 as pb  # noqa: E402  (built by conftest)
from tests import gen  # noqa: E402

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "prism.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(prism_\w+)\s*\(", text)))


def test_header_declares_expected_entry_points():
    names = declared_functions()
    assert set(pb.EXPORTED_SYMBOLS) <= set(names)
    for must in ("prism_estimate", "prism_sparse_attn", "prism_prefill"):
        assert must in names


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", pb.lib_path()], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT\s+(prism_\w+)$", out, flags=re.M))
    for name in declared_functions():
        assert name in exported, f"{name} declared in prism.h but not exported"
        assert hasattr(pb.lib, name)


def test_version_and_status_strings():
    assert pb.prism_version() >= 100
    for code in range(0, -12, -1):
        s = pb.prism_status_str(code)
        assert s and s != "unknown status"
    assert pb.prism_status_str(-999) == "unknown status"


def _cfg(**kw):
    hi, lo = gen.default_bands()
    args = dict(batch=1, hq=4, hkv=2, seqlen=1024, band_hi=hi, band_lo=lo, p=0.95)
    args.update(kw)
    return pb.PrismConfig(**args)


def _ws_size(cfg):
    n = ctypes.c_size_t(0)
    return pb.lib.prism_workspace_size(cfg.ptr(), ctypes.byref(n)), n.value


def test_workspace_size_properties():
    """The workspace grows with the sequence, the heads and the batch, and a
    call with one byte less than the reported size is refused before anything
    is enqueued."""
    s, base = _ws_size(_cfg())
    assert s == 0 and base > 0 and base % 256 == 0
    sizes_n = [_ws_size(_cfg(seqlen=n))[1] for n in (128, 1024, 4096, 32768, 131072)]
    assert all(a < b for a, b in zip(sizes_n, sizes_n[1:])), sizes_n
    sizes_h = [_ws_size(_cfg(hq=hq, hkv=hkv))[1] for hq, hkv in ((1, 1), (2, 1), (4, 2), (8, 2), (32, 8))]
    assert all(a < b for a, b in zip(sizes_h, sizes_h[1:])), sizes_h
    assert _ws_size(_cfg(batch=2))[1] > base
    # every pooled value needs at least 3 x 2 bytes per kept dim: a floor that any layout meets
    assert base >= 6 * (4 + 2) * 8 * 128
    a = 1 << 20
    cfg = _cfg()
    assert pb.lib.prism_estimate(cfg.ptr(), a, a, a, a, base - 1, None, None) == -7
    assert pb.lib.prism_prefill(cfg.ptr(), a, a, a, a, a, a, base - 1, None) == -7


@pytest.mark.parametrize("kw,code", [
    (dict(hq=3, hkv=2), -2), (dict(batch=0), -2), (dict(seqlen=0), -2),
    (dict(head_dim=64), -6), (dict(block=64), -6), (dict(causal=0), -6), (dict(tau_mode=7), -6),
    (dict(p=0.0), -5), (dict(p=-1.0), -5), (dict(p=float("nan")), -5),
    (dict(band_hi=[]), -4), (dict(band_lo=[0, 0]), -4), (dict(band_hi=[128]), -4), (dict(band_lo=[-1]), -4),
    (dict(tau_mode=1, tau_hi=0.0), -11), (dict(tau_mode=1, tau_lo=float("inf")), -11),
    (dict(seqlen=128 * 16385), -6),
])
def test_bad_config_rejected_on_host(kw, code):
    s, _ = _ws_size(_cfg(**kw))
    assert s == code, pb.prism_status_str(s)
    # the compute entry points reject the same config before any CUDA call
    fake = 1 << 20
    assert pb.lib.prism_estimate(_cfg(**kw).ptr(), fake, fake, fake, fake, 1 << 40, None, None) == code
    assert pb.lib.prism_sparse_attn(_cfg(**kw).ptr(), fake, fake, fake, fake, fake, None) == code
    assert pb.lib.prism_prefill(_cfg(**kw).ptr(), fake, fake, fake, None, fake, fake, 1 << 40, None) == code


def test_seqlens_validated_and_layout_sized():
    base = _ws_size(_cfg())[1]
    ok = _cfg(batch=3, seqlens=[1024, 1, 500])
    s, n = _ws_size(ok)
    assert s == 0 and n == _ws_size(_cfg(batch=3))[1]  # the workspace follows the padded layout
    for bad in ([0, 5, 5], [1025, 5, 5], [-3, 5, 5]):
        assert _ws_size(_cfg(batch=3, seqlens=bad))[0] == -2
    assert _ws_size(_cfg(batch=257, seqlens=[7] * 257))[0] == -6
    assert base > 0


def test_null_pointers_workspace_and_alignment_rejected():
    cfg = _cfg()
    _, ws = _ws_size(cfg)
    a = 1 << 20
    assert pb.lib.prism_workspace_size(None, ctypes.byref(ctypes.c_size_t())) == -1
    assert pb.lib.prism_workspace_size(cfg.ptr(), None) == -1
    assert pb.lib.prism_estimate(cfg.ptr(), None, a, a, a, ws, None, None) == -1
    assert pb.lib.prism_estimate(cfg.ptr(), a, a, None, a, ws, None, None) == -1
    assert pb.lib.prism_estimate(cfg.ptr(), a, a, a, None, ws, None, None) == -7
    assert pb.lib.prism_estimate(cfg.ptr(), a, a, a, a, ws - 1, None, None) == -7
    assert pb.lib.prism_estimate(cfg.ptr(), a + 8, a, a, a, ws, None, None) == -3
    assert pb.lib.prism_estimate(cfg.ptr(), a, a, a, a + 16, ws, None, None) == -3
    assert pb.lib.prism_sparse_attn(cfg.ptr(), a, a, a, a, None, None) == -1
    assert pb.lib.prism_sparse_attn(cfg.ptr(), a, a, a + 2, a, a, None) == -3
    assert pb.lib.prism_prefill(cfg.ptr(), a, a, a, None, a, None, ws, None) == -7
    assert pb.lib.prism_prefill(cfg.ptr(), a, a, a, a + 2, a, a, ws, None) == -3  # masks: 4-byte words


def test_python_binding_rejects_host_tensors():
    import torch
    cfg = _cfg()
    q = torch.zeros(1, 4, 1024, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        pb.prism_sparse_attn(cfg, q, q, q, q, q, stream=0)


def test_plain_pooling_config_is_one_band_without_temperature():
    cfg = pb.plain_pooling_config(1, 4, 2, 1024, 0.9)
    assert cfg.c.n_hi == cfg.c.n_lo == 128
    assert [cfg.c.band_hi[i] for i in range(128)] == list(range(128))
    assert cfg.c.tau_mode == pb.PRISM_TAU_EXPLICIT and cfg.c.tau_hi == cfg.c.tau_lo == 1.0
    s, n = _ws_size(cfg)
    assert s == 0 and n > 0


def test_short_last_block_is_accepted():
    """seqlen need not be a multiple of the block: ceil(seqlen / 128) blocks."""
    s, n = _ws_size(_cfg(seqlen=1000))
    assert s == 0 and n > 0
    assert _cfg(seqlen=1000).nb == 8 and _cfg(seqlen=1000).words == 1


def test_force_blocks_flags_validated():
    s, _ = _ws_size(_cfg(force_blocks=pb.PRISM_FORCE_SINK | pb.PRISM_FORCE_DIAG))
    assert s == 0
    s, _ = _ws_size(_cfg(force_blocks=4))
    assert s == -6
