"""Python binding of the Prism B200 library (include/prism.h).

Argument marshalling only: every step of the estimator and the attention runs
in the CUDA kernels of ``libprism_b200.so``; PyTorch provides device memory and
streams.  The functions carry the C names; each raises ``PrismError`` when the
library returns a non-zero status.  There is no CPU fallback: importing this
package fails if the library has not been built
(``python block_sparse_attention_band_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

__all__ = [
    "PrismError", "PrismConfig", "plain_pooling_config", "rope_band_sets", "lib", "lib_path", "prism_version", "prism_status_str",
    "prism_workspace_size", "prism_estimate", "prism_sparse_attn", "prism_prefill",
    "prism_get_last_device_error", "prism_estimate_noalloc", "prism_noalloc_scratch_bytes",
    "prism_selftest_wait_timeout",
    "PRISM_TAU_RMS", "PRISM_TAU_EXPLICIT", "PRISM_FORCE_SINK", "PRISM_FORCE_DIAG", "EXPORTED_SYMBOLS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libprism_b200.so")

PRISM_TAU_RMS = 0
PRISM_TAU_EXPLICIT = 1
PRISM_FORCE_SINK = 1  # keep key block 0 in every row (optional, not part of the method)
PRISM_FORCE_DIAG = 2  # keep the diagonal block in every row (optional)

EXPORTED_SYMBOLS = (
    "prism_workspace_size", "prism_estimate", "prism_sparse_attn", "prism_prefill",
    "prism_get_last_device_error", "prism_status_str", "prism_version", "prism_estimate_noalloc",
    "prism_noalloc_scratch_bytes", "prism_selftest_wait_timeout",
)


def lib_path() -> str:
    return _LIB_PATH


if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"{_LIB_PATH} is missing: build the CUDA library first "
        "(python block_sparse_attention_band_b200/build.py); there is no CPU fallback")

lib = ctypes.CDLL(_LIB_PATH)


class _Config(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int), ("hq", ctypes.c_int), ("hkv", ctypes.c_int),
        ("seqlen", ctypes.c_int), ("head_dim", ctypes.c_int), ("block", ctypes.c_int),
        ("band_hi", ctypes.POINTER(ctypes.c_int32)), ("n_hi", ctypes.c_int),
        ("band_lo", ctypes.POINTER(ctypes.c_int32)), ("n_lo", ctypes.c_int),
        ("p", ctypes.c_float), ("causal", ctypes.c_int), ("tau_mode", ctypes.c_int),
        ("tau_hi", ctypes.c_float), ("tau_lo", ctypes.c_float), ("softmax_scale", ctypes.c_float),
        ("force_blocks", ctypes.c_int),
        ("seqlens", ctypes.POINTER(ctypes.c_int32)),
    ]


class _Debug(ctypes.Structure):
    _fields_ = [("scores", ctypes.c_void_p), ("weights", ctypes.c_void_p), ("tau", ctypes.c_void_p),
                ("pooled", ctypes.c_void_p)]


_vp = ctypes.c_void_p
_cfgp = ctypes.POINTER(_Config)
lib.prism_version.restype = ctypes.c_int
lib.prism_status_str.restype = ctypes.c_char_p
lib.prism_status_str.argtypes = [ctypes.c_int]
lib.prism_workspace_size.restype = ctypes.c_int
lib.prism_workspace_size.argtypes = [_cfgp, ctypes.POINTER(ctypes.c_size_t)]
lib.prism_estimate.restype = ctypes.c_int
lib.prism_estimate.argtypes = [_cfgp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp, ctypes.POINTER(_Debug)]
lib.prism_sparse_attn.restype = ctypes.c_int
lib.prism_sparse_attn.argtypes = [_cfgp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.prism_prefill.restype = ctypes.c_int
lib.prism_prefill.argtypes = [_cfgp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
lib.prism_estimate_noalloc.restype = ctypes.c_int
lib.prism_estimate_noalloc.argtypes = [_cfgp, _vp, _vp, _vp, _vp]
lib.prism_noalloc_scratch_bytes.restype = ctypes.c_size_t
lib.prism_noalloc_scratch_bytes.argtypes = []
lib.prism_selftest_wait_timeout.restype = ctypes.c_int
lib.prism_selftest_wait_timeout.argtypes = [_vp, ctypes.c_uint]
lib.prism_get_last_device_error.restype = ctypes.c_int
lib.prism_get_last_device_error.argtypes = [_vp]


class PrismError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: status {status} ({prism_status_str(status)})")


class PrismConfig:
    """Owns a ``prism_config`` and the band index arrays it points to."""

    def __init__(self, batch: int, hq: int, hkv: int, seqlen: int, band_hi: Sequence[int],
                 band_lo: Sequence[int], p: float, head_dim: int = 128, block: int = 128,
                 causal: int = 1, tau_mode: int = PRISM_TAU_RMS, tau_hi: float = 1.0,
                 tau_lo: float = 1.0, softmax_scale: float = 0.0, force_blocks: int = 0,
                 seqlens: Optional[Sequence[int]] = None):
        """``seqlens``: tokens of each batch element when they differ (padded
        layout of ``seqlen`` tokens; padding zero in q and k, finite in v)."""
        self._hi = (ctypes.c_int32 * max(len(band_hi), 1))(*band_hi)
        self._lo = (ctypes.c_int32 * max(len(band_lo), 1))(*band_lo)
        self._sl = (ctypes.c_int32 * len(seqlens))(*seqlens) if seqlens is not None else None
        self.c = _Config(batch, hq, hkv, seqlen, head_dim, block,
                         ctypes.cast(self._hi, ctypes.POINTER(ctypes.c_int32)), len(band_hi),
                         ctypes.cast(self._lo, ctypes.POINTER(ctypes.c_int32)), len(band_lo),
                         p, causal, tau_mode, tau_hi, tau_lo, softmax_scale, force_blocks,
                         ctypes.cast(self._sl, ctypes.POINTER(ctypes.c_int32)) if self._sl is not None
                         else ctypes.POINTER(ctypes.c_int32)())

    @property
    def nb(self) -> int:
        return -(-self.c.seqlen // self.c.block)  # the last block may be short

    @property
    def words(self) -> int:
        return (self.nb + 31) // 32

    def ptr(self):
        return ctypes.byref(self.c)


def rope_band_sets(layout: str = "half_split", d_high: int = 64, d_low: int = 96,
                   head_dim: int = 128):
    """(band_hi, band_lo) index sets for a RoPE layout.

    RoPE rotates dimension pairs; pair j turns at theta_j = base^(-2j / D), j = 0
    the fastest.  The high band is the d_high / 2 fastest pairs, the low band the
    d_low / 2 slowest (the review's method step (1) takes the leading d_high and the trailing
    d_low dims, read here in frequency-pair order).  Pair j occupies dims (j, j + D/2) in the
    half-split layout (GPT-NeoX / Llama-style checkpoints) and (2j, 2j + 1) in
    the interleaved layout (GPT-J-style).  RoPE variants that keep the
    frequencies monotone in j -- YaRN's per-band interpolation, M-RoPE's
    temporal / height / width sections of one frequency ladder -- keep these
    sets; only the attenuation of each pair under pooling changes."""
    half = head_dim // 2
    if d_high % 2 or d_low % 2 or not (0 < d_high <= head_dim) or not (0 < d_low <= head_dim):
        raise ValueError("band sizes must be even and in (0, head_dim]")
    hi_pairs = range(0, d_high // 2)
    lo_pairs = range(half - d_low // 2, half)
    if layout == "half_split":
        dims = lambda pairs: sorted([j for j in pairs] + [j + half for j in pairs])
    elif layout == "interleaved":
        dims = lambda pairs: sorted([2 * j for j in pairs] + [2 * j + 1 for j in pairs])
    else:
        raise ValueError(f"unknown RoPE layout {layout!r}")
    return dims(hi_pairs), dims(lo_pairs)


def plain_pooling_config(batch: int, hq: int, hkv: int, seqlen: int, p: float,
                         head_dim: int = 128) -> PrismConfig:
    """The standard coarse-grained block estimator that Prism is set against
    (gist.science, Technical Summary section 1): one band of all dims, no
    temperature, i.e. Top-P of softmax(Q_bar K_bar^T / sqrt(head_dim)) per
    query-block row, mean pooling over each block.  Both Prism bands are set
    to the full index set, so M = M_high = M_low."""
    dims = list(range(head_dim))
    return PrismConfig(batch, hq, hkv, seqlen, dims, dims, p, head_dim=head_dim,
                       tau_mode=PRISM_TAU_EXPLICIT, tau_hi=1.0, tau_lo=1.0)


def _addr(x) -> Optional[int]:
    """Device address of a CUDA tensor (or a raw int address); None -> NULL."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if not x.is_cuda:
        raise ValueError("tensor arguments must be CUDA tensors (the library takes device pointers)")
    if not x.is_contiguous():
        raise ValueError("tensor arguments must be contiguous")
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str) -> None:
    if status != 0:
        raise PrismError(status, where)


def prism_version() -> int:
    return lib.prism_version()


def prism_status_str(status: int) -> str:
    return lib.prism_status_str(status).decode()


def prism_workspace_size(cfg: PrismConfig) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.prism_workspace_size(cfg.ptr(), ctypes.byref(n)), "prism_workspace_size")
    return n.value


def prism_estimate(cfg: PrismConfig, q, k, mask, workspace, stream=None, dbg_scores=None,
                   dbg_tau=None, dbg_weights=None, dbg_pooled=None) -> None:
    """The estimator; the ``dbg_*`` tensors (optional, fp32 on the device)
    receive the members of ``prism_debug`` (include/prism.h)."""
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    dbg = None
    if any(x is not None for x in (dbg_scores, dbg_tau, dbg_weights, dbg_pooled)):
        dbg = ctypes.byref(_Debug(_addr(dbg_scores), _addr(dbg_weights), _addr(dbg_tau), _addr(dbg_pooled)))
    _check(lib.prism_estimate(cfg.ptr(), _addr(q), _addr(k), _addr(mask), _addr(workspace), ws_bytes,
                              _stream(stream), dbg), "prism_estimate")


def prism_sparse_attn(cfg: PrismConfig, q, k, v, mask, o, stream=None) -> None:
    _check(lib.prism_sparse_attn(cfg.ptr(), _addr(q), _addr(k), _addr(v), _addr(mask), _addr(o),
                                 _stream(stream)), "prism_sparse_attn")


def prism_prefill(cfg: PrismConfig, q, k, v, mask_out, o, workspace, stream=None) -> None:
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib.prism_prefill(cfg.ptr(), _addr(q), _addr(k), _addr(v), _addr(mask_out), _addr(o),
                             _addr(workspace), ws_bytes, _stream(stream)), "prism_prefill")


def prism_estimate_noalloc(cfg: PrismConfig, q, k, mask, stream=None) -> None:
    """The estimator on the library's built-in scratch (no workspace argument)."""
    _check(lib.prism_estimate_noalloc(cfg.ptr(), _addr(q), _addr(k), _addr(mask), _stream(stream)),
           "prism_estimate_noalloc")


def prism_noalloc_scratch_bytes() -> int:
    return lib.prism_noalloc_scratch_bytes()


def prism_selftest_wait_timeout(timeout_us: int, stream=None) -> None:
    """Enqueue the failure-path self test (bounded waits that must give up)."""
    _check(lib.prism_selftest_wait_timeout(_stream(stream), timeout_us), "prism_selftest_wait_timeout")


def prism_get_last_device_error(stream=None) -> int:
    return lib.prism_get_last_device_error(_stream(stream))
