"""Planted mistakes: each pin set must fail on a wrong oracle.

Each case below plants one plausible slip in a copy of the oracle's source on
the CPU (a dropped square root, a swapped band, an inverted temperature, an
off-by-one in the causal test, a Top-P scan that counts a block's own mass, a
wrong GQA or batch index, a reversed bit order ...), executes the copy as a
module of its own, points the ``oracle`` package's functions at it and runs
every oracle pin (the pin tests of the pooling closed forms, the hand-worked
example, the temperature invariants, Top-P against brute force, the attention
against the library and the RoPE presets).  At least one pin must fail for
each planted slip; the unmodified oracle must pass them all through the same
harness.  Nothing here touches the CUDA path.
"""
import inspect
import itertools
import pathlib
import types
import warnings

import numpy as np
import pytest

import oracle
import oracle.prism_oracle as oracle_module
from tests import test_oracle_pins, test_rope_presets

SOURCE = pathlib.Path(oracle_module.__file__).read_text()

# (label, text in the oracle, replacement)
MUTANTS = [
    # steps (1)-(2): slicing and pooling
    ("slice takes the other dims", "return x[..., list(dims)]", "return np.delete(x, list(dims), axis=-1)"),
    ("pool sums instead of averaging", "head = x[..., :full, :].reshape(shp).mean(axis=-2)",
     "head = x[..., :full, :].reshape(shp).sum(axis=-2)"),
    ("short block divided by the full block", "tail = x[..., full:, :].mean(axis=-2, keepdims=True)",
     "tail = x[..., full:, :].sum(axis=-2, keepdims=True) / block"),
    ("full band is the high band", "    full = list(range(d))\n", "    full = list(band_hi)\n"),
    ("Q low band pooled from the high dims", "qb_lo = mean_pool(band_slice(qh, band_lo), block)",
     "qb_lo = mean_pool(band_slice(qh, band_hi), block)"),
    ("keys of batch 0 for every element", "kb[kv] = (mean_pool(band_slice(kf[bi, kv], band_hi), block),",
     "kb[kv] = (mean_pool(band_slice(kf[0, kv], band_hi), block),"),
    # step (3): RMS
    ("RMS without the square root", "return np.sqrt(np.mean(pooled_band * pooled_band, axis=(-2, -1)))",
     "return np.mean(pooled_band * pooled_band, axis=(-2, -1))"),
    ("mean absolute value for RMS", "return np.sqrt(np.mean(pooled_band * pooled_band, axis=(-2, -1)))",
     "return np.mean(np.abs(pooled_band), axis=(-2, -1))"),
    ("largest per-block RMS", "return np.sqrt(np.mean(pooled_band * pooled_band, axis=(-2, -1)))",
     "return np.max(np.sqrt(np.mean(pooled_band * pooled_band, axis=-1)), axis=-1)"),
    ("K RMS of the bands swapped", "rk = dict(hi=rms(kbar_hi), lo=rms(kbar_lo), full=rms(kbar_full))",
     "rk = dict(hi=rms(kbar_lo), lo=rms(kbar_hi), full=rms(kbar_full))"),
    ("Q full-spectrum RMS from the high band",
     "rq = dict(hi=rms(qbar_hi), lo=rms(qbar_lo), full=rms(qbar_full))",
     "rq = dict(hi=rms(qbar_hi), lo=rms(qbar_lo), full=rms(qbar_hi))"),
    # step (4): temperature
    ("temperature inverted", "    return num / den\n", "    return den / num\n"),
    ("temperature square-rooted", "    return num / den\n", "    return math.sqrt(num / den)\n"),
    ("temperature from Q twice", "num = rq_z * rk_z", "num = rq_z * rq_z"),
    ("no fallback for a zero RMS", "    if num == 0.0 or den == 0.0:\n        return 1.0\n", ""),
    # step (5): logits and softmax
    ("logits divided by d_z", "lg = (qbar_z @ kbar_z.T) / (tau_z * math.sqrt(d_z))",
     "lg = (qbar_z @ kbar_z.T) / (tau_z * d_z)"),
    ("logits scaled by the head dim", "lg = (qbar_z @ kbar_z.T) / (tau_z * math.sqrt(d_z))",
     "lg = (qbar_z @ kbar_z.T) / (tau_z * math.sqrt(128))"),
    ("logits multiplied by tau", "lg = (qbar_z @ kbar_z.T) / (tau_z * math.sqrt(d_z))",
     "lg = (qbar_z @ kbar_z.T) * tau_z / math.sqrt(d_z)"),
    ("logits without tau", "lg = (qbar_z @ kbar_z.T) / (tau_z * math.sqrt(d_z))",
     "lg = (qbar_z @ kbar_z.T) / math.sqrt(d_z)"),
    ("logits transposed", "lg = (qbar_z @ kbar_z.T)", "lg = (kbar_z @ qbar_z.T)"),
    ("low band divided by the high tau", "lg_lo = band_logits(qbar_lo, kbar_lo, tau_lo)",
     "lg_lo = band_logits(qbar_lo, kbar_lo, tau_hi)"),
    ("diagonal block masked", "lg[np.triu_indices(nb, k=1)] = -np.inf", "lg[np.triu_indices(nb, k=0)] = -np.inf"),
    ("anti-causal block mask", "lg[np.triu_indices(nb, k=1)] = -np.inf", "lg[np.tril_indices(nb, k=-1)] = -np.inf"),
    ("no block mask", "lg[np.triu_indices(nb, k=1)] = -np.inf", "pass"),
    ("softmax normalised over columns", "return e / np.sum(e, axis=-1, keepdims=True)",
     "return e / np.sum(e, axis=0, keepdims=True)"),
    # step (6): Top-P
    ("keep while the mass ahead is <= p", "keep = causal & (c_excl < p)", "keep = causal & (c_excl <= p)"),
    ("mass ahead includes the block itself",
     "c_excl_sorted = np.concatenate([np.zeros((nb, 1)), c_incl[:, :-1]], axis=1)", "c_excl_sorted = c_incl"),
    ("smallest blocks first", "key = np.where(causal, -probs, np.inf)", "key = np.where(causal, probs, np.inf)"),
    ("ties to the higher block index", "order = np.argsort(key, axis=1, kind=\"stable\")",
     "order = (nb - 1) - np.argsort(key[:, ::-1], axis=1, kind=\"stable\")"),
    ("scan in index order", "sorted_p = np.take_along_axis(np.where(causal, probs, 0.0), order, axis=1)",
     "sorted_p = np.where(causal, probs, 0.0)"),
    ("mass ahead left in rank order", "np.put_along_axis(c_excl, order, c_excl_sorted, axis=1)",
     "c_excl[...] = c_excl_sorted"),
    ("p = 1 left to the floating-point sum", "if p >= 1.0:", "if p > 1.0:"),
    # step (7) and the optional forced blocks
    ("intersection instead of union", "mask=keep_hi | keep_lo)", "mask=keep_hi & keep_lo)"),
    ("high band only", "mask=keep_hi | keep_lo)", "mask=keep_hi.copy())"),
    ("GQA by h mod Hkv", "            kv = h // grp\n", "            kv = h % hkv\n"),
    ("sink forced as a row", "forced[:, 0] = True", "forced[0, :] = True"),
    ("diagonal forced as the sink", "forced[np.arange(nbh), np.arange(nbh)] = True", "forced[:, 0] = True"),
    # attention
    ("attention GQA by h mod group", "    kv = h // group\n", "    kv = h % group\n"),
    ("query does not see its own key", "visible = key_pos[None, :] <= q_pos[:, None]",
     "visible = key_pos[None, :] < q_pos[:, None]"),
    ("no token causality in the diagonal block", "visible = key_pos[None, :] <= q_pos[:, None]",
     "visible = np.ones((q_pos.size, key_pos.size), dtype=bool)"),
    ("attention scaled by 1/D", "    scale = 1.0 / math.sqrt(d) if scale is None else scale\n    js",
     "    scale = 1.0 / d if scale is None else scale\n    js"),
    ("block mask ignored", "js = [j for j in range(i + 1) if bool(mask_row[j])]", "js = list(range(i + 1))"),
    ("diagonal block dropped", "js = [j for j in range(i + 1) if bool(mask_row[j])]",
     "js = [j for j in range(i) if bool(mask_row[j])]"),
    ("values read from K", "vf = np.concatenate([to_f64(v[b, kv", "vf = np.concatenate([to_f64(k[b, kv"),
    ("keys of batch 0", "kf = np.concatenate([to_f64(k[b, kv", "kf = np.concatenate([to_f64(k[0, kv"),
    ("values of batch 0", "vf = np.concatenate([to_f64(v[b, kv", "vf = np.concatenate([to_f64(v[0, kv"),
    ("softmax not normalised", "out = (e @ vf) / np.where(den > 0, den, 1.0)", "out = (e @ vf)"),
    ("column maximum subtracted", "m = np.max(s, axis=1, keepdims=True)", "m = np.max(s, axis=0, keepdims=True)"),
    ("dense attention GQA by h mod group", "s = qf[bi, h] @ kf[bi, h // group].T * scale",
     "s = qf[bi, h] @ kf[bi, h % group].T * scale"),
    ("dense attention scaled by 1/D", "    scale = 1.0 / math.sqrt(d) if scale is None else scale\n    out",
     "    scale = 1.0 / d if scale is None else scale\n    out"),
    # mask packing
    ("packed MSB first", "weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))",
     "weights = (np.uint64(1) << np.arange(31, -1, -1, dtype=np.uint64))"),
    ("unpacked MSB first", "shifts = np.arange(32, dtype=np.uint64)", "shifts = np.arange(31, -1, -1, dtype=np.uint64)"),
]


def _pin_cases():
    """Every pin test of the two modules with its parametrize grid expanded."""
    cases = []
    for module in (test_oracle_pins, test_rope_presets):
        for name, fn in inspect.getmembers(module, inspect.isfunction):
            if not name.startswith("test_") or fn.__module__ != module.__name__:
                continue
            grids = []
            for mark in getattr(fn, "pytestmark", []):
                if mark.name != "parametrize":
                    continue
                argnames = mark.args[0]
                argnames = [a.strip() for a in argnames.split(",")] if isinstance(argnames, str) else list(argnames)
                values = [v if len(argnames) > 1 else (v,) for v in mark.args[1]]
                grids.append([dict(zip(argnames, v)) for v in values])
            params = set(inspect.signature(fn).parameters)
            for combo in itertools.product(*grids):
                kwargs = {}
                for part in combo:
                    kwargs.update(part)
                assert set(kwargs) == params, f"{name}: the harness calls pins without fixtures"
                cases.append((f"{module.__name__}::{name}{kwargs or ''}", fn, kwargs))
    return cases


PIN_CASES = _pin_cases()
ORACLE_FUNCTIONS = [n for n in dir(oracle)
                    if getattr(getattr(oracle, n), "__module__", None) == oracle_module.__name__]


def _first_failing_pin():
    for label, fn, kwargs in PIN_CASES:
        try:
            with np.errstate(all="ignore"), warnings.catch_warnings():
                warnings.simplefilter("ignore")
                fn(**kwargs)
        except Exception as exc:  # an assertion or a crash both fail the pin
            return label, type(exc).__name__
    return None


def _install(monkeypatch, source):
    module = types.ModuleType("oracle_with_planted_mistake")
    exec(compile(source, "oracle_with_planted_mistake", "exec"), module.__dict__)
    for name in ORACLE_FUNCTIONS:
        monkeypatch.setattr(oracle, name, getattr(module, name))


def test_harness_runs_every_pin_and_the_oracle_passes(monkeypatch):
    assert len(PIN_CASES) >= 40 and len(ORACLE_FUNCTIONS) >= 10
    _install(monkeypatch, SOURCE)  # the unmodified source through the same path
    assert _first_failing_pin() is None


@pytest.mark.parametrize("label,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(label, old, new, monkeypatch):
    assert SOURCE.count(old) == 1, f"the oracle no longer contains the text this case plants into: {old!r}"
    _install(monkeypatch, SOURCE.replace(old, new))
    failed = _first_failing_pin()
    assert failed is not None, f"no pin fails with the planted mistake '{label}'"
    print(f"{label}: caught by {failed[0]} ({failed[1]})")
