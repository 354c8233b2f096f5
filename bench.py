"""Benchmark: Prism prefill ms/layer at 128K (estimator + block-sparse attention).

One step = one prefill layer through the C ABI (prism_prefill: pool, tau,
scores, Top-P, tcgen05 attention) on the Llama-3-8B-shaped layer (32 Q / 8 KV
heads, head_dim 128) at N = 131072, seeded synthetic post-RoPE inputs.

    python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--impl prism|reference]

Multi-GPU (torchrun, one rank per GPU): the one layer is split across the ranks
by (batch, KV group) units (block_sparse_attention_band_b200.shard: every unit's
estimator and attention need only its own heads), with no data-path collective;
each step every rank runs its share, the step time is the max over ranks and
``value`` is ms per whole layer (strong scaling).  ``--impl reference`` times
the fp64 CPU oracle on a bounded sample of the same layer (rank 0 only).
``--record-traffic CSV`` turns an ncu capture of the DRAM-byte counters into
a record keyed by the hash of the CUDA sources (``--traffic-out``, by default
the ``profiles/dram_traffic.json`` that the roofline objects read).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from tests import gen  # noqa: E402

METRIC = "Prism prefill ms/layer @128K (estimate+sparse attn); estimator overhead %"
UNIT = "ms/layer"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")
KERNEL_SOURCES = ("estimate.cuh", "attention.cuh", "ptx.cuh", "prism.cu")
KERNELS_PER_STEP = 2  # estimator_kernel + sparse_attn_kernel (the queue reset is a memset)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    """sha256 over the CUDA sources, to tell whether profiled counters are stale."""
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "block_sparse_attention_band_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes (read + write) per launch of each kernel for ``workload``,
    from the committed ncu record: the captured workload's bytes per launch
    times the recorded scale factor (the ratio of units the two workloads
    process).  Empty when the record is missing, has no factor for the
    workload, or the CUDA sources differ from the ones profiled."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return {}
    if rec.get("source_sha256_16") != kernel_source_hash():
        return {}
    out = {}
    for kern, d in rec.get("kernels", {}).items():
        scale = d.get("scale_to", {}).get(workload, 1.0 if workload == rec.get("workload") else None)
        if scale is not None:
            out[kern] = (d["dram_read_bytes_per_launch"] + d["dram_write_bytes_per_launch"]) * scale
    return out


def record_traffic(csv_paths, workload: str, scales, out_path: str):
    """Parse ncu --csv --print-units base captures of dram__bytes_read.sum /
    dram__bytes_write.sum and write the per-kernel bytes per launch, with the
    hash of the current CUDA sources, to ``out_path``."""
    import csv
    per = {}
    for path in csv_paths:
        with open(path) as f:
            lines = [ln for ln in f if ln.startswith('"')]
        for row in csv.DictReader(lines):
            name = row.get("Kernel Name", "")
            kern = "estimator_kernel" if "estimator" in name else ("sparse_attn_kernel" if "sparse_attn" in name else None)
            metric = row.get("Metric Name", "")
            if kern is None or metric not in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
                continue
            unit = (row.get("Metric Unit") or "byte").lower()
            mult = {"byte": 1, "kbyte": 1e3, "mbyte": 1e6, "gbyte": 1e9}.get(unit, 1)
            val = float(str(row["Metric Value"]).replace(",", "")) * mult
            d = per.setdefault(kern, {}).setdefault(row["ID"], {})
            d[metric] = val
    kernels = {}
    for kern, launches in per.items():
        rd = [x["dram__bytes_read.sum"] for x in launches.values() if len(x) == 2]
        wr = [x["dram__bytes_write.sum"] for x in launches.values() if len(x) == 2]
        if not rd:
            continue
        kernels[kern] = {"launches": len(rd), "dram_read_bytes_per_launch": sum(rd) / len(rd),
                         "dram_write_bytes_per_launch": sum(wr) / len(wr),
                         "scale_to": {k: v for k, v in scales.items()}}
    rec = {"source_sha256_16": kernel_source_hash(), "workload": workload, "kernels": kernels,
           "note": "ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum --print-units base; "
                   "scale_to: bytes of a launch on another workload = bytes per launch here x factor"}
    with open(out_path, "w") as f:
        json.dump(rec, f, indent=1)
    print(json.dumps(rec))


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        except OSError:
            pass
        finally:
            if self.path and os.path.exists(self.path):
                os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": num(rows[0][2]), "samples": len(rows),
                "power_w_max": max((num(r[3]) or 0.0) for r in rows), "reasons": reasons}


def sample_heads_and_blocks(w, seed: int, n_heads: int = 4, n_blocks: int = 16):
    """The oracle's sample of a layer: one Q head from each of ``n_heads`` KV
    groups spread over the layer (the seed picks the head within its group),
    and query blocks {0, 1, nb/2, nb-1} plus seeded random ones."""
    rng = np.random.default_rng(seed)
    g = w.hq // w.hkv
    n_heads = min(n_heads, w.hkv)
    groups = sorted({round(x * (w.hkv - 1) / max(n_heads - 1, 1)) for x in range(n_heads)})
    heads = [kv * g + int(rng.integers(g)) for kv in groups]
    fixed = sorted({0, min(1, w.nb - 1), w.nb // 2, w.nb - 1})[:n_blocks]
    blocks = set(fixed)
    while len(blocks) < min(n_blocks, w.nb):
        blocks.add(int(rng.integers(w.nb)))
    return heads, sorted(blocks)


def cpu_oracle_sample(q, k, v, mask_words, w, n_heads=4, n_blocks=16, seed=0):
    """Time the fp64 oracle on a bounded sample of the layer and extrapolate to
    a full layer: the estimator on ``n_heads`` Q heads (x Hq / n_heads), the
    attention on those heads x ``n_blocks`` query blocks (x total kept tiles /
    sampled kept tiles).  The numbers are extrapolations, labelled so."""
    import oracle
    hi, lo = gen.default_bands()
    g = w.hq // w.hkv
    heads, blocks = sample_heads_and_blocks(w, seed, n_heads, n_blocks)
    t0 = time.perf_counter()
    own = {}
    for h in heads:
        r = oracle.estimate(q[:, h:h + 1], k[:, h // g:h // g + 1], hi, lo, w.p, keep_dense=False)
        own[h] = r["mask"][0, 0]
    t_est = (time.perf_counter() - t0) * w.hq / len(heads)
    causal = np.tril(np.ones((w.nb, w.nb), dtype=bool))
    if mask_words is not None:  # the layer's mask (all heads): its kept tiles
        m = oracle.unpack_mask(mask_words, w.nb)[0]
        kept_total = int((m & causal).sum())
        rows_of = {h: m[h] for h in heads}
    else:  # the sampled heads' own oracle masks, their mean kept count x Hq
        rows_of = own
        kept_total = int(round(sum(int((own[h] & causal).sum()) for h in heads) * w.hq / len(heads)))
    t0 = time.perf_counter()
    kept_sample = 0
    for h in heads:
        for i in blocks:
            oracle.sparse_attention_block(q, k, v, rows_of[h][i], 0, h, i, g)
            kept_sample += int(rows_of[h][i, : i + 1].sum())
    t_attn = (time.perf_counter() - t0) * kept_total / max(kept_sample, 1)
    sample = (f"extrapolated: estimator on {len(heads)} of {w.hq} Q heads x{w.hq / len(heads):g}; attention on "
              f"{len(heads)} heads x {len(blocks)} query blocks ({kept_sample} kept tiles) "
              f"x{kept_total / max(kept_sample, 1):.0f} (kept-tile ratio"
              f"{'' if mask_words is not None else ', layer kept tiles from the sampled heads'}); "
              f"one {w.seqlen}-token layer")
    return (t_est + t_attn) * 1e3, t_est * 1e3, t_attn * 1e3, sample


def reduce_max(values, dist, device):
    """Max over ranks of each value (the slowest rank sets the job time)."""
    if dist is None:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def reduce_sum(values, dist, device):
    """Sum over ranks of each value (counts: kept tiles, bytes copied, launches)."""
    if dist is None:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return [float(x) for x in t.tolist()]


def blas_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max((d.get("num_threads", 1) for d in info), default=os.cpu_count())
    except Exception:
        return os.cpu_count()


def run_reference(args, w, rank, world):
    """The oracle timed on the host cores (rank 0 only; other ranks exit).
    Each timed step runs the oracle on a fresh sample of the layer (estimator
    on 4 Q heads, attention on those heads x 16 query blocks, with the
    sampled heads' own oracle masks) and extrapolates to the whole layer; the
    warm-up steps run a minimal sample (1 head, 1 block)."""
    if rank != 0:
        return
    q, k, v = gen.make_inputs(w)
    vals = []
    sample = ""
    for step in range(args.warmup + args.steps):
        timed = step >= args.warmup
        tot, _, _, smp = cpu_oracle_sample(q, k, v, None, w, n_heads=4 if timed else 1,
                                           n_blocks=16 if timed else 1, seed=step)
        if timed:
            vals.append(tot)
            sample = smp
    val = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": val, "higher_is_better": False,
        "scaling": "strong", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "hq": w.hq, "hkv": w.hkv, "seq_len": w.seqlen,
                   "head_dim": w.head_dim, "block": w.block, "p": w.p},
        "cpu_baseline": {"value": val, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"median over {args.steps} steps of a fresh sample each; " + sample},
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


TABLE_WORKLOADS = ("tiny_2k", "llama3_8b_32k", "llama3_8b_128k", "qwen3_8b_64k_planted", "sweep_8k",
                   "sweep_16k", "sweep_64k", "sweep_128k", "sweep_256k")


def run_table(args):
    """One JSON line per workload of the five configurations (the sweep's N
    values included): estimator, attention and prefill ms/layer with CUDA
    events, density and both rooflines.  Separate from the headline line."""
    import block_sparse_attention_band_b200 as pb
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    peak_tensor = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    names = args.table.split(",") if args.table != "all" else TABLE_WORKLOADS
    for name in names:
        w = gen.WORKLOADS[name]
        q, k, v = gen.make_inputs(w)
        qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
        del q, k, v
        hi, lo = gen.default_bands()
        cfg = pb.PrismConfig(w.batch, w.hq, w.hkv, w.seqlen, hi, lo, w.p)
        ws = torch.empty(pb.prism_workspace_size(cfg), dtype=torch.uint8, device=dev)
        mask = torch.empty(w.batch, w.hq, w.nb, cfg.words, dtype=torch.int32, device=dev)
        o = torch.empty_like(qd)
        stream = torch.cuda.current_stream(dev)
        flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)  # > L2, written before each estimator run
        steps = args.steps
        for _ in range(max(args.warmup, 3)):
            pb.prism_prefill(cfg, qd, kd, vd, mask, o, ws, stream=stream)
        torch.cuda.synchronize()
        est, att, pre = [], [], []
        for _ in range(steps):
            flush.fill_(1)
            e = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
            e[0].record(stream)
            pb.prism_estimate(cfg, qd, kd, mask, ws, stream=stream)
            e[1].record(stream)
            pb.prism_sparse_attn(cfg, qd, kd, vd, mask, o, stream=stream)
            e[2].record(stream)
            flush.fill_(2)
            e[3].record(stream)
            pb.prism_prefill(cfg, qd, kd, vd, mask, o, ws, stream=stream)
            e[4].record(stream)
            torch.cuda.synchronize()
            est.append(e[0].elapsed_time(e[1]))
            att.append(e[1].elapsed_time(e[2]))
            pre.append(e[3].elapsed_time(e[4]))
        assert pb.prism_get_last_device_error() == 0
        t_est, t_att, t_pre = (statistics.median(x) for x in (est, att, pre))
        words = mask.cpu().numpy().view(np.uint32)
        causal_tiles = w.batch * w.hq * w.nb * (w.nb + 1) // 2
        kept = int(np.unpackbits(words.view(np.uint8)).sum())
        flops = kept * 4 * 128 ** 3
        est_bytes = (w.hq + w.hkv) * w.batch * w.seqlen * 128 * 2 + words.nbytes
        line = {"table": True, "workload": w.name, "seq_len": w.seqlen, "p": w.p, "steps": steps,
                "estimate_ms": t_est, "attention_ms": t_att, "prefill_ms": t_pre,
                "estimator_overhead_pct": 100.0 * t_est / (t_est + t_att), "density": kept / causal_tiles,
                "kept_tiles": kept, "attention_tflops": flops / (t_att * 1e-3) / 1e12,
                "attention_tensor_frac": flops / (t_att * 1e-3) / 1e12 / peak_tensor,
                "effective_tflops_vs_dense": causal_tiles * 4 * 128 ** 3 / (t_pre * 1e-3) / 1e12,
                "estimator_gbs": est_bytes / (t_est * 1e-3) / 1e9,
                "estimator_hbm_frac": est_bytes / (t_est * 1e-3) / 1e9 / peaks["hbm_gbs"],
                "peaks": f"{peak_src}: {peaks['hbm_gbs']} GB/s, {peak_tensor} TFLOP/s bf16 sustained",
                "timing": "CUDA events; a 512 MB buffer written before each estimator run (L2 flush)"}
        print(json.dumps(line), flush=True)
        del qd, kd, vd, ws, mask, o, flush
        torch.cuda.empty_cache()


def causal_mask_words(nb: int, words: int) -> torch.Tensor:
    """[nb, words] int32 rows keeping every causal block (p >= 1)."""
    i = np.arange(nb, dtype=np.int64)[:, None]
    lo = 32 * np.arange(words, dtype=np.int64)[None, :]
    kept = np.clip(i + 1 - lo, 0, 32)  # blocks j <= i in word [lo, lo + 32)
    bits = np.where(kept == 32, np.int64(0xFFFFFFFF), (np.int64(1) << kept) - 1)
    return torch.from_numpy(bits.astype(np.uint32).view(np.int32))


def run_sweep_p(args):
    """Prefill time against the kept-block density: one line per Top-P
    threshold p on one workload, with the same kernel on every causal block
    (dense) as the reference point."""
    import block_sparse_attention_band_b200 as pb
    dev = torch.device("cuda:0")
    w = gen.WORKLOADS[args.workload]
    q, k, v = gen.make_inputs(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    hi, lo = gen.default_bands()
    o = torch.empty_like(qd)
    stream = torch.cuda.current_stream(dev)

    def timed(fn, reps):
        fn()
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    cfg1 = pb.PrismConfig(w.batch, w.hq, w.hkv, w.seqlen, hi, lo, 1.0)
    dense_mask = causal_mask_words(w.nb, cfg1.words).expand(w.batch, w.hq, w.nb, cfg1.words).contiguous().to(dev)
    t_dense = timed(lambda: pb.prism_sparse_attn(cfg1, qd, kd, vd, dense_mask, o, stream=stream), args.steps)
    del dense_mask
    causal_tiles = w.batch * w.hq * w.nb * (w.nb + 1) // 2
    for p in [float(x) for x in args.sweep_p.split(",")]:
        cfg = pb.PrismConfig(w.batch, w.hq, w.hkv, w.seqlen, hi, lo, p)
        ws = torch.empty(pb.prism_workspace_size(cfg), dtype=torch.uint8, device=dev)
        mask = torch.empty(w.batch, w.hq, w.nb, cfg.words, dtype=torch.int32, device=dev)
        t_pre = timed(lambda: pb.prism_prefill(cfg, qd, kd, vd, mask, o, ws, stream=stream), args.steps)
        assert pb.prism_get_last_device_error() == 0
        kept = int(np.unpackbits(mask.cpu().numpy().view(np.uint8)).sum())
        print(json.dumps({"sweep_p": p, "workload": w.name, "density": kept / causal_tiles, "prefill_ms": t_pre,
                          "dense_attention_ms": t_dense, "speedup_vs_dense": t_dense / t_pre,
                          "timing": f"CUDA events, median of {args.steps}"}), flush=True)
        del ws, mask


def run_compare_plain(args):
    """Prism's estimator against the plain mean-pooling estimator (one band of
    all dims, no temperature) on one workload: density, estimator time, and the
    error of the block-sparse attention output (our kernel, each estimator's
    mask) against exact dense causal attention (fp64 oracle) on sampled rows.
    The dense line (p = 1, every causal block) is the kernel's own bf16 floor."""
    import block_sparse_attention_band_b200 as pb
    import oracle
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    w = gen.WORKLOADS[args.compare_plain]
    q, k, v = gen.make_inputs(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    hi, lo = gen.default_bands()
    g = w.hq // w.hkv
    rng = np.random.default_rng(11)
    heads = [kv * g + int(rng.integers(g)) for kv in (0, 2, 5, 7) if kv < w.hkv]
    blocks = sorted({w.nb - 1, w.nb // 2, w.nb // 4} | {int(x) for x in rng.integers(w.nb // 8, w.nb, 3)})
    dense_ref = {(h, i): oracle.sparse_attention_block(q, k, v, np.ones(w.nb, dtype=bool), 0, h, i, g)
                 for h in heads for i in blocks}
    def density_of(cfg):
        ws = torch.empty(pb.prism_workspace_size(cfg), dtype=torch.uint8, device=dev)
        mask = torch.empty(w.batch, w.hq, w.nb, cfg.words, dtype=torch.int32, device=dev)
        pb.prism_estimate(cfg, qd, kd, mask, ws)
        words = mask.cpu().numpy().view(np.uint32)
        return int(np.unpackbits(words.view(np.uint8)).sum()) / (w.batch * w.hq * w.nb * (w.nb + 1) // 2)

    # the plain estimator's p that keeps as many blocks as Prism does (bisection)
    target = density_of(pb.PrismConfig(w.batch, w.hq, w.hkv, w.seqlen, hi, lo, w.p))
    lo_p, hi_p = w.p, 0.99999
    for _ in range(20):
        mid = 0.5 * (lo_p + hi_p)
        if density_of(pb.plain_pooling_config(w.batch, w.hq, w.hkv, w.seqlen, mid)) < target:
            lo_p = mid
        else:
            hi_p = mid
    variants = [("prism", pb.PrismConfig(w.batch, w.hq, w.hkv, w.seqlen, hi, lo, w.p)),
                ("plain_pooling", pb.plain_pooling_config(w.batch, w.hq, w.hkv, w.seqlen, w.p)),
                ("plain_pooling_matched_density", pb.plain_pooling_config(w.batch, w.hq, w.hkv, w.seqlen, hi_p)),
                ("dense", pb.PrismConfig(w.batch, w.hq, w.hkv, w.seqlen, hi, lo, 1.0))]
    for name, cfg in variants:
        ws = torch.empty(pb.prism_workspace_size(cfg), dtype=torch.uint8, device=dev)
        mask = torch.empty(w.batch, w.hq, w.nb, cfg.words, dtype=torch.int32, device=dev)
        o = torch.empty_like(qd)
        for _ in range(3):
            pb.prism_estimate(cfg, qd, kd, mask, ws)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        pb.prism_estimate(cfg, qd, kd, mask, ws)
        e1.record()
        pb.prism_sparse_attn(cfg, qd, kd, vd, mask, o)
        torch.cuda.synchronize()
        assert pb.prism_get_last_device_error() == 0
        words = mask.cpu().numpy().view(np.uint32)
        density = int(np.unpackbits(words.view(np.uint8)).sum()) / (w.batch * w.hq * w.nb * (w.nb + 1) // 2)
        errs = []
        for (h, i), ref in dense_ref.items():
            got = o[0, h, i * 128:(i + 1) * 128].float().cpu().numpy().astype(np.float64)
            errs.append(float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)))
        print(json.dumps({"compare": True, "workload": w.name, "estimator": name, "p": cfg.c.p,
                          "density": density, "estimate_ms": e0.elapsed_time(e1),
                          "attn_rel_l2_err_vs_dense_mean": float(np.mean(errs)),
                          "attn_rel_l2_err_vs_dense_max": float(np.max(errs)),
                          "sampled_rows": f"heads {heads} x query blocks {blocks}"}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="prism", choices=["prism", "reference"])
    ap.add_argument("--workload", default="llama3_8b_128k", choices=sorted(gen.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end passes (profiling runs)")
    ap.add_argument("--compare-plain", default=None, choices=sorted(gen.WORKLOADS),
                    help="Prism vs the plain mean-pooling estimator on one workload (attention error vs dense)")
    ap.add_argument("--table", default=None,
                    help="'all' or a comma list of workloads: per-configuration lines instead of the headline")
    ap.add_argument("--sweep-p", default=None,
                    help="comma list of Top-P thresholds: prefill time and density per p on --workload, vs dense")
    ap.add_argument("--record-traffic", default=None,
                    help="comma list of ncu CSV files (dram__bytes_*.sum, --print-units base) of --workload")
    ap.add_argument("--traffic-out", default=TRAFFIC_FILE,
                    help="with --record-traffic: where to write the record")
    ap.add_argument("--traffic-scale", default="",
                    help="with --record-traffic: comma list workload=factor (bytes per launch there / here)")
    args = ap.parse_args()
    if args.record_traffic:
        scales = dict((kv.split("=")[0], float(kv.split("=")[1])) for kv in args.traffic_scale.split(",") if kv)
        os.makedirs(os.path.dirname(os.path.abspath(args.traffic_out)), exist_ok=True)
        record_traffic(args.record_traffic.split(","), args.workload, scales, args.traffic_out)
        return
    if args.table:
        run_table(args)
        return
    if args.sweep_p:
        run_sweep_p(args)
        return
    if args.compare_plain:
        run_compare_plain(args)
        return
    rank, world, local = dist_env()
    w = gen.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, w, rank, world)
        return

    import block_sparse_attention_band_b200 as pb
    from block_sparse_attention_band_b200 import shard

    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)

    # the one layer, generated identically on every rank; each rank uploads
    # and runs its share: runs of whole KV groups (shard.shard_runs)
    q, k, v = gen.make_inputs(w)
    g = w.hq // w.hkv
    hi, lo = gen.default_bands()
    runs = shard.shard_runs(w.batch, w.hkv, world, rank)
    parts = []
    for r in runs:
        qs, ks, vs, _, _ = shard.run_views(r, g, q, k, v, None, None)
        cfg = pb.PrismConfig(1, qs.shape[1], ks.shape[1], w.seqlen, hi, lo, w.p)
        part = {"run": r, "cfg": cfg, "qh": qs.contiguous(), "kh": ks.contiguous(), "vh": vs.contiguous()}
        part["q"], part["k"], part["v"] = part["qh"].to(dev), part["kh"].to(dev), part["vh"].to(dev)
        part["ws"] = torch.empty(pb.prism_workspace_size(cfg), dtype=torch.uint8, device=dev)
        part["mask"] = torch.empty(1, qs.shape[1], w.nb, cfg.words, dtype=torch.int32, device=dev)
        part["o"] = torch.empty_like(part["q"])
        parts.append(part)
    stream = torch.cuda.current_stream(dev)

    def step():
        for x in parts:
            pb.prism_prefill(x["cfg"], x["q"], x["k"], x["v"], x["mask"], x["o"], x["ws"], stream=stream)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    assert pb.prism_get_last_device_error() == 0

    # ---------------- timed region: K prefill steps -----------------------
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier()
    clocks = clk.summary()
    ms_step = reduce_max([ev0.elapsed_time(ev1) / args.steps], dist, dev)[0]
    assert pb.prism_get_last_device_error() == 0

    # ---------------- stage breakdown (same launches, events in between) ----
    est_ms, attn_ms = [], []
    for _ in range(args.steps):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record(stream)
        for x in parts:
            pb.prism_estimate(x["cfg"], x["q"], x["k"], x["mask"], x["ws"], stream=stream)
        e[1].record(stream)
        for x in parts:
            pb.prism_sparse_attn(x["cfg"], x["q"], x["k"], x["v"], x["mask"], x["o"], stream=stream)
        e[2].record(stream)
        torch.cuda.synchronize()
        est_ms.append(e[0].elapsed_time(e[1]))
        attn_ms.append(e[1].elapsed_time(e[2]))
    t_est_own, t_attn_own = statistics.median(est_ms), statistics.median(attn_ms)
    t_est, t_attn = reduce_max([t_est_own, t_attn_own], dist, dev)
    # the same attention kernel on every causal block (p = 1): the dense
    # prefill the method is set against (context for the speed-up, not timed
    # in the step)
    dense_ms = []
    dense_masks = [causal_mask_words(w.nb, x["cfg"].words).expand(1, x["q"].shape[1], w.nb, x["cfg"].words)
                   .contiguous().to(dev) for x in parts]
    for _ in range(3):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        e[0].record(stream)
        for x, dm in zip(parts, dense_masks):
            pb.prism_sparse_attn(x["cfg"], x["q"], x["k"], x["v"], dm, x["o"], stream=stream)
        e[1].record(stream)
        torch.cuda.synchronize()
        dense_ms.append(e[0].elapsed_time(e[1]))
    t_dense = reduce_max([statistics.median(dense_ms)], dist, dev)[0]
    del dense_masks

    words_parts = [x["mask"].cpu().numpy().view(np.uint32) for x in parts]
    nb = w.nb
    kept_own = sum(int(np.unpackbits(wp.view(np.uint8)).sum()) for wp in words_parts)  # bits j > i are 0
    own_heads = sum(x["q"].shape[1] for x in parts)
    flops_tile = 4 * 128 * 128 * 128
    est_bytes_own = sum((x["q"].shape[1] + x["k"].shape[1]) * w.seqlen * 128 * 2 for x in parts) + \
        sum(wp.nbytes for wp in words_parts)
    kept, est_bytes = reduce_sum([kept_own, est_bytes_own], dist, dev)
    kept = int(kept)
    causal_tiles = w.batch * w.hq * nb * (nb + 1) // 2
    density = kept / causal_tiles
    # per-GPU roofline of this rank's kernels (rank 0 prints its own)
    attn_tflops = kept_own * flops_tile / (t_attn_own * 1e-3) / 1e12 if kept_own else 0.0
    est_gbs = est_bytes_own / (t_est_own * 1e-3) / 1e9 if parts else 0.0

    peaks, peak_src = load_peaks()
    traffic = profiled_traffic(w.name) if world == 1 else {}
    peak_tensor = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    peak_hbm = peaks["hbm_gbs"]

    # ---------------- end to end: pinned host buffers, copies timed ---------
    # Every step uploads its Q, K, V from pinned host memory, runs the prefill
    # through the public API and downloads its whole output O.  Serial: one
    # step at a time on one stream.  Pipelined (the reported value): two device
    # buffer sets and three streams, so step s+1's upload and step s-1's
    # download run beside step s's kernels; timed from the first upload to the
    # last download, divided by the steps.  Each rank moves its own share.
    e2e = None
    if not args.no_e2e:
        for x in parts:
            x["qp"], x["kp"], x["vp"] = x["qh"].pin_memory(), x["kh"].pin_memory(), x["vh"].pin_memory()
            x["op"] = [torch.empty(x["o"].shape, dtype=x["o"].dtype).pin_memory() for _ in range(2)]
        e2e_serial = []
        for it in range(args.steps + 1):
            ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ea.record(stream)
            for x in parts:
                x["q"].copy_(x["qp"], non_blocking=True)
                x["k"].copy_(x["kp"], non_blocking=True)
                x["v"].copy_(x["vp"], non_blocking=True)
            step()
            for x in parts:
                x["op"][0].copy_(x["o"], non_blocking=True)
            eb.record(stream)
            torch.cuda.synchronize()
            if it > 0:
                e2e_serial.append(ea.elapsed_time(eb))
        e2e_serial_ms = reduce_max([statistics.median(e2e_serial)], dist, dev)[0]
        for x in parts:
            x["sets"] = [(x["q"], x["k"], x["v"], x["o"]), (torch.empty_like(x["q"]), torch.empty_like(x["k"]),
                                                           torch.empty_like(x["v"]), torch.empty_like(x["o"]))]
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def pipelined(n_steps):
            ev = {}
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(up)
            for s_ in range(n_steps):
                if s_ >= 2:
                    up.wait_event(ev[("done", s_ - 2)])  # step s-2 has read this input set
                with torch.cuda.stream(up):
                    for x in parts:
                        qx, kx, vx, _ = x["sets"][s_ % 2]
                        qx.copy_(x["qp"], non_blocking=True)
                        kx.copy_(x["kp"], non_blocking=True)
                        vx.copy_(x["vp"], non_blocking=True)
                ev[("in", s_)] = torch.cuda.Event()
                ev[("in", s_)].record(up)
                stream.wait_event(ev[("in", s_)])
                if s_ >= 2:
                    stream.wait_event(ev[("out", s_ - 2)])  # step s-2's output has been downloaded
                for x in parts:
                    qx, kx, vx, ox = x["sets"][s_ % 2]
                    pb.prism_prefill(x["cfg"], qx, kx, vx, x["mask"], ox, x["ws"], stream=stream)
                ev[("done", s_)] = torch.cuda.Event()
                ev[("done", s_)].record(stream)
                down.wait_event(ev[("done", s_)])
                with torch.cuda.stream(down):
                    for x in parts:
                        x["op"][s_ % 2].copy_(x["sets"][s_ % 2][3], non_blocking=True)
                ev[("out", s_)] = torch.cuda.Event()
                ev[("out", s_)].record(down)
            t1.record(down)
            torch.cuda.synchronize()
            return t0.elapsed_time(t1) / n_steps

        pipelined(2)  # warm-up of the streams and the second buffer set
        e2e_ms = reduce_max([pipelined(args.steps)], dist, dev)[0]
        assert pb.prism_get_last_device_error() == 0
        h2d, d2h = reduce_sum([sum(x["qp"].nbytes + x["kp"].nbytes + x["vp"].nbytes for x in parts),
                               sum(x["op"][0].nbytes for x in parts)], dist, dev)
        e2e = {"value": e2e_ms, "unit": UNIT, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "mode": "pipelined: step s+1 upload and step s-1 download beside step s (2 buffer sets, 3 streams)",
               "serial_value": e2e_serial_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tot, ce, ca, sample = cpu_oracle_sample(q, k, v, words_parts[0], w, n_heads=4, n_blocks=16)
        cpu = {"value": tot, "unit": UNIT, "cores": blas_threads(), "kind": "oracle", "sample": sample,
               "estimator_ms": ce, "attention_ms": ca}

    launches = reduce_sum([KERNELS_PER_STEP * len(parts) * args.steps], dist, dev)[0]
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return
    per_rank = [sum(x.kv1 - x.kv0 for x in shard.shard_runs(w.batch, w.hkv, world, r_)) for r_ in range(world)]
    share = f"{world} rank(s), KV groups per rank {per_rank}"
    line = {
        "metric": METRIC, "value": ms_step, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": False, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "hq": w.hq, "hkv": w.hkv, "seq_len": w.seqlen,
                   "head_dim": w.head_dim, "block": w.block, "p": w.p,
                   "l2": "inputs (Q+K+V 1.6 GB) larger than L2; no flush",
                   "parallelism": f"one layer split by KV group over {world} GPU(s), no data-path collective"},
        "estimator_overhead_pct": 100.0 * t_est / (t_est + t_attn),
        "stages": {"estimate_ms": t_est, "attention_ms": t_attn, "prefill_ms": ms_step,
                   "density": density, "kept_tiles": kept, "causal_tiles": causal_tiles,
                   "effective_tflops_vs_dense": causal_tiles * flops_tile / (ms_step * 1e-3) / 1e12,
                   "dense_attention_ms": t_dense, "speedup_vs_dense": t_dense / ms_step,
                   "shards": share},
        "roofline": {"kernel": "sparse_attn_kernel", "bound": "tensor", "achieved": attn_tflops,
                     "peak": peak_tensor, "unit": "TFLOP/s", "frac": attn_tflops / peak_tensor,
                     "traffic": traffic.get("sparse_attn_kernel"),
                     "algorithmic_flops": kept_own * flops_tile,
                     "peak_source": f"bf16 sustained (of {peak_src})", "scope": "rank 0's kernels"},
        "estimator_roofline": {"kernel": "estimator_kernel", "bound": "hbm", "achieved": est_gbs,
                               "peak": peak_hbm, "unit": "GB/s", "frac": est_gbs / peak_hbm,
                               "algorithmic_bytes": est_bytes_own, "traffic": traffic.get("estimator_kernel"),
                               "peak_source": f"copy bandwidth (of {peak_src})", "scope": "rank 0's kernels"},
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
