"""Benchmark of the Hadamard-domain quantized linear layer on B200.

One step = the layer's runtime hot path over one batch: hq_quantize_act
(bf16 load, sigma^-1, block FWHT, centring, per-token int4 quantization)
followed by hq_linear (tcgen05 int8 GEMM + fused epilogue) -- every step of
the layer except the offline weight preparation, which is timed once and
reported separately.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl hq|reference]

Prints one JSON line (rank 0).  `value` is device-timed throughput of the
whole job in TOPS (2*T*K*N integer ops of the layer per step, summed over
ranks, divided by the max over ranks of the time of K steps).  The K steps
run back to back from one CUDA graph between two CUDA events.  Every step
reads a different copy of the token batch (copies totalling more than twice
the L2 size), so activations come from HBM on every step without a flush
inside the timed region.  Ranks are independent data-parallel shards: each
rank owns its own batch of tokens and a replica of the prepared weights; there
is no collective on the data path (weak scaling).
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "HadaNorm W4A4 linear TOPS & quantizer HBM GB/s (fraction of roofline), 1×B200"
DEFAULT_CONFIG = 5          # the large DiT linear: the largest single-GPU W4A4 workload
# the other workloads, measured in the same run (configuration, centering override)
PER_CONFIG = ((1, None), (2, None), (3, None), (3, 0), (4, None), (5, None))
CEILING_K_BLOCKS = 4096     # MMA-only loop: k blocks (4 MMAs each) per CTA
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_OVER_BF16 = 2.0        # nominal dense int8 : bf16 tensor ratio (4.5 : 2.25 PFLOP/s)


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=DEFAULT_CONFIG, choices=sorted(synth.CONFIGS))
    ap.add_argument("--centering", type=int, default=None, choices=[0, 1, 2],
                    help="override the configuration's centering mode (2: the mean removed "
                         "before the rotation)")
    ap.add_argument("--out-order", type=int, default=0, choices=[0, 16, 32, 64],
                    help="run the configuration's shape in the weight-only Hadamard form "
                         "(W rotated along N in blocks of this order; no rotation along K)")
    ap.add_argument("--packed", action="store_true",
                    help="store the activation codes two per byte (3- and 4-bit codes)")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the packed-code variant measured beside the headline")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the records of the other workloads (configs 1-5)")
    ap.add_argument("--impl", default="hq", choices=["hq", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the bounded oracle sample")
    return ap.parse_args(argv)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# algorithmic work per step
# ---------------------------------------------------------------------------

def layer_ops(cfg) -> float:
    return 2.0 * cfg.T * cfg.K * cfg.N


def quantizer_bytes(cfg) -> float:
    """Algorithmic bytes of hq_quantize_act: read X (2 B/elt), write the codes
    (1 B/elt in the int8 container, 1/2 B packed), write scale + mean
    (8 B/token); the per-tensor dynamic mode reads X twice."""
    passes = 2 if cfg.act_gran == 1 else 1
    return cfg.T * cfg.K * (2.0 * passes + cfg.code_bytes()) + 8.0 * cfg.T


def gemm_bytes(cfg) -> float:
    """Algorithmic HBM bytes of hq_linear: A codes + B codes + bf16 Y + per-row
    and per-column fp32 vectors."""
    return (cfg.T * cfg.K * cfg.code_bytes() + cfg.N * cfg.K + 2.0 * cfg.T * cfg.N +
            8.0 * cfg.T + 12.0 * cfg.N)


# ---------------------------------------------------------------------------
# DRAM traffic per launch from a committed ncu summary
# ---------------------------------------------------------------------------

E2E_CHUNKS = 8  # row chunks of the end-to-end pipeline (hq_forward_host)
PROFILES = {("gemm", 2): "gemm_i8_cfg2_pixart_qkv.md", ("quant", 2): "quant_seg_cfg2_pixart_qkv.md",
            ("gemm", 5): "gemm_i8_pair_cfg5_large_dit.md",
            ("quant", 5): "quant_wrow_cfg5_large_dit.md",
            ("gw_gemm", 5): "gw_gemm_cfg5_large_dit.md", ("gw_act", 5): "gw_act_cfg5_large_dit.md"}
KERNEL_SOURCES = {"gemm": ("hq_gemm.cu", "hq_device.cuh", "hq_kernels.h"),
                  "quant": ("hq_quant_act.cu", "hq_quant_common.cuh", "hq_device.cuh",
                            "hq_kernels.h"),
                  "gw_gemm": ("hq_gw.cu", "hq_quant_common.cuh", "hq_device.cuh", "hq_kernels.h"),
                  "gw_act": ("hq_gw.cu", "hq_quant_common.cuh", "hq_device.cuh", "hq_kernels.h")}


def kernel_source_hash(kind, root=ROOT):
    import hashlib
    m = hashlib.sha256()
    for f in KERNEL_SOURCES[kind]:
        with open(os.path.join(root, "hadamard_rotated_bit_token_b200", "csrc", f), "rb") as fh:
            m.update(fh.read())
    return m.hexdigest()[:16]


def profiled_traffic(kind, cfg_index, root=ROOT):
    """dram__bytes_read + dram__bytes_write of one launch of the kernel, as
    recorded in profiles/ for this workload, or None if there is no summary
    or the kernel's sources changed since it was captured."""
    name = PROFILES.get((kind, cfg_index))
    if name is None:
        return None
    try:
        with open(os.path.join(root, "profiles", name)) as fh:
            text = fh.read()
    except OSError:
        return None
    fields = {}
    for line in text.splitlines():
        key, sep, val = line.strip().partition(":")
        if sep and key in ("traffic_bytes_per_launch", "kernel_source_sha256"):
            fields[key] = val.strip()
    if fields.get("kernel_source_sha256") != kernel_source_hash(kind, root):
        return None
    try:
        return int(fields["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------------------
# multi-rank aggregation (one process per GPU, independent token shards)
# ---------------------------------------------------------------------------

def rank_env():
    """(world, rank, local_rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(values, world, dist=None, device=None):
    """Element-wise max over ranks of a list of floats (identity for one rank).
    Every rank must call it with the same number of values."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def shard_seed(cfg, rank):
    """Seed of rank `rank`'s token batch: every rank quantizes and multiplies
    its own tokens (data-parallel shards); the weights are the same on all."""
    return cfg.index + 1000 * rank


def job_throughput(ops_per_step, steps, world, total_ms):
    """Whole-job throughput in units of 1e12 per second: every rank runs
    `steps` steps of `ops_per_step` on its own shard (weak scaling); the
    job's time is the slowest rank's `total_ms`."""
    return world * ops_per_step * steps / (total_ms * 1e-3) / 1e12


# ---------------------------------------------------------------------------
# clocks sampled while the timed region runs
# ---------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle legs
# ---------------------------------------------------------------------------

def oracle_prepare(cfg, Xb, Wb, bb):
    import oracle
    sig = None
    if cfg.use_sigma:
        sig = oracle.sigma(oracle.col_absmax(Xb), oracle.col_absmax(Wb), cfg.alpha)
    if cfg.out_order > 1:
        w = oracle.prepare_weights_wh(Wb, cfg.out_order, cfg.w_bits, bias_bits=bb, sigma=sig,
                                      want_tie=False)
    else:
        w = oracle.prepare_weights(Wb, cfg.had_order, cfg.w_bits, bias_bits=bb, sigma=sig,
                                   want_tie=False)
    return sig, w


def oracle_step(cfg, Xb, sig, w, rows, nthreads):
    """The oracle's runtime path for the listed rows: transform / centre /
    quantize, integer GEMM, epilogue (weight side prepared beforehand)."""
    import oracle
    a = oracle.quantize_act(Xb, cfg.had_order, cfg.a_bits, gran=cfg.act_gran,
                            centering=cfg.centering, sigma=sig, rows=rows, want_tie=False,
                            nthreads=nthreads)
    acc = oracle.gemm_acc(a["codes"], w["codes"], nthreads=nthreads)
    if cfg.out_order > 1:
        oracle.epilogue_wh(acc, cfg.out_order, a["scale"], w["scale"], b_bar=w["b_bar"])
        return
    oracle.epilogue(acc, a["scale"], w["scale"], colsum=oracle.correction(w, cfg.centering),
                    bias=w["bias"],
                    mean=a["mean"] if cfg.centering else None)


def size_oracle_sample(cfg, Xb, sig, w, nthreads, target_s):
    """Number of rows whose oracle step takes about target_s seconds."""
    probe = min(cfg.T, 16)
    rows = synth.sample_rows(cfg.T, probe, tile=max(1, cfg.T // probe), seed=1)
    t0 = time.perf_counter()
    oracle_step(cfg, Xb, sig, w, rows, nthreads)
    dt = max(time.perf_counter() - t0, 1e-4)
    per_row = dt / len(rows)
    n = int(max(8, min(cfg.T, target_s / per_row)))
    return n


def cpu_baseline(cfg, Xb, Wb, bb, target_s):
    nthreads = os.cpu_count() or 1
    sig, w = oracle_prepare(cfg, Xb, Wb, bb)
    n = size_oracle_sample(cfg, Xb, sig, w, nthreads, target_s)
    rows = synth.sample_rows(cfg.T, n, tile=max(1, cfg.T // n), seed=2)
    t0 = time.perf_counter()
    oracle_step(cfg, Xb, sig, w, rows, nthreads)
    dt = time.perf_counter() - t0
    ops = 2.0 * len(rows) * cfg.K * cfg.N
    return {"value": ops / dt / 1e12, "unit": "TOPS", "cores": nthreads, "kind": "oracle",
            "sample": f"{len(rows)} of {cfg.T} tokens (seeded, every tile), full K and N; "
                      f"runtime path only (weights prepared beforehand); {dt:.1f} s"}


# ---------------------------------------------------------------------------
# reference arm: the oracle as it stands, on the host cores
# ---------------------------------------------------------------------------

def run_reference(args):
    _, rank, _ = rank_env()
    if rank != 0:
        return 0
    cfg = workload_config(args)
    Xb, Wb, bb = synth.make_layer(cfg)
    nthreads = os.cpu_count() or 1
    sig, w = oracle_prepare(cfg, Xb, Wb, bb)
    # size each step so that warmup + steps finish within about two minutes
    budget = 120.0 / max(1, args.steps + args.warmup)
    n = size_oracle_sample(cfg, Xb, sig, w, nthreads, budget)
    rows = synth.sample_rows(cfg.T, n, tile=max(1, cfg.T // n), seed=3)
    for _ in range(args.warmup):
        oracle_step(cfg, Xb, sig, w, rows, nthreads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(cfg, Xb, sig, w, rows, nthreads)
    dt = (time.perf_counter() - t0) / args.steps
    ops = 2.0 * len(rows) * cfg.K * cfg.N
    value = ops / dt / 1e12
    sample = f"{len(rows)} of {cfg.T} tokens per step (seeded, every tile), full K and N"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64+int64", "data": "synthetic",
        "config": config_block(cfg, args.gpus),
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": nthreads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(args):
    import dataclasses
    cfg = synth.CONFIGS[args.config]
    if args.centering is not None:
        cfg = dataclasses.replace(cfg, centering=args.centering)
    if args.out_order:
        cfg = cfg.weight_only(args.out_order)
    if getattr(args, "packed", False):
        cfg = cfg.packed()
    return cfg


def config_block(cfg, n_gpus):
    gran = {0: "per_token", 1: "per_tensor_dynamic", 2: "per_tensor_static"}[cfg.act_gran]
    workload = cfg.workload()
    if cfg.centering != synth.CONFIGS[cfg.index].centering and cfg.out_order <= 1:
        workload += f":centering{cfg.centering}"
    return {"workload": workload, "tokens_per_gpu": cfg.T, "K": cfg.K, "N": cfg.N,
            "had_order": cfg.had_order, "bits": f"A{cfg.a_bits}W{cfg.w_bits}",
            "form": (f"weight-only Hadamard (W rotated along N, blocks of {cfg.out_order})"
                     if cfg.out_order > 1 else "double Hadamard (X and W rotated along K)"),
            "act_granularity": gran,
            "activation_codes": "two per byte" if cfg.code_format else "one per byte",
            "centering": {0: "none", 1: "token mean after H", 2: "token mean before H"}[cfg.centering],
            "sigma": cfg.use_sigma,
            "l2": "inputs larger than L2: step i reads copy i % M of the token batch, "
                  "M copies > 2x L2 (weights and intermediate codes stay L2-resident)",
            "timing": "one CUDA graph of K back-to-back steps between two CUDA events; "
                      "per-kernel times from graphs of K launches of that kernel",
            "parallelism": f"dp{n_gpus} (token shards, replicated weights, no collective)"}


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------

def setup_layer(hq, torch, cfg, dev, rank, l2):
    """One workload on the device: replicated weights (same seed on every
    rank), the rank's own token batch, the prepared layer and its buffers,
    and M copies of the token batch (M * |X| > 2 x L2) so that step i can
    read copy i % M from HBM."""
    Wb, bb = synth.make_w(cfg)
    Xb = synth.make_x(cfg, seed=shard_seed(cfg, rank))
    to_dev = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
    X, W, b = to_dev(Xb), to_dev(Wb), to_dev(bb)
    T, K, N = cfg.T, cfg.K, cfg.N
    desc = hq.LayerDesc(K, N, cfg.had_order, a_bits=cfg.a_bits, w_bits=cfg.w_bits,
                        act_gran=cfg.act_gran, centering=cfg.centering,
                        code_format=cfg.code_format, out_order=cfg.out_order)
    stream = torch.cuda.current_stream()
    # offline: calibration + weight preparation (timed once, not part of the step)
    absmax = torch.zeros(K, dtype=torch.float32, device=dev) if cfg.use_sigma else None
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    if absmax is not None:
        hq.hq_calib_act_absmax(desc, X, absmax)
    layer = hq.HadamardQuantLinear(desc, W, b, absmax, cfg.alpha)
    p1.record(stream)
    torch.cuda.synchronize()
    x_bytes = X.numel() * X.element_size()
    n_copies = int(min(512, max(2, -(-2 * l2 // x_bytes) + 1)))
    return {"cfg": cfg, "desc": desc, "layer": layer, "bufs": layer.buffers(T),
            "Y": torch.empty((T, N), dtype=torch.bfloat16, device=dev),
            "Xs": [X] + [X.clone() for _ in range(n_copies - 1)], "W": W, "b": b,
            "absmax": absmax, "Xb": Xb, "Wb": Wb, "bb": bb,
            "sig_inv": layer.sigma_inv if layer.use_sigma else None,
            "prep_ms": p0.elapsed_time(p1),
            "launches_per_step": (2 if cfg.act_gran == 1 else 1) + 1}


def capture_layer_graphs(torch, ctx, steps, warmup):
    """Warm-up, then three CUDA graphs of `steps` launches each: whole steps
    (quantize + GEMM), the quantizer alone, the GEMM alone.  Step i reads
    copy i % M of the token batch, so the activations come from HBM."""
    import hadamard_rotated_bit_token_b200 as hq
    desc, layer, bufs, Xs, Y = (ctx[k] for k in ("desc", "layer", "bufs", "Xs", "Y"))
    mean_in = bufs["a_mean"] if desc.centering else None
    n = len(Xs)

    def quantize_i(i):
        hq.hq_quantize_act(desc, Xs[i % n], ctx["sig_inv"], bufs["a_codes"], bufs["a_scale"],
                           bufs["a_mean"], layer.workspace)

    def linear():
        hq.hq_linear(desc, bufs["a_codes"], bufs["a_scale"], mean_in, layer.w_codes,
                     layer.w_scale, layer.colsum, layer.bias_f32, Y)

    for i in range(warmup):
        quantize_i(i)
        linear()
    torch.cuda.synchronize()
    graphs = []
    for do_q, do_l in ((True, True), (True, False), (False, True)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(steps):
                if do_q:
                    quantize_i(i)
                if do_l:
                    linear()
        g.replay()
        graphs.append(g)
    torch.cuda.synchronize()
    return graphs


def host_call_cost(hq, torch, ctx, calls=200):
    """Host microseconds per eager call of hq_quantize_act and hq_linear
    (launch included, the device not waited for): the per-call host cost a
    caller pays outside a CUDA graph."""
    desc, layer, bufs, Xs, Y = (ctx[k] for k in ("desc", "layer", "bufs", "Xs", "Y"))
    mean_in = bufs["a_mean"] if desc.centering else None
    q = lambda: hq.hq_quantize_act(desc, Xs[0], ctx["sig_inv"], bufs["a_codes"],
                                   bufs["a_scale"], bufs["a_mean"], layer.workspace)
    g = lambda: hq.hq_linear(desc, bufs["a_codes"], bufs["a_scale"], mean_in, layer.w_codes,
                             layer.w_scale, layer.colsum, layer.bias_f32, Y)
    out = {}
    for name, fn in (("hq_quantize_act", q), ("hq_linear", g)):
        fn()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for _ in range(calls):
            fn()
        dt = time.perf_counter() - t0
        torch.cuda.synchronize()
        out[name] = dt / calls * 1e6
    out["what"] = ("host time per eager call through the Python binding, device not waited "
                   "for; tensor maps come from the library's cache after the first call")
    out["tmap_cache"] = hq.hq_debug_tmap_cache()
    return out


def measure_mma_ceiling(hq, torch):
    """The measured int8 tensor-core ceiling: the GEMMs' main loops with
    nothing but the MMAs (hq_debug_mma_ceiling), one CTA per SM, timed with
    CUDA events around each launch (about a millisecond each); best of three
    launches after one warm-up launch."""
    out = {"k_blocks_per_cta": CEILING_K_BLOCKS,
           "what": "MMA-only loop (tcgen05.mma kind::i8 128x256x32 per CTA; pair: cta_group::2 "
                   "256x256x32 per cluster), no loads, no epilogue; operands in shared memory"}
    for name, pair in (("single_cta_TOPS", False), ("cta_pair_TOPS", True)):
        try:
            best = 0.0
            stream = torch.cuda.current_stream()
            for rep in range(4):
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                ctas = hq.hq_debug_mma_ceiling(pair, CEILING_K_BLOCKS)
                e1.record(stream)
                torch.cuda.synchronize()
                ops = ctas * CEILING_K_BLOCKS * 4 * 2.0 * 128 * 256 * 32
                if rep > 0:  # the first launch configures the kernel
                    best = max(best, ops / (e0.elapsed_time(e1) * 1e-3) / 1e12)
            out[name] = best
        except Exception as e:  # pair clusters unavailable on this device
            out[name] = None
            out[name + "_error"] = str(e)
    return out


def kernel_record(hq, cfg, q_ms, g_ms, step_ms, peaks, ceiling):
    """Per-kernel figures of one workload: achieved bytes/s (quantizer) and
    int ops/s (GEMM) against the measured peaks."""
    ops = layer_ops(cfg)
    int8_peak = peaks["bf16_tflops"] * INT8_OVER_BF16
    q_gbs = quantizer_bytes(cfg) / (q_ms * 1e-3) / 1e9
    g_tops = ops / (g_ms * 1e-3) / 1e12
    desc = hq.LayerDesc(cfg.K, cfg.N, cfg.had_order, a_bits=cfg.a_bits, w_bits=cfg.w_bits,
                        act_gran=cfg.act_gran, centering=cfg.centering,
                        code_format=cfg.code_format, out_order=cfg.out_order)
    import torch
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    pair_ok = ceiling.get("cta_pair_TOPS") is not None
    plan = hq.hq_debug_plan(desc, cfg.T, props.multi_processor_count,
                            props.multi_processor_count // 2 if pair_ok else 0)
    ceil = ceiling.get("cta_pair_TOPS" if plan["gemm_pair"] else "single_cta_TOPS")
    return {
        "step_ms": step_ms, "step_TOPS": ops / (step_ms * 1e-3) / 1e12,
        "quantizer": {"ms_per_launch": q_ms, "GB/s": q_gbs, "frac_hbm": q_gbs / peaks["hbm_gbs"],
                      "bytes": quantizer_bytes(cfg), "tile_rows": plan["quant_rows"],
                      "threads": plan["quant_threads"]},
        "gemm": {"ms_per_launch": g_ms, "TOPS": g_tops, "frac_int8": g_tops / int8_peak,
                 "mma_ceiling_TOPS": ceil,
                 "frac_mma_ceiling": (g_tops / ceil) if ceil else None,
                 "kernel": "CTA pair 256x256" if plan["gemm_pair"] else
                           f"single CTA 128x{plan['gemm_bn']}",
                 "hbm_bytes": gemm_bytes(cfg)},
    }


def per_config_records(hq, torch, args, head_cfg, dev, l2, peaks, ceiling, timed, check):
    """The other workloads measured in the same run, the same way as the
    headline (graphs of K launches, rotating inputs), one at a time."""
    import dataclasses
    out = {}
    for index, centering in PER_CONFIG:
        cfg = synth.CONFIGS[index]
        if centering is not None:
            cfg = dataclasses.replace(cfg, centering=centering)
        if cfg == head_cfg:
            continue
        name = cfg.workload() + (f":centering{cfg.centering}" if centering is not None else "")
        ctx = setup_layer(hq, torch, cfg, dev, 0, l2)
        graphs = capture_layer_graphs(torch, ctx, args.steps, args.warmup)
        step_ms, q_ms, g_ms = (timed(g) / args.steps for g in graphs)
        check(f"in {name}")
        out[name] = kernel_record(hq, cfg, q_ms, g_ms, step_ms, peaks, ceiling)
        del graphs, ctx
        torch.cuda.empty_cache()
    return out


GW_GROUP, GW_RANK = 64, 32
FP32_LANES_PER_SM = 128  # fp32 FMA lanes per SM (4 sub-partitions x 32)


def group_wise_record(hq, torch, args, cfg, dev, l2, ceiling, clock_info, timed, check):
    """The group-wise 4-bit form with its rank-32 16-bit branch (include/hq_gw.h)
    on the same layer shape and inputs as the headline: graphs of K steps
    (quantize + GEMM) over rotating inputs, and the two kernels alone.  The
    GEMM's bound is the per-group rescale in its epilogue (two fp32 lane
    operations per output element and group: the product of the two scales
    and the fused multiply-add), so it reports against the fp32 lane rate
    at the sampled SM clock as well as the tensor-core ceiling."""
    Wb, bb = synth.make_w(cfg)
    Xb = synth.make_x(cfg)
    to_dev = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
    X, W, b = to_dev(Xb), to_dev(Wb), to_dev(bb)
    T, K, N = cfg.T, cfg.K, cfg.N
    G = K // GW_GROUP
    desc = hq.GwDesc(K, N, GW_GROUP, GW_RANK, 4, 4)
    absmax = torch.zeros(K, dtype=torch.float32, device=dev)
    hq.hq_calib_act_absmax(hq.LayerDesc(K, N, 1), X, absmax)
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record()
    layer = hq.GroupWiseQuantLinear(desc, W, b, absmax, cfg.alpha)
    p1.record()
    torch.cuda.synchronize()
    bufs = layer.buffers(T)
    Y = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
    n = int(min(512, max(2, -(-2 * l2 // (X.numel() * 2)) + 1)))
    Xs = [X] + [X.clone() for _ in range(n - 1)]
    si = layer.sigma_inv

    def quantize_i(i):
        hq.hq_gw_quantize_act(desc, Xs[i % n], si, layer.l1s, bufs["a_codes"], bufs["a_scale"],
                              bufs["u"], bufs["workspace"])

    def linear():
        hq.hq_gw_linear(desc, bufs["a_codes"], bufs["a_scale"], bufs["u"], layer.w_codes,
                        layer.w_scale, layer.l2b, layer.bias_f32, Y, T=T)

    for i in range(args.warmup):
        quantize_i(i)
        linear()
    torch.cuda.synchronize()
    graphs = []
    for do_q, do_l in ((True, True), (True, False), (False, True)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(args.steps):
                if do_q:
                    quantize_i(i)
                if do_l:
                    linear()
        g.replay()
        graphs.append(g)
    torch.cuda.synchronize()
    step_ms, q_ms, g_ms = (timed(g) / args.steps for g in graphs)
    check("in the group-wise form")
    # the output against the unquantized layer (context: the error of the form)
    ref = torch.matmul(X.float(), W.float().t()) + b.float()
    quantize_i(0)
    linear()
    rel = float(((Y.float() - ref).norm() / ref.norm()).item())
    ops = 2.0 * T * K * N + 2.0 * T * GW_RANK * (K + N)
    q_bytes = T * K * 2 + T * K + T * G * 4 + T * GW_RANK * 2 + GW_RANK * K * 2
    sm_mhz = (clock_info or {}).get("sm_mhz") or 1965.0
    props = torch.cuda.get_device_properties(dev)
    lane_ops = 2.0 * T * N * G + T * N  # scale product + multiply-add per group; branch add
    lane_rate = props.multi_processor_count * FP32_LANES_PER_SM * sm_mhz * 1e6
    g_tops = 2.0 * T * K * N / (g_ms * 1e-3) / 1e12
    del graphs, Xs, layer, bufs
    torch.cuda.empty_cache()
    profiled = cfg == synth.CONFIGS[cfg.index]
    return {
        "workload": f"{cfg.workload()} in the group-wise form: groups of {GW_GROUP} channels "
                    f"(H_{GW_GROUP} and one scale per group), W4A4, rank-{GW_RANK} bf16 branch",
        "step_ms": step_ms, "step_TOPS": ops / (step_ms * 1e-3) / 1e12,
        "weight_prep_ms": p0.elapsed_time(p1),
        "rel_err_vs_unquantized": rel,
        "quantizer": {"ms_per_launch": q_ms, "bytes": q_bytes,
                      "GB/s": q_bytes / (q_ms * 1e-3) / 1e9,
                      "traffic": profiled_traffic("gw_act", cfg.index) if profiled else None,
                      "what": "X read once: the group transform and codes on CUDA cores, "
                              "u = X l1^T on the tensor cores from the same tiles"},
        "gemm": {"ms_per_launch": g_ms, "TOPS": g_tops,
                 "traffic": profiled_traffic("gw_gemm", cfg.index) if profiled else None,
                 "frac_mma_ceiling": g_tops / ceiling["single_cta_TOPS"]
                 if ceiling.get("single_cta_TOPS") else None,
                 "bound": "alu", "alu_lane_ops": lane_ops,
                 "alu_floor_ms": lane_ops / lane_rate * 1e3,
                 "frac_alu": lane_ops / lane_rate / (g_ms * 1e-3),
                 "alu_peak": f"{props.multi_processor_count} SMs x {FP32_LANES_PER_SM} fp32 "
                             f"lanes x {sm_mhz:.0f} MHz (sampled SM clock)",
                 "what": "kind::f8f6f4 MMAs (e4m3 bytes holding the integer codes) into one "
                         "fp32 accumulator per group, rescaled by s_x s_w in registers"},
    }


def run_hq(args):
    import torch
    import torch.distributed as dist

    import hadamard_rotated_bit_token_b200 as hq

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    hq.load_library()
    cfg = workload_config(args)
    stream = torch.cuda.current_stream()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size

    def timed(g):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    def check(where):
        status = hq.hq_check_device_error()
        if status != 0:
            raise RuntimeError(f"device error {where}: {hq.STATUS_NAMES.get(status)}")

    ctx = setup_layer(hq, torch, cfg, dev, rank, l2)
    graphs = capture_layer_graphs(torch, ctx, args.steps, args.warmup)
    check("during warm-up")
    g_step, g_quant, g_linear = graphs

    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.25)
    total_ms = timed(g_step)
    if world > 1:
        dist.barrier()
    clock_info = clocks.stop()
    q_total = timed(g_quant)
    g_total = timed(g_linear)
    check("in the timed region")
    del graphs, g_step, g_quant, g_linear
    T, K, N = cfg.T, cfg.K, cfg.N
    desc, layer, bufs, Xs, Y, W = (ctx[k] for k in ("desc", "layer", "bufs", "Xs", "Y", "W"))
    n_copies = len(Xs)

    # context only, outside the timed step: the same layer unquantized, as one
    # cuBLAS bf16 GEMM (torch.matmul) over the same rotating inputs
    Yc = torch.empty((T, N), dtype=torch.bfloat16, device=dev)

    def cublas_i(i):
        torch.matmul(Xs[i % n_copies], W.t(), out=Yc)

    cublas_i(0)
    torch.cuda.synchronize()
    g_cublas = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_cublas):
        for i in range(args.steps):
            cublas_i(i)
    g_cublas.replay()
    torch.cuda.synchronize()
    c_total = timed(g_cublas)
    del g_cublas, Yc

    # variant beside the headline (same inputs and weights, timed the same
    # way): 3- and 4-bit activation codes stored two per byte, widened to
    # int8 inside the GEMM
    pk_times = [0.0, 0.0, 0.0]
    with_packed = cfg.code_format == 0 and cfg.a_bits <= 4 and not args.no_variants
    if with_packed:
        pctx = dict(ctx)
        pdesc = hq.LayerDesc(K, N, cfg.had_order, a_bits=cfg.a_bits, w_bits=cfg.w_bits,
                             act_gran=cfg.act_gran, centering=cfg.centering,
                             code_format=hq.HQ_CODES_I4_PACKED, out_order=cfg.out_order)
        player = hq.HadamardQuantLinear(pdesc, W, ctx["b"], ctx["absmax"], cfg.alpha)
        pctx.update(desc=pdesc, layer=player, bufs=player.buffers(T))
        pgs = capture_layer_graphs(torch, pctx, args.steps, args.warmup)
        if world > 1:
            dist.barrier()
        pk_times = [timed(g) for g in pgs]
        check("in the packed variant")
        del pgs, player, pctx
    (total_ms, q_total, g_total, c_total, pk_step, pk_q, pk_g) = max_over_ranks(
        [total_ms, q_total, g_total, c_total] + pk_times, world, dist, dev)
    ms_per_step = total_ms / args.steps
    ops = layer_ops(cfg)
    value = job_throughput(ops, args.steps, world, total_ms)

    # end to end through the public API with host buffers (pinned), per step:
    # H2D of X, quantize, GEMM, D2H of Y
    e2e = None
    if not args.no_e2e:
        Xh = torch.from_numpy(ctx["Xb"].view(np.int16)).view(torch.bfloat16).pin_memory()
        Yh = torch.empty((T, N), dtype=torch.bfloat16).pin_memory()
        Xd = torch.empty_like(Xs[0])

        def e2e_body():
            # one public call: uploads, the layer's kernels and downloads of
            # row chunks overlapped on the library's copy streams
            hq.hq_forward_host(desc, Xh, Xd, ctx["sig_inv"], bufs["a_codes"], bufs["a_scale"],
                               bufs["a_mean"], layer.workspace, layer.w_codes, layer.w_scale,
                               layer.colsum, layer.bias_f32, Y, Yh, chunks=E2E_CHUNKS)

        for _ in range(max(1, args.warmup)):
            e2e_body()
        torch.cuda.synchronize()
        g_e2e = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_e2e):
            for _ in range(args.steps):
                e2e_body()
        g_e2e.replay()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e2e_ms = max_over_ranks([timed(g_e2e)], world, dist, dev)[0]
        e2e = {"value": job_throughput(ops, args.steps, world, e2e_ms), "unit": "TOPS",
               "h2d_bytes_per_step": int(Xh.numel() * Xh.element_size()),
               "d2h_bytes_per_step": int(Yh.numel() * Yh.element_size()),
               "ms_per_step": e2e_ms / args.steps}
        check("in the e2e region")
        del g_e2e, Xh, Yh, Xd

    ctx_host = host_call_cost(hq, torch, ctx) if rank == 0 else None

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, peak_src = load_peaks()
    int8_peak = peaks["bf16_tflops"] * INT8_OVER_BF16
    ceiling = measure_mma_ceiling(hq, torch)
    check("in the MMA-only loop")
    headline = kernel_record(hq, cfg, q_total / args.steps, g_total / args.steps,
                             ms_per_step, peaks, ceiling)
    q_med = q_total / args.steps
    g_med = g_total / args.steps
    q_gbs = headline["quantizer"]["GB/s"]
    g_tops = headline["gemm"]["TOPS"]
    # the committed ncu summaries cover the configurations as defined, not overrides
    profiled = cfg == synth.CONFIGS[cfg.index]
    if g_med >= q_med:
        roof = {"kernel": "hq_gemm_i8 (tcgen05 kind::i8 + epilogue, "
                          f"{headline['gemm']['kernel']})", "bound": "tensor",
                "achieved": g_tops, "peak": int8_peak, "unit": "TFLOP/s",
                "frac": g_tops / int8_peak,
                "traffic": profiled_traffic("gemm", cfg.index) if profiled else None,
                "peak_source": f"{peak_src}: 2 x bf16_tflops (burst), dense int8:bf16 = 4.5:2.25",
                "frac_of_mma_ceiling": headline["gemm"]["frac_mma_ceiling"],
                "mma_ceiling_TOPS": headline["gemm"]["mma_ceiling_TOPS"],
                "algorithmic": f"2*T*K*N = {ops:.4g} int ops per launch"}
    else:
        roof = {"kernel": "hq_quantize_act (fused FWHT quantizer)", "bound": "hbm",
                "achieved": q_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": q_gbs / peaks["hbm_gbs"],
                "traffic": profiled_traffic("quant", cfg.index) if profiled else None,
                "peak_source": f"{peak_src} hbm_gbs",
                "algorithmic": f"{quantizer_bytes(cfg):.4g} bytes per launch"}
    kernels = {"quantizer": headline["quantizer"], "gemm": headline["gemm"],
               "weight_prep_ms": ctx["prep_ms"]}
    kernels["quantizer"]["traffic"] = profiled_traffic("quant", cfg.index) if profiled else None
    kernels["gemm"]["traffic"] = profiled_traffic("gemm", cfg.index) if profiled else None
    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8 (s8 x s8 -> s32; fp32 transform)", "data": "synthetic",
        "config": config_block(cfg, world),
        "roofline": roof,
        "kernels": kernels,
        "int8_ceiling": ceiling,
        "context": {"cublas_bf16_gemm": {
            "ms_per_launch": c_total / args.steps,
            "TFLOP/s": ops / (c_total / args.steps * 1e-3) / 1e12,
            "what": "torch.matmul(X, W^T) in bf16 (cuBLAS) on the same shape and inputs, "
                    "unquantized; context only, not on the path"}},
        "gpu_launches": ctx["launches_per_step"] * args.steps,
        "clocks": clock_info,
        "e2e": e2e,
    }
    # host time of one eager call of each entry point (tensor maps from the
    # library's cache after the first call); outside any timed region
    line["host_us_per_call"] = ctx_host
    if with_packed:
        pcfg = cfg.packed()
        line["variants"] = {"packed_codes": {
            "what": "the same layer, inputs and weights with the activation codes stored two "
                    "per byte (HQ_CODES_I4_PACKED) and widened to int8 inside the GEMM; "
                    "outputs bit-identical to the headline's",
            "value": job_throughput(ops, args.steps, world, pk_step), "unit": "TOPS",
            "ms_per_step": pk_step / args.steps,
            **kernel_record(hq, pcfg, pk_q / args.steps, pk_g / args.steps,
                            pk_step / args.steps, peaks, ceiling)}}
    host = (ctx["Xb"], ctx["Wb"], ctx["bb"])
    del ctx, layer, bufs, Xs, Y, W
    torch.cuda.empty_cache()
    if not args.no_per_config and world == 1:
        line["per_config"] = per_config_records(hq, torch, args, cfg, dev, l2, peaks, ceiling,
                                                timed, check)
    if not args.no_variants and world == 1 and cfg.K % GW_GROUP == 0 and cfg.N % 16 == 0:
        line["group_wise"] = group_wise_record(hq, torch, args, cfg, dev, l2, ceiling,
                                               clock_info, timed, check)
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(cfg, *host, args.cpu_seconds)
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_hq(args)


if __name__ == "__main__":
    sys.exit(main())
