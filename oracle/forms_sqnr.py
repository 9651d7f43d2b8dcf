"""Output SQNR of each form of the quantized layer on the synthetic
workloads, computed with the oracle only (test infrastructure; nothing here
runs on the GPU).

    python oracle/forms_sqnr.py [--rows 256] [--configs 1 2 3 5]

For a seeded sample of each configuration's tokens, every form's output is
computed with the oracle in fp64 and compared with the exact X W + b:
  SQNR = 10 log10( sum y^2 / sum (y_q - y)^2 )  (HaTQ Eq. (10) on the output).
Forms, each at the configuration's activation and weight widths:
  HadaNorm R1 / R3   per-channel weights, per-token activations, H of the
                     configuration's order with sigma (HadaNorm review,
                     Eq. (1)-(3)); per-token mean removed after (R1) or
                     before (R3) the rotation
  weight-only H64    HaTQ Eq. (17): X unrotated, W rotated along the outputs
                     in blocks of 64
  group-wise r0/r32  the blog's group-wise form: groups of 64 with an H_64
                     block each, sigma, and no or a rank-32 16-bit branch
                     (factors from the singular value decomposition of
                     W diag(sigma))
The synthetic weights are Gaussian, with none of a trained layer's low-rank
structure, so the rank-32 branch removes only the top 32 singular values of
a flat spectrum here.
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402


def sqnr_db(y, ref):
    return 10.0 * np.log10(np.sum(ref * ref) / max(np.sum((y - ref) ** 2), 1e-300))


def run(idx, nrows):
    cfg = synth.CONFIGS[idx]
    Xb, Wb, bb = synth.make_layer(cfg)
    rows = synth.sample_rows(cfg.T, min(nrows, cfg.T), tile=1, seed=7)
    exact = oracle.exact_linear(Xb, Wb, bb, rows=rows)
    out = {}
    for name, cen in (("HadaNorm R1", 1), ("HadaNorm R3", 2)):
        r = oracle.layer(Xb, Wb, bb, cfg.had_order, cfg.a_bits, cfg.w_bits, gran=0,
                         centering=cen, alpha=cfg.alpha, use_sigma=cfg.use_sigma, rows=rows)
        out[name] = sqnr_db(r["y"], exact)
    r = oracle.layer_wh(Xb, Wb, bb, 64, cfg.a_bits, cfg.w_bits, rows=rows)
    out["weight-only H64"] = sqnr_db(r["y"], exact)
    sig = oracle.sigma(oracle.col_absmax(Xb), oracle.col_absmax(Wb), cfg.alpha)
    for rank in (0, 32):
        L1, L2 = oracle.low_rank_factors(Wb, sig, rank)
        w = oracle.gw_prepare_weights(Wb, 64, cfg.w_bits, rank, L1, L2, bias_bits=bb, sigma=sig,
                                      want_tie=False)
        a = oracle.gw_quantize_act(Xb, 64, cfg.a_bits, rank, w["l1"], sigma=sig, rows=rows,
                                   want_tie=False)
        y, _ = oracle.gw_epilogue(a["codes"], w["codes"], 64, a["gscale"], w["gscale"], a["u"],
                                  w["l2"], bias=w["bias"])
        out[f"group-wise r{rank}"] = sqnr_db(y, exact)
    return cfg, out


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--rows", type=int, default=256)
    ap.add_argument("--configs", type=int, nargs="*", default=[1, 2, 3, 5])
    args = ap.parse_args(argv)
    for idx in args.configs:
        cfg, out = run(idx, args.rows)
        print(f"config {idx} ({cfg.workload()}): " +
              ", ".join(f"{k} {v:.2f} dB" for k, v in out.items()), flush=True)


if __name__ == "__main__":
    main()
