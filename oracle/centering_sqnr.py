"""Output SQNR of the quantized layer under each centring reading, computed
with the oracle only (test infrastructure; nothing here runs on the GPU).

    python oracle/centering_sqnr.py [--rows 256] [--configs 1 2 3 4 5]

For each synthetic configuration and a seeded sample of its tokens, the
layer's output is computed with the oracle in fp64 (codes, integer GEMM,
epilogue) and compared with the exact X W + b:
  SQNR = 10 log10( sum y^2 / sum (y_q - y)^2 )  (HaTQ Eq. (10) on the output).
Readings of the HadaNorm review's mu:
  none    no centring
  R1      per-token mean of the rotated row, removed after H
  R3      per-token mean of Y = X diag(sigma^-1), removed before H
  R2      per-channel mean over the tokens (the appended token), removed before
          H and carried into the bias; calibrated on the configuration's own
          tokens ("cal = same") or on a second draw of them ("cal = other")
  R2+R1, R2+R3   both
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
    sig = None
    if cfg.use_sigma:
        sig = oracle.sigma(oracle.col_absmax(Xb), oracle.col_absmax(Wb), cfg.alpha)
    s = sig if sig is not None else np.ones(cfg.K)
    mu_same = oracle.channel_mean(Xb) / s
    X_other = synth.make_x(cfg, seed=cfg.index + 100)
    mu_other = oracle.channel_mean(X_other) / s
    exact = oracle.exact_linear(Xb, Wb, bb, rows=rows)
    out = {}
    cases = [("none", 0, None), ("R1", 1, None), ("R3", 2, None),
             ("R2 (cal = same)", 0, mu_same), ("R2 (cal = other)", 0, mu_other),
             ("R2+R1", 1, mu_same), ("R2+R3", 2, mu_same)]
    w_plain = oracle.prepare_weights(Wb, cfg.had_order, cfg.w_bits, bias_bits=bb, sigma=sig,
                                     want_tie=False)
    for name, cen, mu in cases:
        if cfg.act_gran != 0 and cen != 0:
            continue  # the per-tensor configuration has no per-token mean
        w = w_plain if mu is None else oracle.prepare_weights(
            Wb, cfg.had_order, cfg.w_bits, bias_bits=bb, sigma=sig, want_tie=False, shift=mu)
        a = oracle.quantize_act(Xb, cfg.had_order, cfg.a_bits, gran=cfg.act_gran, centering=cen,
                                sigma=sig, shift=mu, rows=rows, want_tie=False)
        acc = oracle.gemm_acc(a["codes"], w["codes"])
        y, _ = oracle.epilogue(acc, a["scale"], w["scale"], colsum=oracle.correction(w, cen),
                               bias=w["bias"], mean=a["mean"] if cen else None)
        out[name] = sqnr_db(y, exact)
    return cfg, out


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--rows", type=int, default=256)
    ap.add_argument("--configs", type=int, nargs="*", default=[1, 2, 3, 4, 5])
    args = ap.parse_args(argv)
    for idx in args.configs:
        cfg, out = run(idx, args.rows)
        print(f"config {idx} ({cfg.workload()}): " +
              ", ".join(f"{k} {v:.2f} dB" for k, v in out.items()), flush=True)


if __name__ == "__main__":
    main()
