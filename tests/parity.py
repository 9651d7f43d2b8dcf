"""Helpers for the GPU-vs-oracle parity tests (test-side only).

Bars (from the layer's stated tolerances):
  codes     : identical except +-1 flips where the oracle's scaled value lies
              within TIE_TOL code units of a rounding tie; at configuration
              scale at least 99.99 % identical;
  scales    : relative error <= 1e-6;
  means     : |delta| <= 1e-6 * mean |Z_t|;
  colsum    : |delta| <= 1e-6 * sum_k |W~[n,k]|;
  int32 acc : bit-exact when both sides use the same codes;
  output    : relative Frobenius error <= 1e-3 against the oracle's bf16 output.
"""
from __future__ import annotations

import numpy as np

TIE_TOL = 2.0 ** -10
CODE_MATCH_MIN = 0.9999
SCALE_RTOL = 1e-6
Y_REL_FROB = 1e-3


def to_dev_u16(a, torch):
    """numpy uint16 (bf16 bits) -> torch bfloat16 CUDA tensor, bit for bit."""
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def bf16_bits(t) -> np.ndarray:
    return t.detach().contiguous().cpu().view(__import__("torch").int16).numpy().view(np.uint16)


def check_codes(gpu, ref, tie, what="codes", min_match=None):
    gpu = np.asarray(gpu, dtype=np.int16)
    ref = np.asarray(ref, dtype=np.int16)
    diff = gpu - ref
    bad = diff != 0
    nbad = int(bad.sum())
    if nbad:
        far = np.argwhere(np.abs(diff) > 1)
        if far.size:
            show = [(tuple(int(v) for v in ix), int(gpu[tuple(ix)]), int(ref[tuple(ix)]),
                     float(tie[tuple(ix)])) for ix in far[:8]]
            raise AssertionError(f"{what}: {len(far)} codes differ by more than 1 "
                                 f"(index, gpu, oracle, tie): {show}")
        worst = float(np.max(tie[bad]))
        assert worst < TIE_TOL, f"{what}: mismatch {worst:.3g} code units away from a tie"
    match = 1.0 - nbad / max(1, gpu.size)
    if min_match is not None:
        assert match >= min_match, f"{what}: only {match:.6f} identical"
    return match


def check_rel(gpu, ref, rtol, what):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    denom = np.where(ref == 0, 1.0, np.abs(ref))
    err = np.abs(gpu - ref) / denom
    both_zero = (ref == 0) & (gpu == 0)
    err = np.where(both_zero, 0.0, err)
    worst = float(err.max()) if err.size else 0.0
    assert worst <= rtol, f"{what}: relative error {worst:.3g} > {rtol:g}"
    return worst


def rel_frob(gpu_bits, ref_bits):
    import synth
    g = synth.bf16_bits_to_f32(gpu_bits).astype(np.float64)
    r = synth.bf16_bits_to_f32(ref_bits).astype(np.float64)
    return float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-300))


def check_bf16_outputs(gpu_bits, y64, mag, what="Y"):
    """GPU bf16 outputs against the exact fp64 values y64 of the same epilogue
    inputs.  The epilogue forms fma(acc, fl(s_x s_w), fma(m, c, b)) in fp32:
    three roundings of relative size 2^-24 on terms no larger than
    mag = |acc s_x s_w| + |m c| + |b|, so its fp32 value v lies within
    tol = 4 * 2^-24 * mag of y64, and since rounding to bf16 is monotone the
    output bf16_rne(v) lies between bf16_rne(y64 - tol) and bf16_rne(y64 + tol).
    Outside a tol-wide neighbourhood of a bf16 rounding midpoint that interval
    holds one value, bf16_rne(y64), so the check is exact there."""
    import oracle
    import synth
    gpu = synth.bf16_bits_to_f32(np.asarray(gpu_bits, dtype=np.uint16)).astype(np.float64)
    tol = 4.0 * 2.0 ** -24 * np.asarray(mag, dtype=np.float64)
    lo = synth.bf16_bits_to_f32(oracle.f64_to_bf16(y64 - tol)).astype(np.float64)
    hi = synth.bf16_bits_to_f32(oracle.f64_to_bf16(y64 + tol)).astype(np.float64)
    ok = (gpu >= lo) & (gpu <= hi)
    assert np.all(ok), (f"{what}: {int((~ok).sum())} outputs outside the fp32 epilogue's "
                        f"rounding interval")
    return int((gpu != synth.bf16_bits_to_f32(oracle.f64_to_bf16(y64))).sum())
