"""Plain fp64 CPU oracle for the HadaNorm Hadamard-domain quantized linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference legs of ``bench.py`` may import this module.  The
product library (``hadamard_rotated_bit_token_b200``) never imports, links or
runs anything here, and nothing here imports the product library.

The arithmetic lives in ``hq_oracle.cpp`` (plain C++, fp64, dense block
Hadamard products and triple loops); this file only builds that library with
g++ and marshals numpy arrays through ctypes.

Parity pins: see ``tests/test_oracle_pins.py`` (Hadamard orthogonality and the
Sylvester recursion, the Eq. (1) identity with quantization off, hand-worked
quantizer examples, brute force at K = 4 / 8, closed-form invariants, integer
accumulation; for the group-wise int4 form with its low-rank branch a
hand-worked two-group example, the unquantized identity and brute force of the
group quantizer against the per-token one).  Every function here is pinned
there; none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hq_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_i64p = ctypes.POINTER(ctypes.c_int64)
_f64p = ctypes.POINTER(ctypes.c_double)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_i8p = ctypes.POINTER(ctypes.c_int8)
_u8p = ctypes.POINTER(ctypes.c_uint8)


def build(force: bool = False) -> str:
    """Compiles hq_oracle.cpp into liboracle.so next to it (g++, -O2)."""
    stale = (not os.path.exists(_LIB_PATH)) or (
        os.path.getmtime(_LIB_PATH) < max(os.path.getmtime(_SRC),
                                           os.path.getmtime(os.path.join(_HERE, "hq_oracle.h"))))
    if force or stale:
        tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-Wall",
                               "-o", tmp, _SRC, "-lpthread"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            lib.hqo_hadamard_entry.argtypes = [ctypes.c_int64, ctypes.c_int64]
            lib.hqo_hadamard_entry.restype = ctypes.c_int
            lib.hqo_sylvester.argtypes = [ctypes.c_int64, _i8p]
            lib.hqo_bf16_to_f64.argtypes = [ctypes.c_uint16]
            lib.hqo_bf16_to_f64.restype = ctypes.c_double
            lib.hqo_f64_to_bf16.argtypes = [ctypes.c_double]
            lib.hqo_f64_to_bf16.restype = ctypes.c_uint16
            lib.hqo_rne.argtypes = [ctypes.c_double]
            lib.hqo_rne.restype = ctypes.c_double
            lib.hqo_col_absmax.argtypes = [_u16p, ctypes.c_int64, ctypes.c_int64, _f64p]
            lib.hqo_sigma.argtypes = [ctypes.c_int64, _f64p, _f64p, ctypes.c_double, _f64p]
            lib.hqo_quantize_act.argtypes = [
                ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                _u16p, ctypes.c_int64, _f64p, _f64p, ctypes.c_double, _i64p, ctypes.c_int64,
                _i8p, _f64p, _f64p, _f64p, _f64p, ctypes.c_int]
            lib.hqo_prepare_weights.argtypes = [
                ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                _u16p, _u16p, _f64p, _f64p, _i8p, _f64p, _f64p, _f64p, _f64p, _f64p, _f64p,
                ctypes.c_int]
            lib.hqo_channel_mean.argtypes = [_u16p, ctypes.c_int64, ctypes.c_int64, _f64p]
            _i64 = ctypes.c_int64
            lib.hqo_gw_prepare_weights.argtypes = [
                _i64, _i64, _i64, ctypes.c_int, _i64, _u16p, _u16p, _f64p, _f64p, _f64p,
                _u16p, _u16p, _i8p, _f64p, _f64p, _f64p, _f64p, ctypes.c_int]
            lib.hqo_gw_quantize_act.argtypes = [
                _i64, _i64, ctypes.c_int, _i64, _u16p, _i64, _f64p, _u16p, _i64p, _i64,
                _i8p, _f64p, _u16p, _f64p, _f64p, ctypes.c_int]
            lib.hqo_gw_epilogue.argtypes = [
                _i8p, _i8p, _i64, _i64, _i64, _i64, _f64p, _f64p, _u16p, _u16p, _i64, _f64p,
                _f64p, _u16p, ctypes.c_int]
            lib.hqo_gemm_acc.argtypes = [_i8p, _i8p, ctypes.c_int64, ctypes.c_int64,
                                         ctypes.c_int64, _i64p, ctypes.c_int64, _i64p,
                                         ctypes.c_int]
            lib.hqo_epilogue.argtypes = [_i64p, ctypes.c_int64, ctypes.c_int64, _f64p, _f64p,
                                         _f64p, _f64p, _f64p, _f64p, _u16p]
            lib.hqo_exact_linear.argtypes = [_u16p, _u16p, _u16p, ctypes.c_int64,
                                             ctypes.c_int64, ctypes.c_int64, _i64p,
                                             ctypes.c_int64, _f64p, ctypes.c_int]
            lib.hqo_prepare_weights_wh.argtypes = [
                ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                _u16p, _u16p, _f64p, _i8p, _f64p, _f64p, _f64p, _f64p, ctypes.c_int]
            lib.hqo_epilogue_wh.argtypes = [_i64p, ctypes.c_int64, ctypes.c_int64,
                                            ctypes.c_int64, _f64p, _f64p, _f64p, _f64p, _u16p]
            lib.hqo_output_rotation.argtypes = [_f64p, ctypes.c_int64, ctypes.c_int64,
                                                ctypes.c_int64, _f64p]
            lib.hqo_pack_i4.argtypes = [_i8p, ctypes.c_int64, _u8p]
            lib.hqo_unpack_i4.argtypes = [_u8p, ctypes.c_int64, _i8p]
            for name in ("hqo_pack_i4", "hqo_unpack_i4", "hqo_sylvester", "hqo_col_absmax",
                         "hqo_channel_mean", "hqo_sigma", "hqo_quantize_act",
                         "hqo_gw_prepare_weights", "hqo_gw_quantize_act", "hqo_gw_epilogue",
                         "hqo_prepare_weights", "hqo_gemm_acc", "hqo_epilogue",
                         "hqo_exact_linear", "hqo_prepare_weights_wh", "hqo_epilogue_wh",
                         "hqo_output_rotation"):
                getattr(lib, name).restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a, ctype):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments")


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


# ---------------------------------------------------------------------------
# scalar helpers
# ---------------------------------------------------------------------------

def hadamard_entry(j: int, k: int) -> int:
    return _load().hqo_hadamard_entry(j, k)


def sylvester(n: int) -> np.ndarray:
    out = np.zeros((n, n), dtype=np.int8)
    _check(_load().hqo_sylvester(n, _ptr(out, ctypes.c_int8)), "sylvester")
    return out


def bf16_to_f64(bits) -> np.ndarray:
    bits = np.asarray(bits, dtype=np.uint16)
    lib = _load()
    return np.vectorize(lambda b: lib.hqo_bf16_to_f64(int(b)), otypes=[np.float64])(bits)


def f64_to_bf16(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    lib = _load()
    return np.vectorize(lambda v: lib.hqo_f64_to_bf16(float(v)), otypes=[np.uint16])(x)


def rne(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    lib = _load()
    return np.vectorize(lambda v: lib.hqo_rne(float(v)), otypes=[np.float64])(x)


# ---------------------------------------------------------------------------
# layer steps
# ---------------------------------------------------------------------------

def col_absmax(M_bits: np.ndarray) -> np.ndarray:
    M = _c(M_bits, np.uint16)
    R, C = M.shape
    out = np.zeros(C, dtype=np.float64)
    _check(_load().hqo_col_absmax(_ptr(M, ctypes.c_uint16), R, C, _ptr(out, ctypes.c_double)),
           "col_absmax")
    return out


def channel_mean(M_bits: np.ndarray) -> np.ndarray:
    """Per-channel mean over the rows of a bf16 matrix (fp64)."""
    M = _c(M_bits, np.uint16)
    R, C = M.shape
    out = np.zeros(C, dtype=np.float64)
    _check(_load().hqo_channel_mean(_ptr(M, ctypes.c_uint16), R, C, _ptr(out, ctypes.c_double)),
           "channel_mean")
    return out


def sigma(amax_x: np.ndarray, amax_w: np.ndarray, alpha: float) -> np.ndarray:
    ax = _c(amax_x, np.float64)
    aw = _c(amax_w, np.float64)
    out = np.zeros_like(ax)
    _check(_load().hqo_sigma(ax.size, _ptr(ax, ctypes.c_double), _ptr(aw, ctypes.c_double),
                             float(alpha), _ptr(out, ctypes.c_double)), "sigma")
    return out


def quantize_act(X_bits, n, bits, gran=0, centering=1, sigma=None, static_scale=0.0,
                 rows=None, want_tie=True, want_Z=False, nthreads=None, shift=None):
    """Returns dict(codes int8 [r,K], scale f64 [r], mean f64 [r], tie, Z).
    shift: per-channel vector removed from Y = X diag(sigma^-1) before the
    rotation (the appended-token centring), or None."""
    X = _c(X_bits, np.uint16)
    T, K = X.shape
    sig = _c(sigma, np.float64)
    sh = _c(shift, np.float64)
    r = None if rows is None else _c(rows, np.int64)
    nr = T if r is None else r.size
    codes = np.zeros((nr, K), dtype=np.int8)
    scale = np.zeros(nr, dtype=np.float64)
    mean = np.zeros(nr, dtype=np.float64)
    tie = np.zeros((nr, K), dtype=np.float64) if want_tie else None
    Z = np.zeros((nr, K), dtype=np.float64) if want_Z else None
    rc = _load().hqo_quantize_act(
        K, n, bits, gran, centering, _ptr(X, ctypes.c_uint16), T, _ptr(sig, ctypes.c_double),
        _ptr(sh, ctypes.c_double), float(static_scale), _ptr(r, ctypes.c_int64), nr, _ptr(codes, ctypes.c_int8),
        _ptr(scale, ctypes.c_double), _ptr(mean, ctypes.c_double), _ptr(tie, ctypes.c_double),
        _ptr(Z, ctypes.c_double), nthreads or default_threads())
    _check(rc, "quantize_act")
    return {"codes": codes, "scale": scale, "mean": mean, "tie": tie, "Z": Z}


def prepare_weights(W_bits, n, bits, bias_bits=None, sigma=None, want_tie=True,
                    want_Wt=False, nthreads=None, shift=None):
    """Returns dict(codes int8 [N,K], scale [N], colsum [N], bias [N], tie, Wt).
    shift: the activations' per-channel shift (appended-token centring); its
    product with diag(sigma) W is added to the bias."""
    W = _c(W_bits, np.uint16)
    N, K = W.shape
    b = _c(bias_bits, np.uint16)
    sig = _c(sigma, np.float64)
    sh = _c(shift, np.float64)
    codes = np.zeros((N, K), dtype=np.int8)
    scale = np.zeros(N, dtype=np.float64)
    colsum = np.zeros(N, dtype=np.float64)
    corr_pre = np.zeros(N, dtype=np.float64)
    bias = np.zeros(N, dtype=np.float64)
    tie = np.zeros((N, K), dtype=np.float64) if want_tie else None
    Wt = np.zeros((N, K), dtype=np.float64) if want_Wt else None
    rc = _load().hqo_prepare_weights(
        K, N, n, bits, _ptr(W, ctypes.c_uint16), _ptr(b, ctypes.c_uint16),
        _ptr(sig, ctypes.c_double), _ptr(sh, ctypes.c_double), _ptr(codes, ctypes.c_int8),
        _ptr(scale, ctypes.c_double),
        _ptr(colsum, ctypes.c_double), _ptr(corr_pre, ctypes.c_double),
        _ptr(bias, ctypes.c_double), _ptr(tie, ctypes.c_double),
        _ptr(Wt, ctypes.c_double), nthreads or default_threads())
    _check(rc, "prepare_weights")
    return {"codes": codes, "scale": scale, "colsum": colsum, "corr_pre": corr_pre,
            "bias": bias, "tie": tie, "Wt": Wt}


def correction(w, centering):
    """The correction vector c of the epilogue's m_t * c[n] term for a
    centering mode: colsum(W~) after the rotation (1), sum_k sigma_k W[n,k]
    before it (2)."""
    return w["corr_pre"] if centering == 2 else w["colsum"]


def pack_i4(codes) -> np.ndarray:
    """Codes [..., K] (K even, each in [-8, 7]) -> packed bytes [..., K/2]:
    element 2j in the low nibble of byte j, 2j+1 in the high one, as 4-bit
    two's complement (the packed-code reading of the W4A4 GEMM's 4-bit
    operands, "Data-free 4-bit quantization for diffusion transformers")."""
    c = _c(codes, np.int8)
    if c.shape[-1] % 2:
        raise ValueError("pack_i4 needs an even number of codes per row")
    out = np.empty(c.shape[:-1] + (c.shape[-1] // 2,), dtype=np.uint8)
    _check(_load().hqo_pack_i4(_ptr(c, ctypes.c_int8), c.size, _ptr(out, ctypes.c_uint8)),
           "pack_i4")
    return out


def unpack_i4(packed) -> np.ndarray:
    """Packed bytes [..., K/2] -> codes [..., K] (the inverse of pack_i4)."""
    b = _c(packed, np.uint8)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.int8)
    _check(_load().hqo_unpack_i4(_ptr(b, ctypes.c_uint8), out.size, _ptr(out, ctypes.c_int8)),
           "unpack_i4")
    return out


def gemm_acc(A, B, rows=None, nthreads=None) -> np.ndarray:
    A = _c(A, np.int8)
    B = _c(B, np.int8)
    M, K = A.shape
    N, K2 = B.shape
    if K != K2:
        raise ValueError("K mismatch")
    r = None if rows is None else _c(rows, np.int64)
    nr = M if r is None else r.size
    acc = np.zeros((nr, N), dtype=np.int64)
    _check(_load().hqo_gemm_acc(_ptr(A, ctypes.c_int8), _ptr(B, ctypes.c_int8), M, N, K,
                                _ptr(r, ctypes.c_int64), nr, _ptr(acc, ctypes.c_int64),
                                nthreads or default_threads()), "gemm_acc")
    return acc


def epilogue(acc, sx, sw, colsum=None, bias=None, mean=None):
    """Returns (y f64 [r,N], y_bf16 uint16 [r,N])."""
    acc = _c(acc, np.int64)
    nr, N = acc.shape
    sx = _c(np.broadcast_to(np.asarray(sx, dtype=np.float64), (nr,)), np.float64)
    sw = _c(sw, np.float64)
    m = None if mean is None else _c(np.broadcast_to(np.asarray(mean, dtype=np.float64), (nr,)),
                                     np.float64)
    b = _c(bias, np.float64)
    c = _c(colsum, np.float64)
    y = np.zeros((nr, N), dtype=np.float64)
    yb = np.zeros((nr, N), dtype=np.uint16)
    _check(_load().hqo_epilogue(_ptr(acc, ctypes.c_int64), nr, N, _ptr(sx, ctypes.c_double),
                                _ptr(m, ctypes.c_double), _ptr(sw, ctypes.c_double),
                                _ptr(b, ctypes.c_double), _ptr(c, ctypes.c_double),
                                _ptr(y, ctypes.c_double), _ptr(yb, ctypes.c_uint16)), "epilogue")
    return y, yb


def prepare_weights_wh(W_bits, n_out, bits, bias_bits=None, sigma=None, want_tie=True,
                       want_Wbar=False, nthreads=None):
    """Weight-only Hadamard form (HaTQ Eq. (15)-(17), supplement Eq. (40)):
    Wbar = H_out W diag(sigma) rotated along the output channels (blocks of
    n_out), quantized per row, and b_bar = b H_out.
    Returns dict(codes int8 [N,K], scale [N], b_bar [N], tie, Wbar)."""
    W = _c(W_bits, np.uint16)
    N, K = W.shape
    b = _c(bias_bits, np.uint16)
    sig = _c(sigma, np.float64)
    codes = np.zeros((N, K), dtype=np.int8)
    scale = np.zeros(N, dtype=np.float64)
    b_bar = np.zeros(N, dtype=np.float64)
    tie = np.zeros((N, K), dtype=np.float64) if want_tie else None
    Wbar = np.zeros((N, K), dtype=np.float64) if want_Wbar else None
    rc = _load().hqo_prepare_weights_wh(
        K, N, n_out, bits, _ptr(W, ctypes.c_uint16), _ptr(b, ctypes.c_uint16),
        _ptr(sig, ctypes.c_double), _ptr(codes, ctypes.c_int8), _ptr(scale, ctypes.c_double),
        _ptr(b_bar, ctypes.c_double), _ptr(tie, ctypes.c_double), _ptr(Wbar, ctypes.c_double),
        nthreads or default_threads())
    _check(rc, "prepare_weights_wh")
    return {"codes": codes, "scale": scale, "b_bar": b_bar, "tie": tie, "Wbar": Wbar}


def output_rotation(M, n_out) -> np.ndarray:
    """M H_out for an fp64 matrix [rows, N] (blocks of n_out along N)."""
    M = _c(np.atleast_2d(M), np.float64)
    out = np.zeros_like(M)
    _check(_load().hqo_output_rotation(_ptr(M, ctypes.c_double), M.shape[0], M.shape[1],
                                       n_out, _ptr(out, ctypes.c_double)), "output_rotation")
    return out


def epilogue_wh(acc, n_out, sx, sw, b_bar=None):
    """WH output side (supplement Eq. (41)): (s_x s_w acc + b_bar) H_out.
    Returns (y f64 [r,N], y_bf16 uint16 [r,N])."""
    acc = _c(acc, np.int64)
    nr, N = acc.shape
    sx = _c(np.broadcast_to(np.asarray(sx, dtype=np.float64), (nr,)), np.float64)
    sw = _c(sw, np.float64)
    bb = _c(b_bar, np.float64)
    y = np.zeros((nr, N), dtype=np.float64)
    yb = np.zeros((nr, N), dtype=np.uint16)
    _check(_load().hqo_epilogue_wh(_ptr(acc, ctypes.c_int64), nr, N, n_out,
                                   _ptr(sx, ctypes.c_double), _ptr(sw, ctypes.c_double),
                                   _ptr(bb, ctypes.c_double), _ptr(y, ctypes.c_double),
                                   _ptr(yb, ctypes.c_uint16)), "epilogue_wh")
    return y, yb


def exact_linear(X_bits, W_bits, bias_bits=None, rows=None, nthreads=None) -> np.ndarray:
    X = _c(X_bits, np.uint16)
    W = _c(W_bits, np.uint16)
    T, K = X.shape
    N = W.shape[0]
    b = _c(bias_bits, np.uint16)
    r = None if rows is None else _c(rows, np.int64)
    nr = T if r is None else r.size
    y = np.zeros((nr, N), dtype=np.float64)
    _check(_load().hqo_exact_linear(_ptr(X, ctypes.c_uint16), _ptr(W, ctypes.c_uint16),
                                    _ptr(b, ctypes.c_uint16), T, K, N, _ptr(r, ctypes.c_int64),
                                    nr, _ptr(y, ctypes.c_double), nthreads or default_threads()),
           "exact_linear")
    return y


# ---------------------------------------------------------------------------
# the whole layer, as the pages state it
# ---------------------------------------------------------------------------

def layer(X_bits, W_bits, bias_bits, n, a_bits, w_bits, gran=0, centering=1, alpha=0.5,
          use_sigma=True, rows=None, static_scale=0.0, nthreads=None):
    """Full oracle chain for the listed rows (all rows when rows is None):
    sigma (Eq. 3, calibrated on this X) -> weight fold / quantize -> activation
    transform / centering / quantize -> integer GEMM -> epilogue.
    Returns a dict with every intermediate."""
    sig = None
    if use_sigma:
        sig = sigma(col_absmax(X_bits), col_absmax(W_bits), alpha)
    w = prepare_weights(W_bits, n, w_bits, bias_bits=bias_bits, sigma=sig, nthreads=nthreads)
    a = quantize_act(X_bits, n, a_bits, gran=gran, centering=centering, sigma=sig,
                     static_scale=static_scale, rows=rows, nthreads=nthreads)
    acc = gemm_acc(a["codes"], w["codes"], nthreads=nthreads)
    y, yb = epilogue(acc, a["scale"], w["scale"], colsum=correction(w, centering), bias=w["bias"],
                     mean=a["mean"] if centering else None)
    return {"sigma": sig, "w": w, "a": a, "acc": acc, "y": y, "y_bf16": yb}


def layer_wh(X_bits, W_bits, bias_bits, n_out, a_bits, w_bits, gran=0, alpha=0.5,
             use_sigma=False, rows=None, static_scale=0.0, nthreads=None):
    """Weight-only Hadamard form of the layer (HaTQ Eq. (17) with the bias of
    supplement Eq. (40)-(41)): X quantized in its original basis (no rotation,
    no centering), Wbar = H_out W quantized per row, integer GEMM, then
    (dequantized accumulator + b_bar) H_out.  sigma (Eq. 3 of the HadaNorm
    review) is optional smoothing, off by default as on the HaTQ page."""
    sig = None
    if use_sigma:
        sig = sigma(col_absmax(X_bits), col_absmax(W_bits), alpha)
    w = prepare_weights_wh(W_bits, n_out, w_bits, bias_bits=bias_bits, sigma=sig,
                           nthreads=nthreads)
    a = quantize_act(X_bits, 1, a_bits, gran=gran, centering=0, sigma=sig,
                     static_scale=static_scale, rows=rows, nthreads=nthreads)
    acc = gemm_acc(a["codes"], w["codes"], nthreads=nthreads)
    y, yb = epilogue_wh(acc, n_out, a["scale"], w["scale"], b_bar=w["b_bar"])
    return {"sigma": sig, "w": w, "a": a, "acc": acc, "y": y, "y_bf16": yb}


# ---------------------------------------------------------------------------
# group-wise form with a low-rank branch ("Data-free 4-bit quantization for
# diffusion transformers", "Hadamard rotation: the int4 improvement")
# ---------------------------------------------------------------------------

def _shape(name, a, shape):
    """The C side reads exactly `shape`; anything else is refused here."""
    if a is not None and tuple(np.shape(a)) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(np.shape(a))}")


def low_rank_factors(W_bits, sigma, rank):
    """Rank-r factors of W^ = W diag(sigma) ([N,K]) from its singular value
    decomposition: L2 = U_r diag(S_r) [N,r], L1 = V_r^T [r,K] (fp64), zero
    past min(N, K) components.  A library routine serves as this step (the
    method fixes only L2 L1, the best rank-r approximation)."""
    W = bf16_to_f64(_c(W_bits, np.uint16))
    if sigma is not None:
        W = W * np.asarray(sigma, dtype=np.float64)[None, :]
    N, K = W.shape
    L1 = np.zeros((rank, K))
    L2 = np.zeros((N, rank))
    if rank == 0:
        return L1, L2
    U, S, Vt = np.linalg.svd(W, full_matrices=False)
    k = min(rank, S.size)  # past min(N, K) the factors are zero
    L1[:k] = Vt[:k]
    L2[:, :k] = U[:, :k] * S[:k]
    return L1, L2


def gw_prepare_weights(W_bits, g, bits, rank, L1, L2, bias_bits=None, sigma=None,
                       want_tie=True, want_Rh=False, nthreads=None):
    """Returns dict(codes [N,K], gscale [N,K/g], l1 bf16 bits [r,K], l2 bf16
    bits [N,r], bias [N], tie, Rh)."""
    W = _c(W_bits, np.uint16)
    N, K = W.shape
    b = _c(bias_bits, np.uint16)
    sig = _c(sigma, np.float64)
    _shape("sigma", sig, (K,))
    _shape("bias", b, (N,))
    if rank:
        _shape("L1", L1, (rank, K))
        _shape("L2", L2, (N, rank))
    l1 = np.zeros((rank, K), dtype=np.uint16)
    l2 = np.zeros((N, rank), dtype=np.uint16)
    codes = np.zeros((N, K), dtype=np.int8)
    gscale = np.zeros((N, K // g), dtype=np.float64)
    bias = np.zeros(N, dtype=np.float64)
    tie = np.zeros((N, K), dtype=np.float64) if want_tie else None
    Rh = np.zeros((N, K), dtype=np.float64) if want_Rh else None
    L1c = _c(L1, np.float64) if rank else None
    L2c = _c(L2, np.float64) if rank else None
    rc = _load().hqo_gw_prepare_weights(
        K, N, g, bits, rank, _ptr(W, ctypes.c_uint16), _ptr(b, ctypes.c_uint16),
        _ptr(sig, ctypes.c_double), _ptr(L1c, ctypes.c_double), _ptr(L2c, ctypes.c_double),
        _ptr(l1, ctypes.c_uint16), _ptr(l2, ctypes.c_uint16), _ptr(codes, ctypes.c_int8),
        _ptr(gscale, ctypes.c_double), _ptr(bias, ctypes.c_double), _ptr(tie, ctypes.c_double),
        _ptr(Rh, ctypes.c_double), nthreads or default_threads())
    _check(rc, "gw_prepare_weights")
    return {"codes": codes, "gscale": gscale, "l1": l1, "l2": l2, "bias": bias, "tie": tie,
            "Rh": Rh}


def gw_quantize_act(X_bits, g, bits, rank, l1_bits, sigma=None, rows=None, want_tie=True,
                    want_Z=False, nthreads=None):
    """Returns dict(codes [r,K], gscale [r,K/g], u bf16 bits [r,rank], tie, Z)."""
    X = _c(X_bits, np.uint16)
    T, K = X.shape
    sig = _c(sigma, np.float64)
    l1 = _c(l1_bits, np.uint16) if rank else None
    _shape("sigma", sig, (K,))
    if rank:
        _shape("l1", l1, (rank, K))
    r = None if rows is None else _c(rows, np.int64)
    nr = T if r is None else r.size
    codes = np.zeros((nr, K), dtype=np.int8)
    gscale = np.zeros((nr, K // g), dtype=np.float64)
    u = np.zeros((nr, rank), dtype=np.uint16)
    tie = np.zeros((nr, K), dtype=np.float64) if want_tie else None
    Z = np.zeros((nr, K), dtype=np.float64) if want_Z else None
    rc = _load().hqo_gw_quantize_act(
        K, g, bits, rank, _ptr(X, ctypes.c_uint16), T, _ptr(sig, ctypes.c_double),
        _ptr(l1, ctypes.c_uint16), _ptr(r, ctypes.c_int64), nr, _ptr(codes, ctypes.c_int8),
        _ptr(gscale, ctypes.c_double), _ptr(u, ctypes.c_uint16), _ptr(tie, ctypes.c_double),
        _ptr(Z, ctypes.c_double), nthreads or default_threads())
    _check(rc, "gw_quantize_act")
    return {"codes": codes, "gscale": gscale, "u": u, "tie": tie, "Z": Z}


def gw_epilogue(A, B, g, ascale, wscale, u_bits, l2_bits, bias=None, nthreads=None):
    """(y fp64, y bf16 bits) of the group-wise form's output."""
    A = _c(A, np.int8)
    B = _c(B, np.int8)
    nr, K = A.shape
    N = B.shape[0]
    rank = 0 if u_bits is None else np.asarray(u_bits).shape[1]
    a = _c(ascale, np.float64)
    w = _c(wscale, np.float64)
    u = _c(u_bits, np.uint16) if rank else None
    l2 = _c(l2_bits, np.uint16) if rank else None
    b = _c(bias, np.float64)
    y = np.zeros((nr, N), dtype=np.float64)
    yb = np.zeros((nr, N), dtype=np.uint16)
    rc = _load().hqo_gw_epilogue(
        _ptr(A, ctypes.c_int8), _ptr(B, ctypes.c_int8), nr, N, K, g, _ptr(a, ctypes.c_double),
        _ptr(w, ctypes.c_double), _ptr(u, ctypes.c_uint16), _ptr(l2, ctypes.c_uint16), rank,
        _ptr(b, ctypes.c_double), _ptr(y, ctypes.c_double), _ptr(yb, ctypes.c_uint16),
        nthreads or default_threads())
    _check(rc, "gw_epilogue")
    return y, yb


def layer_gw(X_bits, W_bits, bias_bits, g=64, bits=4, rank=32, sigma=None, rows=None,
             factors=None, nthreads=None):
    """The group-wise form end to end for the listed rows; factors = (L1, L2)
    or None for the rank-r SVD of W diag(sigma)."""
    L1, L2 = factors if factors is not None else low_rank_factors(W_bits, sigma, rank)
    w = gw_prepare_weights(W_bits, g, bits, rank, L1, L2, bias_bits=bias_bits, sigma=sigma,
                           nthreads=nthreads)
    a = gw_quantize_act(X_bits, g, bits, rank, w["l1"], sigma=sigma, rows=rows,
                        nthreads=nthreads)
    y, yb = gw_epilogue(a["codes"], w["codes"], g, a["gscale"], w["gscale"], a["u"], w["l2"],
                        bias=w["bias"], nthreads=nthreads)
    return {"w": w, "a": a, "y": y, "y_bf16": yb, "L1": L1, "L2": L2}
