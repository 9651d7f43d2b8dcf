"""Pins for the CPU oracle: each check compares the oracle with something other
than itself (a second construction, a closed form, a hand-worked value, exact
integer arithmetic, or the unquantized product).  CPU only."""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
POW2 = [1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024]


def kron_sylvester(n):
    """Sylvester matrix as a Kronecker power of [[1,1],[1,-1]] (independent of
    both oracle constructions)."""
    h = np.ones((1, 1), dtype=np.int64)
    base = np.array([[1, 1], [1, -1]], dtype=np.int64)
    while h.shape[0] < n:
        h = np.kron(h, base)
    return h


# --------------------------------------------------------------------------
# Hadamard matrix: HaTQ Eq. (32)-(34), blog step 7
# --------------------------------------------------------------------------

@pytest.mark.parametrize("n", POW2)
def test_sylvester_recursion_matches_popcount_entries(n):
    h_rec = oracle.sylvester(n).astype(np.int64)
    h_pop = np.array([[oracle.hadamard_entry(j, k) for k in range(n)] for j in range(n)]) \
        if n <= 64 else None
    h_kron = kron_sylvester(n)
    assert np.array_equal(h_rec, h_kron)
    if h_pop is not None:
        assert np.array_equal(h_pop, h_kron)
    else:  # spot-check the popcount formula on a seeded sample for large orders
        g = np.random.default_rng(n)
        for j, k in g.integers(0, n, size=(2000, 2)):
            assert oracle.hadamard_entry(int(j), int(k)) == h_kron[j, k]


@pytest.mark.parametrize("n", POW2)
def test_hadamard_orthogonality_exact(n):
    h = oracle.sylvester(n).astype(np.int64)
    assert np.array_equal(h @ h.T, n * np.eye(n, dtype=np.int64))
    assert np.array_equal(h, h.T)  # symmetric, so H^T = H


def test_h64_is_the_kronecker_power_printed_on_the_blog():
    spec = json.load(open(os.path.join(GOLDEN, "hand_examples.json")))["h64_kronecker"]
    f = np.array(spec["factor"], dtype=np.float64)
    h = np.ones((1, 1))
    for _ in range(spec["power"]):
        h = np.kron(h, f)
    h *= spec["scale"]
    # the oracle's normalized block: Z for unit vectors e_j is row j of H_64
    n = spec["n"]
    X = synth.f32_to_bf16_bits(np.eye(n, dtype=np.float32))
    r = oracle.quantize_act(X, n, 8, centering=0, want_Z=True)
    assert np.allclose(r["Z"], h, rtol=0, atol=1e-15)


# --------------------------------------------------------------------------
# scalar helpers
# --------------------------------------------------------------------------

def test_round_half_even():
    xs = [0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 0.49999999999, 0.5000000001, 3.0, -7.5, 6.5, 2.4, -2.6]
    want = [0.0, 2.0, 2.0, -0.0, -2.0, -2.0, 0.0, 1.0, 3.0, -8.0, 6.0, 2.0, -3.0]
    got = oracle.rne(xs)
    assert np.array_equal(got, np.array(want))


def test_bf16_conversions():
    # 1.0, 1 + 2^-8 (tie -> even 1.0), 1 + 3*2^-8 (tie -> even 1 + 2^-6 .. i.e. 0x3F82),
    # -2.0, smallest normal, 65280 (max exact near 2^16), 1/3
    vals = [1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.0, 2.0 ** -126, 65280.0, 1.0 / 3.0]
    bits = [0x3F80, 0x3F80, 0x3F82, 0xC000, 0x0080, 0x477F, 0x3EAB]
    assert list(oracle.f64_to_bf16(vals)) == bits
    assert np.array_equal(oracle.bf16_to_f64(np.array(bits[:6], dtype=np.uint16)),
                          np.array([1.0, 1.0, 1.0 + 2 ** -6, -2.0, 2.0 ** -126, 65280.0]))
    # agreement with the float32 path of the generator on random data
    g = np.random.default_rng(0)
    x = g.standard_normal(5000) * 10.0 ** g.uniform(-3, 3, 5000)
    assert np.array_equal(oracle.f64_to_bf16(x.astype(np.float32).astype(np.float64)),
                          synth.f32_to_bf16_bits(x.astype(np.float32)))


# --------------------------------------------------------------------------
# hand-worked quantizer examples (golden)
# --------------------------------------------------------------------------

def test_hand_worked_examples():
    spec = json.load(open(os.path.join(GOLDEN, "hand_examples.json")))
    for ex in spec["examples"]:
        X = synth.f32_to_bf16_bits(np.array([ex["x"]], dtype=np.float32))
        r = oracle.quantize_act(X, ex["n"], ex["bits"], centering=ex["centering"], want_Z=True)
        assert np.allclose(r["Z"][0], ex["Z"], atol=1e-15), ex["name"]
        assert abs(r["mean"][0] - ex["mean"]) < 1e-15, ex["name"]
        assert abs(r["scale"][0] - ex["scale"]) < 1e-15, ex["name"]
        assert list(r["codes"][0]) == ex["codes"], ex["name"]


# --------------------------------------------------------------------------
# Eq. (1) identity with quantization off
# --------------------------------------------------------------------------

def _bf16(x):
    return synth.bf16_bits_to_f32(x).astype(np.float64)


@pytest.mark.parametrize("K,n,N,T", [(16, 4, 8, 5), (64, 16, 24, 9), (256, 64, 40, 7),
                                     (1152, 128, 32, 4), (3072, 1024, 16, 3)])
@pytest.mark.parametrize("centering", [0, 1, 2])
def test_eq1_identity_unquantized(K, n, N, T, centering):
    g = np.random.default_rng(K + n + centering)
    X = synth.f32_to_bf16_bits(g.standard_normal((T, K)) * 2 + g.standard_normal((T, 1)) * 3)
    W = synth.f32_to_bf16_bits(g.standard_normal((N, K)) * 0.05)
    b = synth.f32_to_bf16_bits(g.standard_normal(N) * 0.1)
    sig = oracle.sigma(oracle.col_absmax(X), oracle.col_absmax(W), 0.5)
    assert np.all(sig > 0) and not np.allclose(sig, 1.0)
    a = oracle.quantize_act(X, n, 8, centering=centering, sigma=sig, want_Z=True)
    w = oracle.prepare_weights(W, n, 8, bias_bits=b, sigma=sig, want_Wt=True)
    # X~ = X diag(s^-1) H - mu: mu removed after the rotation (centering 1) or
    # before it (centering 2, where Z is already (Y - mu_t) H)
    shift = a["mean"] if centering == 1 else np.zeros(T)
    V = a["Z"] - shift[:, None]
    c = oracle.correction(w, centering)
    y_tilde = V @ w["Wt"].T + w["bias"][None, :] + a["mean"][:, None] * c[None, :]
    y = _bf16(X) @ _bf16(W).T + _bf16(b)[None, :]          # XW + b
    rel = np.linalg.norm(y_tilde - y) / np.linalg.norm(y)
    assert rel <= 1e-10, rel
    # the layer's own exact reference agrees with the numpy product
    assert np.allclose(oracle.exact_linear(X, W, b), y, rtol=0, atol=1e-10 * np.abs(y).max())


# --------------------------------------------------------------------------
# closed-form invariants
# --------------------------------------------------------------------------

@pytest.mark.parametrize("K,n", [(64, 16), (1152, 128), (320, 64), (2048, 1024)])
def test_invariants(K, n):
    T, N = 6, 10
    g = np.random.default_rng(K)
    X = synth.f32_to_bf16_bits(g.standard_normal((T, K)) + 2.0)
    W = synth.f32_to_bf16_bits(g.standard_normal((N, K)) * 0.02)
    sig = oracle.sigma(oracle.col_absmax(X), oracle.col_absmax(W), 0.5)
    a = oracle.quantize_act(X, n, 4, centering=1, sigma=sig, want_Z=True)
    w = oracle.prepare_weights(W, n, 4, sigma=sig, want_Wt=True)
    Y = _bf16(X) / sig[None, :]
    Z = a["Z"]
    B = K // n
    rn = math.sqrt(n)
    # HaTQ Eq. (23): the constant-basis coordinate is sqrt(n) times the block mean
    for blk in range(B):
        assert np.allclose(Z[:, blk * n], rn * Y[:, blk * n:(blk + 1) * n].mean(axis=1),
                           rtol=1e-12, atol=1e-12)
    # column sums of H~ vanish except the first: m_t = (sqrt(n)/K) sum_b Y[t, b n]
    assert np.allclose(a["mean"], rn / K * Y[:, ::n].sum(axis=1), rtol=1e-12, atol=1e-12)
    # same for the weight fold: c_n = sqrt(n) sum_b sigma_{bn} W[n, bn]
    Wf = _bf16(W)
    assert np.allclose(w["colsum"], rn * (Wf[:, ::n] * sig[None, ::n]).sum(axis=1),
                       rtol=1e-11, atol=1e-12)
    # centred activations sum to zero; the rotation preserves each block's norm
    V = Z - a["mean"][:, None]
    assert np.allclose(V.sum(axis=1), 0.0, atol=1e-10 * np.abs(Z).max())
    for blk in range(B):
        s = slice(blk * n, (blk + 1) * n)
        assert np.allclose(np.linalg.norm(Z[:, s], axis=1), np.linalg.norm(Y[:, s], axis=1),
                           rtol=1e-12)


@pytest.mark.parametrize("K,n", [(64, 16), (1152, 128), (320, 64), (2048, 1024)])
def test_invariants_pre_rotation_centering(K, n):
    """Centering 2 removes mean_k Y[t,k] before the rotation.  Because every
    column of H~ but each block's first sums to zero, this changes only the
    first channel of each block, by -sqrt(n) mu_t, and those channels then
    sum to zero; the weight-side correction is sum_k sigma_k W[n,k]."""
    T, N = 6, 10
    g = np.random.default_rng(K + 1)
    X = synth.f32_to_bf16_bits(g.standard_normal((T, K)) + 2.0)
    W = synth.f32_to_bf16_bits(g.standard_normal((N, K)) * 0.02)
    sig = oracle.sigma(oracle.col_absmax(X), oracle.col_absmax(W), 0.5)
    a2 = oracle.quantize_act(X, n, 4, centering=2, sigma=sig, want_Z=True)
    a0 = oracle.quantize_act(X, n, 4, centering=0, sigma=sig, want_Z=True)
    w = oracle.prepare_weights(W, n, 4, sigma=sig)
    Y = _bf16(X) / sig[None, :]
    mu = Y.mean(axis=1)
    assert np.allclose(a2["mean"], mu, rtol=1e-13, atol=1e-13)
    diff = a2["Z"] - a0["Z"]
    first = np.zeros(K, dtype=bool)
    first[::n] = True
    assert np.allclose(diff[:, ~first], 0.0, atol=1e-12)
    assert np.allclose(diff[:, first], -math.sqrt(n) * mu[:, None], rtol=1e-12, atol=1e-12)
    assert np.allclose(a2["Z"][:, first].sum(axis=1), 0.0, atol=1e-10 * np.abs(a0["Z"]).max())
    assert np.allclose(w["corr_pre"], (_bf16(W) * sig[None, :]).sum(axis=1), rtol=1e-12,
                       atol=1e-13)
    # and in terms of the rotated weights: sqrt(n) times their blocks' first channels
    w2 = oracle.prepare_weights(W, n, 4, sigma=sig, want_Wt=True)
    assert np.allclose(w["corr_pre"], math.sqrt(n) * w2["Wt"][:, first].sum(axis=1),
                       rtol=1e-11, atol=1e-12)


def test_pre_rotation_centering_removes_the_token_offset():
    """On the configurations' token-offset data, removing the mean before the
    rotation leaves a much smaller max |V| than removing it after (which only
    moves the mean of V), so its output is closer to the exact product."""
    for idx in (1, 2):
        cfg = synth.CONFIGS[idx].with_tokens(64)
        Xb, Wb, bb = synth.make_layer(cfg)
        y_ex = oracle.exact_linear(Xb, Wb, bb)

        def sqnr(c):
            r = oracle.layer(Xb, Wb, bb, cfg.had_order, cfg.a_bits, cfg.w_bits, centering=c,
                             alpha=cfg.alpha, use_sigma=cfg.use_sigma)
            return 10 * np.log10(np.linalg.norm(y_ex) ** 2 / np.linalg.norm(r["y"] - y_ex) ** 2)

        assert sqnr(2) > sqnr(1) + 6.0, idx


# --------------------------------------------------------------------------
# brute force at K = 8: exact integer decision of every code
# --------------------------------------------------------------------------

def _exact_codes_int(x_int, n, q, centering):
    """Exact codes for integer inputs with sigma = 1, decided in integer
    arithmetic.  Z_hat = x H~ is an integer vector and Z = Z_hat / sqrt(n);
    the codes depend only on V / max|V|, so scale V by K*sqrt(n):
    U = K*Z_hat - sum(Z_hat) (centred) or K*Z_hat (not centred).
    code = rne(q * U / max|U|).  Returns (codes, is_exact_tie)."""
    B = x_int.shape[1] // n
    H = kron_sylvester(n)
    zh = np.concatenate([x_int[:, b * n:(b + 1) * n] @ H for b in range(B)], axis=1)
    K = x_int.shape[1]
    if centering == 2:
        # K (x - mean(x)) H~ = K Z_hat - sum(x) (n at each block's first
        # channel, 0 elsewhere); sum(x) = sum of the blocks' first channels
        U = K * zh
        U[:, ::n] -= n * zh[:, ::n].sum(axis=1, keepdims=True)
    else:
        U = K * zh - (zh.sum(axis=1, keepdims=True) if centering else 0)
    D = np.abs(U).max(axis=1, keepdims=True)
    num = q * U
    den = np.where(D == 0, 1, D)
    f = np.floor_divide(num, den)
    r = num - f * den
    two_r = 2 * r
    up = two_r > den
    tie = two_r == den
    codes = f + up + (tie & (f % 2 != 0))
    codes = np.where(D == 0, 0, codes)
    return codes, tie & (D != 0), (U / K if centering == 2 else zh)


@pytest.mark.parametrize("n", [4, 8])
@pytest.mark.parametrize("bits,centering", [(4, 1), (3, 1), (4, 0), (4, 2), (3, 2), (2, 0), (2, 1)])
def test_bruteforce_k8(n, bits, centering):
    vals = np.arange(-2, 3)
    x_int = np.array(list(itertools.product(vals, repeat=8)), dtype=np.int64)  # 5^8 rows
    X = synth.f32_to_bf16_bits(x_int.astype(np.float32))
    q = 2 ** (bits - 1) - 1
    r = oracle.quantize_act(X, n, bits, centering=centering, want_Z=True)
    want, tie, zh = _exact_codes_int(x_int, n, q, centering)
    # the dense transform equals an independent evaluation of HaTQ Eq. (8)
    assert np.allclose(r["Z"], zh / math.sqrt(n), rtol=0, atol=1e-13)
    codes = r["codes"].astype(np.int64)
    off = codes != want
    # away from exact ties the decision is unique
    assert not np.any(off & ~tie)
    # at exact ties (fp64 cannot see them when q/n makes the scale inexact) the
    # oracle must still pick one of the two neighbours
    assert np.all(np.abs(codes - want)[tie] <= 1)
    assert np.all(np.abs(codes) <= q)
    # exhaustive arg-min over the 2q+1 grid levels agrees with the code
    levels = np.arange(-q, q + 1)
    V = r["Z"] - (r["mean"][:, None] if centering == 1 else 0.0)
    s = r["scale"][:, None]
    safe = np.where(s == 0, 1.0, s)
    dist = np.abs((V / safe)[..., None] - levels[None, None, :])
    best = levels[np.argmin(dist + 1e-9 * (np.abs(levels) % 2)[None, None, :], axis=2)]
    best = np.where(s == 0, 0, best)
    assert np.array_equal(best[~tie], codes[~tie])


def test_integer_accumulation_all_int4_vectors():
    levels = np.arange(-7, 8, dtype=np.int8)
    A = np.array(list(itertools.product(levels, repeat=4)), dtype=np.int8)  # 15^4 rows
    g = np.random.default_rng(4)
    B = g.integers(-8, 8, size=(6, 4)).astype(np.int8)
    B[0] = 7
    B[1] = -7
    acc = oracle.gemm_acc(A, B)
    assert np.array_equal(acc, A.astype(np.int64) @ B.astype(np.int64).T)


def test_integer_accumulation_full_int8_range():
    g = np.random.default_rng(5)
    A = g.integers(-128, 128, size=(37, 300)).astype(np.int8)
    B = g.integers(-128, 128, size=(19, 300)).astype(np.int8)
    A[0] = -128
    B[0] = -128
    rows = np.array([0, 5, 36])
    acc = oracle.gemm_acc(A, B, rows=rows)
    assert np.array_equal(acc, (A.astype(np.int64) @ B.astype(np.int64).T)[rows])


# --------------------------------------------------------------------------
# lossless case: the quantized chain reproduces XW + b exactly
# --------------------------------------------------------------------------

def test_dyadic_lossless_chain_equals_exact_product():
    """Build X and W whose rotated (and centred) values sit exactly on their
    grids, so quantization loses nothing: then s_x s_w acc + b + m c must equal
    XW + b (HadaNorm Eq. (1) with the HaTQ Eq. (18) accumulator scale).  A
    dropped term, wrong sign or transposed operand breaks the equality."""
    n, K, N, T = 4, 8, 5, 4
    H = kron_sylvester(n) / 2.0                      # H~_4 / sqrt(4), exact
    Hb = np.kron(np.eye(K // n), H)
    g = np.random.default_rng(11)
    X_rows, m_list = [], []
    for t in range(T):
        c = g.integers(-6, 7, size=K)
        c[0] = 7
        c[-1] = -(c[:-1].sum())                      # sum of V = 0
        if abs(c[-1]) > 7:
            c[1:-1] = 0
            c[-1] = -7
        s = 0.25
        m = float(g.integers(-8, 9)) * 0.125
        Z = s * c + m
        X_rows.append(Z @ Hb.T)                      # X = Z H^T (H orthogonal)
        m_list.append(m)
    Xf = np.array(X_rows)
    Wq = g.integers(-7, 8, size=(N, K))
    Wq[:, 0] = 7
    Wt = 0.125 * Wq
    Wf = Wt @ Hb.T                                   # W~ = W H  =>  W = W~ H^T
    bf = g.integers(-4, 5, size=N) * 0.0625
    X = synth.f32_to_bf16_bits(Xf.astype(np.float32))
    W = synth.f32_to_bf16_bits(Wf.astype(np.float32))
    b = synth.f32_to_bf16_bits(bf.astype(np.float32))
    assert np.array_equal(_bf16(X), Xf) and np.array_equal(_bf16(W), Wf)
    out = oracle.layer(X, W, b, n, 4, 4, centering=1, use_sigma=False)
    assert np.allclose(out["a"]["mean"], m_list, atol=0)
    y_exact = oracle.exact_linear(X, W, b)
    assert np.array_equal(out["y"], y_exact), np.abs(out["y"] - y_exact).max()
    assert np.array_equal(out["y_bf16"], oracle.f64_to_bf16(y_exact))


# --------------------------------------------------------------------------
# granularities and row sampling
# --------------------------------------------------------------------------

def test_per_tensor_and_static_scales():
    cfg = synth.CONFIGS[4].with_tokens(64)
    X = synth.make_x(cfg)
    tok = oracle.quantize_act(X, 64, 8, gran=0, centering=0)
    ten = oracle.quantize_act(X, 64, 8, gran=1, centering=0)
    assert np.allclose(ten["scale"], tok["scale"].max(), rtol=1e-15)
    st = oracle.quantize_act(X, 64, 8, gran=2, centering=0, static_scale=ten["scale"][0])
    assert np.array_equal(st["codes"], ten["codes"])
    # sampled rows of a per-tensor quantization still use the whole-tensor scale
    rows = np.array([3, 17, 63])
    sub = oracle.quantize_act(X, 64, 8, gran=1, centering=0, rows=rows)
    assert np.array_equal(sub["codes"], ten["codes"][rows])
    assert np.all(sub["scale"] == ten["scale"][0])


def test_row_subset_matches_full():
    cfg = synth.CONFIGS[2].with_tokens(40)
    X = synth.make_x(cfg)
    full = oracle.quantize_act(X, 128, 4)
    rows = np.array([0, 7, 39])
    sub = oracle.quantize_act(X, 128, 4, rows=rows)
    assert np.array_equal(sub["codes"], full["codes"][rows])
    assert np.array_equal(sub["scale"], full["scale"][rows])
    assert np.array_equal(sub["mean"], full["mean"][rows])


def test_zero_row_gives_zero_codes_and_scale():
    X = np.zeros((2, 64), dtype=np.uint16)
    X[1] = synth.f32_to_bf16_bits(np.linspace(-1, 1, 64).astype(np.float32))
    r = oracle.quantize_act(X, 64, 4)
    assert r["scale"][0] == 0.0 and not r["codes"][0].any()
    assert r["scale"][1] > 0.0


def test_quantization_noise_is_within_grid_bound():
    """|V - s * code| <= s / 2 for every element (HaTQ Eq. (3) with rne)."""
    cfg = synth.CONFIGS[3].with_tokens(16)
    X = synth.make_x(cfg)
    r = oracle.quantize_act(X, 256, 3, want_Z=True)
    V = r["Z"] - r["mean"][:, None]
    err = np.abs(V - r["scale"][:, None] * r["codes"])
    assert np.all(err <= r["scale"][:, None] / 2 * (1 + 1e-12))


# --------------------------------------------------------------------------
# weight-only Hadamard form: HaTQ Eq. (15)-(17), supplement Eq. (40)-(41)
# --------------------------------------------------------------------------

def _block_h(N, n_out):
    """Normalized block-diagonal Sylvester matrix built from the Kronecker
    power (independent of the oracle's popcount construction)."""
    return np.kron(np.eye(N // n_out), kron_sylvester(n_out) / math.sqrt(n_out))


@pytest.mark.parametrize("N,n_out", [(4, 2), (32, 16), (64, 64), (96, 32)])
def test_wh_weights_are_the_output_side_rotation(N, n_out):
    """Wbar = H_out W diag(sigma) and b_bar = b H_out against explicit
    matrices; the codes quantize Wbar row by row."""
    K = 24
    g = np.random.default_rng(N + n_out)
    W = synth.f32_to_bf16_bits(g.standard_normal((N, K)).astype(np.float32))
    b = synth.f32_to_bf16_bits(g.standard_normal(N).astype(np.float32))
    sig = 10.0 ** g.uniform(-0.5, 0.5, size=K)
    w = oracle.prepare_weights_wh(W, n_out, 8, bias_bits=b, sigma=sig, want_Wbar=True)
    Hout = _block_h(N, n_out)
    Wf = synth.bf16_bits_to_f32(W).astype(np.float64)
    bf = synth.bf16_bits_to_f32(b).astype(np.float64)
    assert np.allclose(w["Wbar"], Hout @ (Wf * sig[None, :]), rtol=0, atol=1e-12)
    assert np.allclose(w["b_bar"], bf @ Hout, rtol=0, atol=1e-12)
    s = np.abs(w["Wbar"]).max(axis=1) / 127.0
    assert np.allclose(w["scale"], s, rtol=1e-15)
    assert np.all(np.abs(w["codes"]).max(axis=1) == 127)
    # codes from the unnormalized +-1 sums (the normalization cancels in Wbar / max|Wbar|)
    S = np.kron(np.eye(N // n_out), kron_sylvester(n_out)) @ (Wf * sig[None, :])
    x = S * 127.0 / np.abs(S).max(axis=1)[:, None]
    assert np.array_equal(w["codes"], np.clip(oracle.rne(x), -127, 127))


@pytest.mark.parametrize("n_out", [1, 2, 16, 64])
def test_wh_identity_unquantized(n_out):
    """Eq. (16) / (41) with quantization off: (X Wbar^T + b_bar) H_out = X W^T + b."""
    T, K, N = 7, 40, 128
    g = np.random.default_rng(n_out)
    X = synth.f32_to_bf16_bits(g.standard_normal((T, K)).astype(np.float32))
    W = synth.f32_to_bf16_bits(g.standard_normal((N, K)).astype(np.float32))
    b = synth.f32_to_bf16_bits(g.standard_normal(N).astype(np.float32))
    w = oracle.prepare_weights_wh(W, n_out, 8, bias_bits=b, want_Wbar=True)
    Xf = synth.bf16_bits_to_f32(X).astype(np.float64)
    y = oracle.output_rotation(Xf @ w["Wbar"].T + w["b_bar"][None, :], n_out)
    ex = oracle.exact_linear(X, W, b)
    assert np.allclose(y, ex, rtol=0, atol=1e-11 * np.abs(ex).max())


def test_wh_hand_worked_example():
    """N = 2, n_out = 2, K = 1, W = [3, 1]^T, b = [1, -1], 4-bit codes:
    Wbar = H_2 W = [4, 2] / sqrt(2), b_bar = b H_2 = [0, 2] / sqrt(2);
    row scales Wbar / 7 put both codes at 7.  With X = [[2]] quantized per
    token (code 7, scale 2/7), acc = [49, 49] and the bracket of Eq. (41) is
    [2 * 4/sqrt(2), 2 * 2/sqrt(2) + 2/sqrt(2)] = [8, 6] / sqrt(2); times H_2
    gives [14, 2] / 2 = [7, 1] = X W^T + b exactly (2*3 + 1, 2*1 - 1)."""
    W = synth.f32_to_bf16_bits(np.array([[3.0], [1.0]], dtype=np.float32))
    b = synth.f32_to_bf16_bits(np.array([1.0, -1.0], dtype=np.float32))
    X = synth.f32_to_bf16_bits(np.array([[2.0]], dtype=np.float32))
    r = oracle.layer_wh(X, W, b, 2, 4, 4)
    r2 = math.sqrt(2.0)
    assert np.allclose(r["w"]["scale"], [4 / r2 / 7, 2 / r2 / 7], rtol=1e-15)
    assert np.array_equal(r["w"]["codes"], [[7], [7]])
    assert np.allclose(r["w"]["b_bar"], [0.0, 2 / r2], atol=1e-15)
    assert np.array_equal(r["a"]["codes"], [[7]])
    assert np.array_equal(r["acc"], [[49, 49]])
    assert np.allclose(r["y"], [[7.0, 1.0]], atol=1e-14)


def test_wh_order_one_is_the_plain_quantized_product():
    """n_out = 1: no rotation on either side; the WH layer is then the
    per-token quantized product dequantized column by column, recomputed here
    with integer numpy arithmetic."""
    T, K, N = 9, 48, 20
    g = np.random.default_rng(3)
    X = synth.f32_to_bf16_bits(g.standard_normal((T, K)).astype(np.float32))
    W = synth.f32_to_bf16_bits(g.standard_normal((N, K)).astype(np.float32))
    b = synth.f32_to_bf16_bits(g.standard_normal(N).astype(np.float32))
    r = oracle.layer_wh(X, W, b, 1, 4, 4)
    Xf = synth.bf16_bits_to_f32(X).astype(np.float64)
    Wf = synth.bf16_bits_to_f32(W).astype(np.float64)
    sx = np.abs(Xf).max(axis=1) / 7.0
    sw = np.abs(Wf).max(axis=1) / 7.0

    def exact_codes(M):
        # rne(7 m / max|row|) in exact rational arithmetic (bf16 values are dyadic)
        out = np.zeros(M.shape, dtype=np.int64)
        for i, row in enumerate(M):
            a = max(abs(Fraction(float(v))) for v in row)
            for j, v in enumerate(row):
                x = Fraction(float(v)) * 7 / a
                f = math.floor(x)
                c = f + 1 if x - f > Fraction(1, 2) else (f if x - f < Fraction(1, 2) else
                                                         (f if f % 2 == 0 else f + 1))
                out[i, j] = max(-7, min(7, c))
        return out

    ax, aw = exact_codes(Xf), exact_codes(Wf)
    y = (ax @ aw.T) * sx[:, None] * sw[None, :] + synth.bf16_bits_to_f32(b)[None, :]
    assert np.array_equal(r["a"]["codes"], ax) and np.array_equal(r["w"]["codes"], aw)
    assert np.allclose(r["y"], y, rtol=0, atol=1e-12 * np.abs(y).max())


@pytest.mark.parametrize("n_out", [16, 64])
def test_wh_epilogue_against_explicit_matrices(n_out):
    """The WH epilogue on random integer accumulators equals
    (diag(sx) acc diag(sw) + b_bar) H_out built from the Kronecker power."""
    nr, N = 5, 128
    g = np.random.default_rng(n_out + 1)
    acc = g.integers(-5000, 5000, size=(nr, N)).astype(np.int64)
    sx, sw, bb = g.random(nr) + 0.1, g.random(N) * 0.01, g.standard_normal(N)
    y, _ = oracle.epilogue_wh(acc, n_out, sx, sw, bb)
    ref = (sx[:, None] * acc * sw[None, :] + bb[None, :]) @ _block_h(N, n_out)
    assert np.allclose(y, ref, rtol=0, atol=1e-12 * np.abs(ref).max())


# ---------------------------------------------------------------- packed codes
# Two 3- or 4-bit codes per byte, element 2j in the low nibble of byte j and
# element 2j+1 in the high nibble, each a 4-bit two's-complement value (the
# storage reading for the 4-bit operands of the W4A4 GEMM in "Data-free 4-bit
# quantization for diffusion transformers", which fixes no layout).

def test_packed_codes_hand_worked_bytes():
    # the int4 and int3 hand-worked quantizer examples above, packed by hand:
    #   [7, -2 | -4, -1]: 0x7 + 16 * 0xE = 0xE7, 0xC + 16 * 0xF = 0xFC
    #   [3, -1 | -2,  0]: 0x3 + 16 * 0xF = 0xF3, 0xE + 16 * 0x0 = 0x0E
    assert oracle.pack_i4(np.array([[7, -2, -4, -1]])).tolist() == [[0xE7, 0xFC]]
    assert oracle.pack_i4(np.array([[3, -1, -2, 0]])).tolist() == [[0xF3, 0x0E]]
    assert oracle.unpack_i4(np.array([[0xE7, 0xFC]], np.uint8)).tolist() == [[7, -2, -4, -1]]


def test_packed_codes_are_a_bijection_on_all_bytes():
    every_byte = np.arange(256, dtype=np.uint8)
    codes = oracle.unpack_i4(every_byte)
    assert codes.min() == -8 and codes.max() == 7
    assert np.array_equal(oracle.pack_i4(codes), every_byte)
    pairs = np.array(list(itertools.product(range(-8, 8), repeat=2)), dtype=np.int8).reshape(-1)
    assert np.array_equal(oracle.unpack_i4(oracle.pack_i4(pairs)), pairs)


def test_packed_nibbles_are_arithmetic_shifts_of_the_signed_byte():
    # independent reading of the layout: the byte as int8, shifted right
    # arithmetically by 4, is the high code; shifted left by 4 first (a wrap
    # in int8), the low code
    every_byte = np.arange(256, dtype=np.uint8)
    codes = oracle.unpack_i4(every_byte)
    signed = every_byte.view(np.int8)
    assert np.array_equal(codes[1::2], signed >> 4)
    assert np.array_equal(codes[0::2], (every_byte << 4).astype(np.uint8).view(np.int8) >> 4)


def test_packed_codes_reject_out_of_range_values():
    with pytest.raises(ValueError):
        oracle.pack_i4(np.array([8, 0], dtype=np.int8))
    with pytest.raises(ValueError):
        oracle.pack_i4(np.array([0, -9], dtype=np.int8))
    with pytest.raises(ValueError):
        oracle.pack_i4(np.array([1, 2, 3], dtype=np.int8))


# --------------------------------------------------------------------------
# Calibration: HadaNorm review, "What carries the argument", Eq. (3)
# sigma_i = max|X_i|^alpha / max|W_i|^(1-alpha), with max over the tokens of
# input channel i for X and over the output channels of input channel i for W
# --------------------------------------------------------------------------

def _bf16_bits(values):
    """bf16 bit patterns of values that bf16 holds exactly (hand-checked)."""
    table = {1.0: 0x3F80, -1.0: 0xBF80, 2.0: 0x4000, -2.0: 0xC000, 0.5: 0x3F00,
             0.25: 0x3E80, -3.5: 0xC060, -4.0: 0xC080, 3.0: 0x4040, 0.0: 0x0000,
             4.0: 0x4080}
    out = []
    for v in values:
        if isinstance(v, str):  # "-0": the negative zero bit pattern
            out.append(0x8000)
        else:
            out.append(table[v])
    return out


def test_col_absmax_hand_built_matrix():
    """max over rows of |M[r, c]| for a 3 x 4 bf16 matrix written out by
    hand: negative entries, a column of +0 and -0 only, the largest magnitude
    in the first, middle and last row.  A signed max (no absolute value)
    would give [1, 0, 0.5, 3]; a max along rows instead of columns has
    three entries, not four."""
    rows = [[1.0, "-0", -3.5, 3.0],
            [-2.0, 0.0, 0.5, -1.0],
            [0.25, "-0", -4.0, 2.0]]
    M = np.array([_bf16_bits(r) for r in rows], dtype=np.uint16)
    got = oracle.col_absmax(M)
    assert got.shape == (4,)
    assert got.tolist() == [2.0, 0.0, 4.0, 3.0]
    assert not np.signbit(got[1])  # |-0| is +0
    # a single row is its own absolute value; no rows leaves the zero start
    assert oracle.col_absmax(M[1:2]).tolist() == [2.0, 0.0, 0.5, 1.0]
    assert oracle.col_absmax(M[:0]).tolist() == [0.0, 0.0, 0.0, 0.0]


def test_sigma_hand_worked_values_of_eq3():
    """sigma = amax_x^alpha / amax_w^(1-alpha), worked by hand:
      amax_x = 4,  amax_w = 1/4, alpha = 1/2:  2 / (1/2)        = 4
      amax_x = 16, amax_w = 81,  alpha = 1/4:  16^(1/4) / 81^(3/4) = 2 / 27
    The second case separates the plausible slips: swapping alpha and
    1 - alpha gives 16^(3/4) / 81^(1/4) = 8/3, the inverted ratio 27/2."""
    ax = np.array([4.0, 16.0])
    aw = np.array([0.25, 81.0])
    s = oracle.sigma(ax, aw, 0.5)
    assert s[0] == pytest.approx(4.0, rel=1e-15)
    s = oracle.sigma(ax, aw, 0.25)
    assert s[1] == pytest.approx(2.0 / 27.0, rel=1e-14)
    assert s[1] != pytest.approx(8.0 / 3.0) and s[1] != pytest.approx(27.0 / 2.0)


def test_sigma_end_points_of_alpha():
    """alpha = 0 leaves only the weight term, sigma = 1 / amax_w; alpha = 1
    only the activation term, sigma = amax_x (HadaNorm review Eq. (3) at the
    ends of its range)."""
    ax = np.array([3.0, 0.5, 12.0, 1.0])
    aw = np.array([0.02, 4.0, 0.125, 1.0])
    assert np.allclose(oracle.sigma(ax, aw, 0.0), 1.0 / aw, rtol=1e-15, atol=0)
    assert np.allclose(oracle.sigma(ax, aw, 1.0), ax, rtol=1e-15, atol=0)


def test_sigma_is_one_when_a_maximum_is_zero():
    """A channel that is identically zero on either side has no scale to
    balance: sigma = 1 there (the oracle's guard; the pages are silent), and
    the neighbouring channels keep their Eq. (3) values."""
    ax = np.array([0.0, 4.0, 0.0, 4.0])
    aw = np.array([0.25, 0.0, 0.0, 0.25])
    s = oracle.sigma(ax, aw, 0.5)
    assert s.tolist() == [1.0, 1.0, 1.0, pytest.approx(4.0, rel=1e-15)]
    assert np.all(np.isfinite(oracle.sigma(ax, aw, 0.3)))


def test_sigma_balances_the_channel_maxima():
    """The point of Eq. (3): after X diag(sigma^-1) and diag(sigma) W the
    channel maxima satisfy max|X_i / sigma_i| = amax_x^(1-alpha) amax_w^(1-alpha)
    and max|sigma_i W_i| = amax_x^alpha amax_w^alpha, so at alpha = 1/2 both
    sides share the maximum sqrt(amax_x amax_w) (SmoothQuant-style balance)."""
    g = np.random.default_rng(5)
    X = synth.f32_to_bf16_bits((g.standard_normal((64, 48)) * np.exp(g.standard_normal(48))).astype(np.float32))
    W = synth.f32_to_bf16_bits((g.standard_normal((32, 48)) * 0.02).astype(np.float32))
    ax, aw = oracle.col_absmax(X), oracle.col_absmax(W)
    for alpha in (0.5, 0.3):
        s = oracle.sigma(ax, aw, alpha)
        xs = np.max(np.abs(oracle.bf16_to_f64(X)) / s, axis=0)
        ws = np.max(np.abs(oracle.bf16_to_f64(W)) * s, axis=0)
        assert np.allclose(xs, ax ** (1 - alpha) * aw ** (1 - alpha), rtol=1e-12)
        assert np.allclose(ws, ax ** alpha * aw ** alpha, rtol=1e-12)
        if alpha == 0.5:
            assert np.allclose(xs, ws, rtol=1e-12)


# --------------------------------------------------------------------------
# Per-channel centring over tokens: HadaNorm review, Figure 2 caption (mu, sigma
# in R^d) and Desk Editor's Note (the bias absorbed into an appended token).
# mu_k = mean_t Y[t,k] is removed before the rotation, V = (Y - mu) H, and its
# product with the weights, mu diag(sigma) W, is the same for every token: a
# bias term.
# --------------------------------------------------------------------------

def test_channel_mean_hand_built_matrix():
    """Mean over the rows of each column of a 4 x 4 bf16 matrix written out
    by hand (dyadic values, so the means are exact); a mean along rows would
    give (1 + -2 + 0.5 + 3) / 4 = 0.625 first."""
    vals = [[1.0, -2.0, 0.5, 3.0],
            [3.0, 2.0, "-0", 1.0],
            [0.0, 0.25, 0.5, -4.0],
            [-2.0, -1.0, 3.0, 0.0]]
    M = np.array([_bf16_bits(r) for r in vals], dtype=np.uint16)
    assert oracle.channel_mean(M).tolist() == [0.5, -0.1875, 1.0, 0.0]


def _two_token_layer():
    # X = [[1,2,3,4],[3,2,1,0]] in bf16, sigma = 1, n = K = 4
    X = np.array([_bf16_bits([1.0, 2.0, 3.0, 4.0]), _bf16_bits([3.0, 2.0, 1.0, 0.0])],
                 dtype=np.uint16)
    return X


def test_channel_centring_hand_worked_example():
    """Worked by hand: the channel mean is mu = [2, 2, 2, 2]; Y - mu =
    [-1, 0, 1, 2] and its negation; with H = H~_4 / 2 the rotated rows are
    V = [1, -1, -2, 0] and [-1, 1, 2, 0], max |V| = 2.
      int4 (q = 7): V * 7 / 2 = [3.5, -3.5, -7, 0] -> half to even [4, -4, -7, 0]
      int3 (q = 3): V * 3 / 2 = [1.5, -1.5, -3, 0] -> [2, -2, -3, 0]
    With the token mean also removed before H (centring 2): row 0 becomes
    [-1.5, -0.5, 0.5, 1.5], V = [0, -1, -2, 0], int4 codes [0, -4, -7, 0],
    reported mean 0.5.  The weight side adds mu diag(sigma) W to the bias:
    W = [1, 0, -1, 0.5], b = 0.25 -> 0.25 + 2 * 0.5 = 1.25."""
    X = _two_token_layer()
    mu = oracle.channel_mean(X)
    assert mu.tolist() == [2.0, 2.0, 2.0, 2.0]
    a4 = oracle.quantize_act(X, 4, 4, centering=0, shift=mu, want_Z=True)
    assert a4["Z"].tolist() == [[1.0, -1.0, -2.0, 0.0], [-1.0, 1.0, 2.0, 0.0]]
    assert a4["codes"].tolist() == [[4, -4, -7, 0], [-4, 4, 7, 0]]
    assert a4["scale"].tolist() == pytest.approx([2.0 / 7.0, 2.0 / 7.0], rel=1e-15)
    assert a4["mean"].tolist() == [0.0, 0.0]
    assert np.all(a4["tie"][:, :2] == 0.0)  # 3.5 and -3.5 lie exactly on ties
    a3 = oracle.quantize_act(X, 4, 3, centering=0, shift=mu)
    assert a3["codes"].tolist() == [[2, -2, -3, 0], [-2, 2, 3, 0]]
    a42 = oracle.quantize_act(X[:1], 4, 4, centering=2, shift=mu, want_Z=True)
    assert a42["Z"].tolist() == [[0.0, -1.0, -2.0, 0.0]]
    assert a42["codes"].tolist() == [[0, -4, -7, 0]]
    assert a42["mean"].tolist() == [0.5]
    W = np.array([_bf16_bits([1.0, 0.0, -1.0, 0.5])], dtype=np.uint16)
    b = np.array(_bf16_bits([0.25]), dtype=np.uint16)
    w = oracle.prepare_weights(W, 4, 4, bias_bits=b, shift=mu)
    assert w["bias"].tolist() == [1.25]
    assert oracle.prepare_weights(W, 4, 4, bias_bits=b)["bias"].tolist() == [0.25]


@pytest.mark.parametrize("K,n,N,T", [(64, 16, 24, 9), (256, 64, 40, 7), (1152, 128, 16, 5)])
@pytest.mark.parametrize("centering", [0, 1, 2])
def test_eq1_identity_with_channel_centring(K, n, N, T, centering):
    """With quantization off the layer is exact: the rotated, centred
    activations times W~ plus the bias (which now carries mu diag(sigma) W)
    plus the per-token mean's correction reproduce X W + b (HadaNorm review
    Eq. (1)), to 1e-10 relative, with any per-token centring on top."""
    g = np.random.default_rng(K + T + centering)
    X = synth.f32_to_bf16_bits((g.standard_normal((T, K)) + g.standard_normal(K) * 3.0)
                               .astype(np.float32))
    W = synth.f32_to_bf16_bits((g.standard_normal((N, K)) * 0.05).astype(np.float32))
    b = synth.f32_to_bf16_bits((g.standard_normal(N) * 0.1).astype(np.float32))
    sig = oracle.sigma(oracle.col_absmax(X), oracle.col_absmax(W), 0.5)
    mu = oracle.channel_mean(X) / sig  # the mean of Y = X diag(sigma^-1)
    a = oracle.quantize_act(X, n, 8, centering=centering, sigma=sig, shift=mu, want_Z=True)
    w = oracle.prepare_weights(W, n, 8, bias_bits=b, sigma=sig, shift=mu, want_Wt=True)
    Z = a["Z"]
    m = a["mean"] if centering else np.zeros(T)
    y = (Z - (m[:, None] if centering == 1 else 0.0)) @ w["Wt"].T + w["bias"][None, :]
    if centering:
        y += m[:, None] * oracle.correction(w, centering)[None, :]
    exact = oracle.exact_linear(X, W, b)
    assert np.linalg.norm(y - exact) <= 1e-10 * np.linalg.norm(exact)


def test_channel_centring_zeroes_every_channel_sum():
    """When mu is the channel mean of the same tokens, every channel of
    Y - mu sums to zero over the tokens, and so does every rotated channel
    of V = (Y - mu) H (H is linear)."""
    g = np.random.default_rng(11)
    X = synth.f32_to_bf16_bits((g.standard_normal((33, 256)) + 2.0).astype(np.float32))
    mu = oracle.channel_mean(X)
    a = oracle.quantize_act(X, 64, 8, centering=0, shift=mu, want_Z=True)
    col = a["Z"].sum(axis=0)
    assert np.max(np.abs(col)) <= 1e-11 * np.max(np.abs(a["Z"])) * 33
    # without the shift the channel sums are far from zero
    a0 = oracle.quantize_act(X, 64, 8, centering=0, want_Z=True)
    assert np.max(np.abs(a0["Z"].sum(axis=0))) > 10.0


# --------------------------------------------------------------------------
# Group-wise int4 with a 16-bit low-rank branch: "Data-free 4-bit quantization
# for diffusion transformers", "Hadamard rotation: the int4 improvement",
# steps 1-7 (W^ = L2 L1 + R; y ~ L2 (L1 x^) + Q(R H) Q(H x^); one H_g block and
# one scale per group of g input channels)
# --------------------------------------------------------------------------

def test_group_wise_hand_worked_example():
    """Worked by hand with g = 4, K = 8, rank 1, sigma = 1, H_4 = H~_4 / 2:
      L1 = [0.5 0.5 0.5 0.5 0 0 0 0], L2 = [2, 0]^T; W row 0 = [1 1 1 1 2 0 0 2],
      row 1 = [0 0 0 0 1 1 1 1]; so R row 0 = [0 0 0 0 2 0 0 2], row 1 = W row 1.
      R H per group: row 0 -> [0 0 0 0 | 2 0 0 2] (group 0 all zero: scale 0),
      row 1 -> [0 0 0 0 | 2 0 0 0]; int4 codes [. | 7 0 0 7] and [. | 7 0 0 0],
      scales 2/7.
      x = [1 2 3 4 1 0 0 1]: x H per group = [5 -1 -2 0 | 1 0 0 1], codes
      rne([7, -1.4, -2.8, 0]) = [7 -1 -3 0] and [7 0 0 7], scales 5/7, 1/7;
      u = L1 x = 0.5 * 10 = 5.
      y0 = (1/7)(2/7)(49 + 49) + 5 * 2 + 0.5 = 14.5 = W0 x + b0 exactly;
      y1 = (1/7)(2/7) 49 - 0.25 = 1.75 = W1 x + b1 exactly."""
    W = np.array([_bf16_bits([1.0, 1.0, 1.0, 1.0, 2.0, 0.0, 0.0, 2.0]),
                  _bf16_bits([0.0, 0.0, 0.0, 0.0, 1.0, 1.0, 1.0, 1.0])], dtype=np.uint16)
    b = np.array(_bf16_bits([0.5]) + [0xBE80], dtype=np.uint16)  # 0.5, -0.25
    X = np.array([_bf16_bits([1.0, 2.0, 3.0, 4.0, 1.0, 0.0, 0.0, 1.0])], dtype=np.uint16)
    L1 = np.array([[0.5, 0.5, 0.5, 0.5, 0.0, 0.0, 0.0, 0.0]])
    L2 = np.array([[2.0], [0.0]])
    out = oracle.layer_gw(X, W, b, g=4, bits=4, rank=1, factors=(L1, L2))
    w, a = out["w"], out["a"]
    assert w["codes"].tolist() == [[0, 0, 0, 0, 7, 0, 0, 7], [0, 0, 0, 0, 7, 0, 0, 0]]
    assert w["gscale"].tolist() == [[0.0, pytest.approx(2 / 7)], [0.0, pytest.approx(2 / 7)]]
    assert a["codes"].tolist() == [[7, -1, -3, 0, 7, 0, 0, 7]]
    assert a["gscale"].tolist() == [[pytest.approx(5 / 7), pytest.approx(1 / 7)]]
    assert oracle.bf16_to_f64(a["u"]).tolist() == [[5.0]]
    assert out["y"].tolist() == [[pytest.approx(14.5, abs=1e-12), pytest.approx(1.75, abs=1e-12)]]


@pytest.mark.parametrize("K,g,N,T,rank", [(128, 64, 16, 5, 4), (256, 16, 24, 3, 0),
                                          (512, 64, 32, 4, 32)])
def test_group_wise_identity_unquantized(K, g, N, T, rank):
    """With the codes replaced by the values they quantize, the form is
    exact: R H times x^ H (H H = I) plus the 16-bit branch's l2 (l1 X) (its
    sum unrounded) plus b reproduces X W^T + b to 1e-10 relative -- whatever
    the factors and sigma, because R is what the rounded factors leave."""
    gen = np.random.default_rng(K + g + rank)
    X = synth.f32_to_bf16_bits((gen.standard_normal((T, K)) * 2).astype(np.float32))
    W = synth.f32_to_bf16_bits((gen.standard_normal((N, K)) * 0.05).astype(np.float32))
    b = synth.f32_to_bf16_bits((gen.standard_normal(N) * 0.1).astype(np.float32))
    sig = oracle.sigma(oracle.col_absmax(X), oracle.col_absmax(W), 0.5)
    L1, L2 = oracle.low_rank_factors(W, sig, rank)
    w = oracle.gw_prepare_weights(W, g, 4, rank, L1, L2, bias_bits=b, sigma=sig, want_Rh=True)
    a = oracle.gw_quantize_act(X, g, 4, rank, w["l1"], sigma=sig, want_Z=True)
    Xf = oracle.bf16_to_f64(X)
    lr = (Xf @ oracle.bf16_to_f64(w["l1"]).T) @ oracle.bf16_to_f64(w["l2"]).T if rank else 0.0
    y = a["Z"] @ w["Rh"].T + lr + w["bias"][None, :]
    exact = oracle.exact_linear(X, W, b)
    assert np.linalg.norm(y - exact) <= 1e-10 * np.linalg.norm(exact)


@pytest.mark.parametrize("bits", [4, 3, 2])
def test_group_quantizer_is_the_token_quantizer_per_group(bits):
    """Brute force over every x in {-2..2}^8 with g = 4: each group's codes
    and scale equal the (independently pinned) per-token quantizer applied to
    that group's 4 values alone (n = K = 4, no centring), at every code width
    the group-wise form takes."""
    vals = np.array(list(itertools.product([-2, -1, 0, 1, 2], repeat=8)), dtype=np.float32)
    X = synth.f32_to_bf16_bits(vals)
    a = oracle.gw_quantize_act(X, 4, bits, 0, None, want_tie=False)
    for j in range(2):
        ref = oracle.quantize_act(np.ascontiguousarray(X[:, 4 * j:4 * j + 4]), 4, bits, gran=0,
                                  centering=0, want_tie=False)
        assert np.array_equal(a["codes"][:, 4 * j:4 * j + 4], ref["codes"])
        assert np.allclose(a["gscale"][:, j], ref["scale"], rtol=1e-15, atol=0)
    assert np.abs(a["codes"]).max() == 2 ** (bits - 1) - 1


def test_group_weight_quantizer_is_the_token_quantizer_per_group():
    """The weight side, brute force over every row in {-2..2}^8 with g = 4 and
    no branch (R = W, sigma = 1): each (row, group) scale and its codes equal
    the per-token quantizer applied to that group's 4 weights alone, at 4 and
    at 3 bits."""
    vals = np.array(list(itertools.product([-2, -1, 0, 1, 2], repeat=8)), dtype=np.float32)
    W = synth.f32_to_bf16_bits(vals)
    for bits in (4, 3):
        w = oracle.gw_prepare_weights(W, 4, bits, 0, None, None, want_tie=False)
        for j in range(2):
            ref = oracle.quantize_act(np.ascontiguousarray(W[:, 4 * j:4 * j + 4]), 4, bits,
                                      gran=0, centering=0, want_tie=False)
            assert np.array_equal(w["codes"][:, 4 * j:4 * j + 4], ref["codes"])
            assert np.allclose(w["gscale"][:, j], ref["scale"], rtol=1e-15, atol=0)


def test_low_rank_factors_are_the_best_rank_r_approximation():
    """L2 L1 from the decomposition equals the truncated SVD of W diag(sigma)
    (Eckart-Young: the residual's Frobenius norm is the root of the sum of
    the dropped squared singular values)."""
    gen = np.random.default_rng(3)
    W = synth.f32_to_bf16_bits(gen.standard_normal((48, 96)).astype(np.float32))
    sig = np.exp(gen.standard_normal(96) * 0.3)
    L1, L2 = oracle.low_rank_factors(W, sig, 8)
    What = oracle.bf16_to_f64(W) * sig[None, :]
    s = np.linalg.svd(What, compute_uv=False)
    assert np.isclose(np.linalg.norm(What - L2 @ L1), np.sqrt(np.sum(s[8:] ** 2)), rtol=1e-10)
    assert np.allclose(L1 @ L1.T, np.eye(8), atol=1e-12)  # orthonormal rows


def test_group_wise_inputs_of_the_wrong_shape_are_refused():
    """The C side reads exactly the shapes the description implies: the
    wrappers refuse factors, sigma or l1 of any other shape (a rank above
    min(N, K) is zero-padded by low_rank_factors, not truncated)."""
    W = synth.f32_to_bf16_bits(np.ones((4, 8), dtype=np.float32))
    L1, L2 = oracle.low_rank_factors(W, None, 6)  # rank 6 > min(N, K) = 4
    assert L1.shape == (6, 8) and L2.shape == (4, 6)
    assert np.all(L1[4:] == 0) and np.all(L2[:, 4:] == 0)
    with pytest.raises(ValueError):
        oracle.gw_prepare_weights(W, 4, 4, 6, L1[:4], L2)
    with pytest.raises(ValueError):
        oracle.gw_prepare_weights(W, 4, 4, 6, L1, L2[:, :4])
    with pytest.raises(ValueError):
        oracle.gw_prepare_weights(W, 4, 4, 6, L1, L2, sigma=np.ones(7))
    X = synth.f32_to_bf16_bits(np.ones((2, 8), dtype=np.float32))
    with pytest.raises(ValueError):
        oracle.gw_quantize_act(X, 4, 4, 2, np.zeros((3, 8), dtype=np.uint16))
