"""GPU parity of the group-wise 4-bit form with the 16-bit low-rank branch
(include/hq_gw.h) against the oracle's group-wise functions, element by
element on the same seeded inputs.  Needs a B200."""
import numpy as np
import pytest

import oracle
import synth
from parity import Y_REL_FROB, bf16_bits, check_codes, check_rel, rel_frob, to_dev_u16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

A_SCALE_RTOL = 1e-6


def _check_w_scales(gpu, ref, W, sig, what="weight scales"):
    """R = (W - l2 l1) sigma is formed in fp32, where W - l2 l1 cancels when the
    branch carries most of W: each element is off by a few units of 2^-24 of
    |W sigma|, and max |R H| over a group by at most 8 times that (64 terms,
    1/8).  So |ds| <= 1e-6 s + 2^-18 max_group |W sigma| / q."""
    Wf = oracle.bf16_to_f64(W) * (1.0 if sig is None else sig[None, :])
    N, K = Wf.shape
    gmax = np.abs(Wf).reshape(N, K // 64, 64).max(axis=2)
    tol = 1e-6 * np.abs(ref) + 2.0 ** -18 * gmax
    bad = np.abs(np.asarray(gpu, dtype=np.float64) - ref) > tol
    assert not bad.any(), f"{what}: {int(bad.sum())} outside the fp32 bound"


@pytest.fixture(scope="module")
def hq():
    import hadamard_rotated_bit_token_b200 as hq_mod
    from hadamard_rotated_bit_token_b200 import build as hq_build
    hq_build.build()
    hq_mod.load_library()
    return hq_mod


def _inputs(T, K, N, seed, outliers=True):
    """X ~ N(0,1) with a few channels x30 and a per-token offset (the DiT
    activation recipe), W ~ N(0, 0.02), b ~ N(0, 0.01), all bf16 bits."""
    g = np.random.default_rng(seed)
    x = g.standard_normal((T, K)).astype(np.float32)
    if outliers:
        x[:, g.choice(K, size=max(1, K // 100), replace=False)] *= 30.0
    x += (g.standard_normal((T, 1)) * 1.5).astype(np.float32)
    w = (g.standard_normal((N, K)) * 0.02).astype(np.float32)
    b = (g.standard_normal(N) * 0.01).astype(np.float32)
    return synth.f32_to_bf16_bits(x), synth.f32_to_bf16_bits(w), synth.f32_to_bf16_bits(b)


def _sigma(X, W, use_sigma):
    """sigma from the oracle's Eq. (3), handed to the GPU as fp32 sigma^-1;
    the oracle then uses exactly the sigma that fp32 value stands for."""
    if not use_sigma:
        return None, None
    s = oracle.sigma(oracle.col_absmax(X), oracle.col_absmax(W), 0.5)
    si = (1.0 / s).astype(np.float32)
    return si, 1.0 / si.astype(np.float64)


def _factors(W, sig, rank):
    """Rank-r factors of W diag(sigma) (fp64 SVD), rounded to fp32: both sides
    get the same fp32 values."""
    L1, L2 = oracle.low_rank_factors(W, sig, rank)
    return L1.astype(np.float32), L2.astype(np.float32)


def _dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t if dtype is None else t.to(dtype)


def _codes_int(t):
    """e4m3 code bytes -> integer codes (every value must be an integer)."""
    v = t.float().cpu().numpy()
    assert np.all(v == np.round(v)), "a code is not an integer"
    return v.astype(np.int16)


def _gpu_prepare(hq, desc, W, b, si, L1, L2):
    K, N, r = desc.K, desc.N, desc.rank
    w_codes = torch.full((N, K), 100.0, device="cuda").to(torch.float8_e4m3fn)  # poison
    w_scale = torch.full((K // 64, N), float("nan"), device="cuda")
    l1s = torch.empty((r, K), dtype=torch.bfloat16, device="cuda") if r else None
    l2b = torch.empty((N, r), dtype=torch.bfloat16, device="cuda") if r else None
    bias_f32 = torch.full((N,), float("nan"), device="cuda")
    hq.hq_gw_prepare_weights(desc, to_dev_u16(W, torch), None if b is None else to_dev_u16(b, torch),
                             None if si is None else _dev(si),
                             _dev(L1) if r else None, _dev(L2) if r else None,
                             w_codes, w_scale, l1s, l2b, bias_f32)
    assert hq.hq_check_device_error() == 0
    return {"codes": w_codes, "scale": w_scale, "l1s": l1s, "l2b": l2b, "bias": bias_f32}


def _gpu_quantize(hq, desc, X, si, l1s, workspace=True):
    """workspace: give the call the workspace that lets small batches split
    each token block over two CTAs (poisoned, since the call must not rely
    on its contents)."""
    T, K = X.shape
    r = desc.rank
    ld = hq.hq_gw_scale_ld(T)
    a_codes = torch.full((T, K), 100.0, device="cuda").to(torch.float8_e4m3fn)
    a_scale = torch.full((K // 64, ld), float("nan"), device="cuda")
    u = torch.full((T, r), float("nan"), dtype=torch.bfloat16, device="cuda") if r else None
    ws = None
    nbytes = hq.hq_gw_quantize_act_workspace_bytes(desc, T)
    if workspace and nbytes:
        ws = torch.full((nbytes,), 0x7F, dtype=torch.uint8, device="cuda")
    Xd = to_dev_u16(X, torch)
    hq.hq_gw_quantize_act(desc, Xd, None if si is None else _dev(si), l1s, a_codes, a_scale, u,
                          ws)
    assert hq.hq_check_device_error() == 0
    return {"codes": a_codes, "scale": a_scale, "u": u, "X": Xd}


def _oracle(X, W, b, sig, L1, L2, rank, bits_a, bits_w, rows=None):
    w = oracle.gw_prepare_weights(W, 64, bits_w, rank, L1.astype(np.float64),
                                  L2.astype(np.float64), bias_bits=b, sigma=sig)
    a = oracle.gw_quantize_act(X, 64, bits_a, rank, w["l1"], sigma=sig, rows=rows)
    y, yb = oracle.gw_epilogue(a["codes"], w["codes"], 64, a["gscale"], w["gscale"],
                               a["u"] if rank else None, w["l2"] if rank else None, bias=w["bias"])
    return w, a, y, yb


def _check_u(u_gpu, X, l1_bits, what="u"):
    """u = bf16 of a tensor-core fp32 sum of K products against the exact sum
    u64 (fp64 of the same bf16 inputs): within the bf16 rounding of u64 plus
    the accumulation error, 2^-20 of sum_k |X_k l1_k| (a margin over K * 2^-24
    for K <= 16384), which dominates where the terms cancel; and in most
    places the bf16 of the exact sum itself."""
    Xf = oracle.bf16_to_f64(X)
    Lf = oracle.bf16_to_f64(l1_bits)
    u64 = Xf @ Lf.T
    mag = np.abs(Xf) @ np.abs(Lf).T
    g = synth.bf16_bits_to_f32(u_gpu).astype(np.float64)
    tol = 2.0 ** -8 * np.abs(u64) + 2.0 ** -20 * mag
    bad = np.abs(g - u64) > tol
    assert not bad.any(), f"{what}: {int(bad.sum())} values outside the fp32 accumulation bound"
    same = np.mean(u_gpu == oracle.f64_to_bf16(u64))
    assert same >= 0.98, f"{what}: only {same:.4f} equal to bf16 of the exact sum"


CASES = [
    # T, K, N, rank, bits_a, bits_w, use_sigma
    (1, 64, 16, 32, 4, 4, True),
    (7, 128, 48, 0, 4, 4, False),
    (129, 256, 272, 32, 4, 4, True),
    (300, 1152, 512, 32, 4, 4, True),
    (200, 576, 256, 0, 3, 4, True),
    (130, 1024, 528, 32, 3, 4, False),
    (257, 2048, 784, 32, 4, 3, True),
    (96, 512, 80, 32, 2, 2, True),  # 2-bit codes on both sides
    (64, 64 * 65, 32, 32, 4, 4, True),
    (130, 16384, 48, 32, 4, 4, True),  # the largest K (sigma^-1 takes 64 KB of shared memory)
]


@pytest.mark.parametrize("T,K,N,rank,bits_a,bits_w,use_sigma", CASES)
def test_gw_layer_matches_oracle(hq, T, K, N, rank, bits_a, bits_w, use_sigma):
    X, W, b = _inputs(T, K, N, seed=T * 7 + K + N)
    si, sig = _sigma(X, W, use_sigma)
    L1, L2 = _factors(W, sig, rank)
    desc = hq.GwDesc(K, N, 64, rank, bits_a, bits_w)
    w_ref, a_ref, y_ref, yb_ref = _oracle(X, W, b, sig, L1, L2, rank, bits_a, bits_w)

    wp = _gpu_prepare(hq, desc, W, b, si, L1, L2)
    if rank:
        assert np.array_equal(bf16_bits(wp["l1s"]), w_ref["l1"]), "l1 (bf16) differs"
        assert np.array_equal(bf16_bits(wp["l2b"]), w_ref["l2"]), "l2 (bf16) differs"
    check_codes(_codes_int(wp["codes"]), w_ref["codes"], w_ref["tie"], "weight codes")
    _check_w_scales(wp["scale"].cpu().numpy().T, w_ref["gscale"], W, sig)
    check_rel(wp["bias"].cpu().numpy(), w_ref["bias"], 0.0, "bias")

    ap = _gpu_quantize(hq, desc, X, si, wp["l1s"])
    check_codes(_codes_int(ap["codes"]), a_ref["codes"], a_ref["tie"], "activation codes")
    ld = hq.hq_gw_scale_ld(T)
    check_rel(ap["scale"].cpu().numpy()[:, :T].T, a_ref["gscale"], A_SCALE_RTOL,
              "activation scales")
    assert ld % 4 == 0 and ld >= T
    if rank:
        _check_u(bf16_bits(ap["u"]), X, w_ref["l1"])

    Y = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    hq.hq_gw_linear(desc, ap["codes"], ap["scale"], ap["u"], wp["codes"], wp["scale"], wp["l2b"],
                    wp["bias"], Y)
    assert hq.hq_check_device_error() == 0
    err = rel_frob(bf16_bits(Y), yb_ref)
    assert err <= Y_REL_FROB, f"output relative Frobenius error {err:.3g}"


@pytest.mark.parametrize("T,K,N,rank", [(129, 256, 272, 0), (300, 1152, 512, 32), (1, 64, 16, 32)])
def test_gw_gemm_exact_sums_on_the_oracles_codes(hq, T, K, N, rank):
    """The GEMM fed the oracle's codes with unit scales returns the exact
    integer sums (every partial sum is an integer below 2^24), and with the
    oracle's scales, u, l2 and bias it matches the oracle's fp64 epilogue to
    fp32 accuracy."""
    X, W, b = _inputs(T, K, N, seed=K + N + rank)
    si, sig = _sigma(X, W, True)
    L1, L2 = _factors(W, sig, rank)
    w_ref, a_ref, y_ref, _ = _oracle(X, W, b, sig, L1, L2, rank, 4, 4)
    desc = hq.GwDesc(K, N, 64, rank, 4, 4)
    G = K // 64
    ld = hq.hq_gw_scale_ld(T)
    A = _dev(a_ref["codes"].astype(np.float32)).to(torch.float8_e4m3fn)
    B = _dev(w_ref["codes"].astype(np.float32)).to(torch.float8_e4m3fn)
    ones_a = torch.ones((G, ld), device="cuda")
    ones_w = torch.ones((G, N), device="cuda")
    Y32 = torch.full((T, N), float("nan"), device="cuda")
    d0 = hq.GwDesc(K, N, 64, 0, 4, 4)
    hq.hq_gw_debug_linear_f32(d0, A, ones_a, None, B, ones_w, None, None, Y32)
    assert hq.hq_check_device_error() == 0
    exact = a_ref["codes"].astype(np.int64) @ w_ref["codes"].astype(np.int64).T
    assert np.array_equal(Y32.cpu().numpy().astype(np.int64), exact), "integer sums differ"

    sa = np.zeros((G, ld), dtype=np.float32)
    sa[:, :T] = a_ref["gscale"].T
    u = to_dev_u16(a_ref["u"], torch) if rank else None
    l2 = to_dev_u16(w_ref["l2"], torch) if rank else None
    hq.hq_gw_debug_linear_f32(desc, A, _dev(sa), u, B, _dev(w_ref["gscale"].T.astype(np.float32)),
                              l2, _dev(w_ref["bias"].astype(np.float32)), Y32)
    assert hq.hq_check_device_error() == 0
    y32 = Y32.cpu().numpy().astype(np.float64)
    # fp32 rounding of the scales (2^-24 each) and of G + rank + 1 running sums
    mag = np.abs(a_ref["gscale"]) @ (np.abs(w_ref["gscale"]) * 64 * 49).T
    if rank:
        mag += np.abs(oracle.bf16_to_f64(a_ref["u"])) @ np.abs(oracle.bf16_to_f64(w_ref["l2"])).T
    mag += np.abs(w_ref["bias"])[None, :]
    assert np.all(np.abs(y32 - y_ref) <= 8 * (G + rank + 2) * 2.0 ** -24 * mag)


def test_gw_zero_tokens_and_zero_groups(hq):
    """T = 0 is a no-op; an all-zero group gets scale 0 and zero codes, and a
    zero input row gives the bias alone."""
    K, N = 256, 32
    X, W, b = _inputs(3, K, N, seed=5, outliers=False)
    X[1, :] = 0
    X[2, 64:128] = 0
    desc = hq.GwDesc(K, N, 64, 32, 4, 4)
    L1, L2 = _factors(W, None, 32)
    wp = _gpu_prepare(hq, desc, W, b, None, L1, L2)
    spare = torch.full((64,), 7.0, dtype=torch.float32, device="cuda")  # never written for T = 0
    hq.hq_gw_quantize_act(desc, spare, None, wp["l1s"], spare, spare, spare, T=0)
    assert hq.hq_gw_quantize_act_workspace_bytes(desc, 0) == 0
    assert hq.hq_gw_quantize_act_workspace_bytes(hq.GwDesc(K, N, 64, 0, 4, 4), 1000) == 0
    hq.hq_gw_linear(desc, spare, spare, spare, wp["codes"], wp["scale"], wp["l2b"], wp["bias"],
                    spare, T=0)
    torch.cuda.synchronize()
    assert torch.all(spare == 7.0)
    ap = _gpu_quantize(hq, desc, X, None, wp["l1s"])
    codes = _codes_int(ap["codes"])
    sc = ap["scale"].cpu().numpy()
    assert np.all(codes[1] == 0) and np.all(sc[:, 1] == 0)
    assert np.all(codes[2, 64:128] == 0) and sc[1, 2] == 0
    Y = torch.empty((3, N), dtype=torch.bfloat16, device="cuda")
    hq.hq_gw_linear(desc, ap["codes"], ap["scale"], ap["u"], wp["codes"], wp["scale"], wp["l2b"],
                    wp["bias"], Y)
    assert hq.hq_check_device_error() == 0
    bias = synth.bf16_bits_to_f32(b)
    y1 = synth.bf16_bits_to_f32(bf16_bits(Y)[1])
    assert np.array_equal(y1, synth.bf16_bits_to_f32(oracle.f64_to_bf16(bias.astype(np.float64))))


def test_gw_layer_module(hq):
    """GroupWiseQuantLinear (sigma on the device, factors from the device SVD)
    against the oracle given the module's sigma and fp32 factors."""
    T, K, N = 257, 1152, 528
    X, W, b = _inputs(T, K, N, seed=11)
    act = torch.from_numpy(oracle.col_absmax(X).astype(np.float32)).cuda()
    desc = hq.GwDesc(K, N, 64, 32, 4, 4)
    layer = hq.GroupWiseQuantLinear(desc, to_dev_u16(W, torch), to_dev_u16(b, torch), act, 0.5)
    Y = layer(to_dev_u16(X, torch))
    assert hq.hq_check_device_error() == 0
    si = layer.sigma_inv.cpu().numpy()
    sig = 1.0 / si.astype(np.float64)
    s_ref = oracle.sigma(oracle.col_absmax(X), oracle.col_absmax(W), 0.5)
    check_rel(si, 1.0 / s_ref, 1e-6, "sigma_inv")
    L1, L2 = (f.cpu().numpy() for f in layer.factors)
    w_ref, a_ref, y_ref, yb_ref = _oracle(X, W, b, sig, L1, L2, 32, 4, 4)
    assert np.array_equal(bf16_bits(layer.l1s), w_ref["l1"])
    check_codes(_codes_int(layer.w_codes), w_ref["codes"], w_ref["tie"], "module weight codes")
    bufs = layer.buffers(T)
    check_codes(_codes_int(bufs["a_codes"]), a_ref["codes"], a_ref["tie"], "module codes")
    _check_u(bf16_bits(bufs["u"]), X, w_ref["l1"], "module u")
    err = rel_frob(bf16_bits(Y), yb_ref)
    assert err <= Y_REL_FROB, f"module output relative Frobenius error {err:.3g}"
    # W4A4 with smoothing and the branch stays within 25 % of the exact layer
    exact = oracle.exact_linear(X, W, b)
    assert np.linalg.norm(y_ref - exact) <= 0.25 * np.linalg.norm(exact)


@pytest.mark.parametrize("cfg_index", [2, 5])
def test_gw_full_layer_sampled_rows(hq, cfg_index):
    """The PixArt-Sigma qkv layer (T = 8192, K = 1152, N = 3456) and the large
    DiT linear (T = 16384, K = 3072, N = 12288) in the group-wise form with
    rank 32: the GPU computes every row; the oracle computes the weights in
    full and the activations and outputs of sampled rows (first and last
    tiles included)."""
    cfg = synth.CONFIGS[cfg_index]
    X, W, b = synth.make_layer(cfg)
    T, K, N = X.shape[0], X.shape[1], W.shape[0]
    si, sig = _sigma(X, W, True)
    L1, L2 = _factors(W, sig, 32)
    rows = synth.sample_rows(T, 12, seed=3)
    w_ref, a_ref, y_ref, yb_ref = _oracle(X, W, b, sig, L1, L2, 32, 4, 4, rows=rows)
    desc = hq.GwDesc(K, N, 64, 32, 4, 4)
    wp = _gpu_prepare(hq, desc, W, b, si, L1, L2)
    assert np.array_equal(bf16_bits(wp["l1s"]), w_ref["l1"])
    check_codes(_codes_int(wp["codes"]), w_ref["codes"], w_ref["tie"], "weight codes",
                min_match=0.9999)
    ap = _gpu_quantize(hq, desc, X, si, wp["l1s"])
    check_codes(_codes_int(ap["codes"])[rows], a_ref["codes"], a_ref["tie"], "activation codes",
                min_match=0.9999)
    check_rel(ap["scale"].cpu().numpy()[:, rows].T, a_ref["gscale"], A_SCALE_RTOL, "scales")
    _check_u(bf16_bits(ap["u"])[rows], X[rows], w_ref["l1"])
    Y = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    hq.hq_gw_linear(desc, ap["codes"], ap["scale"], ap["u"], wp["codes"], wp["scale"], wp["l2b"],
                    wp["bias"], Y)
    assert hq.hq_check_device_error() == 0
    err = rel_frob(bf16_bits(Y)[rows], yb_ref)
    assert err <= Y_REL_FROB, f"output relative Frobenius error {err:.3g}"


def test_gw_wait_timeout_is_reported(hq):
    """The fault hook withholds the first X tile of the activation kernel: its
    bounded waits run out, the kernel returns and the error word says so; the
    context stays usable."""
    K, N, T = 256, 32, 130
    X, W, b = _inputs(T, K, N, seed=9)
    desc = hq.GwDesc(K, N, 64, 32, 4, 4)
    L1, L2 = _factors(W, None, 32)
    wp = _gpu_prepare(hq, desc, W, b, None, L1, L2)
    hq.hq_debug_set_wait_limit(20_000_000)  # 20 ms
    hq.hq_debug_inject_fault(hq.HQ_FAULT_QUANT_WITHHOLD_ROW)
    try:
        a_codes = torch.empty((T, K), dtype=torch.float8_e4m3fn, device="cuda")
        a_scale = torch.empty((K // 64, hq.hq_gw_scale_ld(T)), device="cuda")
        u = torch.empty((T, 32), dtype=torch.bfloat16, device="cuda")
        hq.hq_gw_quantize_act(desc, to_dev_u16(X, torch), None, wp["l1s"], a_codes, a_scale, u)
        torch.cuda.synchronize()
        assert hq.hq_check_device_error() == 5  # HQ_ERR_TIMEOUT, blocks whole
        ws = torch.empty(hq.hq_gw_quantize_act_workspace_bytes(desc, T), dtype=torch.uint8,
                         device="cuda")
        hq.hq_gw_quantize_act(desc, to_dev_u16(X, torch), None, wp["l1s"], a_codes, a_scale, u,
                              ws)
        torch.cuda.synchronize()
        assert hq.hq_check_device_error() == 5  # HQ_ERR_TIMEOUT
    finally:
        hq.hq_debug_inject_fault(hq.HQ_FAULT_NONE)
        hq.hq_debug_set_wait_limit(0)
    assert hq.hq_check_device_error() == 0
    ap = _gpu_quantize(hq, desc, X, None, wp["l1s"])
    assert _codes_int(ap["codes"]).shape == (T, K)


@pytest.mark.parametrize("T,K,rank", [(300, 1152, 32), (8192, 1152, 32), (129, 256, 0)])
def test_gw_split_blocks_match_whole_blocks(hq, T, K, rank):
    """With a workspace, small batches split each 128-token block's groups
    over two CTAs: codes and scales are identical to the unsplit call, and u
    (its fp32 sum taken in two parts) meets the same bound as the unsplit u."""
    N = 64
    X, W, b = _inputs(T, K, N, seed=T + K)
    si, sig = _sigma(X, W, True)
    L1, L2 = _factors(W, sig, rank)
    desc = hq.GwDesc(K, N, 64, rank, 4, 4)
    wp = _gpu_prepare(hq, desc, W, b, si, L1, L2)
    whole = _gpu_quantize(hq, desc, X, si, wp["l1s"], workspace=False)
    split = _gpu_quantize(hq, desc, X, si, wp["l1s"], workspace=True)
    assert torch.equal(whole["codes"].view(torch.uint8), split["codes"].view(torch.uint8))
    assert torch.equal(whole["scale"][:, :T], split["scale"][:, :T])
    if rank:
        # both within the fp32 accumulation bound of the exact sum (a value
        # near zero may change sign between the two summation orders)
        _check_u(bf16_bits(whole["u"]), X, bf16_bits(wp["l1s"]), "u, whole blocks")
        _check_u(bf16_bits(split["u"]), X, bf16_bits(wp["l1s"]), "u, split blocks")
