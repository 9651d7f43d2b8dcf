"""GPU parity: the sm_100a kernels (through the C ABI) against the CPU oracle,
element by element on the same seeded inputs.  Needs a B200."""
import numpy as np
import pytest

import oracle
import synth
from parity import (CODE_MATCH_MIN, SCALE_RTOL, TIE_TOL, Y_REL_FROB, bf16_bits, check_codes,
                    check_rel, rel_frob, to_dev_u16)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def hq():
    import hadamard_rotated_bit_token_b200 as hq_mod
    from hadamard_rotated_bit_token_b200 import build as hq_build
    hq_build.build()
    hq_mod.load_library()
    return hq_mod


def _sigma_case(K, seed):
    g = np.random.default_rng(seed)
    return 10.0 ** g.uniform(-0.7, 0.7, size=K)


def _gpu_quantize(hq, desc, X_bits, sigma_inv_f32=None, static_scale=None):
    T, K = X_bits.shape
    X = to_dev_u16(X_bits, torch)
    codes = torch.full((T, K), 0x55, dtype=torch.int8, device="cuda")  # poison
    per_row = desc.act_gran == hq.HQ_PER_TOKEN
    scale = torch.full((T if per_row else 1,), float("nan"), dtype=torch.float32, device="cuda")
    if static_scale is not None:
        scale.fill_(static_scale)
    mean = torch.full((T,), float("nan"), dtype=torch.float32, device="cuda")
    si = None if sigma_inv_f32 is None else torch.from_numpy(sigma_inv_f32).cuda()
    ws_bytes = hq.hq_quantize_act_workspace_bytes(desc, T)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda") if ws_bytes else None
    hq.hq_quantize_act(desc, X, si, codes, scale, mean, ws)
    assert hq.hq_check_device_error() == 0
    return codes.cpu().numpy(), scale.cpu().numpy().astype(np.float64), mean.cpu().numpy()


def _check_act(ref, codes, scale, mean, per_row=True, min_match=None, what="act"):
    check_codes(codes, ref["codes"], ref["tie"], what + " codes", min_match=min_match)
    if per_row:
        check_rel(scale, ref["scale"], SCALE_RTOL, what + " scale")
    else:
        check_rel(scale[:1], ref["scale"][:1], SCALE_RTOL, what + " tensor scale")
    if ref["Z"] is not None:
        tol = 1e-6 * (np.mean(np.abs(ref["Z"]), axis=1) + np.abs(ref["mean"])) + 1e-30
        assert np.all(np.abs(mean - ref["mean"]) <= tol), what + " mean"


# ---------------------------------------------------------------------------
# activation quantizer, small shapes spanning several tiles and ragged tails
# ---------------------------------------------------------------------------

SMALL = []
# K below 1024 (several rows per warp), K = 1024 .. 4096 in whole warps of
# slices (one row per warp, one to four slices a lane), and other K (rows
# spanning warps)
for i, (n, B) in enumerate([(16, 4), (16, 12), (32, 2), (32, 6), (64, 1), (64, 5), (128, 1),
                            (128, 9), (256, 1), (256, 3), (512, 2), (1024, 1), (1024, 3),
                            (16, 128), (128, 16), (1024, 2), (64, 64), (256, 16), (512, 8),
                            (1024, 5)]):
    for T in (1, 7, 129, 300):
        bits = (4, 3, 8)[(i + T) % 3]
        SMALL.append((n * B, n, T, bits, (i + T) % 2, (i % 3) != 0))


# the mean removed before the rotation (HQ_CENTER_TOKEN_MEAN_PRE), every order
SMALL_PRE = [(n * B, n, T, (4, 3, 8)[i % 3], 2, i % 2 == 0)
             for i, (n, B, T) in enumerate([(16, 4, 129), (32, 6, 7), (64, 5, 300), (128, 9, 129),
                                            (256, 3, 300), (512, 2, 7), (1024, 3, 129),
                                            (128, 16, 129), (1024, 4, 7), (1024, 5, 129)])]


# K a multiple of 16 but not of 32 (n = 16: the row's last slice holds 16
# channels), and rows longer than 8192 channels
SMALL_ENVELOPE = [(80, 16, T, 4, c, True) for T, c in ((1, 0), (7, 1), (300, 2))] + \
                 [(144, 16, 129, 3, 1, False), (16 * 27, 16, 65, 8, 0, True)] + \
                 [(12288, n, T, 4, c, True) for n, T, c in ((1024, 7, 1), (256, 33, 2),
                                                           (128, 3, 0))]

# rows of 75-160 slices over enough tokens that the launch plan takes the
# one-CTA segment variant (three rows a tile) or wider two-CTA tiles
SMALL_PLAN = [(4608, 256, 1000, 3, 1, True), (4608, 256, 1000, 4, 2, False),
              (2400, 32, 4000, 4, 1, True), (2816, 256, 700, 8, 0, True)]


@pytest.mark.parametrize("K,n,T,bits,center,use_sigma",
                         SMALL + SMALL_PRE + SMALL_ENVELOPE + SMALL_PLAN)
def test_quantize_small(hq, K, n, T, bits, center, use_sigma):
    g = np.random.default_rng(K * 1000 + T)
    x = g.standard_normal((T, K)).astype(np.float32)
    x[:, g.choice(K, size=max(1, K // 64), replace=False)] *= 30.0
    x += g.standard_normal((T, 1)).astype(np.float32) * 2.0
    X = synth.f32_to_bf16_bits(x)
    sigma = _sigma_case(K, T) if use_sigma else None
    ref = oracle.quantize_act(X, n, bits, gran=0, centering=center, sigma=sigma, want_Z=True)
    desc = hq.LayerDesc(K, 16, n, a_bits=bits, w_bits=4, act_gran=hq.HQ_PER_TOKEN,
                        centering=center)
    si = None if sigma is None else (1.0 / sigma).astype(np.float32)
    codes, scale, mean = _gpu_quantize(hq, desc, X, si)
    _check_act(ref, codes, scale, mean)
    if not center:
        assert np.all(mean == 0.0)


@pytest.mark.parametrize("gran", [1, 2])
@pytest.mark.parametrize("K,n,T,center", [(320, 64, 300, 0), (256, 256, 129, 1), (1024, 1024, 77, 0),
                                            (1152, 128, 200, 2)])
def test_quantize_per_tensor(hq, gran, K, n, T, center):
    cfg = synth.CONFIGS[4]
    g = np.random.default_rng(K + T)
    x = (g.laplace(0, 1, size=(T, K)) * 10.0 ** g.uniform(-1, 1, size=K)).astype(np.float32)
    X = synth.f32_to_bf16_bits(x)
    dyn = oracle.quantize_act(X, n, 8, gran=1, centering=center, want_Z=True)
    desc = hq.LayerDesc(K, 16, n, a_bits=8, w_bits=8, act_gran=gran, centering=center)
    if gran == 1:
        codes, scale, mean = _gpu_quantize(hq, desc, X)
        _check_act(dyn, codes, scale, mean, per_row=False)
    else:
        s32 = float(np.float32(dyn["scale"][0] * 0.75))  # a scale that forces clamping
        ref = oracle.quantize_act(X, n, 8, gran=2, centering=center, static_scale=s32, want_Z=True)
        codes, scale, mean = _gpu_quantize(hq, desc, X, static_scale=s32)
        check_codes(codes, ref["codes"], ref["tie"], "static codes")
        assert np.abs(codes).max() == 127
    del cfg


def test_exact_ties_are_rounded_half_to_even(hq):
    """Dyadic rows whose centred rotated values sit exactly on rounding ties;
    both sides compute them exactly, so the codes must agree bit for bit."""
    n, K, T, bits = 64, 128, 32, 3
    H = np.ones((1, 1))
    for _ in range(6):
        H = np.kron(H, np.array([[1.0, 1.0], [1.0, -1.0]]))
    Hn = np.kron(np.eye(K // n), H / 8.0)
    g = np.random.default_rng(7)
    rows = []
    for t in range(T):
        V = np.zeros(K)
        pos = g.choice(K, size=6, replace=False)
        vals = [3.0, g.choice([0.5, 1.5, 2.5]), g.choice([0.5, 1.5, 2.5])]
        for j, v in enumerate(vals):
            V[pos[2 * j]] = v
            V[pos[2 * j + 1]] = -v
        m = [0.0, 0.25, -0.5][t % 3]
        rows.append((V + m) @ Hn.T)
    xf = np.array(rows)
    X = synth.f32_to_bf16_bits(xf.astype(np.float32))
    assert np.array_equal(synth.bf16_bits_to_f32(X).astype(np.float64), xf)
    ref = oracle.quantize_act(X, n, bits, gran=0, centering=1, want_Z=True)
    assert np.sum(ref["tie"] == 0.0) >= 4 * T  # many exact ties
    desc = hq.LayerDesc(K, 16, n, a_bits=bits, act_gran=hq.HQ_PER_TOKEN, centering=1)
    codes, scale, mean = _gpu_quantize(hq, desc, X)
    assert np.array_equal(codes, ref["codes"])
    assert np.array_equal(scale, ref["scale"])


# ---------------------------------------------------------------------------
# weight preparation
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("N,K,n,w_bits,use_sigma,center",
                         [(48, 64, 16, 4, True, 1), (160, 256, 64, 8, True, 1),
                          (64, 1152, 128, 4, True, 1), (32, 3072, 1024, 4, True, 1),
                          (320, 320, 64, 8, False, 0), (1024, 1024, 1024, 4, True, 1),
                          (64, 1152, 128, 4, True, 2), (48, 512, 16, 8, False, 2),
                          (32, 3072, 1024, 4, True, 2),
                          # K a multiple of 16 only (n = 16), and K above 8192
                          (48, 80, 16, 4, True, 1), (32, 144, 16, 8, True, 2),
                          (16, 12288, 1024, 4, True, 1), (16, 12288, 256, 4, True, 2),
                          (32, 4096, 512, 4, True, 1), (32, 2048, 64, 8, False, 0)])
def test_prepare_weights(hq, N, K, n, w_bits, use_sigma, center):
    g = np.random.default_rng(N + K)
    Xb = synth.f32_to_bf16_bits(g.standard_normal((64, K)).astype(np.float32) *
                                (1 + 20 * (g.random(K) < 0.02)).astype(np.float32))
    Wb = synth.f32_to_bf16_bits(g.standard_normal((N, K)).astype(np.float32) * 0.02)
    bb = synth.f32_to_bf16_bits(g.standard_normal(N).astype(np.float32) * 0.01)
    sig = oracle.sigma(oracle.col_absmax(Xb), oracle.col_absmax(Wb), 0.5) if use_sigma else None
    ref = oracle.prepare_weights(Wb, n, w_bits, bias_bits=bb, sigma=sig, want_Wt=True)
    desc = hq.LayerDesc(K, N, n, a_bits=4, w_bits=w_bits, centering=center)
    X = to_dev_u16(Xb, torch)
    W = to_dev_u16(Wb, torch)
    b = to_dev_u16(bb, torch)
    absmax = None
    if use_sigma:
        absmax = torch.zeros(K, dtype=torch.float32, device="cuda")
        hq.hq_calib_act_absmax(desc, X, absmax)
        assert np.array_equal(absmax.cpu().numpy().astype(np.float64), oracle.col_absmax(Xb))
    w_codes = torch.full((N, K), 0x55, dtype=torch.int8, device="cuda")
    w_scale = torch.empty(N, dtype=torch.float32, device="cuda")
    colsum = torch.empty(N, dtype=torch.float32, device="cuda")
    sigma_inv = torch.empty(K, dtype=torch.float32, device="cuda")
    bias_f32 = torch.empty(N, dtype=torch.float32, device="cuda")
    hq.hq_prepare_weights(desc, W, b, absmax, 0.5, w_codes, w_scale, colsum, sigma_inv, bias_f32)
    assert hq.hq_check_device_error() == 0
    if use_sigma:
        check_rel(sigma_inv.cpu().numpy(), 1.0 / sig, SCALE_RTOL, "sigma_inv")
    else:
        assert np.all(sigma_inv.cpu().numpy() == 1.0)
    check_codes(w_codes.cpu().numpy(), ref["codes"], ref["tie"], "w_codes")
    check_rel(w_scale.cpu().numpy(), ref["scale"], SCALE_RTOL, "w_scale")
    if center == 2:   # sum_k sigma_k W[n,k]: bound by the sum of its terms' magnitudes
        sw = synth.bf16_bits_to_f32(Wb).astype(np.float64) * (sig if sig is not None else 1.0)
        tol = 1e-6 * np.abs(sw).sum(axis=1)
    else:
        tol = 1e-6 * np.abs(ref["Wt"]).sum(axis=1)
    want = oracle.correction(ref, center)
    assert np.all(np.abs(colsum.cpu().numpy() - want) <= tol), "colsum"
    assert np.array_equal(bias_f32.cpu().numpy().astype(np.float64), ref["bias"])


# ---------------------------------------------------------------------------
# integer GEMM: bit-exact accumulators, epilogue
# ---------------------------------------------------------------------------

GEMM_SHAPES = [(1, 16, 32), (127, 48, 160), (128, 192, 128), (129, 320, 320), (300, 512, 1152),
               (256, 1024, 1024), (200, 3456, 256), (131, 160, 4608), (513, 64, 96)]


@pytest.fixture(params=["single_cta", "cta_pair"])
def gemm_variant(request, hq):
    """Runs the test once per GEMM kernel; the automatic choice is restored after."""
    v = {"single_cta": hq.HQ_GEMM_SINGLE_CTA, "cta_pair": hq.HQ_GEMM_CTA_PAIR}[request.param]
    hq.hq_debug_set_gemm_variant(v)
    yield v
    hq.hq_debug_set_gemm_variant(hq.HQ_GEMM_AUTO)


@pytest.mark.parametrize("T,N,K", GEMM_SHAPES)
def test_gemm_accumulators_bit_exact(hq, gemm_variant, T, N, K):
    g = np.random.default_rng(T * N + K)
    A = g.integers(-128, 128, size=(T, K)).astype(np.int8)
    B = g.integers(-128, 128, size=(N, K)).astype(np.int8)
    A[0, :] = -128
    B[0, :] = -128
    acc_ref = oracle.gemm_acc(A, B)
    sx = (g.random(T) * 0.1 + 1e-3)
    sw = (g.random(N) * 0.01 + 1e-4)
    cs = g.standard_normal(N)
    bias = g.standard_normal(N) * 0.1
    mean = g.standard_normal(T)
    sx32, sw32, cs32, b32, m32 = (v.astype(np.float32) for v in (sx, sw, cs, bias, mean))
    _, y_ref = oracle.epilogue(acc_ref, sx32.astype(np.float64), sw32.astype(np.float64),
                               colsum=cs32.astype(np.float64), bias=b32.astype(np.float64),
                               mean=m32.astype(np.float64))
    desc = hq.LayerDesc(K, N, 16, a_bits=8, w_bits=8, act_gran=hq.HQ_PER_TOKEN)
    d = {k: torch.from_numpy(v).cuda() for k, v in
         dict(A=A, B=B, sx=sx32, sw=sw32, cs=cs32, b=b32, m=m32).items()}
    Y = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    acc = torch.full((T, N), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    hq.hq_linear(desc, d["A"], d["sx"], d["m"], d["B"], d["sw"], d["cs"], d["b"], Y, acc)
    assert hq.hq_check_device_error() == 0
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), acc_ref)
    err = rel_frob(bf16_bits(Y), y_ref)
    assert err <= 1e-5, err


def test_gemm_many_tiles_per_cta(hq, gemm_variant):
    """Several output tiles per persistent CTA (both tensor-memory accumulators
    reused, ring phases wrapping many times) with ragged rows, columns and K;
    accumulators checked exactly on a seeded sample of rows from every
    256-row tile, all columns."""
    T, N, K = 4100, 4112, 320
    g = np.random.default_rng(7)
    A = g.integers(-8, 9, size=(T, K)).astype(np.int8)
    B = g.integers(-8, 9, size=(N, K)).astype(np.int8)
    sx = (g.random(T) * 0.1 + 1e-3).astype(np.float32)
    sw = (g.random(N) * 0.01 + 1e-4).astype(np.float32)
    desc = hq.LayerDesc(K, N, 64, a_bits=5, w_bits=5, act_gran=hq.HQ_PER_TOKEN)
    Y = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    acc = torch.full((T, N), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    dev = lambda v: torch.from_numpy(v).cuda()
    hq.hq_linear(desc, dev(A), dev(sx), None, dev(B), dev(sw), None, None, Y, acc)
    assert hq.hq_check_device_error() == 0
    rows = synth.sample_rows(T, 400, tile=256, seed=3)
    acc_ref = oracle.gemm_acc(A[rows], B)
    assert np.array_equal(acc.cpu().numpy()[rows].astype(np.int64), acc_ref)
    _, y_ref = oracle.epilogue(acc_ref, sx[rows].astype(np.float64), sw.astype(np.float64))
    assert rel_frob(bf16_bits(Y)[rows], y_ref) <= 1e-5


def test_gemm_worst_case_int4_accumulation(hq, gemm_variant):
    T, N, K = 256, 256, 4608
    A = np.full((T, K), 7, dtype=np.int8)
    A[1::2] = -7
    B = np.full((N, K), 7, dtype=np.int8)
    B[::3] = -7
    acc_ref = oracle.gemm_acc(A, B)
    desc = hq.LayerDesc(K, N, 256, act_gran=hq.HQ_PER_TENSOR_STATIC)
    one = torch.ones(1, dtype=torch.float32, device="cuda")
    sw = torch.ones(N, dtype=torch.float32, device="cuda")
    Y = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    acc = torch.empty((T, N), dtype=torch.int32, device="cuda")
    hq.hq_linear(desc, torch.from_numpy(A).cuda(), one, None, torch.from_numpy(B).cuda(), sw, None,
                 None, Y, acc)
    assert hq.hq_check_device_error() == 0
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), acc_ref)


# ---------------------------------------------------------------------------
# whole layer
# ---------------------------------------------------------------------------

def _gpu_layer(hq, cfg, Xb, Wb, bb):
    T, K = Xb.shape
    N = Wb.shape[0]
    desc = hq.LayerDesc(K, N, cfg.had_order, a_bits=cfg.a_bits, w_bits=cfg.w_bits,
                        act_gran=cfg.act_gran, centering=cfg.centering)
    X = to_dev_u16(Xb, torch)
    W = to_dev_u16(Wb, torch)
    b = to_dev_u16(bb, torch)
    absmax = None
    if cfg.use_sigma:
        absmax = torch.zeros(K, dtype=torch.float32, device="cuda")
        hq.hq_calib_act_absmax(desc, X, absmax)
    layer = hq.HadamardQuantLinear(desc, W, b, absmax, cfg.alpha)
    acc = torch.empty((T, N), dtype=torch.int32, device="cuda")
    Y = layer(X, acc_debug=acc)
    assert hq.hq_check_device_error() == 0
    bufs = layer.buffers(T)
    return layer, bufs, Y, acc


def _oracle_layer(cfg, Xb, Wb, bb, rows=None, cols=None):
    sig = None
    if cfg.use_sigma:
        sig = oracle.sigma(oracle.col_absmax(Xb), oracle.col_absmax(Wb), cfg.alpha)
    Wsel = Wb if cols is None else Wb[cols]
    bsel = bb if cols is None else bb[cols]
    w = oracle.prepare_weights(Wsel, cfg.had_order, cfg.w_bits, bias_bits=bsel, sigma=sig)
    a = oracle.quantize_act(Xb, cfg.had_order, cfg.a_bits, gran=cfg.act_gran,
                            centering=cfg.centering, sigma=sig, rows=rows, want_Z=True)
    acc = oracle.gemm_acc(a["codes"], w["codes"])
    y, yb = oracle.epilogue(acc, a["scale"], w["scale"], colsum=oracle.correction(w, cfg.centering),
                            bias=w["bias"], mean=a["mean"] if cfg.centering else None)
    return {"w": w, "a": a, "acc": acc, "y": y, "y_bf16": yb, "sigma": sig}


@pytest.mark.parametrize("idx,T", [(1, 300), (2, 257), (3, 130), (4, 1000), (5, 129)])
def test_layer_reduced_tokens(hq, idx, T):
    cfg = synth.CONFIGS[idx].with_tokens(T)
    Xb, Wb, bb = synth.make_layer(cfg)
    if idx == 5:
        Wb, bb = Wb[:768], bb[:768]          # keep the CPU oracle quick
    layer, bufs, Y, acc = _gpu_layer(hq, cfg, Xb, Wb, bb)
    ref = _oracle_layer(cfg, Xb, Wb, bb)
    check_codes(bufs["a_codes"].cpu().numpy(), ref["a"]["codes"], ref["a"]["tie"], "a_codes")
    check_codes(layer.w_codes.cpu().numpy(), ref["w"]["codes"], ref["w"]["tie"], "w_codes")
    err = rel_frob(bf16_bits(Y), ref["y_bf16"])
    assert err <= Y_REL_FROB, err
    # accumulators are exact whenever both sides chose the same codes
    same = (np.all(bufs["a_codes"].cpu().numpy() == ref["a"]["codes"]) and
            np.all(layer.w_codes.cpu().numpy() == ref["w"]["codes"]))
    if same:
        assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref["acc"])


@pytest.mark.parametrize("idx,T", [(1, 300), (2, 257), (3, 130), (5, 129)])
def test_layer_pre_rotation_centering(hq, idx, T):
    """The mean removed before the rotation (HQ_CENTER_TOKEN_MEAN_PRE): codes,
    the correction sum_k sigma_k W[n,k] and the layer output against the
    oracle, and its output is closer to the exact product than the default."""
    import dataclasses
    cfg = dataclasses.replace(synth.CONFIGS[idx].with_tokens(T), centering=2)
    Xb, Wb, bb = synth.make_layer(cfg)
    if idx == 5:
        Wb, bb = Wb[:768], bb[:768]
    layer, bufs, Y, acc = _gpu_layer(hq, cfg, Xb, Wb, bb)
    ref = _oracle_layer(cfg, Xb, Wb, bb)
    check_codes(bufs["a_codes"].cpu().numpy(), ref["a"]["codes"], ref["a"]["tie"], "a_codes")
    check_codes(layer.w_codes.cpu().numpy(), ref["w"]["codes"], ref["w"]["tie"], "w_codes")
    err = rel_frob(bf16_bits(Y), ref["y_bf16"])
    assert err <= Y_REL_FROB, err
    y_exact = oracle.exact_linear(Xb, Wb, bb)
    ref1 = _oracle_layer(dataclasses.replace(cfg, centering=1), Xb, Wb, bb)
    gpu_err = np.linalg.norm(synth.bf16_bits_to_f32(bf16_bits(Y)).astype(np.float64) - y_exact)
    assert gpu_err < np.linalg.norm(ref1["y"] - y_exact)


def test_centering_off_variant_of_w4a3(hq):
    cfg = synth.CONFIGS[3].with_tokens(200)
    import dataclasses
    cfg = dataclasses.replace(cfg, centering=0)
    Xb, Wb, bb = synth.make_layer(cfg)
    layer, bufs, Y, _ = _gpu_layer(hq, cfg, Xb, Wb, bb)
    ref = _oracle_layer(cfg, Xb, Wb, bb)
    check_codes(bufs["a_codes"].cpu().numpy(), ref["a"]["codes"], ref["a"]["tie"], "a_codes")
    assert rel_frob(bf16_bits(Y), ref["y_bf16"]) <= Y_REL_FROB


@pytest.mark.parametrize("idx", [1, 2, 3, 4, 5])
def test_layer_full_size_sampled(hq, idx):
    """Full configuration sizes in the benchmark's launch configuration; the
    oracle checks a seeded sample of rows (every 128-row tile) and of output
    channels (every 256-column tile)."""
    cfg = synth.CONFIGS[idx]
    Xb, Wb, bb = synth.make_layer(cfg)
    layer, bufs, Y, acc = _gpu_layer(hq, cfg, Xb, Wb, bb)
    rows = synth.sample_rows(cfg.T, 512, tile=128, seed=idx)
    cols = synth.sample_rows(cfg.N, 384, tile=256, seed=100 + idx)
    ref = _oracle_layer(cfg, Xb, Wb, bb, rows=rows, cols=cols)
    a_codes = bufs["a_codes"].cpu().numpy()[rows]
    w_codes = layer.w_codes.cpu().numpy()[cols]
    check_codes(a_codes, ref["a"]["codes"], ref["a"]["tie"], "a_codes", min_match=CODE_MATCH_MIN)
    check_codes(w_codes, ref["w"]["codes"], ref["w"]["tie"], "w_codes", min_match=CODE_MATCH_MIN)
    per_row = cfg.act_gran == 0
    sc = bufs["a_scale"].cpu().numpy().astype(np.float64)
    check_rel(sc[rows] if per_row else sc[:1], ref["a"]["scale"] if per_row else ref["a"]["scale"][:1],
              SCALE_RTOL, "a_scale")
    Ys = bf16_bits(Y)[np.ix_(rows, cols)]
    err = rel_frob(Ys, ref["y_bf16"])
    assert err <= Y_REL_FROB, err
    acc_s = acc.cpu().numpy()[np.ix_(rows, cols)].astype(np.int64)
    # exact wherever both the row's and the column's codes agree
    ra = np.all(a_codes == ref["a"]["codes"], axis=1)
    ca = np.all(w_codes == ref["w"]["codes"], axis=1)
    assert np.array_equal(acc_s[np.ix_(ra, ca)], ref["acc"][np.ix_(ra, ca)])


def test_gemm_fed_oracle_codes_is_bit_exact(hq, gemm_variant):
    cfg = synth.CONFIGS[2].with_tokens(384)
    Xb, Wb, bb = synth.make_layer(cfg)
    ref = _oracle_layer(cfg, Xb, Wb[:512], bb[:512])
    T, K = Xb.shape
    N = 512
    desc = hq.LayerDesc(K, N, cfg.had_order, act_gran=0, centering=1)
    f32 = lambda v: torch.from_numpy(np.asarray(v, dtype=np.float32)).cuda()
    Y = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    acc = torch.empty((T, N), dtype=torch.int32, device="cuda")
    hq.hq_linear(desc, torch.from_numpy(ref["a"]["codes"]).cuda(), f32(ref["a"]["scale"]),
                 f32(ref["a"]["mean"]), torch.from_numpy(ref["w"]["codes"]).cuda(),
                 f32(ref["w"]["scale"]), f32(ref["w"]["colsum"]), f32(ref["w"]["bias"]), Y, acc)
    assert hq.hq_check_device_error() == 0
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref["acc"])
    assert rel_frob(bf16_bits(Y), ref["y_bf16"]) <= 1e-4


# ---------------------------------------------------------------------------
# edge cases and the error path
# ---------------------------------------------------------------------------

def test_empty_and_zero_rows(hq):
    desc = hq.LayerDesc(128, 16, 128, a_bits=4)
    X = torch.zeros((0, 128), dtype=torch.bfloat16, device="cuda")
    codes = torch.empty((0, 128), dtype=torch.int8, device="cuda")
    sc = torch.empty(1, dtype=torch.float32, device="cuda")
    hq.hq_quantize_act(desc, X, None, codes, sc, None, T=0)
    Xz = np.zeros((5, 128), dtype=np.uint16)
    Xz[3] = synth.f32_to_bf16_bits(np.linspace(-1, 1, 128).astype(np.float32))
    codes, scale, mean = _gpu_quantize(hq, desc, Xz)
    assert np.all(codes[[0, 1, 2, 4]] == 0) and np.all(scale[[0, 1, 2, 4]] == 0)
    ref = oracle.quantize_act(Xz, 128, 4)
    assert np.array_equal(codes, ref["codes"])


def test_bounded_wait_reports_timeout_and_context_survives(hq):
    desc = hq.LayerDesc(1152, 16, 128, a_bits=4)
    Xb = synth.make_x(synth.CONFIGS[2].with_tokens(64))
    hq.hq_debug_set_wait_limit(2_000_000)  # 2 ms
    hq.hq_debug_inject_fault(hq.HQ_FAULT_QUANT_WITHHOLD_ROW)
    try:
        X = to_dev_u16(Xb, torch)
        codes = torch.empty((64, 1152), dtype=torch.int8, device="cuda")
        sc = torch.empty(64, dtype=torch.float32, device="cuda")
        hq.hq_quantize_act(desc, X, None, codes, sc, None)
        assert hq.hq_check_device_error() == 5  # HQ_ERR_TIMEOUT
    finally:
        hq.hq_debug_inject_fault(hq.HQ_FAULT_NONE)
        hq.hq_debug_set_wait_limit(0)
    # the context is still usable and the word was cleared
    assert hq.hq_check_device_error() == 0
    codes2, scale2, _ = _gpu_quantize(hq, desc, Xb)
    ref = oracle.quantize_act(Xb, 128, 4)
    check_codes(codes2, ref["codes"], ref["tie"], "after timeout")


# ---------------------------------------------------------------------------
# steps issued back to back on one stream
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("variant", ["auto", "cta_pair"])
def test_back_to_back_steps_match_isolated_steps(hq, variant):
    """quantize -> linear -> quantize -> ... with no synchronization between
    launches (eagerly and from one CUDA graph), one codes buffer reused by
    every step, must give bit-identical results to the same steps run one at
    a time."""
    cfg = synth.CONFIGS[2].with_tokens(1000)
    Xb, Wb, bb = synth.make_layer(cfg)
    T, K = Xb.shape
    N = Wb.shape[0]
    desc = hq.LayerDesc(K, N, cfg.had_order, a_bits=cfg.a_bits, w_bits=cfg.w_bits,
                        act_gran=cfg.act_gran, centering=cfg.centering)
    hq.hq_debug_set_gemm_variant(hq.HQ_GEMM_CTA_PAIR if variant == "cta_pair" else hq.HQ_GEMM_AUTO)
    try:
        X0 = to_dev_u16(Xb, torch)
        absmax = torch.zeros(K, dtype=torch.float32, device="cuda")
        hq.hq_calib_act_absmax(desc, X0, absmax)
        layer = hq.HadamardQuantLinear(desc, to_dev_u16(Wb, torch), to_dev_u16(bb, torch), absmax,
                                       cfg.alpha)
        # three different token batches: the rows of X rotated
        Xs = [torch.roll(X0, shifts=s * 97, dims=0).contiguous() for s in range(3)]
        iso = []
        for X in Xs:
            Y = layer(X)
            assert hq.hq_check_device_error() == 0
            iso.append(Y.clone())
        # eager, no synchronization between steps (one codes buffer reused:
        # each quantize overwrites what the previous GEMM reads)
        outs = [torch.empty((T, N), dtype=torch.bfloat16, device="cuda") for _ in Xs]
        bufs = layer.buffers(T)
        mean = bufs["a_mean"] if cfg.centering else None

        def steps():
            for X, Y in zip(Xs, outs):
                hq.hq_quantize_act(desc, X, layer.sigma_inv, bufs["a_codes"], bufs["a_scale"],
                                   bufs["a_mean"], layer.workspace)
                hq.hq_linear(desc, bufs["a_codes"], bufs["a_scale"], mean, layer.w_codes,
                             layer.w_scale, layer.colsum, layer.bias_f32, Y)

        steps()
        assert hq.hq_check_device_error() == 0
        for Y, R in zip(outs, iso):
            assert torch.equal(Y.view(torch.int16), R.view(torch.int16))
        for Y in outs:
            Y.fill_(float("nan"))
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            steps()
        g.replay()
        assert hq.hq_check_device_error() == 0
        for Y, R in zip(outs, iso):
            assert torch.equal(Y.view(torch.int16), R.view(torch.int16))
    finally:
        hq.hq_debug_set_gemm_variant(hq.HQ_GEMM_AUTO)


# ---------------------------------------------------------------------------
# no input-side rotation and the weight-only Hadamard form (HaTQ Eq. (15)-(17))
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("K,T,bits,gran", [(320, 300, 8, 1), (1024, 129, 4, 0), (1152, 77, 3, 0),
                                           (320, 513, 8, 0)])
def test_quantize_without_rotation(hq, K, T, bits, gran):
    """had_order 1: the activations are quantized in their own basis."""
    g = np.random.default_rng(K + T)
    x = (g.laplace(0, 1, size=(T, K)) * 10.0 ** g.uniform(-1, 1, size=K)).astype(np.float32)
    X = synth.f32_to_bf16_bits(x)
    ref = oracle.quantize_act(X, 1, bits, gran=gran, centering=0, want_Z=True)
    desc = hq.LayerDesc(K, 16, 1, a_bits=bits, w_bits=8, act_gran=gran, centering=0)
    codes, scale, mean = _gpu_quantize(hq, desc, X)
    _check_act(ref, codes, scale, mean, per_row=(gran == 0))
    assert np.all(mean == 0.0)


WH_CASES = [(320, 320, 64, 8, False), (1152, 3456, 32, 4, True), (256, 128, 16, 8, True),
            (3072, 1024, 64, 4, False)]


@pytest.mark.parametrize("K,N,m,w_bits,use_sigma", WH_CASES)
def test_wh_prepare_weights(hq, K, N, m, w_bits, use_sigma):
    """Wbar = H_out W diag(sigma) quantized per row, against the oracle."""
    g = np.random.default_rng(K + N + m)
    Wb = synth.f32_to_bf16_bits(g.standard_normal((N, K)).astype(np.float32) *
                                (1 + 10 * (g.random(N) < 0.05)).astype(np.float32)[:, None])
    bb = synth.f32_to_bf16_bits(g.standard_normal(N).astype(np.float32))
    absmax_np = None
    sig = None
    if use_sigma:
        absmax_np = (np.abs(g.standard_normal(K)) * 3 + 0.1).astype(np.float32)
        sig = oracle.sigma(absmax_np.astype(np.float64), oracle.col_absmax(Wb), 0.5)
    ref = oracle.prepare_weights_wh(Wb, m, w_bits, bias_bits=bb, sigma=sig)
    desc = hq.LayerDesc(K, N, 1, a_bits=8, w_bits=w_bits, centering=0, out_order=m)
    absmax = None if absmax_np is None else torch.from_numpy(absmax_np).cuda()
    layer = hq.HadamardQuantLinear(desc, to_dev_u16(Wb, torch), to_dev_u16(bb, torch), absmax)
    assert hq.hq_check_device_error() == 0
    check_codes(layer.w_codes.cpu().numpy(), ref["codes"], ref["tie"], "wh w_codes",
                min_match=0.999)
    check_rel(layer.w_scale.cpu().numpy(), ref["scale"], SCALE_RTOL, "wh w_scale")
    assert np.all(layer.colsum.cpu().numpy() == 0.0)
    assert np.array_equal(layer.bias_f32.cpu().numpy(),
                          synth.bf16_bits_to_f32(bb).astype(np.float32))


@pytest.mark.parametrize("T,K,N,m", [(300, 320, 320, 64), (129, 1152, 640, 32), (513, 256, 128, 16),
                                     (200, 512, 1024, 64)])
def test_wh_gemm_fed_oracle_codes(hq, gemm_variant, T, K, N, m):
    """The oracle's codes through hq_linear in the weight-only form: int32
    accumulators bit-exact (in the Hadamard basis), output against the
    oracle's (dequantized accumulator + b_bar) H_out.  The form always runs
    the single-CTA kernel, whichever variant is asked for."""
    g = np.random.default_rng(T + K + N)
    Xb = synth.f32_to_bf16_bits(g.standard_normal((T, K)).astype(np.float32))
    Wb = synth.f32_to_bf16_bits(g.standard_normal((N, K)).astype(np.float32) * 0.05)
    bb = synth.f32_to_bf16_bits(g.standard_normal(N).astype(np.float32))
    r = oracle.layer_wh(Xb, Wb, bb, m, 8, 8)
    desc = hq.LayerDesc(K, N, 1, a_bits=8, w_bits=8, centering=0, out_order=m)
    d = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in dict(
        A=r["a"]["codes"], B=r["w"]["codes"], sx=r["a"]["scale"].astype(np.float32),
        sw=r["w"]["scale"].astype(np.float32),
        b=synth.bf16_bits_to_f32(bb).astype(np.float32)).items()}
    Y = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    acc = torch.full((T, N), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    hq.hq_linear(desc, d["A"], d["sx"], None, d["B"], d["sw"], None, d["b"], Y, acc)
    assert hq.hq_check_device_error() == 0
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), r["acc"])
    # the same accumulators and fp32-rounded scales through the oracle's output side
    _, y_ref = oracle.epilogue_wh(r["acc"], m, r["a"]["scale"].astype(np.float32).astype(np.float64),
                                  r["w"]["scale"].astype(np.float32).astype(np.float64),
                                  b_bar=r["w"]["b_bar"])
    # fp32 against fp64 on both sides of the bf16 rounding: the fp32 transform
    # over m columns is off by about log2(m) sqrt(m) 2^-24 of an output
    # (~3e-6 for m = 64), which moves an output across a bf16 rounding
    # boundary for ~2 * 3e-6 / 2^-8 ~ 0.15% of outputs, each by one bf16 ulp
    # (2^-8 relative): a Frobenius error of about sqrt(1.5e-3) * 2^-8 ~ 1e-4
    err = rel_frob(bf16_bits(Y), y_ref)
    assert err <= 1e-4, err


@pytest.mark.parametrize("T,K,N,m,a_bits,w_bits,gran,use_sigma",
                         [(1000, 320, 320, 64, 8, 8, 1, False), (257, 1152, 3456, 32, 4, 4, 0, False),
                          (300, 256, 512, 16, 8, 8, 0, True), (129, 3072, 1024, 64, 4, 4, 0, False)])
def test_wh_layer(hq, T, K, N, m, a_bits, w_bits, gran, use_sigma):
    """The whole weight-only Hadamard layer on the GPU against oracle.layer_wh."""
    g = np.random.default_rng(T + N)
    x = (g.laplace(0, 1, size=(T, K)) * (1 + 8 * (g.random(K) < 0.02))).astype(np.float32)
    x += np.abs(g.standard_normal((T, 1))).astype(np.float32)  # a nonzero channel mean
    Xb = synth.f32_to_bf16_bits(x)
    Wb = synth.f32_to_bf16_bits(g.standard_normal((N, K)).astype(np.float32) * 0.03)
    bb = synth.f32_to_bf16_bits(g.standard_normal(N).astype(np.float32) * 0.1)
    ref = oracle.layer_wh(Xb, Wb, bb, m, a_bits, w_bits, gran=gran, use_sigma=use_sigma)
    desc = hq.LayerDesc(K, N, 1, a_bits=a_bits, w_bits=w_bits, act_gran=gran, centering=0,
                        out_order=m)
    X = to_dev_u16(Xb, torch)
    absmax = None
    if use_sigma:
        absmax = torch.zeros(K, dtype=torch.float32, device="cuda")
        hq.hq_calib_act_absmax(desc, X, absmax)
    layer = hq.HadamardQuantLinear(desc, to_dev_u16(Wb, torch), to_dev_u16(bb, torch), absmax)
    acc = torch.empty((T, N), dtype=torch.int32, device="cuda")
    Y = layer(X, acc_debug=acc)
    assert hq.hq_check_device_error() == 0
    bufs = layer.buffers(T)
    check_codes(bufs["a_codes"].cpu().numpy(), ref["a"]["codes"], ref["a"]["tie"], "wh a_codes")
    check_codes(layer.w_codes.cpu().numpy(), ref["w"]["codes"], ref["w"]["tie"], "wh w_codes")
    err = rel_frob(bf16_bits(Y), ref["y_bf16"])
    assert err <= Y_REL_FROB, err
    same = (np.all(bufs["a_codes"].cpu().numpy() == ref["a"]["codes"]) and
            np.all(layer.w_codes.cpu().numpy() == ref["w"]["codes"]))
    if same:
        assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref["acc"])


def test_no_rotation_double_form_layer(hq):
    """had_order 1 with no output transform: the plain per-token quantized
    product, through the same library calls."""
    T, K, N = 300, 1024, 512
    g = np.random.default_rng(11)
    Xb = synth.f32_to_bf16_bits(g.standard_normal((T, K)).astype(np.float32))
    Wb = synth.f32_to_bf16_bits(g.standard_normal((N, K)).astype(np.float32) * 0.05)
    bb = synth.f32_to_bf16_bits(g.standard_normal(N).astype(np.float32))
    ref = oracle.layer(Xb, Wb, bb, 1, 8, 8, centering=0, use_sigma=False)
    desc = hq.LayerDesc(K, N, 1, a_bits=8, w_bits=8, centering=0)
    layer = hq.HadamardQuantLinear(desc, to_dev_u16(Wb, torch), to_dev_u16(bb, torch), None)
    Y = layer(to_dev_u16(Xb, torch))
    assert hq.hq_check_device_error() == 0
    check_codes(layer.w_codes.cpu().numpy(), ref["w"]["codes"], ref["w"]["tie"], "w_codes")
    assert np.all(layer.colsum.cpu().numpy() == 0.0)
    assert rel_frob(bf16_bits(Y), ref["y_bf16"]) <= Y_REL_FROB


# ---------------------------------------------------------------------------
# hq_forward_host: uploads, kernels and downloads overlapped by row chunks
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("idx,T,over,chunks", [(2, 8192, {}, 8), (2, 1000, {}, 8),
                                               (2, 4099, {"centering": 2}, 3),
                                               (4, 65536, {}, 8), (4, 6000, {"act_gran": 2}, 4),
                                               (4, 8192, {"out_order": 64}, 8), (3, 300, {}, 1)])
def test_forward_host_equals_the_device_path(hq, idx, T, over, chunks):
    """Y_host from hq_forward_host equals upload + quantize + GEMM + download
    done one after the other, bit for bit, eagerly and from a CUDA graph
    replayed on fresh input data each time (a stale upload or an early
    download would show as another replay's output)."""
    import dataclasses
    cfg = synth.CONFIGS[idx].with_tokens(T)
    cfg = (cfg.weight_only(over["out_order"]) if "out_order" in over
           else dataclasses.replace(cfg, **over))
    Xb, Wb, bb = synth.make_layer(cfg)
    K, N = Xb.shape[1], Wb.shape[0]
    desc = hq.LayerDesc(K, N, cfg.had_order, a_bits=cfg.a_bits, w_bits=cfg.w_bits,
                        act_gran=cfg.act_gran, centering=cfg.centering, out_order=cfg.out_order)
    X0 = to_dev_u16(Xb, torch)
    absmax = None
    if cfg.use_sigma:
        absmax = torch.zeros(K, dtype=torch.float32, device="cuda")
        hq.hq_calib_act_absmax(desc, X0, absmax)
    static = 0.02 if cfg.act_gran == hq.HQ_PER_TENSOR_STATIC else None
    layer = hq.HadamardQuantLinear(desc, to_dev_u16(Wb, torch), to_dev_u16(bb, torch), absmax,
                                   cfg.alpha, static_scale=static)
    inputs = [X0, torch.roll(X0, 131, dims=0).contiguous(), (X0 * 0.5).contiguous()]

    def reference(X):
        Y = layer.forward(X)     # device path: hq_quantize_act then hq_linear
        torch.cuda.synchronize()
        return Y.cpu()

    refs = [reference(X) for X in inputs]
    X_host = torch.empty((T, K), dtype=torch.bfloat16).pin_memory()
    Y_host = torch.empty((T, N), dtype=torch.bfloat16).pin_memory()
    for X, R in zip(inputs, refs):                              # eager
        X_host.copy_(X.cpu())
        Y_host.fill_(float("nan"))
        layer.forward_host(X_host, Y_host, chunks=chunks)
        torch.cuda.synchronize()
        assert hq.hq_check_device_error() == 0
        assert torch.equal(Y_host.view(torch.int16), R.view(torch.int16))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer.forward_host(X_host, Y_host, chunks=chunks)
    for X, R in zip(inputs[::-1], refs[::-1]):                  # graph, fresh data each replay
        X_host.copy_(X.cpu())
        Y_host.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(Y_host.view(torch.int16), R.view(torch.int16))


def test_tensor_maps_are_reused_across_calls(hq):
    """Repeated calls on the same buffers and shapes take their tensor maps
    from the library's cache (no host encoding per call) and still compute
    the same output; a new output buffer costs one new map."""
    cfg = synth.CONFIGS[2].with_tokens(300)
    Xb, Wb, bb = synth.make_layer(cfg)
    T, K = Xb.shape
    N = Wb.shape[0]
    desc = hq.LayerDesc(K, N, cfg.had_order, a_bits=cfg.a_bits, w_bits=cfg.w_bits,
                        act_gran=cfg.act_gran, centering=cfg.centering)
    X = to_dev_u16(Xb, torch)
    layer = hq.HadamardQuantLinear(desc, to_dev_u16(Wb, torch), to_dev_u16(bb, torch), None)
    Y1 = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    layer(X, Y1)
    torch.cuda.synchronize()
    c0 = hq.hq_debug_tmap_cache()
    for _ in range(3):
        layer(X, Y1)
    torch.cuda.synchronize()
    c1 = hq.hq_debug_tmap_cache()
    # three GEMM maps and one quantizer map per step, all from the cache
    assert c1["misses"] == c0["misses"] and c1["hits"] - c0["hits"] == 3 * 4
    Y2 = torch.empty_like(Y1)
    layer(X, Y2)
    torch.cuda.synchronize()
    c2 = hq.hq_debug_tmap_cache()
    assert c2["misses"] == c1["misses"] + 1
    assert hq.hq_check_device_error() == 0
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))


@pytest.mark.parametrize("K,n,N,T,gran", [(80, 16, 48, 130, 0), (144, 16, 64, 33, 1),
                                         (12288, 1024, 256, 129, 0), (12288, 256, 128, 40, 1)])
def test_layer_at_the_shape_envelope(hq, K, n, N, T, gran):
    """The whole layer where K is a multiple of 16 only, and where K exceeds
    8192: codes, exact accumulators and output against the oracle."""
    g = np.random.default_rng(K + N + T)
    x = g.standard_normal((T, K)).astype(np.float32)
    x[:, g.choice(K, size=max(1, K // 100), replace=False)] *= 25.0
    x += g.standard_normal((T, 1)).astype(np.float32)
    Xb = synth.f32_to_bf16_bits(x)
    Wb = synth.f32_to_bf16_bits((g.standard_normal((N, K)) * 0.02).astype(np.float32))
    bb = synth.f32_to_bf16_bits((g.standard_normal(N) * 0.01).astype(np.float32))
    ref = oracle.layer(Xb, Wb, bb, n, 4, 4, gran=gran, centering=1)
    desc = hq.LayerDesc(K, N, n, a_bits=4, w_bits=4, act_gran=gran, centering=1)
    X = to_dev_u16(Xb, torch)
    absmax = torch.zeros(K, dtype=torch.float32, device="cuda")
    hq.hq_calib_act_absmax(desc, X, absmax)
    layer = hq.HadamardQuantLinear(desc, to_dev_u16(Wb, torch), to_dev_u16(bb, torch), absmax, 0.5)
    acc = torch.empty((T, N), dtype=torch.int32, device="cuda")
    Y = layer(X, acc_debug=acc)
    assert hq.hq_check_device_error() == 0
    check_codes(layer.w_codes.cpu().numpy(), ref["w"]["codes"], ref["w"]["tie"], "w_codes")
    codes = layer.buffers(T)["a_codes"].cpu().numpy()
    check_codes(codes, ref["a"]["codes"], ref["a"]["tie"], "a_codes")
    same = np.all(codes == ref["a"]["codes"], axis=1)
    wsame = np.all(layer.w_codes.cpu().numpy() == ref["w"]["codes"], axis=1)
    a = acc.cpu().numpy()
    assert np.array_equal(a[np.ix_(same, wsame)], ref["acc"][np.ix_(same, wsame)])
    assert rel_frob(bf16_bits(Y), ref["y_bf16"]) <= Y_REL_FROB
