"""GPU parity of packed activation codes (two 3/4-bit codes per byte, element
2j in the low nibble): the quantizer's packed output, the GEMM that widens
packed tiles in shared memory, and the layer end to end.  Needs a B200."""
import numpy as np
import pytest

import oracle
import synth
from parity import (Y_REL_FROB, bf16_bits, check_bf16_outputs, check_codes, check_rel, rel_frob,
                    to_dev_u16)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

PACKED = 1  # HQ_CODES_I4_PACKED


@pytest.fixture(scope="module")
def hq():
    import hadamard_rotated_bit_token_b200 as hq_mod
    from hadamard_rotated_bit_token_b200 import build as hq_build
    hq_build.build()
    hq_mod.load_library()
    return hq_mod


def _quantize(hq, desc, X, sigma_inv=None, static_scale=None):
    """One GPU quantize call; returns (codes as stored, scale, mean) on the host."""
    T, K = X.shape
    if desc.code_format == PACKED:
        codes = torch.full((T, K // 2), 0x55, dtype=torch.uint8, device="cuda")  # poison
    else:
        codes = torch.full((T, K), 0x55, dtype=torch.int8, device="cuda")
    per_row = desc.act_gran == hq.HQ_PER_TOKEN
    scale = torch.full((T if per_row else 1,), float("nan"), dtype=torch.float32, device="cuda")
    if static_scale is not None:
        scale.fill_(static_scale)
    mean = torch.full((T,), float("nan"), dtype=torch.float32, device="cuda")
    ws_bytes = hq.hq_quantize_act_workspace_bytes(desc, T)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda") if ws_bytes else None
    hq.hq_quantize_act(desc, X, sigma_inv, codes, scale, mean, ws)
    assert hq.hq_check_device_error() == 0
    return codes.cpu().numpy(), scale.cpu().numpy(), mean.cpu().numpy()


# (K, n, T, bits, centering, granularity): every store path of the quantizer --
# in-register slices with shuffles (n <= 128), the shared-memory transpose
# (n >= 256), no rotation (n = 1), several blocks per slice (n = 16), and the
# per-tensor passes
QUANT_CASES = [(1152, 128, 257, 4, 1, 0), (4608, 256, 130, 3, 1, 0), (3072, 1024, 129, 4, 2, 0),
               (320, 64, 300, 4, 0, 1), (320, 64, 300, 3, 1, 2), (1024, 1, 129, 4, 0, 0),
               (512, 16, 65, 3, 1, 0), (1024, 32, 100, 4, 1, 0), (2048, 512, 33, 4, 0, 1),
               (4608, 256, 1000, 3, 1, 0)]


@pytest.mark.parametrize("K,n,T,bits,center,gran", QUANT_CASES)
def test_packed_quantize(hq, K, n, T, bits, center, gran):
    g = np.random.default_rng(K + 7 * T + n)
    Xf = g.standard_normal((T, K)) * 2.0
    Xf[:, g.choice(K, 3, replace=False)] *= 20  # a few outlier channels
    Xf[5] = 0                                   # an all-zero token
    X = synth.f32_to_bf16_bits(Xf.astype(np.float32))
    Xd = to_dev_u16(X, torch)
    static = 0.37 if gran == 2 else None
    d8 = hq.LayerDesc(K, 16, n, a_bits=bits, act_gran=gran, centering=center)
    d4 = hq.LayerDesc(K, 16, n, a_bits=bits, act_gran=gran, centering=center, code_format=PACKED)
    c8, s8, m8 = _quantize(hq, d8, Xd, static_scale=static)
    c4, s4, m4 = _quantize(hq, d4, Xd, static_scale=static)
    assert c4.shape == (T, K // 2)
    # the packed bytes hold exactly the codes of the one-per-byte form ...
    assert np.array_equal(oracle.unpack_i4(c4), c8)
    assert np.array_equal(s4.view(np.uint32), s8.view(np.uint32))
    assert np.array_equal(m4.view(np.uint32), m8.view(np.uint32))
    # ... and those are the oracle's codes (ties aside)
    ref = oracle.quantize_act(X, n, bits, gran=gran, centering=center,
                              static_scale=static if static is not None else 0.0)
    check_codes(oracle.unpack_i4(c4), ref["codes"], ref["tie"], "packed codes")
    if gran != 2:
        check_rel(s4[:T if gran == 0 else 1], ref["scale"][:T if gran == 0 else 1], 1e-6, "scale")


# (T, N, K): single and ragged tiles, K tails below one 128-code block, long K
PACKED_GEMM_SHAPES = [(1, 16, 32), (127, 48, 160), (128, 192, 128), (129, 320, 320),
                      (300, 512, 1152), (200, 3456, 256), (131, 160, 4608), (513, 64, 96),
                      (257, 3456, 1152)]


def _linear_packed(hq, A, B, sx, sw, a_bits, w_bits, cs=None, bias=None, mean=None):
    """hq_linear (per-token scales) on oracle-packed A; returns (Y, acc_debug)
    on the device."""
    T, K = A.shape
    N = B.shape[0]
    desc = hq.LayerDesc(K, N, 16, a_bits=a_bits, w_bits=w_bits, act_gran=0, centering=1,
                        code_format=PACKED)
    dev = lambda v: None if v is None else torch.from_numpy(np.ascontiguousarray(v)).cuda()
    Y = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    acc = torch.full((T, N), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    hq.hq_linear(desc, dev(oracle.pack_i4(A)), dev(sx), dev(mean), dev(B), dev(sw), dev(cs),
                 dev(bias), Y, acc, T=T)
    assert hq.hq_check_device_error() == 0
    return Y, acc


@pytest.mark.parametrize("w_bits", [4, 8])
@pytest.mark.parametrize("T,N,K", PACKED_GEMM_SHAPES)
def test_packed_gemm_bit_exact(hq, T, N, K, w_bits):
    g = np.random.default_rng(T * N + K + w_bits)
    A = g.integers(-8, 8, size=(T, K)).astype(np.int8)          # every 4-bit value
    qb = 8 if w_bits == 4 else 128
    B = g.integers(-qb, qb, size=(N, K)).astype(np.int8)
    A[0, :] = -8
    B[0, :] = -qb
    acc_ref = oracle.gemm_acc(A, B)
    f32 = lambda v: np.asarray(v, dtype=np.float32)
    sx, sw = f32(g.random(T) * 0.1 + 1e-3), f32(g.random(N) * 0.01 + 1e-4)
    cs, bias, mean = f32(g.standard_normal(N)), f32(g.standard_normal(N) * 0.1), f32(g.standard_normal(T))
    d = lambda v: v.astype(np.float64)
    y64, _ = oracle.epilogue(acc_ref, d(sx), d(sw), colsum=d(cs), bias=d(bias), mean=d(mean))
    mag = (np.abs(acc_ref * np.outer(d(sx), d(sw))) + np.abs(np.outer(d(mean), d(cs))) +
           np.abs(d(bias))[None, :])
    Y, acc = _linear_packed(hq, A, B, sx, sw, 4, w_bits, cs=cs, bias=bias, mean=mean)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), acc_ref)
    check_bf16_outputs(bf16_bits(Y), y64, mag)


def test_packed_gemm_many_tiles_and_worst_case(hq):
    """Several tiles per persistent CTA with ragged rows, columns and K (rows
    sampled from every tile), then all-extreme codes at K = 4608, where the
    epilogue takes the general integer conversion."""
    T, N, K = 4100, 4112, 320
    g = np.random.default_rng(11)
    A = g.integers(-8, 8, size=(T, K)).astype(np.int8)
    B = g.integers(-8, 8, size=(N, K)).astype(np.int8)
    sx = (g.random(T) * 0.1 + 1e-3).astype(np.float32)
    sw = (g.random(N) * 0.01 + 1e-4).astype(np.float32)
    Y, acc = _linear_packed(hq, A, B, sx, sw, 4, 4)
    rows = synth.sample_rows(T, 400, tile=128, seed=5)
    acc_ref = oracle.gemm_acc(A[rows], B)
    assert np.array_equal(acc.cpu().numpy()[rows].astype(np.int64), acc_ref)
    y64, _ = oracle.epilogue(acc_ref, sx[rows].astype(np.float64), sw.astype(np.float64))
    check_bf16_outputs(bf16_bits(Y)[rows], y64, np.abs(y64))

    T, N, K = 256, 256, 4608
    A = np.full((T, K), -8, dtype=np.int8)
    A[1::2] = 7
    B = np.full((N, K), -8, dtype=np.int8)
    B[::3] = 7
    one = np.ones(T, dtype=np.float32)
    Y, acc = _linear_packed(hq, A, B, one, np.ones(N, dtype=np.float32), 4, 4)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), oracle.gemm_acc(A, B))


def _layer(hq, cfg, Xb, Wb, bb, code_format, out_order=0):
    T, K = Xb.shape
    N = Wb.shape[0]
    desc = hq.LayerDesc(K, N, 1 if out_order else cfg.had_order, a_bits=cfg.a_bits,
                        w_bits=cfg.w_bits, act_gran=cfg.act_gran,
                        centering=0 if out_order else cfg.centering, code_format=code_format,
                        out_order=out_order)
    X = to_dev_u16(Xb, torch)
    absmax = None
    if cfg.use_sigma:
        absmax = torch.zeros(K, dtype=torch.float32, device="cuda")
        hq.hq_calib_act_absmax(desc, X, absmax)
    layer = hq.HadamardQuantLinear(desc, to_dev_u16(Wb, torch), to_dev_u16(bb, torch), absmax,
                                   cfg.alpha)
    acc = torch.empty((T, N), dtype=torch.int32, device="cuda")
    Y = layer(X, acc_debug=acc)
    assert hq.hq_check_device_error() == 0
    return layer, Y, acc


@pytest.mark.parametrize("idx,T,out_order", [(1, 300, 0), (2, 257, 0), (3, 130, 0), (5, 129, 0),
                                             (2, 300, 32), (3, 129, 64)])
def test_packed_layer_equals_one_code_per_byte(hq, idx, T, out_order):
    """The packed path computes the same layer bit for bit: the same codes,
    the same exact accumulators, the same bf16 outputs; and those meet the
    oracle's output bar."""
    cfg = synth.CONFIGS[idx].with_tokens(T)
    Xb, Wb, bb = synth.make_layer(cfg)
    if idx == 5:
        Wb, bb = Wb[:768], bb[:768]
    l8, Y8, acc8 = _layer(hq, cfg, Xb, Wb, bb, 0, out_order)
    l4, Y4, acc4 = _layer(hq, cfg, Xb, Wb, bb, PACKED, out_order)
    b8, b4 = l8.buffers(T), l4.buffers(T)
    assert np.array_equal(oracle.unpack_i4(b4["a_codes"].cpu().numpy()),
                          b8["a_codes"].cpu().numpy())
    assert torch.equal(acc4, acc8)
    assert torch.equal(Y4.view(torch.int16), Y8.view(torch.int16))
    if out_order == 0:
        sig = None
        if cfg.use_sigma:
            sig = oracle.sigma(oracle.col_absmax(Xb), oracle.col_absmax(Wb), cfg.alpha)
        w = oracle.prepare_weights(Wb, cfg.had_order, cfg.w_bits, bias_bits=bb, sigma=sig)
        a = oracle.quantize_act(Xb, cfg.had_order, cfg.a_bits, gran=cfg.act_gran,
                                centering=cfg.centering, sigma=sig)
        _, yb = oracle.epilogue(oracle.gemm_acc(a["codes"], w["codes"]), a["scale"], w["scale"],
                                colsum=oracle.correction(w, cfg.centering), bias=w["bias"],
                                mean=a["mean"] if cfg.centering else None)
        assert rel_frob(bf16_bits(Y4), yb) <= Y_REL_FROB


def test_packed_forward_host_equals_the_device_path(hq):
    cfg = synth.CONFIGS[2].with_tokens(1000)
    Xb, Wb, bb = synth.make_layer(cfg)
    layer, Y, _ = _layer(hq, cfg, Xb, Wb, bb, PACKED)
    X_host = torch.from_numpy(Xb.view(np.int16)).view(torch.bfloat16).pin_memory()
    Y_host = layer.forward_host(X_host, chunks=8)
    torch.cuda.synchronize()
    assert hq.hq_check_device_error() == 0
    assert torch.equal(Y_host.view(torch.int16), Y.cpu().view(torch.int16))
