"""The prepared-weights blob (HadamardQuantLinear.export_prepared /
from_prepared): format round trip and rejection of damaged blobs on the CPU;
on the GPU, a reloaded layer gives the same output bit for bit."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")


def _cpu_layer(hq, K=64, N=32, seed=0, static_scale=None, **desc_kw):
    g = np.random.default_rng(seed)
    lay = hq.HadamardQuantLinear.__new__(hq.HadamardQuantLinear)
    lay.desc = hq.LayerDesc(K, N, 16, **desc_kw)
    lay.static_scale = static_scale
    lay.w_codes = torch.from_numpy(g.integers(-7, 8, size=(N, K)).astype(np.int8))
    lay.w_scale = torch.from_numpy(g.random(N).astype(np.float32))
    lay.colsum = torch.from_numpy(g.standard_normal(N).astype(np.float32))
    lay.sigma_inv = torch.from_numpy((g.random(K) + 0.5).astype(np.float32))
    lay.bias_f32 = torch.from_numpy(g.standard_normal(N).astype(np.float32))
    lay.use_sigma = True
    lay.workspace = None
    lay._bufs = {}
    return lay


@pytest.fixture(scope="module")
def hq():
    import hadamard_rotated_bit_token_b200 as hq_mod
    return hq_mod


def test_blob_round_trip_on_cpu(hq):
    lay = _cpu_layer(hq, a_bits=3, w_bits=8, centering=2)
    blob = lay.export_prepared()
    back = hq.HadamardQuantLinear.from_prepared(blob, device="cpu")
    for f in ("K", "N", "had_order", "a_bits", "w_bits", "act_gran", "centering", "code_format",
              "out_order"):
        assert getattr(back.desc, f) == getattr(lay.desc, f)
    for name in ("w_codes", "w_scale", "colsum", "sigma_inv", "bias_f32"):
        assert torch.equal(getattr(back, name), getattr(lay, name)), name
    assert back.use_sigma is True
    assert back.export_prepared() == blob


def test_blob_rejects_damage(hq):
    blob = _cpu_layer(hq).export_prepared()
    load = lambda b: hq.HadamardQuantLinear.from_prepared(b, device="cpu")
    with pytest.raises(ValueError, match="not a prepared"):
        load(b"XXXX" + blob[4:])
    flipped = bytearray(blob)
    flipped[100] ^= 0x01
    with pytest.raises(ValueError, match="checksum"):
        load(bytes(flipped))
    with pytest.raises(ValueError):
        load(blob[:-10])
    with pytest.raises(ValueError):
        load(blob[:20])


def test_blob_keeps_the_static_scale(hq):
    """HQ_PER_TENSOR_STATIC: the scale is part of the prepared layer, so the
    blob carries it and a reload restores it; the other modes store none."""
    lay = _cpu_layer(hq, act_gran=hq.HQ_PER_TENSOR_STATIC, static_scale=0.0390625)
    back = hq.HadamardQuantLinear.from_prepared(lay.export_prepared(), device="cpu")
    assert back.static_scale == 0.0390625
    back = hq.HadamardQuantLinear.from_prepared(_cpu_layer(hq).export_prepared(), device="cpu")
    assert back.static_scale is None


def test_blob_version_1_still_loads(hq):
    """A version-1 blob (no static-scale field) loads as before."""
    import struct
    import zlib
    blob = _cpu_layer(hq).export_prepared()
    body = blob[:-4]
    v1 = body[:4] + struct.pack("<I", 1) + body[8:48] + body[56:]
    v1 += struct.pack("<I", zlib.crc32(v1) & 0xFFFFFFFF)
    back = hq.HadamardQuantLinear.from_prepared(v1, device="cpu")
    assert back.static_scale is None
    assert back.export_prepared() == blob


def test_static_mode_needs_a_scale(hq):
    """The layer refuses HQ_PER_TENSOR_STATIC without a scale (its quantizer
    and GEMM would read an uninitialised a_scale), and a scale in another
    mode; both before any device call."""
    W = torch.zeros((32, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="static_scale"):
        hq.HadamardQuantLinear(hq.LayerDesc(64, 32, 16, act_gran=hq.HQ_PER_TENSOR_STATIC), W)
    with pytest.raises(ValueError, match="positive"):
        hq.HadamardQuantLinear(hq.LayerDesc(64, 32, 16, act_gran=hq.HQ_PER_TENSOR_STATIC), W,
                               static_scale=0.0)
    with pytest.raises(ValueError, match="only used"):
        hq.HadamardQuantLinear(hq.LayerDesc(64, 32, 16), W, static_scale=0.5)
    # a static-mode blob whose scale field is empty (written as 0) is refused
    lay = _cpu_layer(hq, act_gran=hq.HQ_PER_TENSOR_STATIC)
    with pytest.raises(ValueError, match="blob: static_scale"):
        hq.HadamardQuantLinear.from_prepared(lay.export_prepared(), device="cpu")


@pytest.mark.gpu
def test_static_scale_layer_matches_the_oracle(hq):
    """The layer class in HQ_PER_TENSOR_STATIC mode quantizes with the scale
    it was given: codes, accumulators and output against the oracle fed the
    same static scale (HaTQ Sec. IV-E: a frozen activation scale)."""
    import oracle
    import synth
    from parity import bf16_bits, check_codes, rel_frob, to_dev_u16, Y_REL_FROB
    hq.load_library()
    cfg = synth.CONFIGS[2].with_tokens(260)
    Xb, Wb, bb = synth.make_layer(cfg)
    K, N = Xb.shape[1], Wb.shape[0]
    # a scale below the dynamic one, so some codes clamp at +-q
    dyn = oracle.layer(Xb, Wb, bb, cfg.had_order, 4, 4, gran=1, centering=1)
    s = float(np.float32(dyn["a"]["scale"][0] * 0.75))
    ref = oracle.layer(Xb, Wb, bb, cfg.had_order, 4, 4, gran=2, centering=1, static_scale=s)
    desc = hq.LayerDesc(K, N, cfg.had_order, act_gran=hq.HQ_PER_TENSOR_STATIC, centering=1)
    X = to_dev_u16(Xb, torch)
    absmax = torch.zeros(K, dtype=torch.float32, device="cuda")
    hq.hq_calib_act_absmax(desc, X, absmax)
    layer = hq.HadamardQuantLinear(desc, to_dev_u16(Wb, torch), to_dev_u16(bb, torch), absmax,
                                   0.5, static_scale=s)
    acc = torch.empty((X.shape[0], N), dtype=torch.int32, device="cuda")
    Y = layer(X, acc_debug=acc)
    assert hq.hq_check_device_error() == 0
    b = layer.buffers(X.shape[0])
    assert float(b["a_scale"][0]) == s
    codes = b["a_codes"].cpu().numpy()
    check_codes(codes, ref["a"]["codes"], ref["a"]["tie"])
    assert np.abs(codes).max() == 7  # the clamp was reached
    same = np.all(codes == ref["a"]["codes"], axis=1)
    assert same.any()
    # accumulators bit-exact on the rows whose codes agree with the oracle's
    assert np.array_equal(acc.cpu().numpy()[same], ref["acc"][same])
    assert rel_frob(bf16_bits(Y), ref["y_bf16"]) <= Y_REL_FROB
    again = hq.HadamardQuantLinear.from_prepared(layer.export_prepared())
    assert torch.equal(again(X).view(torch.int16), Y.view(torch.int16))


@pytest.mark.gpu
@pytest.mark.parametrize("wh", [False, True])
def test_reloaded_layer_gives_the_same_output(hq, wh):
    import synth
    from parity import to_dev_u16
    hq.load_library()
    cfg = synth.CONFIGS[2].with_tokens(300)
    if wh:
        cfg = cfg.weight_only(64)
    Xb, Wb, bb = synth.make_layer(cfg)
    K, N = Xb.shape[1], Wb.shape[0]
    desc = hq.LayerDesc(K, N, cfg.had_order, a_bits=cfg.a_bits, w_bits=cfg.w_bits,
                        act_gran=cfg.act_gran, centering=cfg.centering, out_order=cfg.out_order)
    X = to_dev_u16(Xb, torch)
    absmax = None
    if cfg.use_sigma:
        absmax = torch.zeros(K, dtype=torch.float32, device="cuda")
        hq.hq_calib_act_absmax(desc, X, absmax)
    layer = hq.HadamardQuantLinear(desc, to_dev_u16(Wb, torch), to_dev_u16(bb, torch), absmax,
                                   cfg.alpha)
    again = hq.HadamardQuantLinear.from_prepared(layer.export_prepared())
    Y1, Y2 = layer(X), again(X)
    assert hq.hq_check_device_error() == 0
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))
