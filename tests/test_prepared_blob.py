"""The prepared-weights blob (HadamardQuantLinear.export_prepared /
from_prepared): format round trip and rejection of damaged blobs on the CPU;
on the GPU, a reloaded layer gives the same output bit for bit."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")


def _cpu_layer(hq, K=64, N=32, seed=0, **desc_kw):
    g = np.random.default_rng(seed)
    lay = hq.HadamardQuantLinear.__new__(hq.HadamardQuantLinear)
    lay.desc = hq.LayerDesc(K, N, 16, **desc_kw)
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
