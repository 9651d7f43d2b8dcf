"""Host-side checks of the C ABI (no GPU needed): the library builds and loads,
exports every entry point include/hq.h declares, and rejects bad arguments
with the documented status codes before touching the device."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def hq():
    from hadamard_rotated_bit_token_b200 import build as hq_build
    hq_build.build()
    import hadamard_rotated_bit_token_b200 as hq_mod
    hq_mod.load_library()
    return hq_mod


def declared_functions():
    names = set()
    for hdr in sorted(glob.glob(os.path.join(ROOT, "include", "*.h"))):
        text = re.sub(r"/\*.*?\*/", "", open(hdr).read(), flags=re.S)
        names |= set(re.findall(r"\b(hq_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_every_declared_symbol_is_exported(hq):
    names = declared_functions()
    assert "hq_quantize_act" in names and "hq_linear" in names and "hq_prepare_weights" in names
    assert "hq_gw_quantize_act" in names and "hq_gw_linear" in names
    lib = hq.load_library()
    for name in names:
        assert hasattr(lib, name), name
    assert set(hq.EXPORTED) >= set(names)


def test_version_and_status_strings(hq):
    assert hq.hq_version() == 10400
    for code, name in hq.STATUS_NAMES.items():
        assert hq.hq_status_string(code) == name
    assert hq.hq_status_string(99) == "HQ_ERR_UNKNOWN"


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every call below fails validation


def _call_quant(hq, desc, X=FAKE, T=4, codes=FAKE, scale=FAKE, ws=None, ws_bytes=0):
    lib = hq.load_library()
    d = None if desc is None else ctypes.byref(desc)
    return lib.hq_quantize_act(d, X, T, None, codes, scale, None, ws, ws_bytes, None)


def test_quantize_validation(hq):
    D = hq.LayerDesc
    assert _call_quant(hq, None) == 1
    assert _call_quant(hq, D(1024, 16, 1024), X=None) == 1
    assert _call_quant(hq, D(1024, 16, 1024), T=-1) == 1
    assert _call_quant(hq, D(1024, 16, 1000)) == 2          # order not a power of two
    assert _call_quant(hq, D(1024, 16, 2048)) == 2          # order above 1024
    assert _call_quant(hq, D(1024, 16, 8)) == 2             # order below 16
    assert _call_quant(hq, D(1000, 16, 8)) == 2
    assert _call_quant(hq, D(96, 16, 64)) == 2              # K not a multiple of the order
    assert _call_quant(hq, D(16384, 16, 1024)) == 2         # K above the limit (15360)
    # K: a multiple of 16 and of the order; up to 15360 with a rotation, 10240
    # without one
    assert _call_quant(hq, D(80, 16, 16), T=0) == 0
    assert _call_quant(hq, D(80, 16, 1, centering=0), T=0) == 0
    assert _call_quant(hq, D(88, 16, 8)) == 2                  # K not a multiple of 16
    assert _call_quant(hq, D(12288, 16, 1024), T=0) == 0
    assert _call_quant(hq, D(15360, 16, 1024), T=0) == 0
    assert _call_quant(hq, D(15872, 16, 512)) == 2
    assert _call_quant(hq, D(10240, 16, 1, centering=0), T=0) == 0
    assert _call_quant(hq, D(10496, 16, 1, centering=0)) == 2
    # two codes per byte need rows of whole 16-byte units (K a multiple of 32)
    assert _call_quant(hq, D(80, 16, 16, code_format=1)) == 2
    assert _call_quant(hq, D(1024, 15, 1024)) == 2          # N not a multiple of 16
    assert _call_quant(hq, D(1024, 16, 1024, a_bits=5)) == 2
    assert _call_quant(hq, D(1024, 16, 1024, w_bits=3)) == 2
    assert _call_quant(hq, D(1024, 16, 1024, act_gran=7)) == 1
    assert _call_quant(hq, D(1024, 16, 1024, centering=3)) == 1
    # packed codes: 3- and 4-bit activations only; other formats unknown
    assert _call_quant(hq, D(1024, 16, 1024, code_format=1), T=0) == 0
    assert _call_quant(hq, D(1024, 16, 1024, a_bits=3, code_format=1), T=0) == 0
    assert _call_quant(hq, D(1024, 16, 1024, a_bits=8, code_format=1)) == 2
    assert _call_quant(hq, D(1024, 16, 1024, code_format=2)) == 2
    assert _call_quant(hq, D(1024, 16, 1024, code_format=-1)) == 2
    assert _call_quant(hq, D(1024, 16, 1024), X=FAKE + 2) == 3   # misaligned
    assert _call_quant(hq, D(1024, 16, 1024), codes=FAKE + 8) == 3
    # per-tensor dynamic needs its workspace
    assert _call_quant(hq, D(1024, 16, 1024, act_gran=1)) == 1
    assert _call_quant(hq, D(1024, 16, 1024, act_gran=1), ws=FAKE + 4, ws_bytes=16) == 3
    # T = 0 with valid arguments is a no-op that never touches the device
    assert _call_quant(hq, D(1024, 16, 1024), T=0) == 0
    # had_order 1: no rotation along K, only without centering
    assert _call_quant(hq, D(1024, 16, 1, centering=0), T=0) == 0
    assert _call_quant(hq, D(1024, 16, 1, centering=1)) == 2
    assert _call_quant(hq, D(1024, 16, 1, centering=2)) == 2
    # weight-only Hadamard form (out_order > 1): had_order 1, no centering, N % out_order == 0
    assert _call_quant(hq, D(1024, 64, 1, centering=0, out_order=64), T=0) == 0
    assert _call_quant(hq, D(1024, 64, 1, centering=0, out_order=1), T=0) == 0
    assert _call_quant(hq, D(1024, 64, 1024, centering=0, out_order=64)) == 2
    assert _call_quant(hq, D(1024, 64, 1, centering=1, out_order=64)) == 2
    assert _call_quant(hq, D(1024, 48, 1, centering=0, out_order=32)) == 2
    assert _call_quant(hq, D(1024, 64, 1, centering=0, out_order=8)) == 2
    assert _call_quant(hq, D(1024, 64, 1, centering=0, out_order=128)) == 2
    assert _call_quant(hq, D(1024, 64, 1, centering=0, out_order=-1)) == 1


def test_workspace_bytes(hq):
    lib = hq.load_library()
    assert lib.hq_quantize_act_workspace_bytes(ctypes.byref(hq.LayerDesc(64, 16, 64)), 10) == 0
    d = hq.LayerDesc(64, 16, 64, act_gran=hq.HQ_PER_TENSOR_DYNAMIC)
    assert lib.hq_quantize_act_workspace_bytes(ctypes.byref(d), 10) == 16


def test_linear_validation(hq):
    lib = hq.load_library()
    D = hq.LayerDesc

    def call(desc, T=8, a=FAKE, sx=FAKE, m=None, w=FAKE, sw=FAKE, cs=None, b=None, y=FAKE, acc=None):
        d = None if desc is None else ctypes.byref(desc)
        return lib.hq_linear(d, T, a, sx, m, w, sw, cs, b, y, acc, None)

    assert call(None) == 1
    assert call(D(1024, 16, 1024), T=-3) == 1
    assert call(D(1024, 16, 1024), a=None) == 1
    assert call(D(1024, 16, 1024), m=FAKE) == 1            # mean without colsum
    assert call(D(1000, 16, 8)) == 2                       # K not a multiple of 16
    assert call(D(1024, 24, 1024)) == 2                    # N not a multiple of 16
    assert call(D(1024, 16, 1024), y=FAKE + 2) == 3
    assert call(D(1024, 16, 1024), sw=FAKE + 4) == 3
    assert call(D(1024, 16, 1024), T=0) == 0
    wh = dict(centering=0, out_order=64)
    assert call(D(1024, 128, 1, **wh), T=0) == 0
    assert call(D(1024, 128, 1, **wh), m=FAKE, cs=FAKE) == 1   # the form has no centering
    assert call(D(1024, 80, 1, **wh)) == 2                     # N not a multiple of out_order
    assert call(D(1024, 128, 1, centering=0, out_order=48)) == 2
    assert call(D(1024, 128, 1, centering=0, out_order=-2)) == 1
    # packed activation codes: at most 4 bits, K / 2 bytes a multiple of 16
    assert call(D(1024, 16, 1024, code_format=1), T=0) == 0
    assert call(D(1024, 16, 1024, a_bits=8, code_format=1)) == 2
    assert call(D(1040, 16, 16, code_format=1)) == 2
    assert call(D(1024, 16, 1024, code_format=5)) == 2


def test_forward_host_validation(hq):
    """hq_forward_host checks both calls' arguments and its own before it
    enqueues anything."""
    lib = hq.load_library()
    D = hq.LayerDesc

    def call(desc, T=4096, Xh=FAKE, Xd=FAKE, a=FAKE, sx=FAKE, m=None, ws=None, wsb=0, w=FAKE,
             sw=FAKE, cs=FAKE, b=None, yd=FAKE, yh=FAKE, chunks=4):
        d = None if desc is None else ctypes.byref(desc)
        return lib.hq_forward_host(d, Xh, T, Xd, None, a, sx, m, ws, wsb, w, sw, cs, b, yd, yh,
                                   chunks, None)

    assert call(None) == 1
    assert call(D(1024, 16, 1024), T=-1) == 1
    assert call(D(1024, 16, 1024), Xh=None) == 1
    assert call(D(1024, 16, 1024), yh=None) == 1
    assert call(D(1024, 16, 1024), w=None) == 1
    assert call(D(1024, 16, 1024), chunks=0) == 1
    assert call(D(1024, 16, 1024), chunks=65) == 1
    assert call(D(1024, 16, 1000)) == 2
    assert call(D(1024, 16, 1024), Xd=FAKE + 2) == 3
    assert call(D(1024, 16, 1024), yd=FAKE + 8) == 3
    assert call(D(1024, 16, 1024), T=0) == 0
    # packed codes: only 3- and 4-bit activations; unknown formats refused
    assert call(D(1024, 16, 1024, a_bits=8, code_format=1)) == 2
    assert call(D(1024, 16, 1024, code_format=7)) == 2
    assert call(D(1024, 16, 1024, code_format=1), T=0) == 0


def test_layer_desc_layout_matches_the_header(hq):
    """The binding's struct has the header's fields, in order, all int32."""
    text = open(os.path.join(ROOT, "include", "hq.h")).read()
    body = re.search(r"typedef struct hq_layer_desc \{(.*?)\} hq_layer_desc;", text, re.S).group(1)
    names = []
    for line in body.strip().splitlines():
        decl = line.strip().rstrip(";")
        assert decl.startswith("int32_t ")
        names += [n.strip() for n in decl[len("int32_t "):].split(",")]
    assert [f[0] for f in hq.LayerDesc._fields_] == names
    assert all(f[1] is ctypes.c_int32 for f in hq.LayerDesc._fields_)
    assert ctypes.sizeof(hq.LayerDesc) == 4 * len(names)


def test_enum_constants_match_the_header(hq):
    """Every HQ_* enumerator and status code in the header has the same value
    in the binding."""
    text = open(os.path.join(ROOT, "include", "hq.h")).read()
    pairs = re.findall(r"\b(HQ_[A-Z0-9_]+)\s*=\s*(\d+)", text)
    assert len(pairs) >= 20
    for name, value in pairs:
        if name.startswith("HQ_ERR_") or name == "HQ_OK":
            assert hq.STATUS_NAMES[int(value)] == name
        else:
            assert getattr(hq, name) == int(value), name


def test_prepare_and_calib_validation(hq):
    lib = hq.load_library()
    D = hq.LayerDesc
    d = D(1024, 16, 1024)
    assert lib.hq_prepare_weights(ctypes.byref(d), None, None, None, 0.5, FAKE, FAKE, FAKE, FAKE,
                                  FAKE, None) == 1
    assert lib.hq_prepare_weights(ctypes.byref(d), FAKE, None, None, 1.5, FAKE, FAKE, FAKE, FAKE,
                                  FAKE, None) == 1
    assert lib.hq_prepare_weights(ctypes.byref(d), FAKE + 2, None, None, 0.5, FAKE, FAKE, FAKE,
                                  FAKE, FAKE, None) == 3
    assert lib.hq_calib_act_absmax(None, FAKE, 4, FAKE, None) == 1
    assert lib.hq_calib_act_absmax(ctypes.byref(D(100, 16, 16)), FAKE, 4, FAKE, None) == 2
    assert lib.hq_calib_act_absmax(ctypes.byref(d), FAKE, 0, FAKE, None) == 0
    assert lib.hq_debug_inject_fault(9) == 1
    assert lib.hq_debug_inject_fault(0) == 0
    assert lib.hq_debug_set_wait_limit(0) == 0
    assert lib.hq_debug_set_gemm_variant(3) == 1
    assert lib.hq_debug_set_gemm_variant(-1) == 1
    for v in (hq.HQ_GEMM_CTA_PAIR, hq.HQ_GEMM_SINGLE_CTA, hq.HQ_GEMM_AUTO):
        assert lib.hq_debug_set_gemm_variant(v) == 0


def test_binding_rejects_host_tensors(hq):
    torch = pytest.importorskip("torch")
    d = hq.LayerDesc(64, 16, 64)
    with pytest.raises(ValueError):
        hq.hq_quantize_act(d, torch.zeros((2, 64), dtype=torch.bfloat16), None,
                           torch.zeros((2, 64), dtype=torch.int8), torch.zeros(2), None, None,
                           stream=0)


def test_library_has_no_cpu_fallback():
    """The product package neither imports nor runs the oracle."""
    pkg = os.path.join(ROOT, "hadamard_rotated_bit_token_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "hq_oracle" not in text and "liboracle" not in text, f


def test_gw_desc_layout_matches_the_header(hq):
    """The binding's GwDesc has hq_gw_desc's fields, in order, all int32."""
    text = open(os.path.join(ROOT, "include", "hq_gw.h")).read()
    body = re.search(r"typedef struct hq_gw_desc \{(.*?)\} hq_gw_desc;", text, re.S).group(1)
    names = [re.match(r"\s*int32_t (\w+);", line).group(1)
             for line in body.strip().splitlines()]
    assert [f[0] for f in hq.GwDesc._fields_] == names
    assert all(f[1] is ctypes.c_int32 for f in hq.GwDesc._fields_)


def _gw_quant(hq, desc, X=FAKE, T=4, codes=FAKE, scale=FAKE, l1s=FAKE, u=FAKE):
    lib = hq.load_library()
    d = None if desc is None else ctypes.byref(desc)
    return lib.hq_gw_quantize_act(d, X, T, None, l1s, codes, scale, u, None, 0, None)


def _gw_linear(hq, desc, T=4, a=FAKE, sa=FAKE, u=FAKE, w=FAKE, sw=FAKE, l2=FAKE, Y=FAKE):
    lib = hq.load_library()
    return lib.hq_gw_linear(ctypes.byref(desc), T, a, sa, u, w, sw, l2, None, Y, None)


def test_gw_validation(hq):
    """Every group-wise entry rejects bad descriptions, pointers and sizes
    before touching the device (so these run without a GPU)."""
    G = hq.GwDesc
    assert _gw_quant(hq, None) == 1
    assert _gw_quant(hq, G(1024, 16), X=None) == 1
    assert _gw_quant(hq, G(1024, 16), T=-1) == 1
    assert _gw_quant(hq, G(1024, 16), X=FAKE + 8) == 3          # misaligned
    assert _gw_quant(hq, G(1024, 16, rank=32), u=None) == 1     # branch without u
    assert _gw_quant(hq, G(1000, 16)) == 2                      # K not whole groups
    assert _gw_quant(hq, G(16384 + 64, 16)) == 2                # K above 16384
    assert _gw_quant(hq, G(1024, 16, group=128)) == 2           # group other than 64
    assert _gw_quant(hq, G(1024, 16, rank=16)) == 2             # rank other than 0 / 32
    assert _gw_quant(hq, G(1024, 16, a_bits=8)) == 2            # codes beyond e4m3's integers
    assert _gw_quant(hq, G(1024, 16, a_bits=1)) == 2
    assert _gw_quant(hq, G(1024, 16), T=0) == 0                 # no-op
    assert _gw_linear(hq, G(1024, 24)) == 2                     # N not a multiple of 16
    assert _gw_linear(hq, G(1024, 16), Y=None) == 1
    assert _gw_linear(hq, G(1024, 16), sw=FAKE + 4) == 3
    assert _gw_linear(hq, G(1024, 16, rank=0), u=None, l2=None, T=0) == 0
    lib = hq.load_library()
    assert lib.hq_gw_prepare_weights(ctypes.byref(G(1024, 16)), FAKE, None, None, None, None,
                                     FAKE, FAKE, None, None, FAKE, None) == 1  # rank 32, no factors
    assert lib.hq_gw_sigma_inv(ctypes.byref(G(1024, 16)), FAKE, None, 1.5, FAKE, None) == 1
    assert hq.hq_gw_scale_ld(0) == 0 and hq.hq_gw_scale_ld(5) == 8 and hq.hq_gw_scale_ld(8) == 8
    # workspace: two fp32 parts of u per token and a ticket per 128-token block
    assert hq.hq_gw_quantize_act_workspace_bytes(G(1024, 16), 300) == 2 * 300 * 32 * 4 + 16
    assert hq.hq_gw_quantize_act_workspace_bytes(G(1024, 16, rank=0), 300) == 0
    assert lib.hq_gw_quantize_act(ctypes.byref(G(1024, 16)), FAKE, 4, None, FAKE, FAKE, FAKE,
                                  FAKE, FAKE + 4, 1 << 20, None) == 3  # misaligned workspace
