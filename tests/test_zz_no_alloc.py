"""GPU check of hq_quantize_act_noalloc, the quantize entry point for callers
that cannot allocate device memory (fixed-memory runtimes, plugins without an
allocator).  It must give the same results as hq_quantize_act with a
caller-provided workspace, call after call, although every call reuses the
library's one fixed scratch array.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest

import synth
from parity import check_codes, to_dev_u16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def hq():
    from hadamard_rotated_bit_token_b200 import build as hq_build
    hq_build.build()
    import hadamard_rotated_bit_token_b200 as hq_mod
    hq_mod.load_library()
    return hq_mod


def _outputs(T, K):
    return (torch.full((T, K), 0x55, dtype=torch.int8, device="cuda"),
            torch.full((1,), float("nan"), dtype=torch.float32, device="cuda"),
            torch.full((T,), float("nan"), dtype=torch.float32, device="cuda"))


def _noalloc(hq, desc, X, codes, scale, mean):
    """Through the C ABI directly: no workspace argument exists."""
    lib = hq.load_library()
    st = torch.cuda.current_stream().cuda_stream
    return lib.hq_quantize_act_noalloc(ctypes.byref(desc), X.data_ptr(), X.shape[0], None,
                                       codes.data_ptr(), scale.data_ptr(), mean.data_ptr(), st)


@pytest.mark.parametrize("K,n,T,center", [(320, 64, 4099, 0), (1024, 1024, 257, 1)])
def test_noalloc_matches_workspace_entry_point_twice(hq, K, n, T, center):
    desc = hq.LayerDesc(K, 16, n, a_bits=8, w_bits=8, act_gran=hq.HQ_PER_TENSOR_DYNAMIC,
                        centering=center)
    ref_codes, ref_scale, ref_mean = _outputs(T, K)
    ws = torch.empty(hq.hq_quantize_act_workspace_bytes(desc, T), dtype=torch.uint8,
                     device="cuda")
    for call, seed in enumerate((11, 12)):   # two calls in a row, different data
        g = np.random.default_rng(seed)
        x = (g.laplace(0, 1, size=(T, K)) * 10.0 ** g.uniform(-1, 1, size=K)).astype(np.float32)
        X = to_dev_u16(synth.f32_to_bf16_bits(x), torch)
        hq.hq_quantize_act(desc, X, None, ref_codes, ref_scale, ref_mean, ws)
        codes, scale, mean = _outputs(T, K)
        assert _noalloc(hq, desc, X, codes, scale, mean) == 0
        assert hq.hq_check_device_error() == 0
        c, rc = codes.cpu().numpy(), ref_codes.cpu().numpy()
        # same kernels on the same data: identical (tie tolerance kept for the record)
        check_codes(c, rc, np.full(c.shape, 0.0), f"call {call}")
        assert np.array_equal(c, rc)
        assert scale.item() == ref_scale.item() and scale.item() > 0
        assert torch.equal(mean, ref_mean)


def test_noalloc_per_token_needs_no_scratch(hq):
    K, n, T = 1152, 128, 300
    desc = hq.LayerDesc(K, 16, n, a_bits=4, act_gran=hq.HQ_PER_TOKEN)
    X = to_dev_u16(synth.make_x(synth.CONFIGS[2].with_tokens(T)), torch)
    a = torch.empty((T, K), dtype=torch.int8, device="cuda")
    b = torch.empty((T, K), dtype=torch.int8, device="cuda")
    sa, sb = (torch.empty(T, dtype=torch.float32, device="cuda") for _ in range(2))
    ma, mb = (torch.empty(T, dtype=torch.float32, device="cuda") for _ in range(2))
    hq.hq_quantize_act(desc, X, None, a, sa, ma)
    hq.hq_quantize_act_noalloc(desc, X, None, b, sb, mb)
    assert hq.hq_check_device_error() == 0
    assert torch.equal(a, b) and torch.equal(sa, sb) and torch.equal(ma, mb)
