"""The library's launch-shape choices (hq_debug_plan: host logic, no GPU):
the quantizer's rows per tile and threads per CTA, and the GEMM kernel and
tile width, for a 148-SM B200 holding 74 CTA-pair clusters."""
import itertools

import pytest

SMS, PAIRS = 148, 74


@pytest.fixture(scope="module")
def hq():
    import hadamard_rotated_bit_token_b200 as hq_mod
    from hadamard_rotated_bit_token_b200 import build as hq_build
    hq_build.build()
    hq_mod.load_library()
    return hq_mod


def _plan(hq, K, N, n, T, **kw):
    return hq.hq_debug_plan(hq.LayerDesc(K, N, n, **kw), T, SMS, PAIRS)


def test_measured_choices_for_the_configurations(hq):
    # config 2: rows of 36 slices span warps (segment kernel): 7-row tiles,
    # 252 consumers in 8 warps plus the producer warp; 192-column GEMM tiles
    assert _plan(hq, 1152, 3456, 128, 8192) == {"quant_rows": 7, "quant_threads": 288,
                                                 "gemm_pair": False, "gemm_bn": 192}
    # config 3: rows of 144 slices; three-row tiles of the one-CTA variant
    # (432 consumers in 14 warps) take 19 tile rounds where one-row tiles of
    # the two-CTA variant take 28; N = 1152 is not a whole number of pair tiles
    p = _plan(hq, 4608, 1152, 256, 8192, a_bits=3)
    assert (p["quant_rows"], p["quant_threads"], p["gemm_pair"], p["gemm_bn"]) == (3, 480, False, 192)
    # ... and with few tokens, where both take one round, the two-CTA variant
    p = _plan(hq, 4608, 1152, 256, 130, a_bits=3)
    assert (p["quant_rows"], p["quant_threads"]) == (1, 192)
    # config 4: rows of 10 slices, three to a warp (warp-row kernel): 24 rows
    # per tile over 8 consumer warps
    p = _plan(hq, 320, 320, 64, 65536, a_bits=8, w_bits=8, act_gran=1, centering=0)
    assert (p["quant_rows"], p["quant_threads"], p["gemm_bn"]) == (24, 288, 192)
    # config 5: three slices a lane, one row per warp, 4 consumer warps;
    # long K over N in whole 256-column tiles takes the CTA pair
    assert _plan(hq, 3072, 12288, 1024, 16384) == {"quant_rows": 4, "quant_threads": 160,
                                                    "gemm_pair": True, "gemm_bn": 256}
    # config 1: one row per warp, 8 consumer warps; one small GEMM wave
    p = _plan(hq, 1024, 1024, 1024, 256)
    assert (p["quant_rows"], p["quant_threads"], p["gemm_bn"]) == (8, 288, 64)


def test_forms_that_exclude_the_pair_or_wide_tiles(hq):
    # packed codes keep A in tensor memory beside two accumulators: <= 192 columns, no pair
    p = _plan(hq, 3072, 12288, 1024, 16384, code_format=1)
    assert not p["gemm_pair"] and p["gemm_bn"] <= 192
    # the weight-only form runs in the single-CTA kernel; 64-column output
    # blocks need whole 64-column halves
    p = _plan(hq, 3072, 12288, 1, 16384, centering=0, out_order=64)
    assert not p["gemm_pair"] and p["gemm_bn"] in (128, 256)
    # no pair clusters on the device: single CTA
    d = hq.LayerDesc(3072, 12288, 1024)
    assert not hq.hq_debug_plan(d, 16384, SMS, 0)["gemm_pair"]


def test_plan_invariants_over_shapes(hq):
    Ks = [64, 320, 1024, 1152, 3072, 4608, 9216, 12288, 15360]
    Ts = [1, 7, 127, 128, 1000, 8192, 65536]
    Ns = [16, 320, 3456, 12288]
    for K, T, N, packed in itertools.product(Ks, Ts, Ns, (0, 1)):
        n = 64 if K % 64 == 0 else 16
        p = _plan(hq, K, N, n, T, code_format=packed)
        S = K // 32
        R, nt = p["quant_rows"], p["quant_threads"]
        assert R >= 1 and nt % 32 == 0
        if S < 32:  # warp-row kernel, several rows per warp, plus the producer warp
            assert R == (nt // 32 - 1) * (32 // S)
        elif S % 32 == 0 and S <= 128:  # warp-row kernel, one row per warp
            assert R == nt // 32 - 1
        else:  # segment kernel: one thread per slice, plus the producer warp
            # (up to 256 slices a tile in the two-CTA variant, 480 in the
            # one-CTA variant, the only one for rows of more than 256 slices)
            assert R * S + 32 <= nt < R * S + 64 and R * S <= 480
        assert p["gemm_bn"] in (64, 128, 192, 256)
        if packed:
            assert not p["gemm_pair"] and p["gemm_bn"] <= 192
        if p["gemm_pair"]:
            assert N % 256 == 0 and p["gemm_bn"] == 256


def _box_ok(RS):
    # one tensor copy of the whole stage, or equal copies of a multiple of 8 rows
    return RS <= 256 or any(RS % b == 0 for b in range(8, 257, 8))


def _rounds(T, R, slots):
    tiles = -(-T // R)
    grid = min(tiles, slots)
    return -(-tiles // grid)


def test_segment_plan_takes_the_fewest_tile_rounds(hq):
    """The segment quantizer is latency-bound, so its plan takes the tile
    shape with the fewest rounds of tiles over the resident CTAs (two CTAs of
    up to 256 consumers an SM, or one of up to 480), the two-CTA variant on a
    tie; never more rounds than another shape that fits."""
    for K in range(1056, 8193, 32 * 7):
        S = K // 32
        if S % 32 == 0 and S <= 128:
            continue  # warp-row kernel
        for T in (1, 100, 1000, 8192, 65536):
            p = _plan(hq, K, 64, 32, T)
            R, nt = p["quant_rows"], p["quant_threads"]
            one_cta = nt > 288
            got = _rounds(T, R, SMS * (1 if one_cta else 2))
            two = [_rounds(T, r, 2 * SMS) for r in range(1, 256 // S + 1) if _box_ok(r * S)]
            one = [_rounds(T, r, SMS) for r in range(1, 480 // S + 1) if _box_ok(r * S)]
            assert got == min(two + one), (K, T, R, nt)
            if one_cta:
                assert not two or min(one) < min(two), (K, T)


def test_plan_validation(hq):
    import ctypes
    lib = hq.load_library()
    D = hq.LayerDesc
    assert lib.hq_debug_plan(None, 8, SMS, PAIRS, None, None, None, None) == 1
    assert lib.hq_debug_plan(ctypes.byref(D(1024, 16, 1024)), 0, SMS, PAIRS, None, None, None,
                             None) == 1
    assert lib.hq_debug_plan(ctypes.byref(D(1024, 16, 1024)), 8, 0, PAIRS, None, None, None,
                             None) == 1
    assert lib.hq_debug_plan(ctypes.byref(D(1000, 16, 8)), 8, SMS, PAIRS, None, None, None,
                             None) == 2
    assert lib.hq_debug_plan(ctypes.byref(D(1024, 16, 1024)), 8, SMS, PAIRS, None, None, None,
                             None) == 0
