"""Host logic of bench.py's workload overrides (CPU only): the packed-code and
weight-only variants change the description, the algorithmic byte counts
and whether a committed ncu summary applies."""
import pytest

import bench
import synth


def _cfg(*argv):
    return bench.workload_config(bench.parse_args(list(argv)))


def test_default_workload_is_the_configuration_itself():
    cfg = _cfg()
    assert cfg == synth.CONFIGS[bench.DEFAULT_CONFIG]
    assert cfg.code_format == 0
    assert bench.config_block(cfg, 1)["activation_codes"] == "one per byte"


def test_packed_codes_halve_the_code_bytes():
    base, packed = _cfg("--config", "2"), _cfg("--config", "2", "--packed")
    assert packed.code_format == 1 and packed.workload().endswith(":packed")
    assert bench.config_block(packed, 1)["activation_codes"] == "two per byte"
    half = base.T * base.K / 2
    assert bench.quantizer_bytes(base) - bench.quantizer_bytes(packed) == half
    assert bench.gemm_bytes(base) - bench.gemm_bytes(packed) == half
    assert bench.layer_ops(base) == bench.layer_ops(packed)
    # a committed ncu summary describes the configuration as defined only
    assert packed != synth.CONFIGS[2]


def test_packed_codes_need_at_most_four_bits():
    assert _cfg("--config", "3", "--packed").a_bits == 3
    with pytest.raises(ValueError):
        _cfg("--config", "4", "--packed")        # A8 per tensor


def test_weight_only_form_override():
    cfg = _cfg("--config", "2", "--out-order", "64")
    assert (cfg.had_order, cfg.centering, cfg.out_order, cfg.use_sigma) == (1, 0, 64, False)
    assert ":WH64:" in cfg.workload()
    block = bench.config_block(cfg, 1)
    assert block["form"].startswith("weight-only Hadamard")
