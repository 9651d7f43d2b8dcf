"""Seeded synthetic inputs for the Hadamard-domain quantized linear layer.

This module only draws data: it holds none of the layer's arithmetic, and both
the CUDA path (tests, benchmark) and the CPU oracle receive the same arrays
from it.  bf16 tensors are returned as uint16 bit patterns (round-half-to-even
from float32).

Workloads (shapes and distributions of the pages' settings; the pages' own
models and datasets are not available, these stand in for them):

  1 single HadaNorm linear          T=256   K=1024 N=1024  n=1024  A4/W4 per token, centred
  2 PixArt-Sigma-shaped qkv         T=8192  K=1152 N=3456  n=128   A4/W4 per token, centred
  3 DiT MLP fc2, W4A3 setting       T=8192  K=4608 N=1152  n=256   A3/W4 per token, centred and not
  4 LIC 1x1 conv, W8A8 double-H     T=65536 K=320  N=320   n=64    A8 per tensor / W8, not centred, sigma = 1
  5 large DiT linear                T=16384 K=3072 N=12288 n=1024  A4/W4 per token, centred

Recipe (seed = config number): numpy PCG64 generator; X base draw, then the
outlier channels (chosen without replacement) are multiplied, then a per-token
offset is added to every channel of the token.  W ~ N(0, 0.02), b ~ N(0, 0.01).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    index: int
    name: str
    T: int
    K: int
    N: int
    had_order: int
    a_bits: int
    w_bits: int
    act_gran: int          # 0 per token, 1 per tensor dynamic, 2 per tensor static
    centering: int         # 1 per-token mean of the rotated activations, 0 none
    use_sigma: bool        # False: sigma = 1 (double-Hadamard form)
    alpha: float
    x_kind: str            # "normal", "gelu", "laplace"
    x_std: float
    outlier_frac: float
    outlier_count: int
    outlier_mult: float
    offset_std: float
    out_order: int = 0     # > 1: the weight-only Hadamard form (had_order 1, W rotated along N)
    code_format: int = 0   # 1: activation codes two per byte (3- and 4-bit codes only)

    def with_tokens(self, T: int) -> "LayerConfig":
        return dataclasses.replace(self, T=T)

    def workload(self) -> str:
        rot = f"WH{self.out_order}" if self.out_order > 1 else f"H{self.had_order}"
        return (f"cfg{self.index}:{self.name}:T{self.T}xK{self.K}xN{self.N}"
                f":{rot}:A{self.a_bits}W{self.w_bits}" + (":packed" if self.code_format else ""))

    def code_bytes(self) -> float:
        """Bytes per activation code as stored: 1, or 1/2 when packed."""
        return 0.5 if self.code_format else 1.0

    def packed(self) -> "LayerConfig":
        """The same layer with its 3- or 4-bit activation codes two per byte."""
        if self.a_bits > 4:
            raise ValueError("packed codes hold 3- and 4-bit activations only")
        return dataclasses.replace(self, code_format=1)

    def weight_only(self, out_order: int) -> "LayerConfig":
        """The same layer shape and inputs in the weight-only Hadamard form:
        no rotation along K, no centering, no smoothing, W rotated along N in
        blocks of out_order."""
        return dataclasses.replace(self, had_order=1, centering=0, use_sigma=False,
                                   out_order=out_order)


CONFIGS = {
    1: LayerConfig(1, "single_hadanorm_linear", 256, 1024, 1024, 1024, 4, 4, 0, 1, True, 0.5,
                   "normal", 1.0, 0.0, 8, 50.0, 2.0),
    2: LayerConfig(2, "pixart_sigma_qkv", 8192, 1152, 3456, 128, 4, 4, 0, 1, True, 0.5,
                   "normal", 1.0, 0.01, 0, 30.0, 1.5),
    3: LayerConfig(3, "dit_mlp_fc2_w4a3", 8192, 4608, 1152, 256, 3, 4, 0, 1, True, 0.5,
                   "gelu", 1.5, 0.01, 0, 20.0, 0.0),
    4: LayerConfig(4, "lic_1x1_conv_w8a8_dh", 65536, 320, 320, 64, 8, 8, 1, 0, False, 0.5,
                   "laplace", 1.0, 0.0, 0, 1.0, 0.0),
    5: LayerConfig(5, "large_dit_linear", 16384, 3072, 12288, 1024, 4, 4, 0, 1, True, 0.5,
                   "normal", 1.0, 0.005, 0, 50.0, 1.5),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float -> bf16 bit pattern, round half to even (via float32)."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    out = rounded.astype(np.uint16)
    nan = np.isnan(f)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _gelu_erf(x: np.ndarray) -> np.ndarray:
    from scipy.special import erf  # data distribution only
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([seed, stream]))


def make_x(cfg: LayerConfig, T: int | None = None, seed: int | None = None) -> np.ndarray:
    """Activations X [T, K] as bf16 bits."""
    T = cfg.T if T is None else T
    seed = cfg.index if seed is None else seed
    g = _rng(seed, 1)
    K = cfg.K
    if cfg.x_kind == "normal":
        x = g.standard_normal((T, K), dtype=np.float32) * np.float32(cfg.x_std)
    elif cfg.x_kind == "gelu":
        x = _gelu_erf(g.standard_normal((T, K), dtype=np.float32).astype(np.float64)
                      * cfg.x_std).astype(np.float32)
    elif cfg.x_kind == "laplace":
        x = g.laplace(0.0, 1.0, size=(T, K)).astype(np.float32)
        chan = 10.0 ** g.uniform(-1.0, 1.0, size=K)
        x *= chan.astype(np.float32)[None, :]
    else:
        raise ValueError(cfg.x_kind)
    n_out = cfg.outlier_count or int(round(cfg.outlier_frac * K))
    if n_out > 0 and cfg.outlier_mult != 1.0:
        idx = g.choice(K, size=n_out, replace=False)
        x[:, idx] *= np.float32(cfg.outlier_mult)
    if cfg.offset_std > 0.0:
        off = g.standard_normal((T, 1), dtype=np.float32) * np.float32(cfg.offset_std)
        x += off
    return f32_to_bf16_bits(x)


def make_w(cfg: LayerConfig, seed: int | None = None) -> tuple[np.ndarray, np.ndarray]:
    """Weight W [N, K] (nn.Linear orientation) and bias b [N], bf16 bits."""
    seed = cfg.index if seed is None else seed
    g = _rng(seed, 2)
    w = g.standard_normal((cfg.N, cfg.K), dtype=np.float32) * np.float32(0.02)
    b = g.standard_normal(cfg.N, dtype=np.float32) * np.float32(0.01)
    return f32_to_bf16_bits(w), f32_to_bf16_bits(b)


def make_layer(cfg: LayerConfig, T: int | None = None, seed: int | None = None):
    X = make_x(cfg, T=T, seed=seed)
    W, b = make_w(cfg, seed=seed)
    return X, W, b


def sample_rows(T: int, count: int, tile: int = 128, seed: int = 0) -> np.ndarray:
    """Seeded sorted row sample touching every `tile`-row block, plus the last row."""
    g = _rng(seed, 3)
    count = min(count, T)
    per_tile = max(1, count // max(1, (T + tile - 1) // tile))
    rows = []
    for t0 in range(0, T, tile):
        hi = min(T, t0 + tile)
        rows.extend(g.choice(np.arange(t0, hi), size=min(per_tile, hi - t0), replace=False))
    rows.append(T - 1)
    return np.unique(np.asarray(rows, dtype=np.int64))


def random_bf16(shape, seed: int, std: float = 1.0) -> np.ndarray:
    g = _rng(seed, 9)
    return f32_to_bf16_bits(g.standard_normal(shape, dtype=np.float32) * np.float32(std))
