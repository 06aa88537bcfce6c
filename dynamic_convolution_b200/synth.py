"""Seeded synthetic inputs for the dynamic-convolution layer configurations.

This module draws random numbers and rounds them to storage types; it holds
none of the method's arithmetic (no pooling, routing, mixing or convolution),
so the CPU oracle and the CUDA path can both take their inputs from it.

Recipe (every layer):
  * generator ``numpy.random.default_rng(seed)``, draws in fp64, in this order:
    x, experts (expert-major), Wr, br, bias;
  * x ~ N(0, 1)  (optionally plus a per-sample, per-channel mean offset drawn
    after everything else, which makes the routing weights differ strongly
    between samples);
  * experts W_i ~ N(0, std^2) with the Kaiming fan-in std sqrt(2 / fan_in),
    fan_in = (C_in/groups) * KH * KW (the large-n layer scales it by 1/sqrt(n));
  * router weights Wr ~ N(0, 1/C_in), router bias br = 0, expert biases
    bias_i ~ N(0, 0.01) (the second argument of N is a variance);
  * x and experts are rounded to the layer's dtype (fp32, or bf16 by
    round-to-nearest-even from fp32); Wr, br and bias are fp32 on every path.
The consumer (oracle or GPU) receives the rounded values, so both sides see
bit-identical inputs.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

SIGMOID = 0
SOFTMAX = 1
F32 = 0
BF16 = 1


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    dtype: int          # F32 or BF16
    B: int
    C_in: int
    C_out: int
    H: int
    W: int
    KH: int
    KW: int
    stride: int
    pad: int
    groups: int
    n: int
    mode: int           # SIGMOID or SOFTMAX
    tau: float
    expert_scale: float = 1.0   # extra factor on the Kaiming std

    @property
    def H_out(self) -> int:
        return (self.H + 2 * self.pad - self.KH) // self.stride + 1

    @property
    def W_out(self) -> int:
        return (self.W + 2 * self.pad - self.KW) // self.stride + 1

    @property
    def Cg(self) -> int:
        return self.C_in // self.groups

    @property
    def weight_elems(self) -> int:
        """|W|: elements of one expert kernel."""
        return self.C_out * self.KH * self.KW * self.Cg

    @property
    def conv_flops(self) -> int:
        """2 * B * H_out * W_out * C_out * (C_in/groups) * KH * KW (conv work only)."""
        return 2 * self.B * self.H_out * self.W_out * self.C_out * self.Cg * self.KH * self.KW

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == F32 else 2

    def scaled(self, **kw) -> "LayerConfig":
        return dataclasses.replace(self, **kw)


# The five layer configurations (the third is a block of two layers).
CONFIGS: dict[str, LayerConfig] = {
    # tiny fp32 CondConv layer
    "tiny_fp32": LayerConfig("tiny_fp32", F32, 2, 8, 8, 8, 8, 3, 3, 1, 1, 1, 4, SIGMOID, 1.0),
    # ResNet-18-style 3x3 layer
    "resnet18_3x3": LayerConfig("resnet18_3x3", BF16, 64, 128, 128, 28, 28, 3, 3, 1, 1, 1, 4,
                                SOFTMAX, 1.0),
    # EfficientNet-B0-style MBConv block: 1x1 expand, then depthwise 5x5
    "effnet_expand_1x1": LayerConfig("effnet_expand_1x1", BF16, 128, 40, 240, 28, 28, 1, 1, 1, 0,
                                     1, 8, SIGMOID, 1.0),
    "effnet_dw_5x5": LayerConfig("effnet_dw_5x5", BF16, 128, 240, 240, 28, 28, 5, 5, 1, 2, 240, 8,
                                 SIGMOID, 1.0),
    # deep 3x3 layer at the start of temperature annealing
    "deep_3x3_tau30": LayerConfig("deep_3x3_tau30", BF16, 256, 256, 256, 14, 14, 3, 3, 1, 1, 1, 16,
                                  SOFTMAX, 30.0),
    # large-n regime
    "large_n64": LayerConfig("large_n64", BF16, 32, 512, 512, 7, 7, 3, 3, 1, 1, 1, 64, SOFTMAX, 1.0,
                             expert_scale=1.0 / 8.0),
}

HEADLINE = "resnet18_3x3"


def bf16_bits(a) -> np.ndarray:
    """Round to bf16 (fp64 -> fp32 RN, then fp32 -> bf16 RN-even); return the uint16 bits."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_to_f64(bits) -> np.ndarray:
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


@dataclasses.dataclass
class LayerInputs:
    """Host arrays for one layer. ``*_store`` hold the exact device storage
    (float32, or uint16 bf16 bits); ``*_f64`` hold the same values upcast."""
    cfg: LayerConfig
    x_store: np.ndarray
    x_f64: np.ndarray
    experts_store: np.ndarray
    experts_f64: np.ndarray
    Wr: np.ndarray      # float32 [n][C_in]
    br: np.ndarray      # float32 [n]
    bias: np.ndarray    # float32 [n][C_out]

    def with_x(self, x_values) -> "LayerInputs":
        """Same parameters, a different input tensor (rounded to the layer dtype)."""
        xs, xf = _round(x_values, self.cfg.dtype)
        return dataclasses.replace(self, x_store=xs, x_f64=xf)


def _round(values, dtype: int):
    if dtype == F32:
        s = np.ascontiguousarray(np.asarray(values, dtype=np.float32))
        return s, s.astype(np.float64)
    s = bf16_bits(values)
    return s, bf16_to_f64(s)


def make_inputs(cfg: LayerConfig, seed: int = 0, structured: float = 0.0) -> LayerInputs:
    """Draw one layer's inputs. ``structured`` > 0 adds a per-(sample, channel)
    mean offset with that std to x (drawn last), so routing differs per sample."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((cfg.B, cfg.H, cfg.W, cfg.C_in))
    fan_in = cfg.Cg * cfg.KH * cfg.KW
    std = math.sqrt(2.0 / fan_in) * cfg.expert_scale
    experts = rng.standard_normal((cfg.n, cfg.C_out, cfg.KH, cfg.KW, cfg.Cg)) * std
    Wr = rng.standard_normal((cfg.n, cfg.C_in)) * math.sqrt(1.0 / cfg.C_in)
    br = np.zeros(cfg.n)
    bias = rng.standard_normal((cfg.n, cfg.C_out)) * 0.1
    if structured > 0.0:
        x = x + rng.standard_normal((cfg.B, 1, 1, cfg.C_in)) * structured
    xs, xf = _round(x, cfg.dtype)
    es, ef = _round(experts, cfg.dtype)
    return LayerInputs(cfg, xs, xf, es, ef, Wr.astype(np.float32), br.astype(np.float32),
                       bias.astype(np.float32))


def make_upstream_grad(cfg: LayerConfig, seed: int = 1):
    """A seeded upstream gradient dy[B][H_out][W_out][C_out] ~ N(0, 1), rounded to
    the layer dtype: (device storage, the same values as float64)."""
    rng = np.random.default_rng(seed)
    return _round(rng.standard_normal((cfg.B, cfg.H_out, cfg.W_out, cfg.C_out)), cfg.dtype)


@dataclasses.dataclass
class CellInputs:
    """Host arrays of one layer built from warehouse cells: the layer's x (as
    make_inputs draws it), a warehouse of n cells of s elements each drawn like
    one expert's elements, the router of cells * n outputs and a static bias."""
    x_store: np.ndarray
    x_f64: np.ndarray
    warehouse_store: np.ndarray   # [n][s]
    warehouse_f64: np.ndarray
    Wr: np.ndarray                # float32 [cells * n][C_in]
    br: np.ndarray                # float32 [cells * n]
    bias: np.ndarray              # float32 [C_out]


def make_cell_inputs(cfg: LayerConfig, cells: int, n: int, seed: int = 0,
                     structured: float = 0.0) -> CellInputs:
    base = make_inputs(cfg, seed=seed, structured=structured)
    rng = np.random.default_rng(seed + 1000)
    wsize = cfg.C_out * cfg.KH * cfg.KW * cfg.Cg
    assert wsize % cells == 0
    std = math.sqrt(2.0 / (cfg.Cg * cfg.KH * cfg.KW)) * cfg.expert_scale
    ws, wf = _round(rng.standard_normal((n, wsize // cells)) * std, cfg.dtype)
    Wr = rng.standard_normal((cells * n, cfg.C_in)) * math.sqrt(1.0 / cfg.C_in)
    br = rng.standard_normal(cells * n) * 0.1
    bias = rng.standard_normal(cfg.C_out) * 0.1
    return CellInputs(base.x_store, base.x_f64, ws, wf, Wr.astype(np.float32),
                      br.astype(np.float32), bias.astype(np.float32))
