"""Helpers for the GPU parity tests: upload seeded inputs, call the C ABI
through the binding, and compare with the oracle element by element."""
from __future__ import annotations

import numpy as np
import torch

import dynamic_convolution_b200 as dc
from dynamic_convolution_b200 import synth

# Tolerances (written here, used by every GPU test):
#  * bf16 layers: relative Frobenius error <= 5e-3, and max abs error <= 3e-2
#    measured in units of max(1, rms(y_ref)) (the bf16 output rounding alone is
#    up to 2^-9 of |y|, which exceeds 3e-2 in absolute terms once |y| > 16);
#  * fp32 layers: relative Frobenius <= 1e-5 and max abs <= 1e-5 * max|y_ref|;
#  * routing weights: max abs <= 1e-6.
BF16_REL_FRO = 5e-3
BF16_MAX_ABS = 3e-2
F32_REL = 1e-5
ALPHA_ABS = 1e-6


def to_device(a: np.ndarray, dtype: int) -> torch.Tensor:
    if dtype == synth.BF16:
        assert a.dtype == np.uint16
        return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def from_device(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


class Layer:
    """Device copies of one layer's inputs plus output buffers."""

    def __init__(self, inp: synth.LayerInputs):
        cfg = inp.cfg
        self.cfg = cfg
        self.inp = inp
        self.x = to_device(inp.x_store, cfg.dtype)
        self.experts = to_device(inp.experts_store, cfg.dtype)
        self.Wr = torch.from_numpy(inp.Wr).cuda()
        self.br = torch.from_numpy(inp.br).cuda()
        self.bias = torch.from_numpy(inp.bias).cuda()
        self.alpha = torch.full((cfg.B, cfg.n), float("nan"), device="cuda")
        tdt = torch.bfloat16 if cfg.dtype == synth.BF16 else torch.float32
        self.y = torch.full((cfg.B, cfg.H_out, cfg.W_out, cfg.C_out), float("nan"),
                            dtype=tdt, device="cuda")

    def desc(self, variant=dc.VARIANT_AUTO):
        return dc.desc_from_config(self.cfg, variant)

    def route(self, stream=None):
        st = dc.dynconv_route(self.desc(), self.x, self.Wr, self.br, self.cfg.mode, self.cfg.tau,
                              self.alpha, stream)
        dc.check(st, "dynconv_route")

    def forward(self, variant=dc.VARIANT_AUTO, alpha=None, bias="default", workspace=None,
                stream=None):
        a = self.alpha if alpha is None else alpha
        b = self.bias if isinstance(bias, str) else bias
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        st = dc.dynconv_forward(self.desc(variant), self.x, self.experts, a, b, self.y,
                                workspace, ws_bytes, stream)
        dc.check(st, "dynconv_forward")


def compare(y_gpu: np.ndarray, y_ref: np.ndarray, dtype: int) -> dict:
    assert y_gpu.shape == y_ref.shape, (y_gpu.shape, y_ref.shape)
    assert np.isfinite(y_gpu).all(), "unwritten or non-finite outputs"
    diff = y_gpu - y_ref
    rel_fro = float(np.linalg.norm(diff) / max(np.linalg.norm(y_ref), 1e-300))
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    rms = float(np.sqrt(np.mean(y_ref ** 2))) if y_ref.size else 0.0
    out = dict(rel_fro=rel_fro, max_abs=max_abs, rms=rms)
    if dtype == synth.BF16:
        out["ok"] = rel_fro <= BF16_REL_FRO and max_abs <= BF16_MAX_ABS * max(1.0, rms)
    else:
        out["ok"] = rel_fro <= F32_REL and max_abs <= F32_REL * max(float(np.abs(y_ref).max()), 1e-30)
    return out


def alpha_f32_rounded(alpha_f64: np.ndarray) -> np.ndarray:
    """The oracle's routing weights as the fp32 values handed to the GPU forward."""
    return alpha_f64.astype(np.float32).astype(np.float64)
