"""The forward entry point that allocates nothing (dynconv_forward_noalloc).

It exists for callers that cannot allocate device memory where they call the
layer -- a plugin or callback of a host framework that owns all device memory
and hands out no workspace, or code that must not call cudaMalloc after
start-up. It runs the mixing-then-convolution (PREMIX) path with the library's
own fixed scratch array instead of a caller workspace, so its output must be
bit-identical to the regular entry point's given a workspace, and it is
compared with the fp64 oracle on sampled whole samples at the same tolerance
as every other bf16 parity test. This file is collected last on purpose; it
passes alone in a fresh process and after the other tests."""
import numpy as np
import pytest
import torch

import dynamic_convolution_b200 as dc
import oracle
from dynamic_convolution_b200 import synth

from .gpu_util import (BF16_MAX_ABS, BF16_REL_FRO, Layer, alpha_f32_rounded, compare,
                       from_device)


def _built():
    from dynamic_convolution_b200 import build
    build.build()
    dc.load()


def _close(a, b):
    rel = np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)
    rms = float(np.sqrt(np.mean(b ** 2)))
    return rel <= BF16_REL_FRO and np.abs(a - b).max() <= BF16_MAX_ABS * max(1.0, rms)


def test_rejects_shapes_beyond_the_builtin_scratch():
    """Checked on the host before anything runs (no GPU needed)."""
    _built()
    cfg = synth.CONFIGS["deep_3x3_tau30"]          # needs 302 MB of scratch
    d = dc.desc_from_config(cfg)
    assert dc.dynconv_workspace_size(d) > dc.NOALLOC_MAX_BYTES
    assert dc.dynconv_forward_noalloc(d, 256, 256, 256, None, 256) == dc.ERR_WORKSPACE
    assert "scratch" in dc.dynconv_last_error()
    assert dc.dynconv_forward_noalloc(d, None, 256, 256, None, 256) == dc.ERR_INVALID_ARG


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["resnet18_3x3", "effnet_expand_1x1"])
def test_noalloc_matches_regular_forward_twice(name):
    _built()
    assert torch.cuda.is_available()
    cfg = synth.CONFIGS[name]
    L = Layer(synth.make_inputs(cfg, seed=4, structured=1.0))
    d = L.desc(dc.VARIANT_PREMIX)
    assert 0 < dc.dynconv_workspace_size(d) <= dc.NOALLOC_MAX_BYTES
    inp = L.inp
    # the oracle's routing weights, as the fp32 values both paths consume
    a64 = alpha_f32_rounded(oracle.route(inp.x_f64, inp.Wr, inp.br, cfg.mode, cfg.tau))
    L.alpha.copy_(torch.from_numpy(a64.astype(np.float32)))
    # regular entry point, caller-provided workspace
    ws = torch.empty(dc.dynconv_workspace_size(d), dtype=torch.uint8, device="cuda")
    dc.check(dc.dynconv_forward(d, L.x, L.experts, L.alpha, L.bias, L.y, ws, ws.numel()),
             "dynconv_forward")
    torch.cuda.synchronize()
    ref = from_device(L.y)
    samples = sorted({0, cfg.B // 2, cfg.B - 1})
    y_oracle = {b: oracle.forward(inp.x_f64, inp.experts_f64, a64, inp.bias, stride=cfg.stride,
                                  pad=cfg.pad, groups=cfg.groups, samples=(b, 1))[0]
                for b in samples}
    # the entry point without scratch, two calls in a row into fresh outputs
    for _ in range(2):
        y = torch.full_like(L.y, float("nan"))
        dc.check(dc.dynconv_forward_noalloc(d, L.x, L.experts, L.alpha, L.bias, y),
                 "dynconv_forward_noalloc")
        assert dc.dynconv_device_status(None) == dc.OK
        got = from_device(y)
        assert np.isfinite(got).all()
        assert _close(got, ref)
        assert torch.equal(y, L.y), "not bit-identical to the PREMIX forward"
        for b, yr in y_oracle.items():
            r = compare(got[b], yr, cfg.dtype)
            assert r["ok"], (name, b, r)
