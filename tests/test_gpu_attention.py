"""GPU parity of the FMDConv channel attentions (input attention, output
attention): dynconv_route_channels against the oracle's routing computation
with one sigmoid output per channel, and dynconv_forward_attn against the
oracle's forward with the per-sample channel factors, for every variant that
takes them; plus the variants that must refuse the input factor."""
import numpy as np
import pytest
import torch

import dynamic_convolution_b200 as dc
import oracle
from dynamic_convolution_b200 import synth

from .gpu_util import ALPHA_ABS, Layer, alpha_f32_rounded, compare, from_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from dynamic_convolution_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _attention_weights(cfg, seed):
    rng = np.random.default_rng(seed)
    Wi = rng.standard_normal((cfg.C_in, cfg.C_in)) / np.sqrt(cfg.C_in)
    bi = rng.standard_normal(cfg.C_in) * 0.1
    Wo = rng.standard_normal((cfg.C_out, cfg.C_in)) / np.sqrt(cfg.C_in)
    bo = rng.standard_normal(cfg.C_out) * 0.1
    return Wi, bi, Wo, bo


def _case(cfg, variant, workspace, use_in=True, use_out=True, seed=21):
    inp = synth.make_inputs(cfg, seed=seed, structured=1.0)
    L = Layer(inp)
    Wi, bi, Wo, bo = _attention_weights(cfg, seed + 1)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()
    a_in = torch.full((cfg.B, cfg.C_in), float("nan"), device="cuda")
    a_out = torch.full((cfg.B, cfg.C_out), float("nan"), device="cuda")
    dc.check(dc.dynconv_route_channels(L.desc(), L.x, dev(Wi), dev(bi), a_in, dev(Wo), dev(bo),
                                       a_out))
    torch.cuda.synchronize()
    ai_ref = oracle.route(inp.x_f64, Wi.astype(np.float32).astype(np.float64),
                          bi.astype(np.float32).astype(np.float64), oracle.SIGMOID, 1.0)
    ao_ref = oracle.route(inp.x_f64, Wo.astype(np.float32).astype(np.float64),
                          bo.astype(np.float32).astype(np.float64), oracle.SIGMOID, 1.0)
    assert np.abs(from_device(a_in) - ai_ref).max() <= ALPHA_ABS
    assert np.abs(from_device(a_out) - ao_ref).max() <= ALPHA_ABS
    # forward with the oracle's (fp32-rounded) attentions
    a = alpha_f32_rounded(oracle.route(inp.x_f64, inp.Wr, inp.br, cfg.mode, cfg.tau))
    ai = alpha_f32_rounded(ai_ref)
    ao = alpha_f32_rounded(ao_ref)
    L.alpha.copy_(torch.from_numpy(a.astype(np.float32)))
    a_in.copy_(torch.from_numpy(ai.astype(np.float32)))
    a_out.copy_(torch.from_numpy(ao.astype(np.float32)))
    d = L.desc(variant)
    ws, wsb = None, 0
    if workspace:
        wsb = dc.dynconv_workspace_size(d)
        ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device="cuda")
    rc = dc.dynconv_forward_attn(d, L.x, L.experts, L.alpha, L.bias, a_in if use_in else None,
                                 a_out if use_out else None, L.y, ws, wsb)
    if rc != dc.OK:
        return rc
    torch.cuda.synchronize()
    assert dc.dynconv_device_status(None) == dc.OK
    y = from_device(L.y)
    for b in sorted({0, cfg.B // 2, cfg.B - 1}):
        ref = oracle.forward_attn(inp.x_f64, inp.experts_f64, a, inp.bias,
                                  ai if use_in else None, ao if use_out else None,
                                  stride=cfg.stride, pad=cfg.pad, groups=cfg.groups,
                                  samples=(b, 1))[0]
        r = compare(y[b], ref, cfg.dtype)
        assert r["ok"], (cfg.name, variant, b, r)
    return rc


@pytest.mark.parametrize("name,variant,workspace", [
    ("resnet18_3x3", dc.VARIANT_PREMIX, True),
    ("effnet_expand_1x1", dc.VARIANT_PREMIX, True),
    ("resnet18_3x3", dc.VARIANT_AUTO, True),
    ("effnet_dw_5x5", dc.VARIANT_DEPTHWISE, False),
    ("tiny_fp32", dc.VARIANT_DIRECT, False),
], ids=["c2-premix", "c3a-premix", "c2-auto", "c3b-depthwise", "c1-direct"])
def test_forward_attn_both_factors(name, variant, workspace):
    assert _case(synth.CONFIGS[name], variant, workspace) == dc.OK


SMALL = [
    synth.LayerConfig("attn_ragged", synth.BF16, 3, 64, 136, 13, 11, 3, 3, 1, 1, 1, 4,
                      synth.SOFTMAX, 1.0),
    synth.LayerConfig("attn_pointwise", synth.BF16, 4, 40, 96, 12, 12, 1, 1, 1, 0, 1, 3,
                      synth.SIGMOID, 1.0),
]


@pytest.mark.parametrize("cfg", SMALL, ids=[c.name for c in SMALL])
@pytest.mark.parametrize("variant", [dc.VARIANT_FUSED, dc.VARIANT_OUTSIDE, dc.VARIANT_PREMIX,
                                     dc.VARIANT_DIRECT])
def test_forward_attn_output_factor_every_variant(cfg, variant):
    assert _case(cfg, variant, variant == dc.VARIANT_PREMIX, use_in=False) == dc.OK


@pytest.mark.parametrize("cfg", SMALL, ids=[c.name for c in SMALL])
@pytest.mark.parametrize("variant", [dc.VARIANT_PREMIX, dc.VARIANT_DIRECT, dc.VARIANT_AUTO])
def test_forward_attn_input_factor(cfg, variant):
    assert _case(cfg, variant, variant != dc.VARIANT_DIRECT, use_out=False) == dc.OK


@pytest.mark.parametrize("variant", [dc.VARIANT_FUSED, dc.VARIANT_OUTSIDE])
def test_forward_attn_input_factor_refused_where_not_folded(variant):
    assert _case(SMALL[0], variant, False) == dc.ERR_UNSUPPORTED


def test_forward_attn_auto_without_workspace_falls_back_to_direct():
    assert _case(SMALL[1], dc.VARIANT_AUTO, False) == dc.OK
