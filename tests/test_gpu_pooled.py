"""GPU tests of the routing pooled in the previous layer (chained layers):
dynconv_forward_pooled writes y exactly as dynconv_forward does plus partial
channel sums of y as stored; dynconv_route_pooled turns those into the next
layer's routing weights. Checked against fp64 sums of the GPU's own output,
against dynconv_route on that output, and against the oracle's routing of it
(the per-layer parity of a chained block takes the GPU's bf16 output of the
first layer as the oracle's input of the second)."""
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


def _pooled_case(cfg, variant, workspace):
    inp = synth.make_inputs(cfg, seed=7, structured=1.0)
    L = Layer(inp)
    L.route()
    d = L.desc(variant)
    ws = None
    wsb = 0
    if workspace:
        wsb = dc.dynconv_workspace_size(d)
        ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device="cuda")
    parts = dc.dynconv_pool_parts(d, wsb)
    assert parts >= 1
    ysum = torch.full((cfg.B, parts, cfg.C_out), float("nan"), device="cuda")
    dc.check(dc.dynconv_forward_pooled(d, L.x, L.experts, L.alpha, L.bias, L.y, ysum, ws, wsb))
    torch.cuda.synchronize()
    assert dc.dynconv_device_status(None) == dc.OK
    y_pooled = L.y.clone()
    L.y.fill_(float("nan"))
    dc.check(dc.dynconv_forward(d, L.x, L.experts, L.alpha, L.bias, L.y, ws, wsb))
    torch.cuda.synchronize()
    assert torch.equal(y_pooled, L.y), "the pooled forward must store the same y"
    y = from_device(L.y)
    s = from_device(ysum)
    assert np.isfinite(s).all(), "every partial sum is written"
    ref = y.reshape(cfg.B, -1, cfg.C_out).sum(axis=1)
    tot = s.sum(axis=1)
    scale = np.abs(y).reshape(cfg.B, -1, cfg.C_out).sum(axis=1) + 1e-30
    # fp32 sums of at most a few thousand terms: error relative to the sum of |y|
    assert (np.abs(tot - ref) / scale).max() <= 5e-5
    return L, y, s, parts


@pytest.mark.parametrize("variant,workspace", [(dc.VARIANT_FUSED, False),
                                               (dc.VARIANT_OUTSIDE, False),
                                               (dc.VARIANT_PREMIX, True),
                                               (dc.VARIANT_AUTO, True)],
                         ids=["fused", "outside", "premix", "auto"])
@pytest.mark.parametrize("name", ["effnet_expand_1x1", "resnet18_3x3"])
def test_forward_pooled_tensor_core(name, variant, workspace):
    _pooled_case(synth.CONFIGS[name], variant, workspace)


def test_forward_pooled_ragged():
    """Row blocks that do not divide the image, a partial channel tile."""
    cfg = synth.LayerConfig("ragged_pool", synth.BF16, 3, 64, 136, 13, 11, 3, 3, 1, 1, 1, 4,
                            synth.SOFTMAX, 1.0)
    for v, ws in ((dc.VARIANT_FUSED, False), (dc.VARIANT_PREMIX, True)):
        _pooled_case(cfg, v, ws)


@pytest.mark.parametrize("name,variant", [("tiny_fp32", dc.VARIANT_DIRECT),
                                          ("effnet_dw_5x5", dc.VARIANT_DEPTHWISE),
                                          ("effnet_dw_5x5", dc.VARIANT_DIRECT)])
def test_forward_pooled_cuda_core(name, variant):
    _, _, _, parts = _pooled_case(synth.CONFIGS[name], variant, False)
    assert parts == 1


def test_chained_block_routes_from_pooled_sums():
    """C3a -> C3b: the 1x1 expand layer's pooled forward feeds the depthwise
    layer's routing; alpha equals dynconv_route on the stored output (fp32, up
    to summation order) and the oracle's routing of that output; the depthwise
    forward with it matches the oracle on the same input."""
    up = synth.CONFIGS["effnet_expand_1x1"]
    dw = synth.CONFIGS["effnet_dw_5x5"]
    L, y_up, s, parts = _pooled_case(up, dc.VARIANT_AUTO, True)
    ysum = torch.from_numpy(s.astype(np.float32)).cuda()
    inp_dw = synth.make_inputs(dw)
    Wr = torch.from_numpy(inp_dw.Wr).cuda()
    br = torch.from_numpy(inp_dw.br).cuda()
    d_dw = dc.desc_from_config(dw)
    a_pool = torch.full((dw.B, dw.n), float("nan"), device="cuda")
    dc.check(dc.dynconv_route_pooled(d_dw, ysum, parts, Wr, br, dw.mode, dw.tau, a_pool))
    a_direct = torch.full((dw.B, dw.n), float("nan"), device="cuda")
    dc.check(dc.dynconv_route(d_dw, L.y, Wr, br, dw.mode, dw.tau, a_direct))
    torch.cuda.synchronize()
    ap, ad = from_device(a_pool), from_device(a_direct)
    assert np.abs(ap - ad).max() <= ALPHA_ABS
    a_ref = oracle.route(y_up, inp_dw.Wr, inp_dw.br, dw.mode, dw.tau)
    assert np.abs(ap - a_ref).max() <= ALPHA_ABS
    # the depthwise layer on the GPU's own stored output, with the pooled alpha
    y_dw = torch.full((dw.B, dw.H_out, dw.W_out, dw.C_out), float("nan"), dtype=torch.bfloat16,
                      device="cuda")
    E = torch.from_numpy(inp_dw.experts_store).view(torch.bfloat16).cuda()
    bias = torch.from_numpy(inp_dw.bias).cuda()
    dc.check(dc.dynconv_forward(d_dw, L.y, E, a_pool, bias, y_dw))
    torch.cuda.synchronize()
    got = from_device(y_dw)
    a32 = alpha_f32_rounded(ap)
    for b in (0, dw.B // 2, dw.B - 1):
        ref = oracle.forward(y_up, inp_dw.experts_f64, a32, inp_dw.bias, stride=1, pad=dw.pad,
                             groups=dw.groups, samples=(b, 1))[0]
        r = compare(got[b], ref, synth.BF16)
        assert r["ok"], (b, r)


def test_route_pooled_argument_errors():
    dw = synth.CONFIGS["effnet_dw_5x5"]
    d = dc.desc_from_config(dw)
    t = torch.zeros(16, device="cuda")
    assert dc.dynconv_route_pooled(d, None, 1, t, t, 0, 1.0, t) == dc.ERR_INVALID_ARG
    assert dc.dynconv_route_pooled(d, t, 0, t, t, 0, 1.0, t) == dc.ERR_INVALID_ARG
    assert dc.dynconv_route_pooled(d, t, 1, t, t, 1, 0.0, t) == dc.ERR_INVALID_ARG
