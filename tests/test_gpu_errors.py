"""Documented refusals on a device: misaligned pointers, shapes a forced
variant cannot take, a too-small PREMIX workspace. Each returns its negative
status before anything is launched (the library's launch counter does not
move) and leaves the device usable."""
import pytest
import torch

import dynamic_convolution_b200 as dc
from dynamic_convolution_b200 import synth

from .gpu_util import Layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def layer():
    from dynamic_convolution_b200 import build
    build.build()
    cfg = synth.LayerConfig("err_case", synth.BF16, 2, 64, 128, 8, 8, 3, 3, 1, 1, 1, 4,
                            synth.SOFTMAX, 1.0)
    L = Layer(synth.make_inputs(cfg, seed=3))
    L.route()
    torch.cuda.synchronize()
    return L


def _refused(status, expected):
    assert status == expected, (dc.dynconv_status_string(status), dc.dynconv_last_error())


@pytest.mark.parametrize("variant", [dc.VARIANT_FUSED, dc.VARIANT_OUTSIDE, dc.VARIANT_PREMIX])
def test_misaligned_pointers(layer, variant):
    L = layer
    d = L.desc(variant)
    ws = torch.empty(dc.dynconv_workspace_size(d) + 64, dtype=torch.uint8, device="cuda")
    wsb = dc.dynconv_workspace_size(d)
    # views 2 bytes past a 16-byte boundary
    x_off = torch.empty(L.x.numel() + 8, dtype=torch.bfloat16, device="cuda")[1:1 + L.x.numel()]
    y_off = torch.empty(L.y.numel() + 8, dtype=torch.bfloat16, device="cuda")[1:1 + L.y.numel()]
    n0 = dc.dynconv_launch_count()
    _refused(dc.dynconv_forward(d, x_off, L.experts, L.alpha, L.bias, L.y, ws, wsb),
             dc.ERR_MISALIGNED)
    _refused(dc.dynconv_forward(d, L.x, L.experts, L.alpha, L.bias, y_off, ws, wsb),
             dc.ERR_MISALIGNED)
    if variant == dc.VARIANT_PREMIX:
        _refused(dc.dynconv_forward(d, L.x, L.experts, L.alpha, L.bias, L.y, ws[1:], wsb),
                 dc.ERR_MISALIGNED)
    assert dc.dynconv_launch_count() == n0
    assert dc.dynconv_device_status(None) == dc.OK


def test_premix_workspace_too_small(layer):
    L = layer
    d = L.desc(dc.VARIANT_PREMIX)
    need = dc.dynconv_workspace_size(d)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    n0 = dc.dynconv_launch_count()
    _refused(dc.dynconv_forward(d, L.x, L.experts, L.alpha, L.bias, L.y, ws, need - 256),
             dc.ERR_WORKSPACE)
    _refused(dc.dynconv_forward(d, L.x, L.experts, L.alpha, L.bias, L.y, None, 0),
             dc.ERR_WORKSPACE)
    assert dc.dynconv_launch_count() == n0


@pytest.mark.parametrize("kw", [dict(stride=2), dict(groups=2, C_in=64, C_out=128),
                                dict(dtype=synth.F32)])
@pytest.mark.parametrize("variant", [dc.VARIANT_FUSED, dc.VARIANT_OUTSIDE,
                                     dc.VARIANT_DEPTHWISE])
def test_forced_variant_outside_its_shapes(layer, kw, variant):
    """A forced tensor-core or depthwise variant on a shape it does not take
    (stride 2, grouped dense, fp32) is refused; AUTO takes the direct kernel."""
    L = layer
    cfg = L.cfg
    base = dict(B=cfg.B, C_in=cfg.C_in, H=cfg.H, W=cfg.W, C_out=cfg.C_out, KH=3, KW=3,
                stride=1, pad=1, groups=1, n=cfg.n, dtype=synth.BF16)
    base.update(kw)
    d = dc.make_desc(variant=variant, **base)
    n0 = dc.dynconv_launch_count()
    _refused(dc.dynconv_forward(d, L.x, L.experts, L.alpha, L.bias, L.y), dc.ERR_UNSUPPORTED)
    assert dc.dynconv_launch_count() == n0
    assert dc.dynconv_select_variant(dc.make_desc(variant=dc.VARIANT_AUTO, **base)) == \
        dc.VARIANT_DIRECT
