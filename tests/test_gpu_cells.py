"""GPU parity of the warehouse-cell path (include/dynconv_cells.h) against the
oracle's kernel cells: dynconv_route_cells (per-cell softmax or sigmoid) and
dynconv_forward_cells (cell mixing, then the convolution on the forward
kernels), on small layers with ragged batches (one-hot chunks of 64 samples
and a tail), depthwise and fp32 layers, with and without bias, and on a
full-size 3x3 layer with a 128-cell warehouse (sampled samples)."""
import numpy as np
import pytest
import torch

import dynamic_convolution_b200 as dc
import oracle
from dynamic_convolution_b200 import synth

from .gpu_util import ALPHA_ABS, alpha_f32_rounded, compare, from_device, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from dynamic_convolution_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _run(cfg, cells, n, bias=True, samples=None, seed=5):
    ci = synth.make_cell_inputs(cfg, cells, n, seed=seed, structured=1.0)
    d = dc.make_desc(cfg.B, cfg.C_in, cfg.H, cfg.W, cfg.C_out, cfg.KH, cfg.KW, cfg.stride,
                     cfg.pad, cfg.groups, n, cfg.dtype)
    x = to_device(ci.x_store, cfg.dtype)
    E = to_device(ci.warehouse_store, cfg.dtype)
    Wr, br = torch.from_numpy(ci.Wr).cuda(), torch.from_numpy(ci.br).cuda()
    alpha = torch.full((cfg.B, cells, n), float("nan"), device="cuda")
    wsb = dc.dynconv_cells_workspace_size(d, cells)
    assert wsb > 0
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    dc.check(dc.dynconv_route_cells(d, cells, x, Wr, br, cfg.mode, cfg.tau, alpha, ws, wsb),
             "route_cells")
    torch.cuda.synchronize()
    a_ref = oracle.route_cells(ci.x_f64, ci.Wr, ci.br, cells, cfg.mode, cfg.tau)
    a_got = from_device(alpha)
    assert np.abs(a_got - a_ref).max() <= ALPHA_ABS, np.abs(a_got - a_ref).max()
    # the forward with the oracle's attentions, as fp32
    a32 = alpha_f32_rounded(a_ref)
    alpha.copy_(torch.from_numpy(a32.astype(np.float32)))
    tdt = torch.bfloat16 if cfg.dtype == synth.BF16 else torch.float32
    y = torch.full((cfg.B, cfg.H_out, cfg.W_out, cfg.C_out), float("nan"), dtype=tdt, device="cuda")
    b = torch.from_numpy(ci.bias).cuda() if bias else None
    dc.check(dc.dynconv_forward_cells(d, cells, x, E, alpha, b, y, ws, wsb), "forward_cells")
    torch.cuda.synchronize()
    assert dc.dynconv_device_status(None) == dc.OK
    got = from_device(y)
    for b0 in (samples or range(cfg.B)):
        ref = oracle.forward_cells(ci.x_f64, ci.warehouse_f64, a32, ci.bias if bias else None,
                                   cfg.C_out, cfg.KH, cfg.KW, cfg.stride, cfg.pad, cfg.groups,
                                   samples=(b0, 1))[0]
        r = compare(got[b0], ref, cfg.dtype)
        assert r["ok"], (cfg.name, b0, r)


LC = synth.LayerConfig
CASES = [
    # ragged: 136 output channels, 13x11, cells of 8 output channels (17 cells)
    (LC("cells_ragged", synth.BF16, 3, 64, 136, 13, 11, 3, 3, 1, 1, 1, 1, synth.SOFTMAX, 1.5), 17, 24),
    # 70 samples: one-hot chunks of 64 and a tail of 6; 120 warehouse cells
    (LC("cells_b70", synth.BF16, 70, 64, 64, 8, 8, 3, 3, 1, 1, 1, 1, synth.SOFTMAX, 1.0), 8, 120),
    # one cell: the ordinary mixture
    (LC("cells_m1", synth.BF16, 4, 64, 96, 10, 10, 3, 3, 1, 1, 1, 1, synth.SIGMOID, 1.0), 1, 6),
    # 1x1, sigmoid attentions, cells of half an output channel
    (LC("cells_1x1", synth.BF16, 5, 64, 48, 9, 9, 1, 1, 1, 0, 1, 1, synth.SIGMOID, 1.0), 96, 16),
    # depthwise 5x5: the depthwise forward kernel, cells of 8 channels
    (LC("cells_dw", synth.BF16, 3, 48, 48, 11, 9, 5, 5, 1, 2, 48, 1, synth.SOFTMAX, 2.0), 6, 32),
    # fp32, stride 2: the direct forward kernel
    (LC("cells_f32", synth.F32, 2, 8, 12, 9, 8, 3, 3, 2, 1, 1, 1, synth.SOFTMAX, 1.0), 4, 10),
]


@pytest.mark.parametrize("cfg,cells,n", CASES, ids=[c[0].name for c in CASES])
def test_cells_small(cfg, cells, n):
    _run(cfg, cells, n)


def test_cells_without_bias():
    cfg, cells, n = CASES[0]
    _run(cfg, cells, n, bias=False)


def test_cells_full_size_3x3_warehouse_128():
    """The 3x3 layer at full size (B=64, 128->128, 28x28) from 16 cells of 8
    output channels each, warehouse of 128 cells; five sampled samples."""
    cfg = synth.CONFIGS["resnet18_3x3"]
    _run(cfg, 16, 128, samples=(0, 1, 31, 62, 63))
