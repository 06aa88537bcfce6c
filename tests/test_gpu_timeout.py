"""Failure detection without a GPU fault: a tensor-core forward is told (test
hook) to withhold one producer arrival in its first CTA, so that CTA's MMA
thread waits on a barrier nothing will complete. Its bounded wait (shortened
here to 20 ms) must expire, the kernel must drain its in-flight copies, free
tensor memory and exit, and the host must read DYNCONV_ERR_TIMEOUT from the
device error word. The context stays usable: the next call is correct."""
import numpy as np
import pytest
import torch

import dynamic_convolution_b200 as dc
import oracle
from dynamic_convolution_b200 import synth

from .gpu_util import Layer, alpha_f32_rounded, compare, from_device

pytestmark = pytest.mark.gpu


def _layer():
    cfg = synth.LayerConfig("timeout_case", synth.BF16, 2, 64, 128, 8, 8, 3, 3, 1, 1, 1, 4,
                            synth.SOFTMAX, 1.0)
    inp = synth.make_inputs(cfg, seed=2, structured=1.0)
    L = Layer(inp)
    a = alpha_f32_rounded(oracle.route(inp.x_f64, inp.Wr, inp.br, cfg.mode, cfg.tau))
    L.alpha.copy_(torch.from_numpy(a.astype(np.float32)))
    return L, inp, a


@pytest.mark.parametrize("variant", [dc.VARIANT_FUSED, dc.VARIANT_OUTSIDE])
def test_withheld_arrival_reports_timeout_and_recovers(variant):
    from dynamic_convolution_b200 import build
    build.build()
    L, inp, a = _layer()
    assert dc.dynconv_device_status(None) == dc.OK
    try:
        assert dc.dynconv_test_hook(1, 20000) == dc.OK   # 20 ms bounded waits
        assert dc.dynconv_test_hook(2, 1) == dc.OK       # withhold one arrival, next launch
        st = dc.dynconv_forward(L.desc(variant), L.x, L.experts, L.alpha, L.bias, L.y, None, 0, None)
        assert st == dc.OK                               # the launch itself is fine
        assert dc.dynconv_device_status(None) == dc.ERR_TIMEOUT
        assert "error word" in dc.dynconv_last_error()
        # cleared on read
        assert dc.dynconv_device_status(None) == dc.OK
    finally:
        dc.dynconv_test_hook(2, 0)
        dc.dynconv_test_hook(1, 0)
    # the context is still usable and correct
    L.forward(variant)
    assert dc.dynconv_device_status(None) == dc.OK
    ref = oracle.forward(inp.x_f64, inp.experts_f64, a, inp.bias, stride=1, pad=1)
    assert compare(from_device(L.y), ref, synth.BF16)["ok"]
