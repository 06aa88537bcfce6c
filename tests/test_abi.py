"""Host-side checks of the C-ABI library that need no GPU: it loads, exports
every function the header declares, validates arguments before touching CUDA,
and fails loudly (DYNCONV_ERR_CUDA) rather than falling back to the CPU when no
device is present."""
import ctypes
import os
import re

import pytest
import torch

import dynamic_convolution_b200 as dc
from dynamic_convolution_b200 import build as dcbuild
from dynamic_convolution_b200 import synth

HEADERS = [os.path.join(dcbuild.ROOT, "include", h)
           for h in ("dynconv.h", "dynconv_backward.h", "dynconv_cells.h")]


@pytest.fixture(scope="module")
def lib():
    dcbuild.build()
    return dc.load()


def declared_functions():
    text = "".join(open(h).read() for h in HEADERS)
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dynconv_[a-z_]+)\s*\(", text)))


def test_header_declares_the_binding_names():
    assert declared_functions() == sorted(dc.SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert dc.dynconv_status_string(code)
    assert dc.dynconv_status_string(12345) == "unknown status"


def _desc(**kw):
    base = dict(B=2, C_in=8, H=8, W=8, C_out=8, KH=3, KW=3, stride=1, pad=1, groups=1, n=4,
                dtype=dc.F32, variant=0)
    base.update(kw)
    return dc.make_desc(**base)


BAD = [dict(C_in=0), dict(H=-1), dict(KH=0), dict(stride=0), dict(pad=-1), dict(groups=3),
       dict(n=0), dict(dtype=7), dict(variant=9), dict(H=1, W=1, pad=0),
       dict(groups=2, C_out=5)]


@pytest.mark.parametrize("kw", BAD)
def test_invalid_descriptors_rejected_on_host(lib, kw):
    d = _desc(**kw)
    assert dc.dynconv_forward(d, 16, 16, 16, None, 16) == dc.ERR_INVALID_ARG
    assert dc.dynconv_route(d, 16, 16, None, dc.SIGMOID, 1.0, 16) == dc.ERR_INVALID_ARG
    assert dc.dynconv_select_variant(d) == dc.ERR_INVALID_ARG
    assert dc.dynconv_workspace_size(d) == 0


def test_null_pointers_and_bad_route_args_rejected(lib):
    d = _desc()
    assert dc.dynconv_forward(d, None, 16, 16, None, 16) == dc.ERR_INVALID_ARG
    assert dc.dynconv_forward(d, 16, 16, 16, None, None) == dc.ERR_INVALID_ARG
    assert dc.dynconv_route(d, 16, None, None, dc.SIGMOID, 1.0, 16) == dc.ERR_INVALID_ARG
    assert dc.dynconv_route(d, 16, 16, None, dc.SOFTMAX, 0.0, 16) == dc.ERR_INVALID_ARG
    assert dc.dynconv_route(d, 16, 16, None, dc.SOFTMAX, -1.0, 16) == dc.ERR_INVALID_ARG
    assert dc.dynconv_route(d, 16, 16, None, 5, 1.0, 16) == dc.ERR_INVALID_ARG


def test_empty_batch_is_a_noop(lib):
    d = _desc(B=0)
    assert dc.dynconv_forward(d, 16, 16, 16, None, 16) == dc.OK
    assert dc.dynconv_route(d, 16, 16, None, dc.SIGMOID, 1.0, 16) == dc.OK


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_no_device_fails_loudly(lib):
    d = _desc()
    assert dc.dynconv_forward(d, 16, 16, 16, None, 16) == dc.ERR_CUDA
    assert dc.dynconv_route(d, 16, 16, None, dc.SIGMOID, 1.0, 16) == dc.ERR_CUDA
    assert dc.dynconv_last_error() != ""


# The forward variant measured fastest on each layer by bench.py's
# per_config.variants_forward_ms (median of 50 cold calls, one B200): with a
# workspace, PREMIX on every dense layer (e.g. 30.7 us against FUSED 55.2 and
# OUTSIDE 96.1 on the 3x3 layer; 184 us against 1933 and 5066 on the n=64
# layer); without one, FUSED before OUTSIDE on every dense layer.
MEASURED_BEST = {
    "tiny_fp32": ("direct", "direct"),
    "resnet18_3x3": ("premix", "fused"),
    "effnet_expand_1x1": ("premix", "fused"),
    "effnet_dw_5x5": ("depthwise", "depthwise"),
    "deep_3x3_tau30": ("premix", "fused"),
    "large_n64": ("premix", "fused"),
}


def test_variant_selection_per_config(lib):
    """AUTO resolves to the measured fastest variant on every layer, with the
    workspace dynconv_workspace_size asks for and with none."""
    for name, cfg in synth.CONFIGS.items():
        d = dc.desc_from_config(cfg)
        ws = dc.dynconv_workspace_size(d)
        with_ws, without = MEASURED_BEST[name]
        assert dc.VARIANT_NAMES[dc.dynconv_select_variant(d, ws)] == with_ws, name
        assert dc.VARIANT_NAMES[dc.dynconv_select_variant(d, 0)] == without, name
    for name in ("deep_3x3_tau30", "large_n64"):
        d = dc.desc_from_config(synth.CONFIGS[name])
        # every sample's mixed kernel, 256-byte aligned
        wb = (synth.CONFIGS[name].B * synth.CONFIGS[name].weight_elems * 2 + 255) // 256 * 256
        assert dc.dynconv_workspace_size(d) == wb + 256   # + the mixing GEMM's tile counter
    # a forced variant is reported as is
    d = dc.desc_from_config(synth.CONFIGS["resnet18_3x3"], variant=dc.VARIANT_OUTSIDE)
    assert dc.dynconv_select_variant(d) == dc.VARIANT_OUTSIDE


def test_shapes_outside_tensor_core_kernels_go_direct(lib):
    # stride 2, odd channel counts, fp32: the CUDA-core direct kernel
    assert dc.dynconv_select_variant(_desc(dtype=dc.BF16, stride=2)) == dc.VARIANT_DIRECT
    assert dc.dynconv_select_variant(_desc(dtype=dc.BF16, C_in=12, C_out=12)) == dc.VARIANT_DIRECT
    assert dc.dynconv_select_variant(_desc(dtype=dc.BF16, groups=2)) == dc.VARIANT_DIRECT


def test_test_hook_arguments(lib):
    assert dc.dynconv_test_hook(1, 0) == dc.OK
    assert dc.dynconv_test_hook(1, -5) == dc.ERR_INVALID_ARG
    assert dc.dynconv_test_hook(99, 0) == dc.ERR_INVALID_ARG
    # depthwise kernel choice, persistent convolution, grouped mixing
    for key in (8, 9, 11):
        assert dc.dynconv_test_hook(key, 4 if key == 8 else 3) == dc.ERR_INVALID_ARG
        assert dc.dynconv_test_hook(key, 0 if key == 8 else 1) == dc.OK
    assert dc.dynconv_test_hook(10, 100) == dc.ERR_INVALID_ARG   # group bytes below 4096
    assert dc.dynconv_test_hook(10, -1) == dc.ERR_INVALID_ARG
    assert dc.dynconv_test_hook(10, 1 << 20) == dc.OK
    assert dc.dynconv_test_hook(10, -(1 << 20)) == dc.OK     # sequential groups of 1 MB
    assert dc.dynconv_test_hook(10, 3) == dc.ERR_INVALID_ARG
    assert dc.dynconv_test_hook(10, 2) == dc.OK
    assert dc.dynconv_test_hook(10, 0) == dc.OK
    assert dc.dynconv_test_hook(12, 2) == dc.ERR_INVALID_ARG
    assert dc.dynconv_test_hook(12, -1) == dc.ERR_INVALID_ARG
    assert dc.dynconv_test_hook(12, 1) == dc.OK
    assert dc.dynconv_test_hook(12, 0) == dc.OK
    assert dc.dynconv_test_hook(14, 257) == dc.ERR_INVALID_ARG
    assert dc.dynconv_test_hook(14, -1) == dc.ERR_INVALID_ARG
    assert dc.dynconv_test_hook(14, 7) == dc.OK
    assert dc.dynconv_test_hook(14, 0) == dc.OK
    assert dc.dynconv_test_hook(18, 3) == dc.ERR_INVALID_ARG
    assert dc.dynconv_test_hook(18, 2) == dc.OK
    assert dc.dynconv_test_hook(18, 0) == dc.OK
    assert dc.dynconv_test_hook(18, 1) == dc.OK
    assert dc.dynconv_test_hook(15, 0) == dc.ERR_INVALID_ARG   # no such key


def test_pooled_entry_points_host_side(lib):
    d = _desc(dtype=dc.BF16)
    assert dc.dynconv_forward_pooled(d, 16, 16, 16, None, 16, None) == dc.ERR_INVALID_ARG
    assert dc.dynconv_route_pooled(d, None, 1, 16, None, dc.SIGMOID, 1.0, 16) == dc.ERR_INVALID_ARG
    assert dc.dynconv_route_pooled(d, 16, 0, 16, None, dc.SIGMOID, 1.0, 16) == dc.ERR_INVALID_ARG
    for kw in BAD:
        assert dc.dynconv_pool_parts(_desc(**kw)) == dc.ERR_INVALID_ARG
    # one partial per sample for the CUDA-core kernels, row blocks for the tensor-core ones
    assert dc.dynconv_pool_parts(dc.desc_from_config(synth.CONFIGS["tiny_fp32"])) == 1
    assert dc.dynconv_pool_parts(dc.desc_from_config(synth.CONFIGS["effnet_dw_5x5"])) == 1
    for name in ("resnet18_3x3", "effnet_expand_1x1"):
        d = dc.desc_from_config(synth.CONFIGS[name])
        parts = dc.dynconv_pool_parts(d, dc.dynconv_workspace_size(d))
        assert 1 <= parts <= synth.CONFIGS[name].H


def test_attention_entry_points_host_side(lib):
    d = _desc(dtype=dc.BF16)
    # neither attention requested, or an output missing for a given weight
    assert dc.dynconv_route_channels(d, 16, None, None, None, None, None, None) == dc.ERR_INVALID_ARG
    assert dc.dynconv_route_channels(d, 16, 16, None, None, None, None, None) == dc.ERR_INVALID_ARG
    assert dc.dynconv_route_channels(d, None, 16, None, 16, None, None, None) == dc.ERR_INVALID_ARG
    assert dc.dynconv_forward_attn(d, None, 16, 16, None, 16, 16, 16) == dc.ERR_INVALID_ARG
    for kw in BAD:
        assert dc.dynconv_forward_attn(_desc(**kw), 16, 16, 16, None, None, None, 16) == \
            dc.ERR_INVALID_ARG


def test_backward_entry_points_host_side(lib):
    """Argument checks of the backward calls, the workspace size (per-sample
    fp32 weight gradients, or transposed experts plus the transposed forward's
    own scratch, whichever is larger), and the loud failure with no device."""
    cfg = synth.CONFIGS["resnet18_3x3"]
    d = dc.desc_from_config(cfg)
    wsize = cfg.C_out * cfg.KH * cfg.KW * cfg.C_in
    need = dc.dynconv_backward_workspace_size(d)
    assert need >= 4 * cfg.B * wsize + 4 * cfg.B * cfg.C_out
    t = dc.make_desc(cfg.B, cfg.C_out, cfg.H, cfg.W, cfg.C_in, 3, 3, 1, 1, 1, cfg.n, cfg.dtype)
    assert need >= 2 * cfg.n * wsize + dc.dynconv_workspace_size(t)
    assert dc.dynconv_backward_workspace_size(dc.make_desc(0, 0, 1, 1, 1, 1, 1)) == 0
    P, ws = 256, need
    bw = dc.dynconv_backward_weight
    assert bw(d, None, P, P, P, P, P, P, P, P, ws) == dc.ERR_INVALID_ARG      # no x
    assert bw(d, P, P, P, P, P, P, None, P, P, ws) == dc.ERR_INVALID_ARG      # bias without dbias
    assert bw(d, P, P, P, P, None, P, P, P, P, ws) == dc.ERR_INVALID_ARG      # dbias without bias
    assert bw(d, P, P, P, P, P, P, P, P, P, ws - 256) == dc.ERR_WORKSPACE
    assert bw(d, P, P, P, P, P, P, P, P, P + 16, ws) == dc.ERR_MISALIGNED     # workspace alignment
    s2 = dc.make_desc(cfg.B, cfg.C_in, cfg.H, cfg.W, cfg.C_out, 3, 3, 2, 1, 1, cfg.n, cfg.dtype,
                      dc.VARIANT_PREMIX)
    assert bw(s2, P, P, P, P, P, P, P, P, P, ws) == dc.ERR_UNSUPPORTED       # forced TC, stride 2
    assert bw(d, P, P, P, P, P, P, P, P, P, ws) == dc.ERR_CUDA               # no device: loud
    rb = dc.dynconv_route_backward
    assert rb(d, P, P, P, P, 2, 1.0, P, P, P, P, ws) == dc.ERR_INVALID_ARG          # bad mode
    assert rb(d, P, P, P, P, dc.SOFTMAX, 0.0, P, P, P, P, ws) == dc.ERR_INVALID_ARG
    assert rb(d, P, None, P, P, dc.SOFTMAX, 1.0, P, P, P, P, ws) == dc.ERR_INVALID_ARG
    assert rb(d, P, P, P, P, dc.SOFTMAX, 1.0, P, None, P, P, ws) == dc.ERR_CUDA     # dbr optional
    assert rb(d, P, P, P, P, dc.SOFTMAX, 1.0, P, P, P) == dc.ERR_CUDA               # no workspace
    bd = dc.dynconv_backward_data
    assert bd(d, None, P, P, None, P, P, ws) == dc.ERR_INVALID_ARG
    assert bd(d, P, P, P, None, P, P, 1024) == dc.ERR_WORKSPACE              # no room for experts
    assert bd(d, P, P, P, None, P, P, ws) == dc.ERR_CUDA
    # shapes off the transposed path take the CUDA-core kernel and need no workspace
    assert bd(s2, P, P, P, None, P, None, 0) == dc.ERR_CUDA
    assert dc.dynconv_last_error() != ""


def test_cells_entry_points_host_side(lib):
    """Shapes the cell path takes, its workspace, argument checks, and the loud
    failure with no device."""
    cfg = synth.CONFIGS["resnet18_3x3"]
    d = dc.make_desc(cfg.B, cfg.C_in, cfg.H, cfg.W, cfg.C_out, 3, 3, 1, 1, 1, 128, cfg.dtype)
    wsize = cfg.C_out * 9 * cfg.C_in
    need = dc.dynconv_cells_workspace_size(d, 16)
    assert need >= 2 * cfg.B * wsize                       # every sample's kernel
    assert dc.dynconv_cells_workspace_size(d, 7) == 0      # cells must divide the kernel
    assert dc.dynconv_cells_workspace_size(d, wsize // 4) == 0   # cells of 4 elements: not 16 bytes
    big = dc.make_desc(cfg.B, cfg.C_in, cfg.H, cfg.W, cfg.C_out, 3, 3, 1, 1, 1, 2048, cfg.dtype)
    assert dc.dynconv_cells_workspace_size(big, 16) == 0   # warehouse above 1024 cells
    P = 256
    fc = dc.dynconv_forward_cells
    assert fc(d, 0, P, P, P, None, P, P, need) == dc.ERR_INVALID_ARG
    assert fc(d, 16, None, P, P, None, P, P, need) == dc.ERR_INVALID_ARG
    assert fc(d, 7, P, P, P, None, P, P, need) == dc.ERR_UNSUPPORTED
    assert fc(d, 16, P, P, P, None, P, P, need - 256) == dc.ERR_WORKSPACE
    assert fc(d, 16, P, P + 2, P, None, P, P, need) == dc.ERR_MISALIGNED
    assert fc(d, 16, P, P, P, None, P, P, need) == dc.ERR_CUDA
    rc = dc.dynconv_route_cells
    assert rc(d, 16, P, P, None, 2, 1.0, P, P, need) == dc.ERR_INVALID_ARG
    assert rc(d, 16, P, P, None, dc.SOFTMAX, 0.0, P, P, need) == dc.ERR_INVALID_ARG
    assert rc(d, 64, P, P, None, dc.SOFTMAX, 1.0, P, P, need) == dc.ERR_UNSUPPORTED  # 64 * 128
    assert rc(d, 16, P, P, None, dc.SOFTMAX, 1.0, P, None, 0) == dc.ERR_WORKSPACE
    assert rc(d, 16, P, P, None, dc.SOFTMAX, 1.0, P, P, need) == dc.ERR_CUDA
