"""GPU parity: the CUDA path, called through the C ABI, against the fp64 oracle
on the same seeded inputs.

* Full-size layer configurations: routing weights on every sample; outputs on
  sampled whole samples (first, middle, last and two more), computed by the
  oracle one sample at a time, in the launch configuration the benchmark uses.
* Small structured cases (per-sample channel offsets, so routing differs
  strongly between samples) with ragged tails: image heights that do not
  divide into row blocks, output channels that do not fill a 128-row tile,
  input channels that do not fill a 64-wide chunk, odd expert counts.
* Every forward variant the library offers is compared, not only the one the
  cost model picks.
"""
import numpy as np
import pytest
import torch

import dynamic_convolution_b200 as dc
import oracle
from dynamic_convolution_b200 import synth

from .gpu_util import ALPHA_ABS, Layer, alpha_f32_rounded, compare, from_device

pytestmark = pytest.mark.gpu

DENSE_TC = ["resnet18_3x3", "effnet_expand_1x1", "deep_3x3_tau30", "large_n64"]


@pytest.fixture(scope="module", autouse=True)
def _built():
    from dynamic_convolution_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


_CACHE = {}


def layer_inputs(name: str) -> synth.LayerInputs:
    """Seeded inputs; the depthwise layer's input is the bf16-rounded ORACLE output
    of the 1x1 expand layer of the same block (never the GPU's)."""
    if name in _CACHE:
        return _CACHE[name]
    cfg = synth.CONFIGS[name]
    inp = synth.make_inputs(cfg)
    if name == "effnet_dw_5x5":
        up = layer_inputs("effnet_expand_1x1")
        a = oracle.route(up.x_f64, up.Wr, up.br, up.cfg.mode, up.cfg.tau)
        y = oracle.forward(up.x_f64, up.experts_f64, a, up.bias, stride=1, pad=0)
        inp = inp.with_x(y)
    _CACHE[name] = inp
    return inp


def sample_ids(B: int):
    return sorted({0, 1, B // 2, B - 2, B - 1} & set(range(B)))


@pytest.mark.parametrize("name", list(synth.CONFIGS))
def test_route_matches_oracle(name):
    inp = layer_inputs(name)
    cfg = inp.cfg
    L = Layer(inp)
    L.route()
    torch.cuda.synchronize()
    got = from_device(L.alpha)
    ref = oracle.route(inp.x_f64, inp.Wr, inp.br, cfg.mode, cfg.tau)
    assert np.abs(got - ref).max() <= ALPHA_ABS, np.abs(got - ref).max()
    if cfg.mode == synth.SOFTMAX:
        assert np.abs(got.sum(axis=1) - 1.0).max() < 1e-6
    # deterministic: a second call gives identical bits
    first = L.alpha.clone()
    L.route()
    torch.cuda.synchronize()
    assert torch.equal(first, L.alpha)


def _forward_case(name, variant, workspace=False):
    inp = layer_inputs(name)
    cfg = inp.cfg
    L = Layer(inp)
    a64 = alpha_f32_rounded(oracle.route(inp.x_f64, inp.Wr, inp.br, cfg.mode, cfg.tau))
    L.alpha.copy_(torch.from_numpy(a64.astype(np.float32)))
    ws = None
    if workspace:
        nbytes = dc.dynconv_workspace_size(L.desc(variant))
        assert nbytes > 0
        ws = torch.empty(nbytes // 2, dtype=torch.bfloat16, device="cuda")
    L.forward(variant, workspace=ws)
    assert dc.dynconv_device_status(None) == dc.OK
    y = from_device(L.y)
    for b in sample_ids(cfg.B):
        ref = oracle.forward(inp.x_f64, inp.experts_f64, a64, inp.bias, stride=cfg.stride,
                             pad=cfg.pad, groups=cfg.groups, samples=(b, 1))[0]
        r = compare(y[b], ref, cfg.dtype)
        assert r["ok"], (name, variant, b, r)
    assert np.isfinite(y).all()


@pytest.mark.parametrize("name", DENSE_TC)
@pytest.mark.parametrize("variant", [dc.VARIANT_FUSED, dc.VARIANT_OUTSIDE, dc.VARIANT_PREMIX])
def test_forward_tensor_core_full_size(name, variant):
    _forward_case(name, variant, workspace=(variant == dc.VARIANT_PREMIX))


def test_forward_tiny_fp32_direct():
    _forward_case("tiny_fp32", dc.VARIANT_DIRECT)


@pytest.mark.parametrize("variant", [dc.VARIANT_DEPTHWISE, dc.VARIANT_DIRECT])
def test_forward_depthwise_full_size(variant):
    _forward_case("effnet_dw_5x5", variant)


@pytest.mark.parametrize("name", list(synth.CONFIGS))
def test_end_to_end_route_then_forward(name):
    """GPU route -> GPU forward (AUTO variant) against oracle route -> oracle forward."""
    inp = layer_inputs(name)
    cfg = inp.cfg
    L = Layer(inp)
    L.route()
    L.forward()
    torch.cuda.synchronize()
    y = from_device(L.y)
    a = oracle.route(inp.x_f64, inp.Wr, inp.br, cfg.mode, cfg.tau)
    for b in sample_ids(cfg.B)[:3]:
        ref = oracle.forward(inp.x_f64, inp.experts_f64, a, inp.bias, stride=cfg.stride,
                             pad=cfg.pad, groups=cfg.groups, samples=(b, 1))[0]
        r = compare(y[b], ref, cfg.dtype)
        assert r["ok"], (name, b, r)


SMALL = [
    # name, B, C_in, C_out, H, W, K, pad, n, mode, tau
    ("ragged_rows", 3, 64, 128, 13, 11, 3, 1, 4, synth.SOFTMAX, 1.0),
    ("two_mtiles_partial", 2, 72, 136, 9, 10, 3, 1, 5, synth.SIGMOID, 1.0),
    ("pointwise_odd_n", 4, 40, 96, 12, 12, 1, 0, 3, synth.SIGMOID, 1.0),
    ("dense_5x5", 2, 32, 64, 10, 9, 5, 2, 2, synth.SOFTMAX, 0.5),
    ("single_expert", 2, 64, 128, 8, 8, 3, 1, 1, synth.SOFTMAX, 1.0),
    ("wide_image", 1, 16, 32, 3, 200, 3, 1, 3, synth.SOFTMAX, 2.0),
]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
@pytest.mark.parametrize("variant", [dc.VARIANT_FUSED, dc.VARIANT_OUTSIDE, dc.VARIANT_PREMIX,
                                     dc.VARIANT_DIRECT])
def test_small_structured_all_variants(case, variant):
    name, B, Cin, Cout, H, W, K, pad, n, mode, tau = case
    cfg = synth.LayerConfig(name, synth.BF16, B, Cin, Cout, H, W, K, K, 1, pad, 1, n, mode, tau)
    inp = synth.make_inputs(cfg, seed=3, structured=1.5)
    L = Layer(inp)
    L.route()
    torch.cuda.synchronize()
    a_gpu = from_device(L.alpha)
    a = oracle.route(inp.x_f64, inp.Wr, inp.br, mode, tau)
    assert np.abs(a_gpu - a).max() <= ALPHA_ABS
    if n > 1:  # structured inputs: routing really differs between samples
        assert B == 1 or np.abs(a - a[0]).max() > 1e-2
    a32 = alpha_f32_rounded(a)
    L.alpha.copy_(torch.from_numpy(a32.astype(np.float32)))
    ws = None
    if variant == dc.VARIANT_PREMIX:
        ws = torch.empty(dc.dynconv_workspace_size(L.desc(variant)) // 2 + 8,
                         dtype=torch.bfloat16, device="cuda")
    L.forward(variant, workspace=ws)
    torch.cuda.synchronize()
    ref = oracle.forward(inp.x_f64, inp.experts_f64, a32, inp.bias, stride=1, pad=pad)
    r = compare(from_device(L.y), ref, synth.BF16)
    assert r["ok"], (name, variant, r)


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_small_structured_streamed_mixing(case):
    """The streamed-mixing PREMIX kernel on the ragged small cases (partial
    channel chunks and channel tiles, odd expert counts, tiny batches)."""
    name, B, Cin, Cout, H, W, K, pad, n, mode, tau = case
    cfg = synth.LayerConfig(name, synth.BF16, B, Cin, Cout, H, W, K, K, 1, pad, 1, n, mode, tau)
    inp = synth.make_inputs(cfg, seed=4, structured=1.5)
    L = Layer(inp)
    a32 = alpha_f32_rounded(oracle.route(inp.x_f64, inp.Wr, inp.br, mode, tau))
    L.alpha.copy_(torch.from_numpy(a32.astype(np.float32)))
    ws = torch.empty(dc.dynconv_workspace_size(L.desc(dc.VARIANT_PREMIX)) // 2 + 8,
                     dtype=torch.bfloat16, device="cuda")
    try:
        assert dc.dynconv_test_hook(6, 1) == dc.OK
        L.forward(dc.VARIANT_PREMIX, workspace=ws)
        torch.cuda.synchronize()
        assert dc.dynconv_device_status(None) == dc.OK
    finally:
        dc.dynconv_test_hook(6, 0)
    ref = oracle.forward(inp.x_f64, inp.experts_f64, a32, inp.bias, stride=1, pad=pad)
    r = compare(from_device(L.y), ref, synth.BF16)
    assert r["ok"], (name, r)


@pytest.mark.parametrize("variant", [dc.VARIANT_FUSED, dc.VARIANT_DIRECT])
def test_no_bias(variant):
    cfg = synth.LayerConfig("nobias", synth.BF16, 2, 64, 64, 7, 7, 3, 3, 1, 1, 1, 3,
                            synth.SIGMOID, 1.0)
    inp = synth.make_inputs(cfg, seed=5, structured=1.0)
    L = Layer(inp)
    a = alpha_f32_rounded(oracle.route(inp.x_f64, inp.Wr, inp.br, cfg.mode, cfg.tau))
    L.alpha.copy_(torch.from_numpy(a.astype(np.float32)))
    L.forward(variant, bias=None)
    torch.cuda.synchronize()
    ref = oracle.forward(inp.x_f64, inp.experts_f64, a, None, stride=1, pad=1)
    assert compare(from_device(L.y), ref, synth.BF16)["ok"]


def test_fp32_general_shapes_direct():
    """fp32 path with stride 2, groups 2 and an odd kernel size."""
    cfg = synth.LayerConfig("f32_general", synth.F32, 3, 6, 8, 11, 9, 5, 5, 2, 2, 2, 3,
                            synth.SOFTMAX, 3.0)
    inp = synth.make_inputs(cfg, seed=9, structured=1.0)
    L = Layer(inp)
    L.route()
    L.forward()
    torch.cuda.synchronize()
    a = oracle.route(inp.x_f64, inp.Wr, inp.br, cfg.mode, cfg.tau)
    assert np.abs(from_device(L.alpha) - a).max() <= ALPHA_ABS
    ref = oracle.forward(inp.x_f64, inp.experts_f64, a, inp.bias, stride=2, pad=2, groups=2)
    r = compare(from_device(L.y), ref, synth.F32)
    assert r["ok"], r


def test_outputs_outside_y_untouched():
    """Canary: the forward writes exactly y, nothing after it."""
    inp = layer_inputs("resnet18_3x3")
    cfg = inp.cfg.scaled(B=4)
    small = synth.make_inputs(cfg)
    L = Layer(small)
    big = torch.full((L.y.numel() + 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
    L.y = big[: L.y.numel()].view(L.y.shape)
    L.route()
    for v in (dc.VARIANT_FUSED, dc.VARIANT_OUTSIDE, dc.VARIANT_DIRECT):
        L.forward(v)
    torch.cuda.synchronize()
    assert torch.all(big[L.y.numel():] == 7.0)


@pytest.mark.parametrize("name", ["resnet18_3x3", "effnet_expand_1x1"])
def test_streamed_mixing_equals_two_kernels(name):
    """PREMIX with the mixing streamed into the convolution (one persistent
    kernel, per-slice counters) gives the same bits as the two-kernel form with
    the same CUDA-core mixer, on three consecutive calls (the counters carry
    over between launches)."""
    inp = layer_inputs(name)
    L = Layer(inp)
    L.route()
    d = L.desc(dc.VARIANT_PREMIX)
    ws = torch.zeros(dc.dynconv_workspace_size(d), dtype=torch.uint8, device="cuda")
    outs = []
    try:
        for stream_mix, mixer, calls in ((1, 0, 3), (0, 2, 1)):
            assert dc.dynconv_test_hook(6, stream_mix) == dc.OK
            assert dc.dynconv_test_hook(7, mixer) == dc.OK
            for _ in range(calls):
                L.y.fill_(float("nan"))
                dc.check(dc.dynconv_forward(d, L.x, L.experts, L.alpha, L.bias, L.y, ws,
                                            ws.numel()))
                assert dc.dynconv_device_status(None) == dc.OK
                outs.append(L.y.clone())
    finally:
        dc.dynconv_test_hook(6, 0)
        dc.dynconv_test_hook(7, 0)
    for o in outs[1:]:
        assert torch.equal(outs[0], o)
    assert torch.isfinite(outs[0].float()).all()


def test_streamed_mixing_more_streams_than_slots():
    """The streamed mixing keeps per-stream counters in a fixed number of
    device slots (64). With more streams than free slots, a stream without a
    slot runs the two-kernel form instead of sharing another stream's
    counters: every stream's output equals the two-kernel output bit for bit."""
    cfg = synth.LayerConfig("slots", synth.BF16, 4, 64, 64, 8, 8, 3, 3, 1, 1, 1, 4,
                            synth.SIGMOID, 1.0)
    inp = synth.make_inputs(cfg, seed=12, structured=1.0)
    L = Layer(inp)
    L.route()
    d = L.desc(dc.VARIANT_PREMIX)
    nbytes = dc.dynconv_workspace_size(d)
    ws0 = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    try:
        assert dc.dynconv_test_hook(7, 2) == dc.OK  # two-kernel form, CUDA-core mixer
        dc.check(dc.dynconv_forward(d, L.x, L.experts, L.alpha, L.bias, L.y, ws0, nbytes))
        torch.cuda.synchronize()
        ref = L.y.clone()
        assert dc.dynconv_test_hook(7, 0) == dc.OK
        assert dc.dynconv_test_hook(6, 1) == dc.OK  # streamed mixing
        streams = [torch.cuda.Stream() for _ in range(72)]
        outs = [torch.full_like(L.y, float("nan")) for _ in streams]
        wss = [torch.zeros(nbytes, dtype=torch.uint8, device="cuda") for _ in streams]
        torch.cuda.synchronize()
        for st, y, ws in zip(streams, outs, wss):
            dc.check(dc.dynconv_forward(d, L.x, L.experts, L.alpha, L.bias, y, ws, nbytes,
                                        st.cuda_stream), "dynconv_forward (streamed)")
        torch.cuda.synchronize()
        assert dc.dynconv_device_status(None) == dc.OK
    finally:
        dc.dynconv_test_hook(6, 0)
        dc.dynconv_test_hook(7, 0)
    for y in outs:
        assert torch.equal(y, ref)


@pytest.mark.parametrize("name", ["resnet18_3x3", "effnet_expand_1x1"])
@pytest.mark.parametrize("mixer", [(0, 1), (0, 2), (1, 0)], ids=["gemm", "cuda-core", "streamed"])
def test_premix_mixers_full_size(name, mixer):
    """PREMIX with each mixing kernel (tensor-core GEMM with a hi/lo split of
    alpha; CUDA-core fp32 mixer; the mixing streamed into the convolution)
    against the oracle on sampled whole samples."""
    stream_mix, which = mixer
    try:
        assert dc.dynconv_test_hook(6, stream_mix) == dc.OK
        assert dc.dynconv_test_hook(7, which) == dc.OK
        _forward_case(name, dc.VARIANT_PREMIX, workspace=True)
    finally:
        dc.dynconv_test_hook(6, 0)
        dc.dynconv_test_hook(7, 0)


@pytest.mark.parametrize("name", ["resnet18_3x3", "deep_3x3_tau30", "large_n64"])
def test_premix_transposed_mixer_full_size(name):
    """PREMIX with the transposed mixing GEMM over the whole batch (test hook
    7 = 3: M = weights, N = samples) against the oracle on sampled whole
    samples."""
    try:
        assert dc.dynconv_test_hook(7, 3) == dc.OK
        _forward_case(name, dc.VARIANT_PREMIX, workspace=True)
    finally:
        dc.dynconv_test_hook(7, 0)


@pytest.mark.parametrize("tiles", [2, 0], ids=["counter", "static"])
@pytest.mark.parametrize("store", [0, 1], ids=["lane-store", "register-store"])
@pytest.mark.parametrize("B", [3, 40, 100, 250],
                         ids=["B3-four-copies", "B40-two-copies", "B100", "B250-ragged-row-tile"])
def test_premix_gemm_small_batches(B, store, tiles):
    """The tensor-core mixing GEMM (test hook 7 = 1) with each epilogue form
    (test hook 12) and tile hand-out (test hook 18): the batch copied into the
    128 accumulator rows (B <= 32: four copies, B <= 64: two), each copy's
    epilogue warps storing a share of the columns; a ragged second row tile
    (B = 250); a kernel size that is not a multiple of the 256-weight tile.
    Against the oracle element by element."""
    cfg = synth.LayerConfig(f"premix_b{B}", synth.BF16, B, 24, 40, 7, 9, 3, 3, 1, 1, 1, 12,
                            synth.SOFTMAX, 2.0)
    inp = synth.make_inputs(cfg, seed=11, structured=1.0)
    a32 = alpha_f32_rounded(oracle.route(inp.x_f64, inp.Wr, inp.br, cfg.mode, cfg.tau))
    L = Layer(inp)
    L.alpha.copy_(torch.from_numpy(a32.astype(np.float32)))
    ws = torch.empty(dc.dynconv_workspace_size(L.desc(dc.VARIANT_PREMIX)), dtype=torch.uint8,
                     device="cuda")
    try:
        assert dc.dynconv_test_hook(7, 1) == dc.OK
        assert dc.dynconv_test_hook(12, store) == dc.OK
        assert dc.dynconv_test_hook(18, tiles) == dc.OK
        L.y.fill_(float("nan"))
        L.forward(dc.VARIANT_PREMIX, workspace=ws)
        assert dc.dynconv_device_status(None) == dc.OK
    finally:
        dc.dynconv_test_hook(7, 0)
        dc.dynconv_test_hook(12, 0)
        dc.dynconv_test_hook(18, 1)
    ref = oracle.forward(inp.x_f64, inp.experts_f64, a32, inp.bias, stride=1, pad=1)
    r = compare(from_device(L.y), ref, synth.BF16)
    assert r["ok"], (B, store, tiles, r)


@pytest.mark.parametrize("name", ["deep_3x3_tau30", "large_n64"])
def test_premix_gemm_tile_order_identical(name):
    """The mixing GEMM with its tiles handed out by the workspace counter (test
    hook 18 = 2) and statically (18 = 0) at full size: each tile's arithmetic
    does not depend on which CTA takes it, so the outputs are bit-identical;
    twice in a row with the counter (it is re-zeroed per call)."""
    inp = layer_inputs(name)
    L = Layer(inp)
    L.route()
    ws = torch.empty(dc.dynconv_workspace_size(L.desc(dc.VARIANT_PREMIX)), dtype=torch.uint8,
                     device="cuda")
    try:
        assert dc.dynconv_test_hook(18, 0) == dc.OK
        L.forward(dc.VARIANT_PREMIX, workspace=ws)
        ref = L.y.clone()
        assert dc.dynconv_test_hook(18, 2) == dc.OK
        for _ in range(2):
            L.y.fill_(float("nan"))
            L.forward(dc.VARIANT_PREMIX, workspace=ws)
            assert dc.dynconv_device_status(None) == dc.OK
            assert torch.equal(L.y, ref)
    finally:
        dc.dynconv_test_hook(18, 1)


def test_premix_cuda_core_mixer_refuses_many_experts():
    inp = layer_inputs("deep_3x3_tau30")
    L = Layer(inp)
    d = L.desc(dc.VARIANT_PREMIX)
    ws = torch.zeros(dc.dynconv_workspace_size(d), dtype=torch.uint8, device="cuda")
    try:
        assert dc.dynconv_test_hook(7, 2) == dc.OK
        rc = dc.dynconv_forward(d, L.x, L.experts, L.alpha, L.bias, L.y, ws, ws.numel())
        assert rc == dc.ERR_UNSUPPORTED
    finally:
        dc.dynconv_test_hook(7, 0)


DEPTHWISE_SHAPES = [
    # name, B, C, H, W, K, pad, n: ragged channel chunks, column bands (wide
    # images), row bands (tall images), windows larger than the image, no
    # padding (output smaller than the input), all three kernel sizes
    ("dw3_small", 2, 24, 7, 9, 3, 1, 3),
    ("dw5_ragged", 3, 40, 13, 11, 5, 2, 4),
    ("dw7_wide", 1, 64, 9, 60, 7, 3, 2),
    ("dw5_tall", 1, 16, 200, 8, 5, 2, 2),
    ("dw3_many_channels", 2, 264, 6, 6, 3, 1, 2),
    ("dw5_tiny_image", 1, 8, 3, 3, 5, 2, 1),
    ("dw3_no_pad", 2, 32, 12, 12, 3, 0, 2),
    ("dw7_odd", 2, 56, 10, 31, 7, 3, 5),
]


@pytest.mark.parametrize("kernel", [0, 1, 2, 3],
                         ids=["pipelined", "per-tile", "pipelined-2col", "pipelined-4col"])
@pytest.mark.parametrize("case", DEPTHWISE_SHAPES, ids=[c[0] for c in DEPTHWISE_SHAPES])
def test_depthwise_kernels_ragged(case, kernel):
    """Every depthwise kernel form (test hook 8: the pipelined kernel with its
    default, 2 or 4 output columns per thread, and the per-tile kernel)
    against the oracle on structured inputs, element by element, with and
    without bias."""
    name, B, C, H, W, K, pad, n = case
    cfg = synth.LayerConfig(name, synth.BF16, B, C, C, H, W, K, K, 1, pad, C, n, synth.SIGMOID, 1.0)
    inp = synth.make_inputs(cfg, seed=6, structured=1.0)
    a = alpha_f32_rounded(oracle.route(inp.x_f64, inp.Wr, inp.br, cfg.mode, cfg.tau))
    L = Layer(inp)
    L.alpha.copy_(torch.from_numpy(a.astype(np.float32)))
    try:
        assert dc.dynconv_test_hook(8, kernel) == dc.OK
        for bias in (True, False):
            L.y.fill_(float("nan"))
            L.forward(dc.VARIANT_DEPTHWISE, bias="default" if bias else None)
            assert dc.dynconv_device_status(None) == dc.OK
            ref = oracle.forward(inp.x_f64, inp.experts_f64, a, inp.bias if bias else None,
                                 stride=1, pad=pad, groups=C)
            r = compare(from_device(L.y), ref, synth.BF16)
            assert r["ok"], (name, kernel, bias, r)
    finally:
        dc.dynconv_test_hook(8, 0)


@pytest.mark.parametrize("kernel", [1, 2, 3], ids=["per-tile", "pipelined-2col", "pipelined-4col"])
def test_depthwise_full_size_kernel_forms(kernel):
    """Each depthwise kernel form at full size (the default form runs in
    test_forward_depthwise_full_size)."""
    try:
        assert dc.dynconv_test_hook(8, kernel) == dc.OK
        _forward_case("effnet_dw_5x5", dc.VARIANT_DEPTHWISE)
    finally:
        dc.dynconv_test_hook(8, 0)


def test_depthwise_pipelined_is_deterministic():
    """Two calls of the pipelined depthwise kernel give identical bits (fixed
    mixing and tap order, no atomics)."""
    inp = layer_inputs("effnet_dw_5x5")
    L = Layer(inp)
    L.route()
    outs = []
    for _ in range(2):
        L.forward(dc.VARIANT_DEPTHWISE)
        outs.append(L.y.clone())
    assert torch.equal(outs[0], outs[1])


GROUPED = [
    # name, B, C_in, C_out, H, W, K, pad, n, mode, tau, group bytes (test hook 10)
    ("samples_ragged", 5, 64, 264, 9, 7, 3, 1, 12, synth.SOFTMAX, 1.0, 65536),
    ("tiles_ragged", 5, 64, 264, 9, 7, 3, 1, 12, synth.SOFTMAX, 1.0, 1 << 20),
    ("tiles_136", 3, 72, 136, 13, 11, 3, 1, 9, synth.SIGMOID, 1.0, 1 << 20),
    ("samples_1x1", 7, 40, 240, 12, 12, 1, 0, 10, synth.SIGMOID, 1.0, 65536),
    # two groups of 75 samples: more than 64 per group, the samples-as-M GEMM
    ("samples_wide", 150, 16, 24, 5, 5, 3, 1, 9, synth.SOFTMAX, 1.0, 691200),
]


@pytest.mark.parametrize("case", GROUPED, ids=[c[0] for c in GROUPED])
@pytest.mark.parametrize("seq", [False, True], ids=["concurrent", "sequential"])
def test_grouped_premix_ragged(case, seq):
    """The grouped mixing pipeline (runs of samples, or runs of 128-channel
    tiles; concurrent: two workspace slots and an internal stream; sequential:
    one slot on the caller's stream) against the oracle element by element,
    next to the one-pass form; each deterministic."""
    name, B, Cin, Cout, H, W, K, pad, n, mode, tau, gbytes = case
    if seq:
        gbytes = -gbytes
    cfg = synth.LayerConfig(name, synth.BF16, B, Cin, Cout, H, W, K, K, 1, pad, 1, n, mode, tau)
    inp = synth.make_inputs(cfg, seed=8, structured=1.5)
    a32 = alpha_f32_rounded(oracle.route(inp.x_f64, inp.Wr, inp.br, mode, tau))
    L = Layer(inp)
    L.alpha.copy_(torch.from_numpy(a32.astype(np.float32)))
    ws = torch.empty(dc.dynconv_workspace_size(L.desc(dc.VARIANT_PREMIX)), dtype=torch.uint8,
                     device="cuda")
    outs = []
    try:
        for hook in (gbytes, 0):
            assert dc.dynconv_test_hook(10, hook) == dc.OK
            for _ in range(2):
                L.y.fill_(float("nan"))
                L.forward(dc.VARIANT_PREMIX, workspace=ws)
                assert dc.dynconv_device_status(None) == dc.OK
                outs.append(L.y.clone())
    finally:
        dc.dynconv_test_hook(10, 0)
    ref = oracle.forward(inp.x_f64, inp.experts_f64, a32, inp.bias, stride=1, pad=pad)
    for o in (outs[0], outs[2]):  # grouped, one pass
        r = compare(from_device(o), ref, synth.BF16)
        assert r["ok"], (name, r)
    # each form is deterministic (the grouped form may mix with the transposed
    # GEMM, whose fp32 sums may differ from the one-pass GEMM's in the last bit)
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[2], outs[3])


@pytest.mark.parametrize("name", ["resnet18_3x3", "effnet_expand_1x1", "deep_3x3_tau30"])
def test_persistent_conv_bit_identical(name):
    """The persistent PREMIX convolution (test hook 9) gives the same bits as
    one CTA per unit: same MMA order over K, same epilogue arithmetic."""
    inp = layer_inputs(name)
    L = Layer(inp)
    L.route()
    d = L.desc(dc.VARIANT_PREMIX)
    ws = torch.empty(dc.dynconv_workspace_size(d), dtype=torch.uint8, device="cuda")
    outs = []
    try:
        for persist in (2, 0):
            assert dc.dynconv_test_hook(9, persist) == dc.OK
            assert dc.dynconv_test_hook(10, 0) == dc.OK
            L.y.fill_(float("nan"))
            dc.check(dc.dynconv_forward(d, L.x, L.experts, L.alpha, L.bias, L.y, ws, ws.numel()))
            assert dc.dynconv_device_status(None) == dc.OK
            outs.append(L.y.clone())
    finally:
        dc.dynconv_test_hook(9, 1)
        dc.dynconv_test_hook(10, 0)
    assert torch.equal(outs[0], outs[1])
    assert torch.isfinite(outs[0].float()).all()


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_small_structured_persistent_conv(case):
    """PREMIX with the persistent convolution forced (hook 9 = 2) on the
    ragged small cases (by default small layers run one CTA per unit)."""
    try:
        assert dc.dynconv_test_hook(9, 2) == dc.OK
        test_small_structured_all_variants(case, dc.VARIANT_PREMIX)
    finally:
        dc.dynconv_test_hook(9, 1)


@pytest.mark.parametrize("mode", [1, 2], ids=["concurrent", "sequential"])
@pytest.mark.parametrize("name", ["deep_3x3_tau30", "large_n64"])
def test_grouped_and_one_pass_full_size(name, mode):
    """At full size the grouped pipeline (test hook 10; off by default) is
    deterministic, matches the oracle on sampled whole samples and agrees
    with the one-pass PREMIX within the bf16 tolerance everywhere."""
    inp = layer_inputs(name)
    cfg = synth.CONFIGS[name]
    L = Layer(inp)
    a32 = alpha_f32_rounded(oracle.route(inp.x_f64, inp.Wr, inp.br, cfg.mode, cfg.tau))
    L.alpha.copy_(torch.from_numpy(a32.astype(np.float32)))
    d = L.desc(dc.VARIANT_PREMIX)
    ws = torch.empty(dc.dynconv_workspace_size(d), dtype=torch.uint8, device="cuda")
    outs = []
    try:
        for hook in (mode, mode, 0):
            assert dc.dynconv_test_hook(10, hook) == dc.OK
            L.y.fill_(float("nan"))
            dc.check(dc.dynconv_forward(d, L.x, L.experts, L.alpha, L.bias, L.y, ws, ws.numel()))
            assert dc.dynconv_device_status(None) == dc.OK
            outs.append(L.y.clone())
    finally:
        dc.dynconv_test_hook(10, 0)
    assert torch.equal(outs[0], outs[1])
    got = from_device(outs[0])
    r = compare(got, from_device(outs[2]), synth.BF16)
    assert r["ok"], (name, r)
    for b in sorted({0, cfg.B // 2 + 1, cfg.B - 1}):
        yr = oracle.forward(inp.x_f64, inp.experts_f64, a32, inp.bias, stride=cfg.stride,
                            pad=cfg.pad, groups=cfg.groups, samples=(b, 1))[0]
        r = compare(got[b], yr, synth.BF16)
        assert r["ok"], (name, b, r)
