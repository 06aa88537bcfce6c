"""Pins for the fp64 CPU oracle, independent of the oracle itself.

Each test checks the oracle against something other than its own formula:
a library convolution for n=1, a second brute-force formulation (explicit
im2col matrix, experts summed on the output side), closed forms (impulse,
constant input, zero input), library activations, and the identities that the
definition implies (linearity in the kernel, batch and expert permutation).
The definition pinned here is the sum of n static kernels, each weighted by an
attention computed from the input (KernelWarehouse: Rethinking the Design of
Dynamic Convolution, abstract), one kernel per example (CondConv:
Conditionally Parameterized Convolutions for Efficient Inference, abstract),
and temperature-scaled softmax attention (FMDConv: Fast multi-attention
dynamic convolution via speed-accuracy trade-off, abstract).
"""
import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from dynamic_convolution_b200 import synth

RTOL = 1e-12


def _rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _rand_layer(rng, B, Cin, Cout, H, W, K, stride, pad, groups, n):
    x = rng.standard_normal((B, H, W, Cin))
    E = rng.standard_normal((n, Cout, K, K, Cin // groups))
    alpha = rng.uniform(0.1, 1.0, (B, n))
    bias = rng.standard_normal((n, Cout))
    return x, E, alpha, bias


def _torch_conv(x, Wb, bb, stride, pad, groups):
    """Library convolution (torch, fp64, CPU): NHWC x, [Cout][KH][KW][Cg] kernel."""
    xt = torch.from_numpy(np.ascontiguousarray(x.transpose(0, 3, 1, 2)))
    wt = torch.from_numpy(np.ascontiguousarray(Wb.transpose(0, 3, 1, 2)))
    bt = None if bb is None else torch.from_numpy(np.ascontiguousarray(bb))
    y = torch.nn.functional.conv2d(xt, wt, bt, stride=stride, padding=pad, groups=groups)
    return y.numpy().transpose(0, 2, 3, 1)


SHAPES = [
    # B, Cin, Cout, H, W, K, stride, pad, groups
    (2, 3, 5, 7, 6, 3, 1, 1, 1),
    (1, 4, 4, 9, 5, 5, 1, 2, 4),      # depthwise
    (2, 6, 3, 8, 8, 1, 1, 0, 1),      # 1x1
    (1, 4, 6, 7, 9, 3, 2, 1, 2),      # stride 2, groups 2
    (3, 2, 2, 5, 5, 3, 2, 0, 1),      # stride 2, no pad
    (1, 5, 5, 6, 7, 5, 1, 1, 5),      # depthwise, pad smaller than K/2
    (2, 3, 4, 4, 4, 3, 1, 2, 1),      # pad larger than K/2
]


@pytest.mark.parametrize("shape", SHAPES)
def test_n1_alpha1_is_static_conv_torch(shape):
    """n=1, alpha=1 reduces to a plain convolution: compare with torch conv2d (fp64)."""
    B, Cin, Cout, H, W, K, s, p, g = shape
    rng = np.random.default_rng(hash(shape) % 2**32)
    x, E, _, bias = _rand_layer(rng, B, Cin, Cout, H, W, K, s, p, g, 1)
    alpha = np.ones((B, 1))
    y = oracle.forward(x, E, alpha, bias, stride=s, pad=p, groups=g)
    ref = _torch_conv(x, E[0], bias[0], s, p, g)
    assert y.shape == ref.shape
    assert _rel(y, ref) < RTOL


@pytest.mark.parametrize("shape", SHAPES)
def test_mixed_kernel_matches_torch_conv(shape):
    """General n: torch conv2d on a kernel mixed with numpy's tensordot, per sample."""
    B, Cin, Cout, H, W, K, s, p, g = shape
    rng = np.random.default_rng(1 + hash(shape) % 2**31)
    n = 3
    x, E, alpha, bias = _rand_layer(rng, B, Cin, Cout, H, W, K, s, p, g, n)
    y = oracle.forward(x, E, alpha, bias, stride=s, pad=p, groups=g)
    for b in range(B):
        Wb = np.tensordot(alpha[b], E, axes=(0, 0))
        bb = alpha[b] @ bias
        ref = _torch_conv(x[b:b + 1], Wb, bb, s, p, g)[0]
        assert _rel(y[b], ref) < RTOL


def _im2col_output_side(x, E, alpha, bias, stride, pad, groups):
    """Second formulation: explicit zero-padded im2col matrix, one matrix product
    per expert, outputs summed with alpha afterwards (output-side order)."""
    B, H, W, Cin = x.shape
    n, Cout, KH, KW, Cg = E.shape
    Ho = (H + 2 * pad - KH) // stride + 1
    Wo = (W + 2 * pad - KW) // stride + 1
    xp = np.zeros((B, H + 2 * pad, W + 2 * pad, Cin))
    xp[:, pad:pad + H, pad:pad + W, :] = x
    y = np.zeros((B, Ho, Wo, Cout))
    Coutg = Cout // groups
    for g in range(groups):
        cols = np.zeros((B, Ho, Wo, KH, KW, Cg))
        for kh in range(KH):
            for kw in range(KW):
                patch = xp[:, kh:kh + stride * (Ho - 1) + 1:stride,
                           kw:kw + stride * (Wo - 1) + 1:stride, g * Cg:(g + 1) * Cg]
                cols[:, :, :, kh, kw, :] = patch
        A = cols.reshape(B, Ho * Wo, KH * KW * Cg)
        for i in range(n):
            Wi = E[i, g * Coutg:(g + 1) * Coutg].reshape(Coutg, -1)     # [Coutg][K]
            yi = A @ Wi.T                                               # [B][P][Coutg]
            y[:, :, :, g * Coutg:(g + 1) * Coutg] += (
                alpha[:, i][:, None, None] * yi).reshape(B, Ho, Wo, Coutg)
    y += (alpha @ bias)[:, None, None, :]
    return y


@pytest.mark.parametrize("seed", range(12))
def test_brute_force_second_formulation(seed):
    """Random tiny shapes: odd sizes, k in {1,3,5}, stride {1,2}, pad {0,1,2},
    groups {1,C}, n in {1,2,5}."""
    rng = np.random.default_rng(100 + seed)
    K = int(rng.choice([1, 3, 5]))
    s = int(rng.choice([1, 2]))
    p = int(rng.choice([0, 1, 2]))
    C = int(rng.integers(1, 6))
    depthwise = bool(rng.integers(0, 2))
    Cin = C
    Cout = C if depthwise else int(rng.integers(1, 6))
    g = C if depthwise else 1
    H = int(rng.integers(K, K + 6)) | 1
    W = int(rng.integers(K, K + 6)) | 1
    n = int(rng.choice([1, 2, 5]))
    B = int(rng.integers(1, 4))
    x, E, alpha, bias = _rand_layer(rng, B, Cin, Cout, H, W, K, s, p, g, n)
    y = oracle.forward(x, E, alpha, bias, stride=s, pad=p, groups=g)
    ref = _im2col_output_side(x, E, alpha, bias, s, p, g)
    assert _rel(y, ref) < RTOL


def test_tiny_config_second_formulation():
    """The tiny fp32 layer configuration, against the im2col formulation."""
    cfg = synth.CONFIGS["tiny_fp32"]
    inp = synth.make_inputs(cfg)
    alpha = oracle.route(inp.x_f64, inp.Wr, inp.br, cfg.mode, cfg.tau)
    y = oracle.forward(inp.x_f64, inp.experts_f64, alpha, inp.bias, stride=1, pad=1)
    ref = _im2col_output_side(inp.x_f64, inp.experts_f64, alpha, inp.bias.astype(np.float64), 1, 1, 1)
    assert _rel(y, ref) < RTOL


def test_linearity_in_the_kernel():
    """conv(x, sum_i a_i W_i) = sum_i a_i conv(x, W_i), each term an n=1 oracle call."""
    rng = np.random.default_rng(7)
    B, Cin, Cout, H, W, K, n = 3, 4, 6, 7, 8, 3, 4
    x, E, alpha, bias = _rand_layer(rng, B, Cin, Cout, H, W, K, 1, 1, 1, n)
    y = oracle.forward(x, E, alpha, bias, stride=1, pad=1)
    acc = np.zeros_like(y)
    for i in range(n):
        yi = oracle.forward(x, E[i:i + 1], np.ones((B, 1)), bias[i:i + 1], stride=1, pad=1)
        acc += alpha[:, i][:, None, None, None] * yi
    assert _rel(y, acc) < RTOL


def test_impulse_pins_orientation():
    """A unit impulse at (h0, w0, c) gives y[h0-kh+p, w0-kw+p, co] = W_b[co,kh,kw,c] + b_b[co]
    (cross-correlation), and b_b[co] everywhere else."""
    rng = np.random.default_rng(3)
    B, Cin, Cout, H, W, K, p, n = 2, 3, 4, 9, 9, 3, 1, 3
    _, E, alpha, bias = _rand_layer(rng, B, Cin, Cout, H, W, K, 1, p, 1, n)
    h0, w0, c0 = 4, 3, 2
    x = np.zeros((B, H, W, Cin))
    x[:, h0, w0, c0] = 1.0
    y = oracle.forward(x, E, alpha, bias, stride=1, pad=p)
    for b in range(B):
        Wb = np.tensordot(alpha[b], E, axes=(0, 0))
        bb = alpha[b] @ bias
        expect = np.broadcast_to(bb, y[b].shape).copy()
        for kh in range(K):
            for kw in range(K):
                expect[h0 - kh + p, w0 - kw + p, :] += Wb[:, kh, kw, c0]
        assert np.abs(y[b] - expect).max() < 1e-13


def test_constant_input_interior_closed_form():
    """A constant-1 input gives y = sum_{kh,kw,ci} W_b + b_b at interior pixels."""
    rng = np.random.default_rng(4)
    B, Cin, Cout, H, W, K, n = 2, 5, 3, 8, 8, 3, 2
    _, E, alpha, bias = _rand_layer(rng, B, Cin, Cout, H, W, K, 1, 1, 1, n)
    x = np.ones((B, H, W, Cin))
    y = oracle.forward(x, E, alpha, bias, stride=1, pad=1)
    for b in range(B):
        Wb = np.tensordot(alpha[b], E, axes=(0, 0))
        expect = Wb.sum(axis=(1, 2, 3)) + alpha[b] @ bias
        assert np.abs(y[b, 1:-1, 1:-1, :] - expect).max() < 1e-12


def test_zero_input_gives_mixed_bias_and_route_of_br():
    """x = 0: GAP = 0 so alpha = act(br); y equals the mixed bias everywhere."""
    rng = np.random.default_rng(5)
    B, C, H, W, n = 3, 6, 5, 5, 4
    x = np.zeros((B, H, W, C))
    Wr = rng.standard_normal((n, C))
    br = rng.standard_normal(n)
    a_sig = oracle.route(x, Wr, br, oracle.SIGMOID)
    assert np.allclose(a_sig, 1.0 / (1.0 + np.exp(-br))[None, :], rtol=0, atol=1e-15)
    tau = 2.5
    a_sm = oracle.route(x, Wr, br, oracle.SOFTMAX, tau)
    assert np.allclose(a_sm, scipy.special.softmax(br / tau)[None, :], rtol=0, atol=1e-15)
    E = rng.standard_normal((n, C, 3, 3, C))
    bias = rng.standard_normal((n, C))
    y = oracle.forward(x, E, a_sm, bias, stride=1, pad=1)
    assert np.abs(y - (a_sm @ bias)[:, None, None, :]).max() < 1e-14


def test_constant_input_route_closed_form():
    """x = c everywhere: g = c, so z_i = c * sum_j Wr[i,j] + br_i."""
    rng = np.random.default_rng(6)
    B, C, H, W, n = 2, 7, 4, 6, 5
    cvals = np.array([0.75, -1.5])
    x = np.broadcast_to(cvals[:, None, None, None], (B, H, W, C)).copy()
    Wr = rng.standard_normal((n, C))
    br = rng.standard_normal(n)
    z = cvals[:, None] * Wr.sum(axis=1)[None, :] + br[None, :]
    assert np.allclose(oracle.route(x, Wr, br, oracle.SIGMOID), scipy.special.expit(z),
                       rtol=0, atol=1e-14)
    assert np.allclose(oracle.route(x, Wr, br, oracle.SOFTMAX, 0.7),
                       scipy.special.softmax(z / 0.7, axis=1), rtol=0, atol=1e-14)


@pytest.mark.parametrize("mode,tau", [(oracle.SIGMOID, 1.0), (oracle.SOFTMAX, 1.0),
                                      (oracle.SOFTMAX, 0.3), (oracle.SOFTMAX, 30.0)])
def test_route_against_library_routines(mode, tau):
    """GAP via numpy mean, FC via a matrix product, activation via scipy."""
    rng = np.random.default_rng(8)
    B, C, H, W, n = 4, 12, 5, 7, 6
    x = rng.standard_normal((B, H, W, C)) + rng.standard_normal((B, 1, 1, C))
    Wr = rng.standard_normal((n, C))
    br = rng.standard_normal(n)
    z = x.mean(axis=(1, 2)) @ Wr.T + br
    ref = scipy.special.expit(z) if mode == oracle.SIGMOID else scipy.special.softmax(z / tau, axis=1)
    got = oracle.route(x, Wr, br, mode, tau)
    assert np.abs(got - ref).max() < 1e-14


def test_route_invariants():
    rng = np.random.default_rng(9)
    B, C, H, W, n = 5, 8, 6, 6, 7
    x = rng.standard_normal((B, H, W, C)) * 3 + rng.standard_normal((B, 1, 1, C)) * 2
    Wr = rng.standard_normal((n, C))
    br = rng.standard_normal(n)
    a = oracle.route(x, Wr, br, oracle.SOFTMAX, 1.0)
    assert np.abs(a.sum(axis=1) - 1.0).max() < 1e-12
    assert (a > 0).all()
    s = oracle.route(x, Wr, br, oracle.SIGMOID)
    assert ((s > 0) & (s < 1)).all()
    # tau -> infinity flattens the softmax to 1/n
    flat = oracle.route(x, Wr, br, oracle.SOFTMAX, 1e12)
    assert np.abs(flat - 1.0 / n).max() < 1e-10


def test_tau30_near_uniform_bound():
    """At tau=30 on the deep layer's input statistics, |alpha_i - 1/n| is bounded by
    the closed form 1/n * (exp(2 max|z|/tau) - 1)."""
    cfg = synth.CONFIGS["deep_3x3_tau30"].scaled(B=8)
    inp = synth.make_inputs(cfg)
    a = oracle.route(inp.x_f64, inp.Wr, inp.br, cfg.mode, cfg.tau)
    g = inp.x_f64.mean(axis=(1, 2))
    zmax = np.abs(g @ inp.Wr.astype(np.float64).T).max()
    bound = (1.0 / cfg.n) * (math.exp(2 * zmax / cfg.tau) - 1.0)
    assert np.abs(a - 1.0 / cfg.n).max() <= bound
    assert np.abs(a - 1.0 / cfg.n).max() < 1e-3


def test_batch_permutation():
    rng = np.random.default_rng(10)
    B, Cin, Cout, H, W, K, n = 4, 3, 5, 6, 6, 3, 3
    x, E, alpha, bias = _rand_layer(rng, B, Cin, Cout, H, W, K, 1, 1, 1, n)
    perm = np.array([2, 0, 3, 1])
    y = oracle.forward(x, E, alpha, bias, stride=1, pad=1)
    yp = oracle.forward(x[perm], E, alpha[perm], bias, stride=1, pad=1)
    assert np.array_equal(y[perm], yp)
    Wr = rng.standard_normal((n, Cin))
    br = rng.standard_normal(n)
    a = oracle.route(x, Wr, br, oracle.SOFTMAX, 1.0)
    assert np.array_equal(a[perm], oracle.route(x[perm], Wr, br, oracle.SOFTMAX, 1.0))


def test_expert_permutation():
    """Permuting experts together with Wr rows, br and bias leaves alpha-weighted y unchanged."""
    rng = np.random.default_rng(11)
    B, Cin, Cout, H, W, K, n = 2, 4, 4, 6, 5, 3, 5
    x, E, _, bias = _rand_layer(rng, B, Cin, Cout, H, W, K, 1, 1, 1, n)
    Wr = rng.standard_normal((n, Cin))
    br = rng.standard_normal(n)
    perm = np.array([3, 1, 4, 0, 2])
    for mode in (oracle.SIGMOID, oracle.SOFTMAX):
        a = oracle.route(x, Wr, br, mode, 1.0)
        ap = oracle.route(x, Wr[perm], br[perm], mode, 1.0)
        assert np.abs(ap - a[:, perm]).max() < 1e-15
        y = oracle.forward(x, E, a, bias, stride=1, pad=1)
        yp = oracle.forward(x, E[perm], ap, bias[perm], stride=1, pad=1)
        assert _rel(y, yp) < RTOL


def test_sample_subset_matches_full():
    rng = np.random.default_rng(12)
    x, E, alpha, bias = _rand_layer(rng, 5, 3, 4, 6, 6, 3, 1, 1, 1, 2)
    full = oracle.forward(x, E, alpha, bias, stride=1, pad=1)
    part = oracle.forward(x, E, alpha, bias, stride=1, pad=1, samples=(2, 2))
    assert np.array_equal(full[2:4], part)


def test_assemble_matches_tensordot():
    rng = np.random.default_rng(13)
    E = rng.standard_normal((6, 4, 3, 3, 5))
    a = rng.standard_normal(6)
    assert _rel(oracle.assemble(E, a), np.tensordot(a, E, axes=(0, 0))) < RTOL


def test_no_bias_means_zero_bias():
    rng = np.random.default_rng(14)
    x, E, alpha, _ = _rand_layer(rng, 2, 3, 3, 5, 5, 3, 1, 1, 1, 2)
    y0 = oracle.forward(x, E, alpha, None, stride=1, pad=1)
    y1 = oracle.forward(x, E, alpha, np.zeros((2, 3)), stride=1, pad=1)
    assert np.array_equal(y0, y1)


def test_rejects_bad_arguments():
    x = np.zeros((1, 4, 4, 3))
    with pytest.raises(ValueError):
        oracle.route(x, np.zeros((2, 3)), np.zeros(2), oracle.SOFTMAX, 0.0)
    with pytest.raises(ValueError):
        oracle.route(x, np.zeros((2, 3)), np.zeros(2), 7, 1.0)


def test_synth_recipe_statistics():
    """The generator matches its stated recipe (variance reading of N(0, v))."""
    cfg = synth.CONFIGS["resnet18_3x3"].scaled(B=8)
    inp = synth.make_inputs(cfg)
    assert inp.x_store.dtype == np.uint16
    assert abs(inp.x_f64.std() - 1.0) < 0.01
    assert abs(inp.experts_f64.std() - math.sqrt(2.0 / (9 * 128))) / math.sqrt(2.0 / 1152) < 0.01
    assert abs(inp.Wr.std() - math.sqrt(1.0 / 128)) / math.sqrt(1.0 / 128) < 0.12  # 512 draws
    assert np.all(inp.br == 0)
    # bf16 rounding is round-to-nearest-even and exact on representable values
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0])
    assert np.array_equal(synth.bf16_to_f64(synth.bf16_bits(v)), [1.0, 1.0, 1.0 + 2 ** -6, -2.5, 0.0])


def test_row_band_matches_full_forward():
    rng = np.random.default_rng(15)
    x, E, alpha, bias = _rand_layer(rng, 3, 4, 5, 9, 7, 3, 2, 1, 1, 3)
    full = oracle.forward(x, E, alpha, bias, stride=2, pad=1)
    for b, oh0, noh in [(0, 0, 1), (2, 1, 3), (1, 0, full.shape[1])]:
        band = oracle.forward_rows(x, E, alpha, bias, b, oh0, noh, stride=2, pad=1)
        assert np.array_equal(band, full[b, oh0:oh0 + noh])


# ---- FMDConv channel attentions (input attention, output attention: FMDConv,
# abstract; the page gives no formula, the reading is a per-channel factor of
# the sample's input and output)

@pytest.mark.parametrize("shape", SHAPES)
def test_channel_attention_matches_torch_conv(shape):
    """torch conv2d (fp64) on the input scaled by a_in channel by channel, with
    the mixed kernel and bias, then scaled by a_out channel by channel."""
    B, Cin, Cout, H, W, K, s, p, g = shape
    rng = np.random.default_rng(7 + hash(shape) % 2**31)
    n = 3
    x, E, alpha, bias = _rand_layer(rng, B, Cin, Cout, H, W, K, s, p, g, n)
    a_in = rng.uniform(0.05, 1.0, (B, Cin))
    a_out = rng.uniform(0.05, 1.0, (B, Cout))
    y = oracle.forward_attn(x, E, alpha, bias, a_in, a_out, stride=s, pad=p, groups=g)
    for b in range(B):
        Wb = np.tensordot(alpha[b], E, axes=(0, 0))
        bb = alpha[b] @ bias
        xs = x[b:b + 1] * a_in[b][None, None, None, :]
        ref = _torch_conv(xs, Wb, bb, s, p, g)[0] * a_out[b][None, None, :]
        assert _rel(y[b], ref) < RTOL


def test_channel_attention_absent_or_ones_is_the_plain_forward():
    rng = np.random.default_rng(11)
    x, E, alpha, bias = _rand_layer(rng, 2, 4, 6, 6, 5, 3, 1, 1, 1, 2)
    plain = oracle.forward(x, E, alpha, bias, pad=1)
    assert np.array_equal(oracle.forward_attn(x, E, alpha, bias, None, None, pad=1), plain)
    ones = oracle.forward_attn(x, E, alpha, bias, np.ones((2, 4)), np.ones((2, 6)), pad=1)
    assert _rel(ones, plain) < RTOL


def test_channel_attention_scale_invariance_without_bias():
    """Without bias, c * a_in with a_out / c leaves y unchanged (bilinearity)."""
    rng = np.random.default_rng(12)
    x, E, alpha, _ = _rand_layer(rng, 2, 3, 4, 5, 6, 3, 1, 1, 1, 2)
    a_in = rng.uniform(0.1, 1.0, (2, 3))
    a_out = rng.uniform(0.1, 1.0, (2, 4))
    y1 = oracle.forward_attn(x, E, alpha, None, a_in, a_out, pad=1)
    y2 = oracle.forward_attn(x, E, alpha, None, 2.5 * a_in, a_out / 2.5, pad=1)
    assert _rel(y2, y1) < RTOL


def test_channel_attention_zero_input_gives_scaled_bias():
    """x = 0: y[b, ., ., co] = a_out[b, co] * sum_i alpha_bi bias_i[co] exactly."""
    rng = np.random.default_rng(13)
    _, E, alpha, bias = _rand_layer(rng, 2, 3, 4, 5, 5, 3, 1, 1, 1, 2)
    x = np.zeros((2, 5, 5, 3))
    a_in = rng.uniform(0.1, 1.0, (2, 3))
    a_out = rng.uniform(0.1, 1.0, (2, 4))
    y = oracle.forward_attn(x, E, alpha, bias, a_in, a_out, pad=1)
    ref = (a_out * (alpha @ bias))[:, None, None, :]
    assert np.allclose(y, np.broadcast_to(ref, y.shape), rtol=1e-14, atol=0)


def test_channel_attention_routing_is_sigmoid_of_fc_of_gap():
    """The channel attentions are routing-shaped outputs (sigmoid of a linear
    layer of the pooled input, one per channel): the oracle's routing with
    n = channel count gives the library sigmoid of the library mean's FC."""
    rng = np.random.default_rng(14)
    x = rng.standard_normal((3, 5, 4, 6))
    Wi = rng.standard_normal((6, 6)) / np.sqrt(6)
    bi = rng.standard_normal(6) * 0.1
    a = oracle.route(x, Wi, bi, oracle.SIGMOID, 1.0)
    ref = scipy.special.expit(x.mean(axis=(1, 2)) @ Wi.T + bi)
    assert np.abs(a - ref).max() < 1e-14
