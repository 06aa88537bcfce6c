"""GPU parity of the backward pass against the oracle's backward:
dynconv_backward_weight (tcgen05 and CUDA-core per-sample weight gradients,
then the mixture's gradients), dynconv_route_backward, and
dynconv_backward_data (the transposed problem on every forward variant, and
the generic kernel for strided or grouped layers). Element by element on small
layers with ragged tiles; on sampled outputs at the full layer sizes.

Tolerances (the gradients of experts, biases and attentions are fp32 sums of
exact products of bf16 values, so fp32 rounding bounds them):
  * dexperts, dbias, dalpha: relative Frobenius <= 1e-4, max abs <= 1e-3 of
    the largest reference magnitude;
  * dWr, dbr, dg: relative Frobenius <= 1e-3 (the softmax's gradient subtracts
    the attention-weighted mean from each dalpha);
  * dx: the forward's tolerances for the layer dtype, unchanged (it is a
    convolution with the bf16-rounded mixed kernel, plus dg/(H*W), rounded
    once)."""
import numpy as np
import pytest
import torch

import dynamic_convolution_b200 as dc
import oracle
from dynamic_convolution_b200 import synth

from .gpu_util import (Layer, alpha_f32_rounded, compare,
                       from_device, to_device)

pytestmark = pytest.mark.gpu

GRAD_REL = 1e-4
ROUTER_REL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _built():
    from dynamic_convolution_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _close(got, ref, rel, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.isfinite(got).all(), (what, "unwritten or non-finite")
    err = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    mx = float(np.abs(got - ref).max()) if got.size else 0.0
    assert err <= rel and mx <= 10 * rel * max(float(np.abs(ref).max()), 1e-30), (what, err, mx)


class Case:
    """One layer's inputs on the device, the oracle's attentions, and dy."""

    def __init__(self, cfg, seed=3):
        self.cfg = cfg
        self.inp = synth.make_inputs(cfg, seed=seed, structured=1.0)
        self.L = Layer(self.inp)
        self.a = alpha_f32_rounded(oracle.route(self.inp.x_f64, self.inp.Wr, self.inp.br,
                                                cfg.mode, cfg.tau))
        self.L.alpha.copy_(torch.from_numpy(self.a.astype(np.float32)))
        dys, self.dy_f = synth.make_upstream_grad(cfg, seed + 1)
        self.dy = to_device(dys, cfg.dtype)

    def run(self, wg_variant=dc.VARIANT_AUTO, dx_variant=dc.VARIANT_AUTO, bias=True):
        cfg, L = self.cfg, self.L
        d = dc.desc_from_config(cfg, wg_variant)
        wsb = max(dc.dynconv_backward_workspace_size(d),
                  dc.dynconv_backward_workspace_size(dc.desc_from_config(cfg, dx_variant)))
        ws = torch.empty(max(wsb, 256), dtype=torch.uint8, device="cuda")
        nan = lambda *s: torch.full(s, float("nan"), device="cuda")
        dE = nan(*self.inp.experts_f64.shape)
        dbias = nan(cfg.n, cfg.C_out) if bias else None
        dalpha = nan(cfg.B, cfg.n)
        dc.check(dc.dynconv_backward_weight(d, L.x, self.dy, L.experts, L.alpha,
                                            L.bias if bias else None, dE, dbias, dalpha, ws, wsb),
                 "dynconv_backward_weight")
        dWr, dbr, dg = nan(cfg.n, cfg.C_in), nan(cfg.n), nan(cfg.B, cfg.C_in)
        dc.check(dc.dynconv_route_backward(d, L.x, L.Wr, L.alpha, dalpha, cfg.mode, cfg.tau,
                                           dWr, dbr, dg, ws, wsb), "dynconv_route_backward")
        dx = torch.full_like(L.x, float("nan"))
        dc.check(dc.dynconv_backward_data(dc.desc_from_config(cfg, dx_variant), self.dy,
                                          L.experts, L.alpha, dg, dx, ws, wsb),
                 "dynconv_backward_data")
        torch.cuda.synchronize()
        assert dc.dynconv_device_status(None) == dc.OK
        return {k: from_device(v) for k, v in dict(dexperts=dE, dalpha=dalpha, dWr=dWr, dbr=dbr,
                                                    dg=dg, dx=dx).items()} | (
            {"dbias": from_device(dbias)} if bias else {})

    def reference(self, bias=True):
        cfg = self.cfg
        return oracle.backward(self.inp.x_f64, self.dy_f, self.inp.experts_f64, self.a,
                               self.inp.bias if bias else None, self.inp.Wr, cfg.mode, cfg.tau,
                               stride=cfg.stride, pad=cfg.pad, groups=cfg.groups)


def _check_all(got, ref, cfg):
    _close(got["dexperts"], ref["dexperts"], GRAD_REL, "dexperts")
    if "dbias" in got:
        _close(got["dbias"], ref["dbias"], GRAD_REL, "dbias")
    _close(got["dalpha"], ref["dalpha"], GRAD_REL, "dalpha")
    _close(got["dWr"], ref["dWr"], ROUTER_REL, "dWr")
    _close(got["dbr"], ref["dbr"], ROUTER_REL, "dbr")
    _close(got["dg"], ref["dg"], ROUTER_REL, "dg")
    r = compare(got["dx"], ref["dx"], cfg.dtype)
    assert r["ok"], ("dx", r)


LC = synth.LayerConfig
DENSE = [
    # ragged: 136 output channels (second 128-channel tile of 8), 13x11 image
    # (K tiles of 7 rows x 11 = 77 pixels, the second one partly outside)
    LC("bw_ragged", synth.BF16, 3, 64, 136, 13, 11, 3, 3, 1, 1, 1, 4, synth.SOFTMAX, 1.5),
    # 72 input channels: the second 64-channel block holds 8
    LC("bw_c72", synth.BF16, 2, 72, 64, 9, 8, 3, 3, 1, 1, 1, 3, synth.SIGMOID, 1.0),
    LC("bw_pointwise", synth.BF16, 4, 64, 96, 12, 12, 1, 1, 1, 0, 1, 3, synth.SIGMOID, 1.0),
    # no padding: the transposed problem pads by 2 (not "same": CUDA-core forward)
    LC("bw_pad0", synth.BF16, 2, 64, 64, 10, 10, 3, 3, 1, 0, 1, 2, synth.SOFTMAX, 1.0),
    # 25 taps: seven groups of atoms, the last with one
    LC("bw_5x5", synth.BF16, 2, 64, 64, 8, 8, 5, 5, 1, 2, 1, 2, synth.SIGMOID, 1.0),
]


@pytest.mark.parametrize("wg", [dc.VARIANT_AUTO, dc.VARIANT_DIRECT], ids=["tcgen05", "cuda-core"])
@pytest.mark.parametrize("cfg", DENSE, ids=[c.name for c in DENSE])
def test_backward_dense(cfg, wg):
    c = Case(cfg)
    _check_all(c.run(wg_variant=wg), c.reference(), cfg)


@pytest.mark.parametrize("cfg", DENSE, ids=[c.name for c in DENSE])
def test_backward_dense_cuda_core_mixing_gradient(cfg):
    """The tcgen05 weight gradient with the CUDA-core mixing gradient (test
    hook 11 = 0); the default pairs it with the tensor-core one."""
    c = Case(cfg)
    try:
        assert dc.dynconv_test_hook(11, 0) == dc.OK
        got = c.run()
    finally:
        dc.dynconv_test_hook(11, 1)
    _check_all(got, c.reference(), cfg)


@pytest.mark.parametrize("dxv", [dc.VARIANT_FUSED, dc.VARIANT_OUTSIDE, dc.VARIANT_PREMIX,
                                 dc.VARIANT_DIRECT], ids=["fused", "outside", "premix", "direct"])
def test_backward_data_every_forward_variant(dxv):
    c = Case(DENSE[0])
    got = c.run(dx_variant=dxv)
    r = compare(got["dx"], c.reference()["dx"], synth.BF16)
    assert r["ok"], r


OTHER = [
    LC("bw_depthwise", synth.BF16, 3, 48, 48, 11, 9, 5, 5, 1, 2, 48, 4, synth.SIGMOID, 1.0),
    LC("bw_dw3", synth.BF16, 2, 32, 32, 7, 7, 3, 3, 1, 1, 32, 8, synth.SOFTMAX, 2.0),
    # strided and grouped: the generic input-gradient kernel
    LC("bw_s2g2", synth.BF16, 2, 32, 48, 9, 7, 3, 3, 2, 1, 2, 3, synth.SOFTMAX, 0.7),
    LC("bw_f32_s2", synth.F32, 2, 6, 10, 9, 8, 3, 3, 2, 0, 1, 3, synth.SIGMOID, 1.0),
    # 1x1 with 40 input channels and 48 output channels: tcgen05 boxes wider than
    # the tensor's channel extent (zero fill)
    LC("bw_c40", synth.BF16, 3, 40, 48, 10, 10, 1, 1, 1, 0, 1, 8, synth.SIGMOID, 1.0),
    # 16 output channels; 20 experts (a group of 16 and a partial group of 4)
    LC("bw_c16out", synth.BF16, 2, 64, 16, 9, 9, 3, 3, 1, 1, 1, 20, synth.SOFTMAX, 1.0),
    # grouped, stride 1: tiled expert transposition with groups, CUDA-core forward
    LC("bw_g4", synth.BF16, 2, 64, 64, 8, 8, 3, 3, 1, 1, 4, 3, synth.SIGMOID, 1.0),
    # 16 samples: the mixing gradient splits the samples into groups (partial
    # dexperts added in order)
    LC("bw_b16", synth.BF16, 16, 64, 64, 6, 6, 3, 3, 1, 1, 1, 3, synth.SOFTMAX, 1.0),
    # 12 input channels: rows not a 16-byte multiple (unvectorised sums and adds)
    LC("bw_c12", synth.BF16, 2, 12, 16, 6, 6, 3, 3, 1, 1, 1, 2, synth.SIGMOID, 1.0),
]


@pytest.mark.parametrize("cfg", OTHER + [synth.CONFIGS["tiny_fp32"]],
                         ids=[c.name for c in OTHER] + ["tiny_fp32"])
def test_backward_cuda_core_paths(cfg):
    c = Case(cfg)
    _check_all(c.run(), c.reference(), cfg)


@pytest.mark.parametrize("cfg,wg", [(OTHER[0], dc.VARIANT_DIRECT), (OTHER[1], dc.VARIANT_DEPTHWISE),
                                    (OTHER[4], dc.VARIANT_DIRECT)],
                         ids=["depthwise-generic", "depthwise-forced", "c40-cuda-core"])
def test_backward_forced_weight_kernels(cfg, wg):
    c = Case(cfg)
    _check_all(c.run(wg_variant=wg), c.reference(), cfg)


def test_backward_without_bias():
    c = Case(DENSE[1])
    got = c.run(bias=False)
    ref = c.reference(bias=False)
    assert "dbias" not in got
    _check_all(got, ref, DENSE[1])


def test_backward_is_deterministic():
    c = Case(DENSE[0])
    a, b = c.run(), c.run()
    for k in a:
        assert np.array_equal(a[k], b[k]), k


# Full-size layers: sampled outputs. dalpha of the first and last samples,
# dexperts at 256 random elements, dbias in full, dx of the last sample (its
# pooled-vector gradient from the oracle's dalpha of that sample); the router's
# parameter gradients in full where the oracle's dalpha of every sample takes
# at most ~1e10 multiply-adds.
@pytest.mark.parametrize("name", ["resnet18_3x3", "effnet_expand_1x1", "effnet_dw_5x5",
                                  "deep_3x3_tau30", "large_n64"])
def test_backward_full_size_sampled(name):
    cfg = synth.CONFIGS[name]
    c = Case(cfg, seed=0)
    got = c.run()
    inp, a, s, p, g = c.inp, c.a, cfg.stride, cfg.pad, cfg.groups
    x, E, dy = inp.x_f64, inp.experts_f64, c.dy_f
    B, n = cfg.B, cfg.n
    # dalpha
    for b in (0, B - 1):
        ref = oracle.dalpha(x, dy, E, inp.bias, s, p, g, samples=(b, 1))[0]
        _close(got["dalpha"][b], ref, GRAD_REL, f"dalpha[{b}]")
    # dexperts at sampled elements
    rng = np.random.default_rng(5)
    wsize = E[0].size
    idx = rng.choice(wsize, size=min(256, wsize), replace=False)
    ref = oracle.dexperts_at(x, dy, a, idx, n, cfg.C_out, cfg.KH, cfg.KW, s, p, g)
    _close(got["dexperts"].reshape(n, -1)[:, idx], ref, GRAD_REL, "dexperts (sampled)")
    _close(got["dbias"], oracle.dbias(dy, a), GRAD_REL, "dbias")
    # dx of the last sample
    b = B - 1
    da_b = oracle.dalpha(x, dy, E, inp.bias, s, p, g, samples=(b, 1))
    _, _, dg_b = oracle.route_backward(x[b:b + 1], inp.Wr, a[b:b + 1], da_b, cfg.mode, cfg.tau)
    dg = np.zeros((B, cfg.C_in))
    dg[b] = dg_b[0]
    ref = oracle.backward_data(dy, E, a, dg, cfg.H, cfg.W, s, p, g, samples=(b, 1))[0]
    r = compare(got["dx"][b], ref, cfg.dtype)
    assert r["ok"], ("dx", r)
    # router gradients in full where affordable
    if B * wsize * cfg.H_out * cfg.W_out <= 1e10:
        da = oracle.dalpha(x, dy, E, inp.bias, s, p, g)
        dWr, dbr, dgr = oracle.route_backward(x, inp.Wr, a, da, cfg.mode, cfg.tau)
        _close(got["dWr"], dWr, ROUTER_REL, "dWr")
        _close(got["dbr"], dbr, ROUTER_REL, "dbr")
        _close(got["dg"], dgr, ROUTER_REL, "dg")
    elif cfg.mode == synth.SOFTMAX:
        # softmax gradients sum to zero over experts at any size
        assert abs(got["dbr"].sum()) <= 1e-4 * np.abs(got["dbr"]).sum()


def test_backward_zero_batch():
    cfg = DENSE[1]
    d = dc.make_desc(0, cfg.C_in, cfg.H, cfg.W, cfg.C_out, cfg.KH, cfg.KW, 1, 1, 1, cfg.n,
                     cfg.dtype)
    dE = torch.full((cfg.n, cfg.C_out, 3, 3, cfg.C_in), 7.0, device="cuda")
    db = torch.full((cfg.n, cfg.C_out), 7.0, device="cuda")
    t = torch.zeros(16, device="cuda")
    assert dc.dynconv_backward_weight(d, t, t, t, t, t, dE, db, t, None, 0) == dc.OK
    torch.cuda.synchronize()
    assert not dE.any() and not db.any()
