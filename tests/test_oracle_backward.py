"""Pins for the oracle's backward functions, independent of their formulas.

The per-example kernels and their mixture are learned (CondConv, abstract;
KernelWarehouse, abstract), so the layer's gradients are those of the forward
definition. They are checked against:

* central differences of the (separately pinned) forward oracle, for the loss
  L = <y, dy> as a function of every input: x through both the convolution
  and the router, the experts, the biases, the router's weight and bias, and
  the attentions taken as an input of their own;
* torch autograd of the same definition (a library differentiator, fp64 CPU);
* identities: softmax gradients sum to zero over experts, dy = 0 gives zero
  everywhere, x = 0 leaves only the bias terms, and the pooled vector's
  gradient adds dg/(H*W) on every pixel.
"""
import numpy as np
import pytest
import torch

import oracle

EPS = 1e-5
FD_RTOL = 1e-6

# B, Cin, Cout, H, W, KH, KW, stride, pad, groups, n, mode, tau
CASES = [
    (2, 4, 6, 5, 4, 3, 3, 1, 1, 1, 3, oracle.SOFTMAX, 2.5),
    (2, 3, 5, 6, 5, 3, 2, 1, 1, 1, 2, oracle.SIGMOID, 1.0),    # KH != KW
    (1, 4, 6, 7, 6, 3, 3, 2, 1, 2, 3, oracle.SOFTMAX, 0.7),    # stride 2, groups 2
    (2, 4, 4, 6, 6, 5, 5, 1, 2, 4, 4, oracle.SIGMOID, 1.0),    # depthwise 5x5
    (3, 5, 3, 4, 5, 1, 1, 1, 0, 1, 5, oracle.SOFTMAX, 1.0),    # 1x1
    (1, 2, 3, 5, 5, 3, 3, 2, 0, 1, 2, oracle.SIGMOID, 1.0),    # stride 2, no padding
]
IDS = ["softmax-3x3", "sigmoid-3x2", "stride2-groups2", "depthwise-5x5", "pointwise",
       "stride2-nopad"]


def _layer(case, seed):
    B, Cin, Cout, H, W, KH, KW, s, p, g, n, mode, tau = case
    rng = np.random.default_rng(seed)
    Ho = (H + 2 * p - KH) // s + 1
    Wo = (W + 2 * p - KW) // s + 1
    return dict(
        x=rng.standard_normal((B, H, W, Cin)) + rng.standard_normal((B, 1, 1, Cin)),
        E=rng.standard_normal((n, Cout, KH, KW, Cin // g)) * 0.5,
        bias=rng.standard_normal((n, Cout)),
        Wr=rng.standard_normal((n, Cin)),
        br=rng.standard_normal(n) * 0.3,
        dy=rng.standard_normal((B, Ho, Wo, Cout)),
        rng=rng)


def _loss(L, case, x=None, E=None, bias=None, Wr=None, br=None):
    B, Cin, Cout, H, W, KH, KW, s, p, g, n, mode, tau = case
    x = L["x"] if x is None else x
    alpha = oracle.route(x, L["Wr"] if Wr is None else Wr, L["br"] if br is None else br, mode, tau)
    y = oracle.forward(x, L["E"] if E is None else E, alpha, L["bias"] if bias is None else bias,
                       stride=s, pad=p, groups=g)
    return float(np.sum(y * L["dy"]))


def _grads(L, case):
    B, Cin, Cout, H, W, KH, KW, s, p, g, n, mode, tau = case
    alpha = oracle.route(L["x"], L["Wr"], L["br"], mode, tau)
    return alpha, oracle.backward(L["x"], L["dy"], L["E"], alpha, L["bias"], L["Wr"], mode, tau,
                                  stride=s, pad=p, groups=g)


def _directional(f, P, grad, rng, ndir=3):
    """Central differences of f along random directions against <grad, v>."""
    for _ in range(ndir):
        v = rng.standard_normal(P.shape)
        fd = (f(P + EPS * v) - f(P - EPS * v)) / (2 * EPS)
        an = float(np.sum(grad * v))
        scale = max(abs(an), abs(fd), 1e-3)
        assert abs(fd - an) <= FD_RTOL * scale + 1e-8, (fd, an)


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_central_differences_every_input(case):
    L = _layer(case, 1)
    _, gr = _grads(L, case)
    rng = L["rng"]
    _directional(lambda v: _loss(L, case, x=v), L["x"], gr["dx"], rng)
    _directional(lambda v: _loss(L, case, E=v), L["E"], gr["dexperts"], rng)
    _directional(lambda v: _loss(L, case, bias=v), L["bias"], gr["dbias"], rng)
    _directional(lambda v: _loss(L, case, Wr=v), L["Wr"], gr["dWr"], rng)
    _directional(lambda v: _loss(L, case, br=v), L["br"], gr["dbr"], rng)


@pytest.mark.parametrize("case", CASES[:4], ids=IDS[:4])
def test_central_differences_attention_as_input(case):
    """dalpha: the attentions as an input of their own (router not involved)."""
    B, Cin, Cout, H, W, KH, KW, s, p, g, n, mode, tau = case
    L = _layer(case, 2)
    alpha = L["rng"].uniform(0.05, 1.0, (B, n))
    _, _, dalpha = oracle.backward_weight(L["x"], L["dy"], L["E"], alpha, L["bias"], s, p, g)
    f = lambda a: float(np.sum(oracle.forward(L["x"], L["E"], a, L["bias"], s, p, g) * L["dy"]))
    _directional(f, alpha, dalpha, L["rng"])


def test_central_differences_elementwise_tiny():
    """Every element of x and of Wr on a tiny softmax layer, one at a time."""
    case = (1, 2, 3, 3, 4, 3, 3, 1, 1, 1, 3, oracle.SOFTMAX, 1.7)
    L = _layer(case, 3)
    _, gr = _grads(L, case)
    for name, key in (("x", "dx"), ("Wr", "dWr")):
        P = L[name]
        for idx in np.ndindex(P.shape):
            e = np.zeros_like(P)
            e[idx] = 1.0
            fd = (_loss(L, case, **{name: P + EPS * e}) - _loss(L, case, **{name: P - EPS * e})) / (2 * EPS)
            assert abs(fd - gr[key][idx]) <= FD_RTOL * max(abs(fd), 1e-2), (name, idx, fd, gr[key][idx])


def _torch_grads(L, case):
    """The forward definition in torch ops (fp64, CPU), differentiated by autograd."""
    B, Cin, Cout, H, W, KH, KW, s, p, g, n, mode, tau = case
    t = lambda a: torch.tensor(a, dtype=torch.float64, requires_grad=True)
    x, E, bias, Wr, br = t(L["x"]), t(L["E"]), t(L["bias"]), t(L["Wr"]), t(L["br"])
    z = x.mean(dim=(1, 2)) @ Wr.T + br
    alpha = torch.sigmoid(z) if mode == oracle.SIGMOID else torch.softmax(z / tau, dim=1)
    Wb = torch.einsum("bi,iokhc->bokhc", alpha, E)            # [B][Cout][KH][KW][Cg]
    ys = []
    for b in range(B):
        xb = x[b].permute(2, 0, 1).unsqueeze(0)               # NCHW
        # [Cout][Cg][KH][KW], made contiguous: with a permuted (non-contiguous)
        # kernel inside the graph, torch's CPU conv2d backward returned a wrong
        # kernel gradient for grouped strided layers (central differences
        # disagree with it there and agree with the contiguous form)
        wb = Wb[b].permute(0, 3, 1, 2).contiguous()
        ys.append(torch.nn.functional.conv2d(xb, wb, alpha[b] @ bias, stride=s, padding=p,
                                             groups=g))
    y = torch.cat(ys).permute(0, 2, 3, 1)
    (y * torch.from_numpy(L["dy"])).sum().backward()
    return dict(dx=x.grad.numpy(), dexperts=E.grad.numpy(), dbias=bias.grad.numpy(),
                dWr=Wr.grad.numpy(), dbr=br.grad.numpy())


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_matches_torch_autograd(case):
    L = _layer(case, 4)
    _, gr = _grads(L, case)
    ref = _torch_grads(L, case)
    for k, v in ref.items():
        err = np.linalg.norm(gr[k] - v) / max(np.linalg.norm(v), 1e-300)
        assert err <= 1e-11, (k, err)


def test_softmax_router_gradients_sum_to_zero_over_experts():
    """softmax(z/tau) is unchanged by adding a constant to every logit, so
    sum_i dz_i = 0: the router bias gradients sum to zero, and so does every
    column of the router weight gradient."""
    case = CASES[0]
    L = _layer(case, 5)
    _, gr = _grads(L, case)
    assert abs(gr["dbr"].sum()) <= 1e-12 * np.abs(gr["dbr"]).sum()
    assert np.abs(gr["dWr"].sum(axis=0)).max() <= 1e-12 * np.abs(gr["dWr"]).sum()


@pytest.mark.parametrize("case", CASES[:3], ids=IDS[:3])
def test_zero_upstream_gradient_gives_zero(case):
    L = _layer(case, 6)
    L["dy"] = np.zeros_like(L["dy"])
    _, gr = _grads(L, case)
    for k, v in gr.items():
        assert not np.any(v), k


def test_zero_input_leaves_bias_terms():
    """x = 0: every per-sample weight gradient is zero, so dexperts = 0 and
    dalpha[b,i] = sum_co (sum over pixels of dy[b,.,.,co]) * bias_i[co]."""
    case = CASES[0]
    B, Cin, Cout, H, W, KH, KW, s, p, g, n, mode, tau = case
    L = _layer(case, 7)
    x = np.zeros_like(L["x"])
    alpha = L["rng"].uniform(0.1, 1, (B, n))
    dE, dbias, dalpha = oracle.backward_weight(x, L["dy"], L["E"], alpha, L["bias"], s, p, g)
    assert not np.any(dE)
    S = L["dy"].sum(axis=(1, 2))                               # [B][Cout]
    np.testing.assert_allclose(dalpha, S @ L["bias"].T, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(dbias, alpha.T @ S, rtol=1e-13, atol=1e-13)


def test_pooled_gradient_adds_a_constant_per_channel():
    case = CASES[2]
    B, Cin, Cout, H, W, KH, KW, s, p, g, n, mode, tau = case
    L = _layer(case, 8)
    alpha = L["rng"].uniform(0.1, 1, (B, n))
    dg = L["rng"].standard_normal((B, Cin))
    a = oracle.backward_data(L["dy"], L["E"], alpha, dg, H, W, s, p, g)
    b = oracle.backward_data(L["dy"], L["E"], alpha, None, H, W, s, p, g)
    np.testing.assert_allclose(a - b, np.broadcast_to(dg[:, None, None, :] / (H * W), a.shape),
                               rtol=1e-12, atol=1e-14)


def test_sample_ranges_match_full():
    case = CASES[1]
    B, Cin, Cout, H, W, KH, KW, s, p, g, n, mode, tau = case
    L = _layer(case, 9)
    alpha = L["rng"].uniform(0.1, 1, (B, n))
    full = oracle.backward_data(L["dy"], L["E"], alpha, None, H, W, s, p, g)
    part = oracle.backward_data(L["dy"], L["E"], alpha, None, H, W, s, p, g, samples=(1, 1))
    np.testing.assert_array_equal(full[1:2], part)
    dW, db = oracle.weight_grad(L["x"], L["dy"], KH, KW, s, p, g)
    dW1, db1 = oracle.weight_grad(L["x"], L["dy"], KH, KW, s, p, g, samples=(1, 1))
    np.testing.assert_array_equal(dW[1:2], dW1)
    np.testing.assert_array_equal(db[1:2], db1)
    # the per-sample gradients recombine to the mixture's gradients
    dE, dbias, dalpha = oracle.backward_weight(L["x"], L["dy"], L["E"], alpha, L["bias"], s, p, g)
    np.testing.assert_allclose(dE, np.einsum("bi,b...->i...", alpha, dW), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_restrictions_match_the_full_functions(case):
    """dalpha of a sample range, dexperts at chosen elements and dbias equal the
    corresponding parts of backward_weight (pinned above)."""
    B, Cin, Cout, H, W, KH, KW, s, p, g, n, mode, tau = case
    L = _layer(case, 10)
    alpha = L["rng"].uniform(0.1, 1, (B, n))
    dE, dbias, dalpha = oracle.backward_weight(L["x"], L["dy"], L["E"], alpha, L["bias"], s, p, g)
    np.testing.assert_allclose(oracle.dalpha(L["x"], L["dy"], L["E"], L["bias"], s, p, g),
                               dalpha, rtol=1e-12, atol=1e-12)
    b0 = B - 1
    np.testing.assert_allclose(oracle.dalpha(L["x"], L["dy"], L["E"], L["bias"], s, p, g,
                                             samples=(b0, 1)), dalpha[b0:], rtol=1e-12, atol=1e-12)
    idx = L["rng"].choice(dE[0].size, size=min(17, dE[0].size), replace=False)
    got = oracle.dexperts_at(L["x"], L["dy"], alpha, idx, n, Cout, KH, KW, s, p, g)
    np.testing.assert_allclose(got, dE.reshape(n, -1)[:, idx], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle.dbias(L["dy"], alpha), dbias, rtol=1e-12, atol=1e-12)
