"""Pins for the oracle's kernel cells (the reading of KernelWarehouse:
Rethinking the Design of Dynamic Convolution, abstract; the page gives the
idea of cells shared through a warehouse, not a formula), independent of the
cell code itself:

* m = 1 (one cell) is the ordinary mixture: the pinned oracle forward with the
  warehouse as the n experts, and the pinned routing;
* every cell's attentions are the pinned routing on that cell's rows of the
  router (the activation is taken per cell);
* one-hot attentions pick whole warehouse cells: torch conv2d (fp64, CPU) with
  the kernel put together from them;
* locality: changing one cell's attentions changes only the outputs of the
  output channels that cell holds.
"""
import numpy as np
import pytest
import torch

import oracle


def _torch_conv(x, Wb, bias, stride, pad, groups):
    xt = torch.from_numpy(np.ascontiguousarray(x.transpose(0, 3, 1, 2)))
    wt = torch.from_numpy(np.ascontiguousarray(Wb.transpose(0, 3, 1, 2)))
    bt = None if bias is None else torch.from_numpy(np.ascontiguousarray(bias))
    return torch.nn.functional.conv2d(xt, wt, bt, stride=stride, padding=pad,
                                      groups=groups).numpy().transpose(0, 2, 3, 1)


SHAPES = [
    # B, Cin, Cout, H, W, K, stride, pad, groups, m, n
    (2, 4, 6, 6, 5, 3, 1, 1, 1, 3, 5),     # cells of two output channels
    (1, 6, 4, 7, 7, 3, 2, 1, 2, 6, 4),     # cells of two thirds of an output channel
    (2, 4, 4, 5, 6, 5, 1, 2, 4, 4, 3),     # depthwise, one channel per cell
    (3, 3, 5, 4, 4, 1, 1, 0, 1, 5, 7),
]


def _case(shape, seed):
    B, Cin, Cout, H, W, K, s, p, g, m, n = shape
    rng = np.random.default_rng(seed)
    wsize = Cout * K * K * (Cin // g)
    assert wsize % m == 0
    return dict(x=rng.standard_normal((B, H, W, Cin)), E=rng.standard_normal((n, wsize // m)),
                alpha=rng.uniform(0.0, 1.0, (B, m, n)), bias=rng.standard_normal(Cout), rng=rng)


@pytest.mark.parametrize("shape", SHAPES)
def test_one_cell_is_the_ordinary_mixture(shape):
    B, Cin, Cout, H, W, K, s, p, g, m, n = shape
    c = _case(shape, 1)
    rng = c["rng"]
    E = rng.standard_normal((n, Cout, K, K, Cin // g))
    alpha = rng.uniform(0, 1, (B, 1, n))
    got = oracle.forward_cells(c["x"], E.reshape(n, -1), alpha, None, Cout, K, K, s, p, g)
    ref = oracle.forward(c["x"], E, alpha[:, 0, :], None, s, p, g)
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("mode,tau", [(oracle.SOFTMAX, 1.0), (oracle.SOFTMAX, 3.0),
                                      (oracle.SIGMOID, 1.0)])
def test_cell_routing_is_the_routing_per_cell(mode, tau):
    rng = np.random.default_rng(2)
    B, C, H, W, m, n = 3, 6, 5, 4, 4, 7
    x = rng.standard_normal((B, H, W, C)) + rng.standard_normal((B, 1, 1, C))
    Wr, br = rng.standard_normal((m * n, C)), rng.standard_normal(m * n) * 0.3
    a = oracle.route_cells(x, Wr, br, m, mode, tau)
    for j in range(m):
        ref = oracle.route(x, Wr[j * n:(j + 1) * n], br[j * n:(j + 1) * n], mode, tau)
        np.testing.assert_allclose(a[:, j, :], ref, rtol=1e-14, atol=1e-15)
    if mode == oracle.SOFTMAX:
        np.testing.assert_allclose(a.sum(axis=2), 1.0, rtol=0, atol=1e-13)
    # m = 1 is the ordinary routing over all rows
    np.testing.assert_allclose(oracle.route_cells(x, Wr, br, 1, mode, tau)[:, 0, :],
                               oracle.route(x, Wr, br, mode, tau), rtol=1e-14, atol=1e-15)


@pytest.mark.parametrize("shape", SHAPES)
def test_one_hot_attentions_pick_whole_cells(shape):
    B, Cin, Cout, H, W, K, s, p, g, m, n = shape
    c = _case(shape, 3)
    pick = c["rng"].integers(0, n, (B, m))
    alpha = np.zeros((B, m, n))
    for b in range(B):
        for j in range(m):
            alpha[b, j, pick[b, j]] = 1.0
    got = oracle.forward_cells(c["x"], c["E"], alpha, c["bias"], Cout, K, K, s, p, g)
    for b in range(B):
        Wb = np.concatenate([c["E"][pick[b, j]] for j in range(m)]).reshape(Cout, K, K, Cin // g)
        ref = _torch_conv(c["x"][b:b + 1], Wb, c["bias"], s, p, g)[0]
        np.testing.assert_allclose(got[b], ref, rtol=1e-12, atol=1e-12)


def test_a_cell_changes_only_its_output_channels():
    shape = SHAPES[0]          # 6 output channels, 3 cells of 2 channels each
    B, Cin, Cout, H, W, K, s, p, g, m, n = shape
    c = _case(shape, 4)
    a2 = c["alpha"].copy()
    a2[:, 1, :] = c["rng"].uniform(0, 1, (B, n))
    y1 = oracle.forward_cells(c["x"], c["E"], c["alpha"], c["bias"], Cout, K, K, s, p, g)
    y2 = oracle.forward_cells(c["x"], c["E"], a2, c["bias"], Cout, K, K, s, p, g)
    per = Cout // m
    changed = np.abs(y1 - y2).max(axis=(0, 1, 2)) > 1e-12
    assert list(changed) == [j // per == 1 for j in range(Cout)]


def test_assemble_cells_layout():
    """W_b holds the cells in order, each the attention-weighted warehouse."""
    rng = np.random.default_rng(5)
    E, a = rng.standard_normal((3, 4)), rng.standard_normal((2, 3))
    Wb = oracle.assemble_cells(E, a)
    for j in range(2):
        for e in range(4):
            assert abs(Wb[j * 4 + e] - sum(a[j, i] * E[i, e] for i in range(3))) < 1e-14
