"""fp64 CPU oracle for the per-sample kernel-mixture convolution.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module; the product library never does.

The arithmetic lives in ``dynconv_oracle.c`` (plain C, fp64, direct loops,
threads over samples only). This module compiles it with gcc and marshals
numpy arrays in and out; it adds no arithmetic of its own.

Every forward function here is pinned by ``tests/test_oracle_pins.py`` against
closed forms, a library convolution (n=1), brute force on tiny inputs and the
identities that the pages' definition implies; the backward functions by
``tests/test_oracle_backward.py`` against central differences of the pinned
forward and against torch autograd of the same definition; the warehouse
cells by ``tests/test_oracle_cells.py`` against the pinned ordinary mixture
(one cell), the pinned routing (per cell), torch conv2d (one-hot cells) and
per-cell locality.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dynconv_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

SIGMOID = 0
SOFTMAX = 1

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no GPU, no CUDA) and return the .so path."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
             "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"],
            check=True)
        os.replace(tmp, _LIB)
    return _LIB


def configure(lib):
    """Declare the C signatures on a loaded oracle library and return it."""
    dp = ctypes.POINTER(ctypes.c_double)
    i = ctypes.c_int
    lib.oracle_route.argtypes = [i, i, i, i, dp, i, dp, dp, i, ctypes.c_double, dp, i]
    lib.oracle_route.restype = i
    lib.oracle_forward.argtypes = [i] * 11 + [dp, dp, dp, dp, i, i, dp, i]
    lib.oracle_forward.restype = i
    lib.oracle_forward_attn.argtypes = [i] * 11 + [dp, dp, dp, dp, dp, dp, i, i, dp, i]
    lib.oracle_forward_attn.restype = i
    lib.oracle_forward_rows.argtypes = [i] * 11 + [dp, dp, dp, dp, i, i, i, dp]
    lib.oracle_forward_rows.restype = i
    lib.oracle_assemble.argtypes = [i, ctypes.c_long, dp, dp, dp]
    lib.oracle_assemble.restype = None
    lib.oracle_threads_used.argtypes = [i, i]
    lib.oracle_threads_used.restype = i
    lib.oracle_weight_grad.argtypes = [i] * 10 + [dp, dp, i, i, dp, dp, i]
    lib.oracle_weight_grad.restype = i
    lib.oracle_backward_weight.argtypes = [i] * 11 + [dp, dp, dp, dp, dp, dp, dp, dp, i]
    lib.oracle_backward_weight.restype = i
    lib.oracle_route_backward.argtypes = [i, i, i, i, dp, i, dp, dp, dp, i, ctypes.c_double,
                                          dp, dp, dp]
    lib.oracle_route_backward.restype = i
    lib.oracle_backward_data.argtypes = [i] * 11 + [dp, dp, dp, dp, i, i, dp, i]
    lib.oracle_backward_data.restype = i
    lib.oracle_dalpha.argtypes = [i] * 11 + [dp, dp, dp, dp, i, i, dp, i]
    lib.oracle_dalpha.restype = i
    lib.oracle_dexperts_at.argtypes = [i] * 11 + [dp, dp, dp, i, ctypes.POINTER(ctypes.c_long), dp]
    lib.oracle_dexperts_at.restype = i
    lib.oracle_dbias.argtypes = [i, i, i, i, dp, dp, dp]
    lib.oracle_dbias.restype = i
    lib.oracle_assemble_cells.argtypes = [i, i, ctypes.c_long, dp, dp, dp]
    lib.oracle_assemble_cells.restype = None
    lib.oracle_route_cells.argtypes = [i, i, i, i, dp, i, i, dp, dp, i, ctypes.c_double, dp]
    lib.oracle_route_cells.restype = i
    lib.oracle_forward_cells.argtypes = [i] * 12 + [dp, dp, dp, dp, i, i, dp]
    lib.oracle_forward_cells.restype = i
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = configure(ctypes.CDLL(build()))
    return _lib


def _dp(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def threads_used(nthreads: int, nb: int) -> int:
    return _load().oracle_threads_used(int(nthreads), int(nb))


def route(x, Wr, br, mode: int, tau: float = 1.0, nthreads: int = 0):
    """alpha[B][n] = act(FC(GAP(x_b))) for NHWC x[B][H][W][C]; Wr[n][C], br[n] (or None)."""
    x = _f64(x)
    Wr = _f64(Wr)
    br = _f64(br)
    B, H, W, C = x.shape
    n = Wr.shape[0]
    assert Wr.shape == (n, C)
    assert br is None or br.shape == (n,)
    alpha = np.empty((B, n), dtype=np.float64)
    rc = _load().oracle_route(B, C, H, W, _dp(x), n, _dp(Wr), _dp(br), int(mode), float(tau),
                              _dp(alpha), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_route rejected its arguments (rc={rc})")
    return alpha


def forward(x, experts, alpha, bias=None, stride: int = 1, pad: int = 0, groups: int = 1,
            samples: tuple[int, int] | None = None, nthreads: int = 0):
    """y = conv2d(x_b, sum_i alpha_bi W_i) + sum_i alpha_bi bias_i, NHWC, fp64.

    x[B][H][W][C_in], experts[n][C_out][KH][KW][C_in/groups], alpha[B][n],
    bias[n][C_out] or None.  ``samples=(b0, nb)`` computes only samples
    b0..b0+nb-1 and returns y[nb][H_out][W_out][C_out].
    """
    x = _f64(x)
    experts = _f64(experts)
    alpha = _f64(alpha)
    bias = _f64(bias)
    B, H, W, Cin = x.shape
    n, Cout, KH, KW, Cg = experts.shape
    assert Cg * groups == Cin, "experts' last dim must be C_in/groups"
    assert alpha.shape == (B, n)
    assert bias is None or bias.shape == (n, Cout)
    b0, nb = (0, B) if samples is None else samples
    Ho = (H + 2 * pad - KH) // stride + 1
    Wo = (W + 2 * pad - KW) // stride + 1
    y = np.empty((nb, Ho, Wo, Cout), dtype=np.float64)
    rc = _load().oracle_forward(B, Cin, H, W, Cout, KH, KW, stride, pad, groups, n,
                                _dp(x), _dp(experts), _dp(alpha), _dp(bias), b0, nb, _dp(y),
                                int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_forward rejected its arguments (rc={rc})")
    return y


def forward_attn(x, experts, alpha, bias, a_in, a_out, stride: int = 1, pad: int = 0,
                 groups: int = 1, samples: tuple[int, int] | None = None, nthreads: int = 0):
    """``forward`` with the FMDConv channel attentions: a_in[B][C_in] multiplies
    every input channel of a sample, a_out[B][C_out] every output channel (bias
    included); either may be None (all ones)."""
    x = _f64(x)
    experts = _f64(experts)
    alpha = _f64(alpha)
    bias = _f64(bias)
    a_in = _f64(a_in)
    a_out = _f64(a_out)
    B, H, W, Cin = x.shape
    n, Cout, KH, KW, Cg = experts.shape
    assert Cg * groups == Cin, "experts' last dim must be C_in/groups"
    assert alpha.shape == (B, n)
    assert bias is None or bias.shape == (n, Cout)
    assert a_in is None or a_in.shape == (B, Cin)
    assert a_out is None or a_out.shape == (B, Cout)
    b0, nb = (0, B) if samples is None else samples
    Ho = (H + 2 * pad - KH) // stride + 1
    Wo = (W + 2 * pad - KW) // stride + 1
    y = np.empty((nb, Ho, Wo, Cout), dtype=np.float64)
    rc = _load().oracle_forward_attn(B, Cin, H, W, Cout, KH, KW, stride, pad, groups, n,
                                     _dp(x), _dp(experts), _dp(alpha), _dp(bias), _dp(a_in),
                                     _dp(a_out), b0, nb, _dp(y), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_forward_attn rejected its arguments (rc={rc})")
    return y


def forward_rows(x, experts, alpha, bias, b: int, oh0: int, noh: int, stride: int = 1,
                 pad: int = 0, groups: int = 1):
    """Output rows oh0..oh0+noh-1 of sample b only: y[noh][W_out][C_out] (one thread)."""
    x = _f64(x)
    experts = _f64(experts)
    alpha = _f64(alpha)
    bias = _f64(bias)
    B, H, W, Cin = x.shape
    n, Cout, KH, KW, Cg = experts.shape
    assert Cg * groups == Cin
    Wo = (W + 2 * pad - KW) // stride + 1
    y = np.empty((noh, Wo, Cout), dtype=np.float64)
    rc = _load().oracle_forward_rows(B, Cin, H, W, Cout, KH, KW, stride, pad, groups, n, _dp(x),
                                     _dp(experts), _dp(alpha), _dp(bias), int(b), int(oh0),
                                     int(noh), _dp(y))
    if rc != 0:
        raise ValueError(f"oracle_forward_rows rejected its arguments (rc={rc})")
    return y


def assemble(experts, alpha_b):
    """W_b = sum_i alpha_b[i] * experts[i] (any expert shape), fp64."""
    experts = _f64(experts)
    alpha_b = _f64(alpha_b)
    n = experts.shape[0]
    assert alpha_b.shape == (n,)
    wsize = int(np.prod(experts.shape[1:]))
    out = np.empty(experts.shape[1:], dtype=np.float64)
    _load().oracle_assemble(n, wsize, _dp(experts), _dp(alpha_b), _dp(out))
    return out


# ------------------------------------------------------------------ backward


def weight_grad(x, dy, KH: int, KW: int, stride: int = 1, pad: int = 0, groups: int = 1,
                samples: tuple[int, int] | None = None, nthreads: int = 0):
    """Per-sample gradients of the convolution's weight and bias:
    dW[nb][C_out][KH][KW][C_in/groups] and db[nb][C_out] for samples b0..b0+nb-1."""
    x = _f64(x)
    dy = _f64(dy)
    B, H, W, Cin = x.shape
    Cout = dy.shape[3]
    assert dy.shape[:3] == (B, (H + 2 * pad - KH) // stride + 1, (W + 2 * pad - KW) // stride + 1)
    b0, nb = (0, B) if samples is None else samples
    dW = np.empty((nb, Cout, KH, KW, Cin // groups), dtype=np.float64)
    db = np.empty((nb, Cout), dtype=np.float64)
    rc = _load().oracle_weight_grad(B, Cin, H, W, Cout, KH, KW, stride, pad, groups, _dp(x),
                                    _dp(dy), b0, nb, _dp(dW), _dp(db), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_weight_grad rejected its arguments (rc={rc})")
    return dW, db


def backward_weight(x, dy, experts, alpha, bias=None, stride: int = 1, pad: int = 0,
                    groups: int = 1, nthreads: int = 0):
    """(dexperts[n][C_out][KH][KW][C_in/groups], dbias[n][C_out] or None, dalpha[B][n])."""
    x = _f64(x)
    dy = _f64(dy)
    experts = _f64(experts)
    alpha = _f64(alpha)
    bias = _f64(bias)
    B, H, W, Cin = x.shape
    n, Cout, KH, KW, Cg = experts.shape
    assert Cg * groups == Cin and alpha.shape == (B, n)
    assert bias is None or bias.shape == (n, Cout)
    assert dy.shape == (B, (H + 2 * pad - KH) // stride + 1, (W + 2 * pad - KW) // stride + 1, Cout)
    dexperts = np.empty(experts.shape, dtype=np.float64)
    dbias = None if bias is None else np.empty((n, Cout), dtype=np.float64)
    dalpha = np.empty((B, n), dtype=np.float64)
    rc = _load().oracle_backward_weight(B, Cin, H, W, Cout, KH, KW, stride, pad, groups, n,
                                        _dp(x), _dp(dy), _dp(experts), _dp(alpha), _dp(bias),
                                        _dp(dexperts), _dp(dbias), _dp(dalpha), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_backward_weight rejected its arguments (rc={rc})")
    return dexperts, dbias, dalpha


def route_backward(x, Wr, alpha, dalpha, mode: int, tau: float = 1.0):
    """(dWr[n][C], dbr[n], dg[B][C]) from dalpha[B][n] through the activation and
    the linear layer; dg is the gradient of each sample's pooled vector."""
    x = _f64(x)
    Wr = _f64(Wr)
    alpha = _f64(alpha)
    dalpha = _f64(dalpha)
    B, H, W, C = x.shape
    n = Wr.shape[0]
    assert Wr.shape == (n, C) and alpha.shape == (B, n) and dalpha.shape == (B, n)
    dWr = np.empty((n, C), dtype=np.float64)
    dbr = np.empty(n, dtype=np.float64)
    dg = np.empty((B, C), dtype=np.float64)
    rc = _load().oracle_route_backward(B, C, H, W, _dp(x), n, _dp(Wr), _dp(alpha), _dp(dalpha),
                                       int(mode), float(tau), _dp(dWr), _dp(dbr), _dp(dg))
    if rc != 0:
        raise ValueError(f"oracle_route_backward rejected its arguments (rc={rc})")
    return dWr, dbr, dg


def backward_data(dy, experts, alpha, dg, H: int, W: int, stride: int = 1, pad: int = 0,
                  groups: int = 1, samples: tuple[int, int] | None = None, nthreads: int = 0):
    """dx[nb][H][W][C_in] for samples b0..b0+nb-1: the input gradient through the
    convolution with W_b, plus dg[b][c]/(H*W) when dg is given (else None)."""
    dy = _f64(dy)
    experts = _f64(experts)
    alpha = _f64(alpha)
    dg = _f64(dg)
    B = dy.shape[0]
    n, Cout, KH, KW, Cg = experts.shape
    Cin = Cg * groups
    assert dy.shape == (B, (H + 2 * pad - KH) // stride + 1, (W + 2 * pad - KW) // stride + 1, Cout)
    assert alpha.shape == (B, n) and (dg is None or dg.shape == (B, Cin))
    b0, nb = (0, B) if samples is None else samples
    dx = np.empty((nb, H, W, Cin), dtype=np.float64)
    rc = _load().oracle_backward_data(B, Cin, H, W, Cout, KH, KW, stride, pad, groups, n,
                                      _dp(dy), _dp(experts), _dp(alpha), _dp(dg), b0, nb,
                                      _dp(dx), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_backward_data rejected its arguments (rc={rc})")
    return dx


def backward(x, dy, experts, alpha, bias, Wr, mode: int, tau: float = 1.0, stride: int = 1,
             pad: int = 0, groups: int = 1, nthreads: int = 0):
    """Every gradient of one layer with its router, given dy: a dict with dx,
    dexperts, dbias, dalpha, dWr, dbr, dg (the three steps above in order)."""
    x = _f64(x)
    H, W = x.shape[1], x.shape[2]
    dexperts, dbias, dalpha = backward_weight(x, dy, experts, alpha, bias, stride, pad, groups,
                                              nthreads)
    dWr, dbr, dg = route_backward(x, Wr, alpha, dalpha, mode, tau)
    dx = backward_data(dy, experts, alpha, dg, H, W, stride, pad, groups, nthreads=nthreads)
    return dict(dx=dx, dexperts=dexperts, dbias=dbias, dalpha=dalpha, dWr=dWr, dbr=dbr, dg=dg)


def dalpha(x, dy, experts, bias, stride: int = 1, pad: int = 0, groups: int = 1,
           samples: tuple[int, int] | None = None, nthreads: int = 0):
    """dalpha[nb][n] of samples b0..b0+nb-1 (as backward_weight, restricted)."""
    x = _f64(x)
    dy = _f64(dy)
    experts = _f64(experts)
    bias = _f64(bias)
    B, H, W, Cin = x.shape
    n, Cout, KH, KW, Cg = experts.shape
    b0, nb = (0, B) if samples is None else samples
    out = np.empty((nb, n), dtype=np.float64)
    rc = _load().oracle_dalpha(B, Cin, H, W, Cout, KH, KW, stride, pad, groups, n, _dp(x),
                               _dp(dy), _dp(experts), _dp(bias), b0, nb, _dp(out), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_dalpha rejected its arguments (rc={rc})")
    return out


def dexperts_at(x, dy, alpha, idx, n: int, Cout: int, KH: int, KW: int, stride: int = 1,
                pad: int = 0, groups: int = 1):
    """dexperts[i][idx[k]] -> out[n][len(idx)] for flat indices into
    [C_out][KH][KW][C_in/groups] (as backward_weight, restricted)."""
    x = _f64(x)
    dy = _f64(dy)
    alpha = _f64(alpha)
    B, H, W, Cin = x.shape
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int64))
    out = np.empty((n, len(idx)), dtype=np.float64)
    rc = _load().oracle_dexperts_at(B, Cin, H, W, Cout, KH, KW, stride, pad, groups, n, _dp(x),
                                    _dp(dy), _dp(alpha), len(idx),
                                    idx.ctypes.data_as(ctypes.POINTER(ctypes.c_long)), _dp(out))
    if rc != 0:
        raise ValueError(f"oracle_dexperts_at rejected its arguments (rc={rc})")
    return out


def dbias(dy, alpha):
    """dbias[n][C_out] = sum_b alpha[b][i] * (dy[b] summed over pixels)."""
    dy = _f64(dy)
    alpha = _f64(alpha)
    B, Ho, Wo, Cout = dy.shape
    n = alpha.shape[1]
    out = np.empty((n, Cout), dtype=np.float64)
    rc = _load().oracle_dbias(B, Ho * Wo, Cout, n, _dp(dy), _dp(alpha), _dp(out))
    if rc != 0:
        raise ValueError(f"oracle_dbias rejected its arguments (rc={rc})")
    return out


# ------------------------------------------------------------- kernel cells


def route_cells(x, Wr, br, m: int, mode: int, tau: float = 1.0):
    """alpha[B][m][n]: the router with m*n outputs (Wr[m*n][C], br[m*n] or None),
    its activation taken per cell of n values."""
    x = _f64(x)
    Wr = _f64(Wr)
    br = _f64(br)
    B, H, W, C = x.shape
    assert Wr.shape[0] % m == 0 and Wr.shape[1] == C
    n = Wr.shape[0] // m
    alpha = np.empty((B, m, n), dtype=np.float64)
    rc = _load().oracle_route_cells(B, C, H, W, _dp(x), m, n, _dp(Wr), _dp(br), int(mode),
                                    float(tau), _dp(alpha))
    if rc != 0:
        raise ValueError(f"oracle_route_cells rejected its arguments (rc={rc})")
    return alpha


def assemble_cells(warehouse, alpha_b):
    """W_b (flat, m*s elements) from warehouse[n][s] and alpha_b[m][n]."""
    warehouse = _f64(warehouse)
    alpha_b = _f64(alpha_b)
    n, s = warehouse.shape
    m = alpha_b.shape[0]
    assert alpha_b.shape == (m, n)
    out = np.empty(m * s, dtype=np.float64)
    _load().oracle_assemble_cells(m, n, s, _dp(warehouse), _dp(alpha_b), _dp(out))
    return out


def forward_cells(x, warehouse, alpha, bias, Cout: int, KH: int, KW: int, stride: int = 1,
                  pad: int = 0, groups: int = 1, samples: tuple[int, int] | None = None):
    """y with the kernel assembled from cells: warehouse[n][s], alpha[B][m][n],
    bias[C_out] static (or None); the layer's kernel has m*s elements."""
    x = _f64(x)
    warehouse = _f64(warehouse)
    alpha = _f64(alpha)
    bias = _f64(bias)
    B, H, W, Cin = x.shape
    n, s = warehouse.shape
    m = alpha.shape[1]
    assert alpha.shape == (B, m, n) and m * s == Cout * KH * KW * (Cin // groups)
    assert bias is None or bias.shape == (Cout,)
    b0, nb = (0, B) if samples is None else samples
    Ho = (H + 2 * pad - KH) // stride + 1
    Wo = (W + 2 * pad - KW) // stride + 1
    y = np.empty((nb, Ho, Wo, Cout), dtype=np.float64)
    rc = _load().oracle_forward_cells(B, Cin, H, W, Cout, KH, KW, stride, pad, groups, m, n,
                                      _dp(x), _dp(warehouse), _dp(alpha), _dp(bias), b0, nb,
                                      _dp(y))
    if rc != 0:
        raise ValueError(f"oracle_forward_cells rejected its arguments (rc={rc})")
    return y
