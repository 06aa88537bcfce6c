"""Python binding of the sm_100a dynamic-convolution C ABI (``include/dynconv.h``,
``include/dynconv_backward.h``, ``include/dynconv_cells.h``).

Argument marshalling only: every function forwards to the symbol of the same
name in ``libdynconv.so``; all arithmetic runs in the library's CUDA kernels.
Tensors may be passed as torch CUDA tensors (their data pointers are taken) or
as raw integer device addresses. There is no CPU fallback: if the library is
missing or no sm_100 device is present, the calls raise.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdynconv.so")

# dynconv_dtype / dynconv_mode / dynconv_variant
F32, BF16 = 0, 1
SIGMOID, SOFTMAX = 0, 1
VARIANT_AUTO, VARIANT_FUSED, VARIANT_OUTSIDE, VARIANT_PREMIX, VARIANT_DIRECT, VARIANT_DEPTHWISE = range(6)
VARIANT_NAMES = {0: "auto", 1: "fused", 2: "outside", 3: "premix", 4: "direct", 5: "depthwise"}

# status codes
OK = 0
ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_MISALIGNED, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE = -1, -2, -3, -4, -5, -6

SYMBOLS = ("dynconv_route", "dynconv_forward", "dynconv_forward_noalloc",
           "dynconv_pool_parts", "dynconv_forward_pooled", "dynconv_route_pooled",
           "dynconv_route_channels", "dynconv_forward_attn",
           "dynconv_workspace_size", "dynconv_select_variant",
           "dynconv_status_string", "dynconv_last_error", "dynconv_device_status",
           "dynconv_launch_count", "dynconv_test_hook",
           # include/dynconv_backward.h
           "dynconv_backward_workspace_size", "dynconv_backward_weight",
           "dynconv_route_backward", "dynconv_backward_data",
           # include/dynconv_cells.h
           "dynconv_route_cells", "dynconv_cells_workspace_size", "dynconv_forward_cells")


class dynconv_desc(ctypes.Structure):
    _fields_ = [(f, ctypes.c_int) for f in
                ("B", "C_in", "H", "W", "C_out", "KH", "KW", "stride", "pad", "groups", "n",
                 "dtype", "variant")]


class DynconvError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {dynconv_status_string(status)} ({status}) {dynconv_last_error()}")


_lib = None


def load():
    """Load libdynconv.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m dynamic_convolution_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        P = ctypes.c_void_p
        D = ctypes.POINTER(dynconv_desc)
        lib.dynconv_route.argtypes = [D, P, P, P, ctypes.c_int, ctypes.c_float, P, P]
        lib.dynconv_route.restype = ctypes.c_int
        lib.dynconv_forward.argtypes = [D, P, P, P, P, P, P, ctypes.c_size_t, P]
        lib.dynconv_forward.restype = ctypes.c_int
        lib.dynconv_forward_noalloc.argtypes = [D, P, P, P, P, P, P]
        lib.dynconv_forward_noalloc.restype = ctypes.c_int
        lib.dynconv_route_channels.argtypes = [D, P, P, P, P, P, P, P, P]
        lib.dynconv_route_channels.restype = ctypes.c_int
        lib.dynconv_forward_attn.argtypes = [D, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        lib.dynconv_forward_attn.restype = ctypes.c_int
        lib.dynconv_pool_parts.argtypes = [D, ctypes.c_size_t]
        lib.dynconv_pool_parts.restype = ctypes.c_int
        lib.dynconv_forward_pooled.argtypes = [D, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        lib.dynconv_forward_pooled.restype = ctypes.c_int
        lib.dynconv_route_pooled.argtypes = [D, P, ctypes.c_int, P, P, ctypes.c_int,
                                             ctypes.c_float, P, P]
        lib.dynconv_route_pooled.restype = ctypes.c_int
        lib.dynconv_workspace_size.argtypes = [D]
        lib.dynconv_workspace_size.restype = ctypes.c_size_t
        lib.dynconv_select_variant.argtypes = [D, ctypes.c_size_t]
        lib.dynconv_select_variant.restype = ctypes.c_int
        lib.dynconv_status_string.argtypes = [ctypes.c_int]
        lib.dynconv_status_string.restype = ctypes.c_char_p
        lib.dynconv_last_error.argtypes = []
        lib.dynconv_last_error.restype = ctypes.c_char_p
        lib.dynconv_device_status.argtypes = [P]
        lib.dynconv_device_status.restype = ctypes.c_int
        lib.dynconv_launch_count.argtypes = []
        lib.dynconv_launch_count.restype = ctypes.c_ulonglong
        lib.dynconv_test_hook.argtypes = [ctypes.c_int, ctypes.c_longlong]
        lib.dynconv_test_hook.restype = ctypes.c_int
        lib.dynconv_backward_workspace_size.argtypes = [D]
        lib.dynconv_backward_workspace_size.restype = ctypes.c_size_t
        lib.dynconv_backward_weight.argtypes = [D, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        lib.dynconv_backward_weight.restype = ctypes.c_int
        lib.dynconv_route_backward.argtypes = [D, P, P, P, P, ctypes.c_int, ctypes.c_float, P, P,
                                               P, P, ctypes.c_size_t, P]
        lib.dynconv_route_backward.restype = ctypes.c_int
        lib.dynconv_backward_data.argtypes = [D, P, P, P, P, P, P, ctypes.c_size_t, P]
        lib.dynconv_backward_data.restype = ctypes.c_int
        lib.dynconv_route_cells.argtypes = [D, ctypes.c_int, P, P, P, ctypes.c_int, ctypes.c_float,
                                            P, P, ctypes.c_size_t, P]
        lib.dynconv_route_cells.restype = ctypes.c_int
        lib.dynconv_cells_workspace_size.argtypes = [D, ctypes.c_int]
        lib.dynconv_cells_workspace_size.restype = ctypes.c_size_t
        lib.dynconv_forward_cells.argtypes = [D, ctypes.c_int, P, P, P, P, P, P, ctypes.c_size_t, P]
        lib.dynconv_forward_cells.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s):
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def make_desc(B, C_in, H, W, C_out, KH, KW, stride=1, pad=0, groups=1, n=1, dtype=BF16,
              variant=VARIANT_AUTO) -> dynconv_desc:
    return dynconv_desc(B, C_in, H, W, C_out, KH, KW, stride, pad, groups, n, dtype, variant)


def desc_from_config(cfg, variant=VARIANT_AUTO, B=None) -> dynconv_desc:
    """Descriptor for a ``synth.LayerConfig``."""
    return make_desc(cfg.B if B is None else B, cfg.C_in, cfg.H, cfg.W, cfg.C_out, cfg.KH, cfg.KW,
                     cfg.stride, cfg.pad, cfg.groups, cfg.n, cfg.dtype, variant)


def dynconv_route(desc, x, Wr, br, mode, tau, alpha, stream=None) -> int:
    return load().dynconv_route(ctypes.byref(desc), _ptr(x), _ptr(Wr), _ptr(br), int(mode),
                                float(tau), _ptr(alpha), _stream(stream))


def dynconv_forward(desc, x, experts, alpha, bias, y, workspace=None, workspace_bytes=0,
                    stream=None) -> int:
    return load().dynconv_forward(ctypes.byref(desc), _ptr(x), _ptr(experts), _ptr(alpha),
                                  _ptr(bias), _ptr(y), _ptr(workspace), int(workspace_bytes),
                                  _stream(stream))


def dynconv_route_channels(desc, x, Wi, bi, a_in, Wo, bo, a_out, stream=None) -> int:
    """FMDConv channel attentions a_in [B][C_in], a_out [B][C_out] (sigmoid of a
    linear layer of the average pool; either pair may be None)."""
    return load().dynconv_route_channels(ctypes.byref(desc), _ptr(x), _ptr(Wi), _ptr(bi),
                                         _ptr(a_in), _ptr(Wo), _ptr(bo), _ptr(a_out),
                                         _stream(stream))


def dynconv_forward_attn(desc, x, experts, alpha, bias, a_in, a_out, y, workspace=None,
                         workspace_bytes=0, stream=None) -> int:
    """dynconv_forward with the input / output channel attentions (either None)."""
    return load().dynconv_forward_attn(ctypes.byref(desc), _ptr(x), _ptr(experts), _ptr(alpha),
                                       _ptr(bias), _ptr(a_in), _ptr(a_out), _ptr(y),
                                       _ptr(workspace), int(workspace_bytes), _stream(stream))


def dynconv_pool_parts(desc, workspace_bytes=0) -> int:
    return int(load().dynconv_pool_parts(ctypes.byref(desc), int(workspace_bytes)))


def dynconv_forward_pooled(desc, x, experts, alpha, bias, y, ysum, workspace=None,
                           workspace_bytes=0, stream=None) -> int:
    """dynconv_forward that also writes partial channel sums of y (the next
    layer's routing pool), ysum fp32 [B][P][C_out] with P = dynconv_pool_parts."""
    return load().dynconv_forward_pooled(ctypes.byref(desc), _ptr(x), _ptr(experts), _ptr(alpha),
                                         _ptr(bias), _ptr(y), _ptr(ysum), _ptr(workspace),
                                         int(workspace_bytes), _stream(stream))


def dynconv_route_pooled(desc, ysum, parts, Wr, br, mode, tau, alpha, stream=None) -> int:
    """Routing of the layer `desc` from the previous layer's pooled partial sums."""
    return load().dynconv_route_pooled(ctypes.byref(desc), _ptr(ysum), int(parts), _ptr(Wr),
                                       _ptr(br), int(mode), float(tau), _ptr(alpha),
                                       _stream(stream))


# Bytes of the library's built-in scratch array (DYNCONV_NOALLOC_MAX_BYTES).
NOALLOC_MAX_BYTES = 32 * 1024 * 1024


def dynconv_forward_noalloc(desc, x, experts, alpha, bias, y, stream=None) -> int:
    """dynconv_forward (PREMIX variant) with the library's built-in scratch array
    instead of a caller workspace; for callers that cannot allocate device memory."""
    return load().dynconv_forward_noalloc(ctypes.byref(desc), _ptr(x), _ptr(experts), _ptr(alpha),
                                          _ptr(bias), _ptr(y), _stream(stream))


def dynconv_workspace_size(desc) -> int:
    return int(load().dynconv_workspace_size(ctypes.byref(desc)))


def dynconv_select_variant(desc, workspace_bytes=0) -> int:
    return int(load().dynconv_select_variant(ctypes.byref(desc), int(workspace_bytes)))


def dynconv_status_string(status: int) -> str:
    return load().dynconv_status_string(int(status)).decode()


def dynconv_last_error() -> str:
    return load().dynconv_last_error().decode()


def dynconv_device_status(stream=None) -> int:
    return int(load().dynconv_device_status(_stream(stream)))


def dynconv_launch_count() -> int:
    return int(load().dynconv_launch_count())


def dynconv_test_hook(key: int, value: int) -> int:
    return int(load().dynconv_test_hook(int(key), int(value)))


def check(status: int, where: str = "dynconv") -> None:
    if status != OK:
        raise DynconvError(status, where)


# ------------------------------------------------------------------ backward


def dynconv_backward_workspace_size(desc) -> int:
    return load().dynconv_backward_workspace_size(ctypes.byref(desc))


def dynconv_backward_weight(desc, x, dy, experts, alpha, bias, dexperts, dbias, dalpha,
                            workspace, workspace_bytes, stream=None) -> int:
    """dexperts [n][C_out][KH][KW][C_in/groups], dbias [n][C_out] (None with no
    bias), dalpha [B][n], all fp32, from the forward's x, alpha and dy."""
    return load().dynconv_backward_weight(ctypes.byref(desc), _ptr(x), _ptr(dy), _ptr(experts),
                                          _ptr(alpha), _ptr(bias), _ptr(dexperts), _ptr(dbias),
                                          _ptr(dalpha), _ptr(workspace), int(workspace_bytes),
                                          _stream(stream))


def dynconv_route_backward(desc, x, Wr, alpha, dalpha, mode, tau, dWr, dbr, dg,
                           workspace=None, workspace_bytes=0, stream=None) -> int:
    """dWr [n][C_in], dbr [n] (may be None), dg [B][C_in] (fp32)."""
    return load().dynconv_route_backward(ctypes.byref(desc), _ptr(x), _ptr(Wr), _ptr(alpha),
                                         _ptr(dalpha), int(mode), float(tau), _ptr(dWr),
                                         _ptr(dbr), _ptr(dg), _ptr(workspace),
                                         int(workspace_bytes), _stream(stream))


def dynconv_backward_data(desc, dy, experts, alpha, dg, dx, workspace, workspace_bytes,
                          stream=None) -> int:
    """dx [B][H][W][C_in] in the layer's dtype; dg [B][C_in] or None."""
    return load().dynconv_backward_data(ctypes.byref(desc), _ptr(dy), _ptr(experts), _ptr(alpha),
                                        _ptr(dg), _ptr(dx), _ptr(workspace),
                                        int(workspace_bytes), _stream(stream))


# ------------------------------------------------------------- kernel cells


def dynconv_route_cells(desc, cells, x, Wr, br, mode, tau, alpha, workspace, workspace_bytes,
                        stream=None) -> int:
    """alpha [B][cells][n] (fp32) from Wr [cells*n][C_in], br [cells*n] (or None)."""
    return load().dynconv_route_cells(ctypes.byref(desc), int(cells), _ptr(x), _ptr(Wr), _ptr(br),
                                      int(mode), float(tau), _ptr(alpha), _ptr(workspace),
                                      int(workspace_bytes), _stream(stream))


def dynconv_cells_workspace_size(desc, cells) -> int:
    return load().dynconv_cells_workspace_size(ctypes.byref(desc), int(cells))


def dynconv_forward_cells(desc, cells, x, warehouse, alpha, bias, y, workspace, workspace_bytes,
                          stream=None) -> int:
    """y with the kernel assembled from `cells` cells of the warehouse [n][s];
    bias [C_out] static (or None)."""
    return load().dynconv_forward_cells(ctypes.byref(desc), int(cells), _ptr(x), _ptr(warehouse),
                                        _ptr(alpha), _ptr(bias), _ptr(y), _ptr(workspace),
                                        int(workspace_bytes), _stream(stream))
