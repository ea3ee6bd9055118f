"""INT8 ConvRot linear layer on NVIDIA B200 (sm_100a).

Thin ctypes binding over ``libconvrot.so`` (C ABI in ``include/convrot.h``).
Every function here only marshals torch tensors into device pointers and
sizes and calls the C entry point of the same name; all arithmetic runs in
the library's CUDA kernels.  There is no CPU fallback: if the library is
missing or the device is not a B200, calls raise.

Typical use::

    w = quantize_weight(w_bf16)                 # offline, QuantizedWeight
    ws = make_workspace(m, w)                   # zero-filled scratch
    y = linear_int8(x_bf16, w, ws)              # BF16 [m, n]
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libconvrot.so")
GROUP = 256

_STATUS = {
    0: "CONVROT_OK", 1: "CONVROT_ERR_INVALID_ARG", 2: "CONVROT_ERR_ALIGNMENT",
    3: "CONVROT_ERR_UNSUPPORTED_SHAPE", 4: "CONVROT_ERR_UNSUPPORTED_ARCH",
    5: "CONVROT_ERR_WORKSPACE", 6: "CONVROT_ERR_CUDA", 7: "CONVROT_ERR_DEVICE_TIMEOUT",
    8: "CONVROT_WARN_INEXACT_DOMAIN",
}


class ConvrotError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s failed: %s" % (where, _STATUS.get(status, "status %d" % status)))


class convrot_weight_t(ctypes.Structure):
    """Mirror of the C struct: a view of (q int8 [n,k], scale fp32 [n])."""
    _fields_ = [("q", ctypes.c_void_p), ("scale", ctypes.c_void_p),
                ("n", ctypes.c_int64), ("k", ctypes.c_int64), ("group", ctypes.c_int32)]


class convrot_linear_job_t(ctypes.Structure):
    """Mirror of the C struct: one linear of a batched call."""
    _fields_ = [("x_bf16", ctypes.c_void_p), ("w", ctypes.POINTER(convrot_weight_t)),
                ("y_bf16", ctypes.c_void_p), ("bias_bf16", ctypes.c_void_p)]


class convrot_weight4_t(ctypes.Structure):
    """Mirror of the C struct: packed INT4 weight (q uint8 [n, k/2], scale fp32 [n])."""
    _fields_ = [("q", ctypes.c_void_p), ("scale", ctypes.c_void_p),
                ("n", ctypes.c_int64), ("k", ctypes.c_int64), ("group", ctypes.c_int32)]


class convrot_linear4_job_t(ctypes.Structure):
    """Mirror of the C struct: one W4A8 linear of a call."""
    _fields_ = [("x_bf16", ctypes.c_void_p), ("w", ctypes.POINTER(convrot_weight4_t)),
                ("y_bf16", ctypes.c_void_p), ("bias_bf16", ctypes.c_void_p)]


class convrot_conv2d_t(ctypes.Structure):
    """Mirror of the C struct: convolution geometry (NHWC input)."""
    _fields_ = [(f, ctypes.c_int32) for f in ("n", "h", "w", "c", "kh", "kw", "stride", "pad", "dilation")]


class convrot_conv2d_plan_t(ctypes.Structure):
    """Mirror of the C struct: how the im2col gather of a convolution runs."""
    _fields_ = [("tiled", ctypes.c_int32), ("th", ctypes.c_int32), ("tw", ctypes.c_int32), ("rh", ctypes.c_int32),
                ("rw", ctypes.c_int32), ("tiles", ctypes.c_int64), ("buf_bytes", ctypes.c_int64)]


class convrot_gemm_plan_t(ctypes.Structure):
    """Mirror of the C struct: how the GEMM kernel tiles a product."""
    _fields_ = [(f, ctypes.c_int32) for f in ("njobs", "swap", "bn", "grid", "full_waves", "full_tiles",
                                               "split_ways", "split_pieces", "rep", "stages", "tmem_cols",
                                               "slots")] + \
               [(f, ctypes.c_int64) for f in ("tail_units", "smem_bytes", "ws_bytes")] + \
               [(f, ctypes.c_int32 * 8) for f in ("tiles_a", "tiles_b", "group_a", "kbpt", "tile_base")] + \
               [("unit0", ctypes.c_int64 * 8)]


class convrot_gemm_job_t(ctypes.Structure):
    """Mirror of the C struct: one product of a batched GEMM call."""
    _fields_ = [("xq", ctypes.c_void_p), ("sx", ctypes.c_void_p), ("w", ctypes.POINTER(convrot_weight_t)),
                ("y_bf16", ctypes.c_void_p), ("acc", ctypes.c_void_p), ("bias_bf16", ctypes.c_void_p)]


# exported symbol -> (argtypes, restype); every name declared in convrot.h
_P, _I64, _I32, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
_WP = ctypes.POINTER(convrot_weight_t)
SIGNATURES = {
    "convrot_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "convrot_version": ([], ctypes.c_int),
    "convrot_build_id": ([], ctypes.c_char_p),
    "convrot_dynamic_group": ([_I64, _I32], _I32),
    "convrot_quantize_tensor": ([_P, _I64, _P, _P, _P], ctypes.c_int),
    "convrot_conv2d_shape": ([_P, _P, _P], ctypes.c_int),
    "convrot_conv2d_gather_plan": ([_P, _I32, _P], ctypes.c_int),
    "convrot_gemm_plan": ([_I64, _I32, _P, _P, _I32, _I32, _P], ctypes.c_int),
    "convrot_quantize_conv_weight": ([_P, _P, _WP, _P], ctypes.c_int),
    "convrot_conv2d_workspace_bytes": ([_P, _WP], _SZ),
    "convrot_conv2d_int8": ([_P, _P, _WP, _P, _P, _SZ, _P], ctypes.c_int),
    "convrot_weight4_init": ([ctypes.POINTER(convrot_weight4_t), _P, _P, _I64, _I64, _I32], ctypes.c_int),
    "convrot_quantize_weight4": ([_P, ctypes.POINTER(convrot_weight4_t), _P], ctypes.c_int),
    "convrot_linear_w4a8": ([_I64, ctypes.c_int, _P, _P, _SZ, _P], ctypes.c_int),
    "convrot_linear_w4a8_workspace_bytes": ([_I64, ctypes.c_int, _P], _SZ),
    "convrot_embed_lookup": ([_P, _I64, _P, _P, _I64, _I64, _P, _P], ctypes.c_int),
    "convrot_last_error_string": ([], ctypes.c_char_p),
    "convrot_weight_init": ([_WP, _P, _P, _I64, _I64, _I32], ctypes.c_int),
    "convrot_quantize_weight": ([_P, _WP, _P], ctypes.c_int),
    "convrot_quantize_act": ([_P, _I64, _I64, _I32, _P, _P, _P], ctypes.c_int),
    "convrot_gemm_workspace_bytes": ([_I64, _I64, _I64], _SZ),
    "convrot_linear_workspace_bytes": ([_I64, _I64, _I64], _SZ),
    "convrot_workspace_init": ([_P, _SZ, _P], ctypes.c_int),
    "convrot_gemm_i8": ([_P, _P, _I64, _WP, _P, _P, _P, _SZ, _P], ctypes.c_int),
    "convrot_linear_int8": ([_P, _I64, _WP, _P, _P, _SZ, _P], ctypes.c_int),
    "convrot_device_status": ([_P], ctypes.c_int),
    "convrot_linear_int8_batch": ([_I64, ctypes.c_int, ctypes.POINTER(convrot_linear_job_t), _P, _SZ, _P],
                                  ctypes.c_int),
    "convrot_linear_batch_workspace_bytes": ([_I64, ctypes.c_int, ctypes.POINTER(convrot_linear_job_t)], _SZ),
    "convrot_gemm_i8_batch": ([_I64, ctypes.c_int, ctypes.POINTER(convrot_gemm_job_t), _P, _SZ, _P], ctypes.c_int),
    "convrot_gemm_batch_workspace_bytes": ([_I64, ctypes.c_int, ctypes.POINTER(convrot_gemm_job_t)], _SZ),
    "convrot_gemm_i8_noalloc": ([_P, _P, _I64, _WP, _P, _P, _P], ctypes.c_int),
}

_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libconvrot.so.  The in-tree library is first rebuilt if it is
    missing or its build id differs from the hash of the sources beside it;
    after loading, its id must equal that hash (ImportError otherwise:
    there is no fallback path)."""
    global _lib
    if _lib is None:
        from . import build as _build
        expected = None
        if os.path.abspath(path) == os.path.abspath(LIB_PATH):
            _build.build()
            expected = _build.source_hash()
        if not os.path.exists(path):
            raise ImportError("libconvrot.so is not built (run rotated_int8_quantized_b200/build.py); "
                              "there is no fallback path")
        lib = ctypes.CDLL(path)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        if expected is not None and lib.convrot_build_id().decode() != expected:
            raise ImportError("libconvrot.so (build %s) was not built from the sources beside it (%s)"
                              % (lib.convrot_build_id().decode(), expected))
        _lib = lib
    return _lib


def build_id() -> str:
    """The loaded library's build id (hash of the sources it was built from)."""
    return load_library().convrot_build_id().decode()


def _check(status: int, where: str) -> None:
    if status != 0:
        err = ConvrotError(status, where)
        if status == 6:
            err.args = (err.args[0] + " (" + load_library().convrot_last_error_string().decode() + ")",)
        raise err


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t: Optional[torch.Tensor]) -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(0)
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("expected a contiguous CUDA tensor")
    return ctypes.c_void_p(t.data_ptr())


@dataclass
class QuantizedWeight:
    """Rotated INT8 weight q [n, k] with FP32 row scales [n] (caller-owned
    device memory) and the C handle viewing them."""
    q: torch.Tensor
    scale: torch.Tensor
    handle: convrot_weight_t

    @property
    def n(self) -> int:
        return self.handle.n

    @property
    def k(self) -> int:
        return self.handle.k

    @property
    def group(self) -> int:
        return self.handle.group


def convrot_status_string(status: int) -> str:
    return load_library().convrot_status_string(status).decode()


def convrot_version() -> int:
    return load_library().convrot_version()


def convrot_weight_init(q: torch.Tensor, scale: torch.Tensor, group: int = GROUP) -> QuantizedWeight:
    n, k = q.shape
    h = convrot_weight_t()
    _check(load_library().convrot_weight_init(ctypes.byref(h), _ptr(q), _ptr(scale), n, k, group),
           "convrot_weight_init")
    return QuantizedWeight(q, scale, h)


def convrot_quantize_weight(w_bf16: torch.Tensor, out: QuantizedWeight, stream=None) -> QuantizedWeight:
    assert w_bf16.dtype == torch.bfloat16 and tuple(w_bf16.shape) == (out.n, out.k)
    _check(load_library().convrot_quantize_weight(_ptr(w_bf16), ctypes.byref(out.handle), _stream(stream)),
           "convrot_quantize_weight")
    return out


def convrot_quantize_act(x_bf16: torch.Tensor, xq: torch.Tensor, sx: torch.Tensor,
                         group: int = GROUP, stream=None) -> None:
    assert x_bf16.dtype == torch.bfloat16 and xq.dtype == torch.int8 and sx.dtype == torch.float32
    m, k = x_bf16.shape
    _check(load_library().convrot_quantize_act(_ptr(x_bf16), m, k, group, _ptr(xq), _ptr(sx),
                                               _stream(stream)), "convrot_quantize_act")


def convrot_gemm_workspace_bytes(m: int, n: int, k: int) -> int:
    return int(load_library().convrot_gemm_workspace_bytes(m, n, k))


def convrot_linear_workspace_bytes(m: int, n: int, k: int) -> int:
    return int(load_library().convrot_linear_workspace_bytes(m, n, k))


def convrot_workspace_init(ws: torch.Tensor, stream=None) -> None:
    _check(load_library().convrot_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "convrot_workspace_init")


def convrot_gemm_i8(xq: torch.Tensor, sx: torch.Tensor, w: QuantizedWeight, y: Optional[torch.Tensor],
                    acc: Optional[torch.Tensor], ws: Optional[torch.Tensor], stream=None) -> None:
    m = xq.shape[0]
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(load_library().convrot_gemm_i8(_ptr(xq), _ptr(sx), m, ctypes.byref(w.handle), _ptr(y), _ptr(acc),
                                          _ptr(ws), ws_bytes, _stream(stream)), "convrot_gemm_i8")


def convrot_linear_int8(x_bf16: torch.Tensor, w: QuantizedWeight, y: torch.Tensor, ws: torch.Tensor,
                        stream=None) -> None:
    m = x_bf16.shape[0]
    _check(load_library().convrot_linear_int8(_ptr(x_bf16), m, ctypes.byref(w.handle), _ptr(y), _ptr(ws),
                                              ws.numel() * ws.element_size(), _stream(stream)),
           "convrot_linear_int8")


def _jobs(xs, ws_, ys, biases=None):
    arr = (convrot_linear_job_t * len(xs))()
    biases = biases or [None] * len(xs)
    for i, (x, w, y, b) in enumerate(zip(xs, ws_, ys, biases)):
        arr[i].x_bf16 = _ptr(x)
        arr[i].w = ctypes.pointer(w.handle)
        arr[i].y_bf16 = _ptr(y)
        arr[i].bias_bf16 = _ptr(b)
    return arr


class LinearBatch:
    """A prepared batched call: the C job array is built once and reused,
    so a step costs one C call (argument marshalling only).  ``biases``: an
    optional BF16 [n] tensor (or None) per linear.  Linears given the same
    input tensor share its rotation."""

    def __init__(self, xs, weights, ys, ws: Optional[torch.Tensor] = None, biases=None):
        self.xs, self.weights, self.ys = list(xs), list(weights), list(ys)
        self.biases = list(biases) if biases is not None else None
        self.m = self.xs[0].shape[0]
        self.jobs = _jobs(self.xs, self.weights, self.ys, self.biases)
        need = int(load_library().convrot_linear_batch_workspace_bytes(self.m, len(self.xs), self.jobs))
        if need == 0:
            raise ConvrotError(1, "convrot_linear_batch_workspace_bytes")
        if ws is None:
            ws = torch.zeros(need, dtype=torch.uint8, device=self.xs[0].device)
        self.ws = ws

    def __call__(self, stream=None) -> None:
        _check(load_library().convrot_linear_int8_batch(self.m, len(self.xs), self.jobs, _ptr(self.ws),
                                                        self.ws.numel(), _stream(stream)),
               "convrot_linear_int8_batch")


def convrot_linear_int8_batch(xs, weights, ys, ws: torch.Tensor, stream=None, biases=None) -> None:
    """Run len(xs) linears with the same token count together."""
    m = xs[0].shape[0]
    jobs = _jobs(xs, weights, ys, biases)
    _check(load_library().convrot_linear_int8_batch(m, len(xs), jobs, _ptr(ws), ws.numel() * ws.element_size(),
                                                    _stream(stream)), "convrot_linear_int8_batch")


def convrot_linear_batch_workspace_bytes(xs, weights, ys, biases=None) -> int:
    return int(load_library().convrot_linear_batch_workspace_bytes(xs[0].shape[0], len(xs),
                                                                   _jobs(xs, weights, ys, biases)))


class GemmBatch:
    """A prepared batched GEMM call (job array built once)."""

    def __init__(self, xqs, sxs, weights, ys, accs=None, ws: Optional[torch.Tensor] = None, biases=None):
        n = len(xqs)
        accs = accs or [None] * n
        biases = biases or [None] * n
        self.keep = (list(xqs), list(sxs), list(weights), list(ys), list(accs), list(biases))
        self.m = xqs[0].shape[0]
        self.jobs = (convrot_gemm_job_t * n)()
        for i in range(n):
            self.jobs[i].xq = _ptr(xqs[i])
            self.jobs[i].sx = _ptr(sxs[i])
            self.jobs[i].w = ctypes.pointer(weights[i].handle)
            self.jobs[i].y_bf16 = _ptr(ys[i])
            self.jobs[i].acc = _ptr(accs[i])
            self.jobs[i].bias_bf16 = _ptr(biases[i])
        need = int(load_library().convrot_gemm_batch_workspace_bytes(self.m, n, self.jobs))
        if need == 0:
            raise ConvrotError(1, "convrot_gemm_batch_workspace_bytes")
        self.ws = ws if ws is not None else torch.zeros(need, dtype=torch.uint8, device=xqs[0].device)

    def __call__(self, stream=None) -> None:
        _check(load_library().convrot_gemm_i8_batch(self.m, len(self.jobs), self.jobs, _ptr(self.ws),
                                                    self.ws.numel(), _stream(stream)), "convrot_gemm_i8_batch")


def convrot_quantize_tensor(w_bf16: torch.Tensor, q: torch.Tensor, scale: torch.Tensor, stream=None) -> None:
    """Tensor-wise simple INT8 (embedding table): q int8 like w, scale a
    one-element fp32 tensor."""
    assert w_bf16.dtype == torch.bfloat16 and q.dtype == torch.int8 and q.numel() == w_bf16.numel()
    assert scale.dtype == torch.float32 and scale.numel() == 1
    _check(load_library().convrot_quantize_tensor(_ptr(w_bf16), w_bf16.numel(), _ptr(q), _ptr(scale),
                                                  _stream(stream)), "convrot_quantize_tensor")


def convrot_embed_lookup(tokens: torch.Tensor, q: torch.Tensor, scale: torch.Tensor, out: torch.Tensor,
                         stream=None) -> None:
    """out[i] = bf16(q[tokens[i]] * scale) for int32 tokens [t], q [vocab, dim]."""
    assert tokens.dtype == torch.int32 and q.dim() == 2 and out.shape == (tokens.numel(), q.shape[1])
    _check(load_library().convrot_embed_lookup(_ptr(tokens), tokens.numel(), _ptr(q), _ptr(scale), q.shape[0],
                                               q.shape[1], _ptr(out), _stream(stream)), "convrot_embed_lookup")


# ---------------------------------------------------------------- INT4 weights (W4A8)
@dataclass
class QuantizedWeight4:
    """Packed INT4 weight q [n, k/2] (uint8) with FP32 row scales [n] and the C handle."""
    q: torch.Tensor
    scale: torch.Tensor
    handle: convrot_weight4_t

    @property
    def n(self) -> int:
        return self.handle.n

    @property
    def k(self) -> int:
        return self.handle.k

    @property
    def group(self) -> int:
        return self.handle.group


def quantize_weight4(w_bf16: torch.Tensor, stream=None, group: int = GROUP, dynamic: bool = False) -> QuantizedWeight4:
    """Offline INT4 ConvRot conversion of a BF16 weight [n, k]."""
    n, k = w_bf16.shape
    if dynamic:
        group = convrot_dynamic_group(k, group)
    q = torch.empty((n, k // 2), dtype=torch.uint8, device=w_bf16.device)
    scale = torch.empty((n,), dtype=torch.float32, device=w_bf16.device)
    h = convrot_weight4_t()
    lib = load_library()
    _check(lib.convrot_weight4_init(ctypes.byref(h), _ptr(q), _ptr(scale), n, k, group), "convrot_weight4_init")
    _check(lib.convrot_quantize_weight4(_ptr(w_bf16), ctypes.byref(h), _stream(stream)), "convrot_quantize_weight4")
    return QuantizedWeight4(q, scale, h)


class LinearBatchW4:
    """A prepared W4A8 call over up to 8 linears with the same token count."""

    def __init__(self, xs, weights, ys, ws: Optional[torch.Tensor] = None, biases=None):
        self.keep = (list(xs), list(weights), list(ys), list(biases) if biases else None)
        self.m = xs[0].shape[0]
        n = len(xs)
        biases = biases or [None] * n
        self.jobs = (convrot_linear4_job_t * n)()
        for i in range(n):
            self.jobs[i].x_bf16 = _ptr(xs[i])
            self.jobs[i].w = ctypes.pointer(weights[i].handle)
            self.jobs[i].y_bf16 = _ptr(ys[i])
            self.jobs[i].bias_bf16 = _ptr(biases[i])
        need = int(load_library().convrot_linear_w4a8_workspace_bytes(self.m, n, self.jobs))
        if need == 0:
            raise ConvrotError(3, "convrot_linear_w4a8_workspace_bytes")
        self.ws = ws if ws is not None else torch.zeros(need, dtype=torch.uint8, device=xs[0].device)

    def __call__(self, stream=None) -> None:
        _check(load_library().convrot_linear_w4a8(self.m, len(self.jobs), self.jobs, _ptr(self.ws),
                                                  self.ws.numel(), _stream(stream)), "convrot_linear_w4a8")


# ---------------------------------------------------------------- convolutions
def conv2d_geometry(x_shape, kh: int, kw: int, stride: int = 1, pad: int = 0, dilation: int = 1) -> convrot_conv2d_t:
    n, h, w, c = x_shape
    return convrot_conv2d_t(n, h, w, c, kh, kw, stride, pad, dilation)


def gemm_plan(m: int, ns, ks, w4: bool = False, sms: int = 148) -> convrot_gemm_plan_t:
    """How the GEMM kernel tiles one product (len(ns) == 1) or a batched
    launch of several (host only)."""
    count = len(ns)
    n_arr = (ctypes.c_int64 * count)(*ns)
    k_arr = (ctypes.c_int64 * count)(*ks)
    out = convrot_gemm_plan_t()
    _check(load_library().convrot_gemm_plan(m, count, n_arr, k_arr, 1 if w4 else 0, sms, ctypes.byref(out)),
           "convrot_gemm_plan")
    return out


def conv2d_gather_plan(x_shape, kh: int, kw: int, stride: int = 1, pad: int = 0, dilation: int = 1,
                       sms: int = 148) -> convrot_conv2d_plan_t:
    """The im2col gather's launch plan for a convolution (host only)."""
    g = conv2d_geometry(x_shape, kh, kw, stride, pad, dilation)
    out = convrot_conv2d_plan_t()
    _check(load_library().convrot_conv2d_gather_plan(ctypes.byref(g), sms, ctypes.byref(out)),
           "convrot_conv2d_gather_plan")
    return out


def quantize_conv_weight(w_oihw_bf16: torch.Tensor, stride: int = 1, pad: int = 0, dilation: int = 1,
                         group: Optional[int] = None, stream=None) -> QuantizedWeight:
    """Offline INT8 ConvRot conversion of a BF16 OIHW weight; the group
    defaults to the largest power of two <= 256 dividing the channels."""
    o, c, kh, kw = w_oihw_bf16.shape
    group = group or convrot_dynamic_group(c)
    k = kh * kw * c
    q = torch.empty((o, k), dtype=torch.int8, device=w_oihw_bf16.device)
    scale = torch.empty((o,), dtype=torch.float32, device=w_oihw_bf16.device)
    wt = convrot_weight_init(q, scale, group)
    g = convrot_conv2d_t(1, kh, kw, c, kh, kw, 1, 0, 1)      # only c, kh, kw matter for the weight
    _check(load_library().convrot_quantize_conv_weight(_ptr(w_oihw_bf16), ctypes.byref(g), ctypes.byref(wt.handle),
                                                       _stream(stream)), "convrot_quantize_conv_weight")
    return wt


def conv2d_int8(x_nhwc: torch.Tensor, w: QuantizedWeight, kh: int, kw: int, stride: int = 1, pad: int = 0,
                dilation: int = 1, y: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
    """INT8 ConvRot convolution: NHWC BF16 in, NHWC BF16 out."""
    g = conv2d_geometry(x_nhwc.shape, kh, kw, stride, pad, dilation)
    lib = load_library()
    oh, ow = ctypes.c_int32(), ctypes.c_int32()
    _check(lib.convrot_conv2d_shape(ctypes.byref(g), ctypes.byref(oh), ctypes.byref(ow)), "convrot_conv2d_shape")
    if y is None:
        y = torch.empty((g.n, oh.value, ow.value, w.n), dtype=torch.bfloat16, device=x_nhwc.device)
    if ws is None:
        need = int(lib.convrot_conv2d_workspace_bytes(ctypes.byref(g), ctypes.byref(w.handle)))
        if need == 0:
            raise ConvrotError(3, "convrot_conv2d_workspace_bytes")
        ws = torch.zeros(need, dtype=torch.uint8, device=x_nhwc.device)
    _check(lib.convrot_conv2d_int8(_ptr(x_nhwc), ctypes.byref(g), ctypes.byref(w.handle), _ptr(y), _ptr(ws),
                                   ws.numel(), _stream(stream)), "convrot_conv2d_int8")
    return y


def convrot_device_status(stream=None) -> None:
    _check(load_library().convrot_device_status(_stream(stream)), "convrot_device_status")


# ---------------------------------------------------------------- helpers
def convrot_dynamic_group(k: int, max_group: int = GROUP) -> int:
    """The group --dynamic-convrot picks for k input features (0: none)."""
    return int(load_library().convrot_dynamic_group(k, max_group))


def quantize_weight(w_bf16: torch.Tensor, stream=None, group: int = GROUP, dynamic: bool = False) -> QuantizedWeight:
    """Allocate q/scale and run the offline rotate+quantise kernel; with
    dynamic=True the group is the largest power of two <= group dividing k."""
    n, k = w_bf16.shape
    if dynamic:
        group = convrot_dynamic_group(k, group)
    q = torch.empty((n, k), dtype=torch.int8, device=w_bf16.device)
    scale = torch.empty((n,), dtype=torch.float32, device=w_bf16.device)
    return convrot_quantize_weight(w_bf16, convrot_weight_init(q, scale, group), stream)


def make_workspace(m: int, w: QuantizedWeight, device=None, linear: bool = True) -> torch.Tensor:
    """A zero-filled workspace big enough for convrot_linear_int8 (or, with
    linear=False, convrot_gemm_i8) at m rows against w."""
    nbytes = (convrot_linear_workspace_bytes if linear else convrot_gemm_workspace_bytes)(m, w.n, w.k)
    return torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device or w.q.device)


def linear_int8(x_bf16: torch.Tensor, w: QuantizedWeight, ws: torch.Tensor, y: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
    if y is None:
        y = torch.empty((x_bf16.shape[0], w.n), dtype=torch.bfloat16, device=x_bf16.device)
    convrot_linear_int8(x_bf16, w, y, ws, stream)
    return y
