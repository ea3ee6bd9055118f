"""CPU oracle for the INT8 ConvRot linear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or calls it, and it shares no code
with that path.

The arithmetic lives in ``convrot_oracle.c`` (plain C, compiled with gcc, no
fast-math, no FMA contraction); this module only compiles it and marshals
numpy arrays through ctypes.  What each function computes, and the passage of
the source pages it follows, is stated in the C file:

* grouped Hadamard rotation, group 256, Sylvester order, 1/16 normalisation,
  exact FP64 sum rounded once to FP32  (0539edu.com "minimax-h3-nvfp4-convrot",
  section 4 "INT8 ConvRot"; zskr.cn "Qwen3-VL-32B ... INT8-ConvRot",
  "INT8 ConvRot quantisation details")
* row-wise symmetric INT8 round-to-nearest-even quantisation
  (zskr.cn conversion command ``--int8 --scaling_mode row``; 0539edu.com
  section 5, ``--simple`` = RTN)
* exact INT8 x INT8 -> INT32 GEMM and FP32 dequantisation to BF16
  (0539edu.com section 4 and summary item 3), with an optional BF16 bias
  (an extension; the pages' projections carry none)
* the group --dynamic-convrot picks: the largest power of two <= 256 that
  divides k, with rotations of such groups (0539edu.com section 4, item 3)
* tensor-wise simple INT8 of the embedding table and the lookup from it
  (zskr.cn quantisation configuration and conversion command)
* 2-D convolutions as the ConvRot layer on their im2col matrix (NHWC input,
  taps outer, channels inner; the VAE's int8_convrot)
* INT4 ConvRot weights (levels -7..7, row scale a/7) packed two per byte,
  with INT8 activations: the W4A4 variant's Blackwell route (0539edu.com
  sections 5 and 7)

Every function here is pinned by the ``-m "not gpu"`` tests against
something other than itself (scipy's Hadamard, closed forms, brute force,
numpy integer matmul, hand-worked tie cases).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "convrot_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_LIB_OMP = os.path.join(_HERE, "liboracle_omp.so")
_CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c99", "-Wall",
           "-shared", "-fPIC"]

_libs = {}
_parallel = False


def build(force: bool = False, openmp: bool = False) -> str:
    """Compile ``convrot_oracle.c`` into ``liboracle.so`` next to it (with
    ``openmp``: ``liboracle_omp.so``, the same source built with -fopenmp,
    rows split over threads, for the timed all-cores CPU baseline)."""
    lib = _LIB_OMP if openmp else _LIB
    if force or not os.path.exists(lib) or (
            os.path.getmtime(lib) < os.path.getmtime(_SRC)):
        tmp = lib + ".tmp.%d" % os.getpid()
        extra = ["-fopenmp"] if openmp else []
        subprocess.check_call(["gcc", *_CFLAGS, *extra, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, lib)
    return lib


def set_parallel(on: bool) -> None:
    """Route the calls below to the OpenMP build (all host cores, or
    OMP_NUM_THREADS) or back to the single-threaded one."""
    global _parallel
    _parallel = bool(on)


def _load():
    if _parallel not in _libs:
        lib = ctypes.CDLL(build(openmp=_parallel))
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        lib.oracle_sylvester_hadamard.argtypes = [ctypes.c_int, P]
        lib.oracle_sylvester_hadamard.restype = ctypes.c_int
        lib.oracle_rotate_rows.argtypes = [P, I64, I64, ctypes.c_int, P, P]
        lib.oracle_rotate_rows.restype = ctypes.c_int
        lib.oracle_rotate_rows_f64.argtypes = [P, I64, I64, ctypes.c_int, P]
        lib.oracle_rotate_rows_f64.restype = ctypes.c_int
        lib.oracle_quantize_rows.argtypes = [P, I64, I64, P, P]
        lib.oracle_quantize_rows.restype = I64
        lib.oracle_gemm_i32.argtypes = [P, P, I64, I64, I64, P]
        lib.oracle_gemm_i32.restype = I64
        lib.oracle_dequant_bf16.argtypes = [P, P, P, I64, I64, P]
        lib.oracle_quantize_tensor.argtypes = [P, I64, P, P]
        lib.oracle_quantize_tensor.restype = I64
        lib.oracle_embed_lookup.argtypes = [P, I64, P, ctypes.c_float, I64, I64, P]
        lib.oracle_embed_lookup.restype = I64
        lib.oracle_quantize_rows4.argtypes = [P, I64, I64, P, P]
        lib.oracle_quantize_rows4.restype = I64
        lib.oracle_pack_int4.argtypes = [P, I64, I64, P]
        lib.oracle_unpack_int4.argtypes = [P, I64, I64, P]
        lib.oracle_rotate_quantize4.argtypes = [P, I64, I64, ctypes.c_int, P, P]
        lib.oracle_rotate_quantize4.restype = I64
        lib.oracle_im2col_nhwc.argtypes = [P, I64, I64, I64, I64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, I64, I64, P]
        lib.oracle_conv_weight_rows.argtypes = [P, I64, I64, ctypes.c_int, ctypes.c_int, P]
        lib.oracle_dynamic_group.argtypes = [I64, ctypes.c_int]
        lib.oracle_dynamic_group.restype = ctypes.c_int
        lib.oracle_dequant_bf16_bias.argtypes = [P, P, P, P, I64, I64, P]
        lib.oracle_dequant_bf16.restype = None
        lib.oracle_rotate_quantize.argtypes = [P, I64, I64, ctypes.c_int, P, P]
        lib.oracle_rotate_quantize.restype = I64
        lib.oracle_linear_int8.argtypes = [P, I64, I64, ctypes.c_int, P, P, I64,
                                           P, P, P, P]
        lib.oracle_linear_int8.restype = ctypes.c_int
        lib.oracle_matmul_nt_f64.argtypes = [P, P, I64, I64, I64, P]
        lib.oracle_matmul_nt_f64.restype = None
        lib.oracle_float_to_bf16.argtypes = [ctypes.c_float]
        lib.oracle_float_to_bf16.restype = ctypes.c_uint16
        _libs[_parallel] = lib
    return _libs[_parallel]


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _bf16_bits(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("BF16 inputs are passed as their uint16 bit patterns")
    return a


class OracleError(RuntimeError):
    pass


def sylvester_hadamard(n: int) -> np.ndarray:
    """H_n by Sylvester's recursion, int32 [n, n]."""
    H = np.empty((n, n), dtype=np.int32)
    if _load().oracle_sylvester_hadamard(n, _ptr(H)) != 0:
        raise OracleError("n must be a power of two")
    return H


def dynamic_group(k: int, max_group: int = 256) -> int:
    """The largest power of two <= max_group dividing k (--dynamic-convrot)."""
    return int(_load().oracle_dynamic_group(k, max_group))


def rotate_rows(a_bf16: np.ndarray, group: int = 256):
    """Grouped Hadamard rotation of BF16 rows, exact then rounded to FP32.

    Returns ``(y_fp32, inexact_groups)``.
    """
    a = _bf16_bits(a_bf16)
    rows, k = a.shape
    y = np.empty((rows, k), dtype=np.float32)
    bad = ctypes.c_int64(0)
    if _load().oracle_rotate_rows(_ptr(a), rows, k, group, _ptr(y),
                                  ctypes.byref(bad)) != 0:
        raise OracleError("group must be a power of two dividing k")
    return y, int(bad.value)


def rotate_rows_f64(a: np.ndarray, group: int = 256) -> np.ndarray:
    """The same rotation on FP64 rows, kept in FP64."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    rows, k = a.shape
    y = np.empty((rows, k), dtype=np.float64)
    if _load().oracle_rotate_rows_f64(_ptr(a), rows, k, group, _ptr(y)) != 0:
        raise OracleError("group must be a power of two dividing k")
    return y


def quantize_rows(y: np.ndarray):
    """Row-wise absmax INT8 RTN of FP32 rows.  Returns ``(q, s, ties)``."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    rows, k = y.shape
    q = np.empty((rows, k), dtype=np.int8)
    s = np.empty((rows,), dtype=np.float32)
    ties = _load().oracle_quantize_rows(_ptr(y), rows, k, _ptr(q), _ptr(s))
    return q, s, int(ties)


def rotate_quantize(a_bf16: np.ndarray, group: int = 256):
    """Rotate then quantise BF16 rows (weights offline, activations online).

    Returns ``(q int8 [rows,k], s fp32 [rows])``; raises if a group's
    rotation could not be evaluated exactly.
    """
    a = _bf16_bits(a_bf16)
    rows, k = a.shape
    q = np.empty((rows, k), dtype=np.int8)
    s = np.empty((rows,), dtype=np.float32)
    bad = _load().oracle_rotate_quantize(_ptr(a), rows, k, group, _ptr(q), _ptr(s))
    if bad < 0:
        raise OracleError("group must be a power of two dividing k")
    if bad > 0:
        raise OracleError("%d rotation groups span more than 37 binades" % bad)
    return q, s


def quantize_tensor(a_bf16: np.ndarray):
    """Tensor-wise simple INT8 (embedding table): ``(q int8, s fp32 scalar,
    ties)`` with one scale for the whole tensor, no rotation."""
    a = _bf16_bits(a_bf16)
    q = np.empty(a.shape, dtype=np.int8)
    s = np.empty((1,), dtype=np.float32)
    ties = _load().oracle_quantize_tensor(_ptr(a), a.size, _ptr(q), _ptr(s))
    if ties < 0:
        raise OracleError("out of memory")
    return q, s[0], int(ties)


def embed_lookup(tokens: np.ndarray, q: np.ndarray, s) -> np.ndarray:
    """out[i] = bf16(q[tokens[i]] * s) as BF16 bits; zero rows for tokens
    outside the table."""
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    q = np.ascontiguousarray(q, dtype=np.int8)
    vocab, dim = q.shape
    out = np.empty((tokens.size, dim), dtype=np.uint16)
    _load().oracle_embed_lookup(_ptr(tokens), tokens.size, _ptr(q), float(np.float32(s)), vocab, dim, _ptr(out))
    return out


def quantize_rows4(y: np.ndarray):
    """Row-wise absmax INT4 RTN (levels -7..7) of FP32 rows: ``(q int8, s, ties)``."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    rows, k = y.shape
    q = np.empty((rows, k), dtype=np.int8)
    s = np.empty((rows,), dtype=np.float32)
    ties = _load().oracle_quantize_rows4(_ptr(y), rows, k, _ptr(q), _ptr(s))
    return q, s, int(ties)


def pack_int4(q: np.ndarray) -> np.ndarray:
    """INT4 codes [rows, k] (int8 holding -8..7) -> packed uint8 [rows, k/2]."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    rows, k = q.shape
    assert k % 16 == 0
    out = np.empty((rows, k // 2), dtype=np.uint8)
    _load().oracle_pack_int4(_ptr(q), rows, k, _ptr(out))
    return out


def unpack_int4(packed: np.ndarray) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    rows, half = packed.shape
    out = np.empty((rows, 2 * half), dtype=np.int8)
    _load().oracle_unpack_int4(_ptr(packed), rows, 2 * half, _ptr(out))
    return out


def rotate_quantize4(a_bf16: np.ndarray, group: int = 256):
    """Rotate, INT4-quantise and pack BF16 weight rows: ``(packed uint8 [rows, k/2], s fp32 [rows])``."""
    a = _bf16_bits(a_bf16)
    rows, k = a.shape
    packed = np.empty((rows, k // 2), dtype=np.uint8)
    s = np.empty((rows,), dtype=np.float32)
    bad = _load().oracle_rotate_quantize4(_ptr(a), rows, k, group, _ptr(packed), _ptr(s))
    if bad < 0:
        raise OracleError("group must be a power of two dividing k, k % 16 == 0")
    if bad > 0:
        raise OracleError("%d rotation groups span more than 37 binades" % bad)
    return packed, s


def linear_w4a8(x_bf16: np.ndarray, packed: np.ndarray, sw: np.ndarray, group: int = 256, bias=None):
    """W4A8 layer: the activations as in linear_int8 (INT8 rows), the weight
    codes unpacked from INT4; exact INT32 GEMM; the same dequantisation."""
    wq = unpack_int4(packed)
    return linear_int8(x_bf16, wq, sw, group=group, bias=bias)


def conv_out_size(size: int, k: int, stride: int, pad: int, dil: int) -> int:
    return (size + 2 * pad - dil * (k - 1) - 1) // stride + 1


def im2col_nhwc(x_bf16: np.ndarray, kh: int, kw: int, stride: int = 1, pad: int = 0, dil: int = 1) -> np.ndarray:
    """BF16 bits [n, h, w, c] -> im2col rows [n*oh*ow, kh*kw*c] (taps outer, channels inner)."""
    x = _bf16_bits(x_bf16)
    n, h, w, c = x.shape
    oh, ow = conv_out_size(h, kh, stride, pad, dil), conv_out_size(w, kw, stride, pad, dil)
    out = np.empty((n * oh * ow, kh * kw * c), dtype=np.uint16)
    _load().oracle_im2col_nhwc(_ptr(x), n, h, w, c, kh, kw, stride, pad, dil, oh, ow, _ptr(out))
    return out


def conv_weight_rows(w_bf16: np.ndarray) -> np.ndarray:
    """BF16 bits [o, c, kh, kw] (OIHW) -> rows [o, kh*kw*c] in the im2col order."""
    w = _bf16_bits(w_bf16)
    o, c, kh, kw = w.shape
    out = np.empty((o, kh * kw * c), dtype=np.uint16)
    _load().oracle_conv_weight_rows(_ptr(w), o, c, kh, kw, _ptr(out))
    return out


def conv2d_int8(x_nhwc_bf16: np.ndarray, w_oihw_bf16: np.ndarray, stride: int = 1, pad: int = 0, dil: int = 1,
                group: int = 256):
    """INT8 ConvRot 2-D convolution: the linear layer on the im2col matrix.
    Returns the linear_int8 dict with ``y`` reshaped to NHWC [n, oh, ow, o]."""
    n, h, w, c = x_nhwc_bf16.shape
    o, _, kh, kw = w_oihw_bf16.shape
    oh, ow = conv_out_size(h, kh, stride, pad, dil), conv_out_size(w, kw, stride, pad, dil)
    wq, sw = rotate_quantize(conv_weight_rows(w_oihw_bf16), group)
    out = linear_int8(im2col_nhwc(x_nhwc_bf16, kh, kw, stride, pad, dil), wq, sw, group=group)
    out["y"] = out["y"].reshape(n, oh, ow, o)
    out["wq"], out["sw"] = wq, sw
    return out


def gemm_i32(xq: np.ndarray, wq: np.ndarray) -> np.ndarray:
    """acc = xq @ wq.T, exact, int32 (raises on overflow)."""
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    wq = np.ascontiguousarray(wq, dtype=np.int8)
    m, k = xq.shape
    n, k2 = wq.shape
    assert k == k2
    acc = np.empty((m, n), dtype=np.int32)
    if _load().oracle_gemm_i32(_ptr(xq), _ptr(wq), m, n, k, _ptr(acc)) != 0:
        raise OracleError("INT32 overflow in the INT8 GEMM")
    return acc


def dequant_bf16(acc: np.ndarray, sx: np.ndarray, sw: np.ndarray, bias=None) -> np.ndarray:
    """Y = bf16(((float)acc * sx[m]) * sw[n] [+ bias[n]]) as uint16 bit
    patterns; ``bias`` is BF16 bits [n] or None."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    sx = np.ascontiguousarray(sx, dtype=np.float32)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    m, n = acc.shape
    y = np.empty((m, n), dtype=np.uint16)
    if bias is None:
        _load().oracle_dequant_bf16(_ptr(acc), _ptr(sx), _ptr(sw), m, n, _ptr(y))
    else:
        b = _bf16_bits(np.asarray(bias).reshape(-1))
        assert b.shape == (n,)
        _load().oracle_dequant_bf16_bias(_ptr(acc), _ptr(sx), _ptr(sw), _ptr(b), m, n, _ptr(y))
    return y


def linear_int8(x_bf16: np.ndarray, wq: np.ndarray, sw: np.ndarray,
                group: int = 256, bias=None):
    """Forward of the layer on pre-quantised weights (optional BF16 bias
    bits [n], added in FP32 before the rounding to BF16).

    Returns a dict with ``y`` (BF16 bits [m,n]), ``xq``, ``sx`` and ``acc``.
    """
    x = _bf16_bits(x_bf16)
    wq = np.ascontiguousarray(wq, dtype=np.int8)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    m, k = x.shape
    n = wq.shape[0]
    y = np.empty((m, n), dtype=np.uint16)
    xq = np.empty((m, k), dtype=np.int8)
    sx = np.empty((m,), dtype=np.float32)
    acc = np.empty((m, n), dtype=np.int32)
    rc = _load().oracle_linear_int8(_ptr(x), m, k, group, _ptr(wq), _ptr(sw), n,
                                    _ptr(y), _ptr(xq), _ptr(sx), _ptr(acc))
    if rc != 0:
        raise OracleError({-1: "bad arguments", -2: "inexact rotation group",
                           -3: "INT32 overflow"}[rc])
    if bias is not None:
        y = dequant_bf16(acc, sx, sw, bias)
    return {"y": y, "xq": xq, "sx": sx, "acc": acc}


def matmul_nt_f64(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """c = a @ b.T in FP64, plain triple loop."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    b = np.ascontiguousarray(b, dtype=np.float64)
    m, k = a.shape
    n, _ = b.shape
    c = np.empty((m, n), dtype=np.float64)
    _load().oracle_matmul_nt_f64(_ptr(a), _ptr(b), m, n, k, _ptr(c))
    return c


def float_to_bf16(f: float) -> int:
    """Nearest-even BF16 bit pattern of one binary32 value."""
    return int(_load().oracle_float_to_bf16(ctypes.c_float(f)))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen BF16 bit patterns to FP64 (exact)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
