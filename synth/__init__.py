"""Seeded synthetic inputs for the INT8 ConvRot linear layer.

This module holds none of the layer's arithmetic (no rotation, no
quantisation, no GEMM).  It only draws the BF16 activations X [M, K] and
weights W [N, K] that both the CUDA path and the CPU oracle consume, so the
two sides read identical bytes.

Generator (counter-based, so any element or row can be regenerated alone):

* ``splitmix64``: the i-th output (0-based) of the stream with state ``key``
  is ``mix(key + (i + 1) * 0x9E3779B97F4A7C15)`` with Vigna's finaliser
  ``z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27;
  z *= 0x94D049BB133111EB; z ^= z >> 31`` (all mod 2^64).
* Normal deviates: the top 16 bits of an output index a table of the 65536
  equiprobable quantiles ``Phi^-1((i + 0.5) / 65536)`` of N(0, 1), held as
  FP32.  This is a 16-bit discretisation of N(0, 1) (|z| <= 4.33, no zeros);
  it needs only integer arithmetic and a table lookup, so host (numpy) and
  device (torch) draws are bit-identical.
* A drawn element is ``bf16_rne(fp32(table[idx] * sigma) * scale[channel])``
  with FP32 products, then rounded once to BF16 (nearest-even).

Shapes and distributions follow the workloads the source pages describe
(Qwen3-VL-32B hidden 5120 with 12 conditioning tokens -- zskr.cn
"Qwen3-VL-32B ... INT8-ConvRot", validation section; MiniMax-H3
attn.qkv_proj in_features 5376 -- 0539edu.com section 4), with outlier
input channels to exercise the rotation's purpose of spreading outlier
energy.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Sequence, Tuple

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
MIX1 = 0xBF58476D1CE4E5B9
MIX2 = 0x94D049BB133111EB
MASK64 = (1 << 64) - 1

# ---------------------------------------------------------------------------
# normal quantile table
# ---------------------------------------------------------------------------
_TABLE: Optional[np.ndarray] = None


def normal_table() -> np.ndarray:
    """FP32 [65536]: Phi^-1((i + 0.5) / 65536)."""
    global _TABLE
    if _TABLE is None:
        from scipy.special import ndtri
        p = (np.arange(65536, dtype=np.float64) + 0.5) / 65536.0
        _TABLE = ndtri(p).astype(np.float32)
        _TABLE.setflags(write=False)
    return _TABLE


# ---------------------------------------------------------------------------
# splitmix64 (numpy, uint64 wrap-around arithmetic)
# ---------------------------------------------------------------------------
def splitmix64_at(key: int, idx: np.ndarray) -> np.ndarray:
    """Outputs number ``idx`` (uint64 array) of the stream with state ``key``."""
    with np.errstate(over="ignore"):
        z = np.uint64(key & MASK64) + (idx.astype(np.uint64) + np.uint64(1)) * np.uint64(GAMMA)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(MIX1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(MIX2)
        z = z ^ (z >> np.uint64(31))
    return z


def splitmix64_scalar(key: int, i: int) -> int:
    z = (key + (i + 1) * GAMMA) & MASK64
    z = ((z ^ (z >> 30)) * MIX1) & MASK64
    z = ((z ^ (z >> 27)) * MIX2) & MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, tensor_id: int) -> int:
    """Key of an independent stream for one tensor of one seeded workload."""
    return splitmix64_scalar(splitmix64_scalar(seed & MASK64, 0), tensor_id)


def f32_to_bf16_bits(f: np.ndarray) -> np.ndarray:
    """Nearest-even rounding of finite FP32 values to BF16 bit patterns."""
    u = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_f32_at(key: int, idx: np.ndarray) -> np.ndarray:
    z = splitmix64_at(key, idx)
    return normal_table()[(z >> np.uint64(48)).astype(np.int64)]


def draw_rows_np(key: int, rows: Sequence[int] | np.ndarray, cols: int,
                 sigma: float = 1.0,
                 channel_scale: Optional[np.ndarray] = None) -> np.ndarray:
    """BF16 bits [len(rows), cols] of the given rows of a drawn matrix."""
    rows = np.asarray(rows, dtype=np.int64)
    idx = rows[:, None] * np.int64(cols) + np.arange(cols, dtype=np.int64)[None, :]
    v = normal_f32_at(key, idx.reshape(-1)).reshape(len(rows), cols)
    if sigma != 1.0:
        v = (v * np.float32(sigma)).astype(np.float32)
    if channel_scale is not None:
        v = (v * channel_scale.astype(np.float32)[None, :]).astype(np.float32)
    return f32_to_bf16_bits(v)


def draw_np(key: int, rows: int, cols: int, sigma: float = 1.0,
            channel_scale: Optional[np.ndarray] = None) -> np.ndarray:
    """BF16 bits [rows, cols] of a whole drawn matrix (host)."""
    out = np.empty((rows, cols), dtype=np.uint16)
    step = max(1, (1 << 22) // max(cols, 1))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        out[r0:r1] = draw_rows_np(key, np.arange(r0, r1), cols, sigma, channel_scale)
    return out


# ---------------------------------------------------------------------------
# the same draws with torch (CPU or CUDA), bit-identical to the numpy ones
# ---------------------------------------------------------------------------
def _s64(c: int) -> int:
    c &= MASK64
    return c - (1 << 64) if c >= (1 << 63) else c


def _srl(z, s: int):
    return (z >> s) & ((1 << (64 - s)) - 1)


_TORCH_TABLES = {}


def _torch_table(device):
    import torch
    key = str(device)
    if key not in _TORCH_TABLES:
        _TORCH_TABLES[key] = torch.from_numpy(normal_table().copy()).to(device)
    return _TORCH_TABLES[key]


def draw_torch(key: int, rows: int, cols: int, sigma: float = 1.0,
               channel_scale: Optional[np.ndarray] = None, device="cpu",
               out=None, row_chunk: Optional[int] = None):
    """torch.bfloat16 [rows, cols] on ``device``, identical to ``draw_np``."""
    import torch
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.bfloat16, device=device)
    table = _torch_table(device)
    cs = None
    if channel_scale is not None:
        cs = torch.from_numpy(np.ascontiguousarray(channel_scale, dtype=np.float32)).to(device)
    if row_chunk is None:
        row_chunk = max(1, (1 << 24) // max(cols, 1))
    col_idx = torch.arange(cols, dtype=torch.int64, device=device)
    for r0 in range(0, rows, row_chunk):
        r1 = min(rows, r0 + row_chunk)
        idx = torch.arange(r0, r1, dtype=torch.int64, device=device)[:, None] * cols + col_idx[None, :]
        z = (idx + 1) * _s64(GAMMA) + _s64(key)
        z = (z ^ _srl(z, 30)) * _s64(MIX1)
        z = (z ^ _srl(z, 27)) * _s64(MIX2)
        z = z ^ _srl(z, 31)
        v = table[_srl(z, 48)]
        del z, idx
        if sigma != 1.0:
            v = v * torch.tensor(sigma, dtype=torch.float32, device=device)
        if cs is not None:
            v = v * cs[None, :]
        out[r0:r1] = v.to(torch.bfloat16)
    return out


# ---------------------------------------------------------------------------
# channel scales (outlier patterns); host only, K values
# ---------------------------------------------------------------------------
def outlier_scale_fixed(k: int, channels: Sequence[int], factor: float) -> np.ndarray:
    cs = np.ones(k, dtype=np.float32)
    cs[np.asarray(channels, dtype=np.int64)] = np.float32(factor)
    return cs


def outlier_scale_fraction(key: int, k: int, fraction: float, factor: float) -> np.ndarray:
    """The first ceil(fraction * k) channels of a seeded permutation get ``factor``."""
    order = np.argsort(splitmix64_at(key, np.arange(k, dtype=np.int64)), kind="stable")
    count = int(math.ceil(fraction * k))
    cs = np.ones(k, dtype=np.float32)
    cs[order[:count]] = np.float32(factor)
    return cs


def student_t3_scale(key: int, k: int, lo: float = 2.0 ** -6, hi: float = 2.0 ** 6) -> np.ndarray:
    """|t_3| per channel, t_3 = z / sqrt(chi2_3 / 3) from four table normals,
    clipped to [lo, hi] so every rotation group stays exactly summable."""
    base = np.arange(k, dtype=np.int64) * 4
    z = normal_f32_at(key, base).astype(np.float64)
    c2 = sum(normal_f32_at(key, base + j).astype(np.float64) ** 2 for j in (1, 2, 3))
    t = z / np.sqrt(c2 / 3.0)
    return np.clip(np.abs(t), lo, hi).astype(np.float32)


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------
# (name, K = in_features, N = out_features) of the seven linears of one
# Qwen3-VL-32B decoder layer (hidden 5120, 64 query / 8 kv heads of 128,
# MLP 25600).
QWEN_LINEARS: List[Tuple[str, int, int]] = [
    ("q", 5120, 8192), ("k", 5120, 1024), ("v", 5120, 1024),
    ("o", 8192, 5120), ("gate", 5120, 25600), ("up", 5120, 25600),
    ("down", 25600, 5120),
]
MINIMAX_QKV = ("qkv", 5376, 16128)
W_SIGMA = 0.02


@dataclass
class Linear:
    """One linear of a workload: shapes, seed and how X and W are drawn."""
    name: str
    m: int
    k: int
    n: int
    seed: int
    x_scale: np.ndarray = field(repr=False, default=None)
    group: int = 256

    @property
    def x_key(self) -> int:
        return stream_key(self.seed, 0)

    @property
    def w_key(self) -> int:
        return stream_key(self.seed, 1)

    def x_np(self) -> np.ndarray:
        return draw_np(self.x_key, self.m, self.k, 1.0, self.x_scale)

    def w_np(self) -> np.ndarray:
        return draw_np(self.w_key, self.n, self.k, W_SIGMA, None)

    def x_rows_np(self, rows) -> np.ndarray:
        return draw_rows_np(self.x_key, rows, self.k, 1.0, self.x_scale)

    def w_rows_np(self, rows) -> np.ndarray:
        return draw_rows_np(self.w_key, rows, self.k, W_SIGMA, None)

    def x_torch(self, device="cpu", out=None):
        return draw_torch(self.x_key, self.m, self.k, 1.0, self.x_scale, device, out)

    def w_torch(self, device="cpu", out=None):
        return draw_torch(self.w_key, self.n, self.k, W_SIGMA, None, device, out)

    @property
    def weight_bytes(self) -> int:
        return self.n * self.k


def tiny() -> List[Linear]:
    """M=4, K=512 (2 groups), N=256; X ~ N(0,1) with channels 3, 130, 300,
    511 scaled x50; W ~ N(0, 0.02); seed 0."""
    k = 512
    return [Linear("tiny", 4, k, 256, 0, outlier_scale_fixed(k, (3, 130, 300, 511), 50.0))]


def qwen_layer(m: int, seed_base: int = 1) -> List[Linear]:
    """The seven Qwen3-VL-32B-shaped linears at M tokens; X ~ N(0,1) with
    1% outlier channels x30 (seeded permutation); W ~ N(0, 0.02); seed
    ``seed_base + matrix index``."""
    out = []
    for i, (name, k, n) in enumerate(QWEN_LINEARS):
        seed = seed_base + i
        cs = outlier_scale_fraction(stream_key(seed, 2), k, 0.01, 30.0)
        out.append(Linear(name, m, k, n, seed, cs))
    return out


def minimax_qkv(m: int, seed: int = 4) -> List[Linear]:
    """MiniMax-H3-shaped attn.qkv_proj: K=5376 (21 groups), N=16128; X =
    z * c_k with heavy-tailed Student-t(3) channel scales; W ~ N(0, 0.02)."""
    name, k, n = MINIMAX_QKV
    return [Linear(name, m, k, n, seed, student_t3_scale(stream_key(seed, 2), k))]


def qwen_stack(m: int, layers: int = 50) -> List[Linear]:
    """``layers`` x the seven Qwen linears, seed 1000 + layer."""
    out = []
    for layer in range(layers):
        for lin in qwen_layer(m, seed_base=1000 + layer * 7):
            lin.name = "L%d.%s" % (layer, lin.name)
            out.append(lin)
    return out


WORKLOADS = {
    "tiny": lambda: tiny(),
    "qwen_decode_m12": lambda: qwen_layer(12),
    "qwen_prefill_m4096": lambda: qwen_layer(4096),
    "minimax_qkv_m8192": lambda: minimax_qkv(8192),
    "minimax_qkv_m32768": lambda: minimax_qkv(32768),
}
