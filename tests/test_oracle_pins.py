"""Pins for the CPU oracle, each against something other than the oracle.

The oracle (``oracle/``) is the parity reference for the CUDA path, so every
function in it is checked here against a library routine, a closed form,
hand-worked values under ``tests/golden/``, an invariant of the mathematics,
or brute force on tiny inputs.  These run without a GPU.
"""
import os

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append(line)
    return rows


def _f32_to_bf16_torch(f):
    """Nearest-even BF16 via torch's own conversion (a library routine)."""
    t = torch.from_numpy(np.ascontiguousarray(f, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _bf16_from_f32_exact(v):
    """BF16 bits of values that are exactly representable in BF16."""
    b = _f32_to_bf16_torch(np.asarray(v, dtype=np.float32))
    assert np.array_equal(synth.bf16_bits_to_f32(b), np.asarray(v, dtype=np.float32))
    return b


# ---------------------------------------------------------------------------
# Hadamard matrix
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 32, 64, 128, 256])
def test_hadamard_matches_scipy(n):
    assert np.array_equal(oracle.sylvester_hadamard(n), scipy.linalg.hadamard(n))


def test_hadamard_8_golden():
    H8 = np.array([[int(v) for v in r.split()] for r in _golden_rows("hadamard_8.txt")])
    assert np.array_equal(oracle.sylvester_hadamard(8), H8)


def test_hadamard_256_orthogonal_and_closed_form():
    H = oracle.sylvester_hadamard(256).astype(np.int64)
    assert np.array_equal(H @ H.T, 256 * np.eye(256, dtype=np.int64))
    assert np.array_equal(H, H.T)
    i = np.arange(256)
    pc = np.vectorize(lambda v: bin(v).count("1"))(i[:, None] & i[None, :])
    assert np.array_equal(H, np.where(pc % 2 == 0, 1, -1))


def test_hadamard_rejects_non_power_of_two():
    with pytest.raises(oracle.OracleError):
        oracle.sylvester_hadamard(12)


# ---------------------------------------------------------------------------
# rotation
# ---------------------------------------------------------------------------
def _block_rotation_np(x64, group):
    """Block-diagonal H/sqrt(G) applied with numpy's matmul and scipy's H."""
    H = scipy.linalg.hadamard(group).astype(np.float64) / np.sqrt(group)
    rows, k = x64.shape
    return (x64.reshape(rows, k // group, group) @ H).reshape(rows, k)


def test_rotation_matches_library_matmul_exactly():
    # products with +-1 are exact and the group sums are exact (within 37
    # binades), so numpy's FP64 matmul gives the exact value whatever its
    # summation order; rounding it once to FP32 must equal the oracle.
    lin = synth.tiny()[0]
    x = lin.x_np()
    y, bad = oracle.rotate_rows(x)
    assert bad == 0
    ref = _block_rotation_np(oracle.bf16_bits_to_f64(x), 256).astype(np.float32)
    assert np.array_equal(y, ref)
    w = lin.w_np()
    yw, bad = oracle.rotate_rows(w)
    assert bad == 0
    assert np.array_equal(yw, _block_rotation_np(oracle.bf16_bits_to_f64(w), 256).astype(np.float32))


def test_rotation_one_hot_golden():
    for line in _golden_rows("one_hot_rotation.txt"):
        i, c, ys, qs = [p.strip() for p in line.split("|")]
        i, c = int(i), float(c)
        yv = [float(v) for v in ys.split()]
        qv = [int(v) for v in qs.split()]
        row = np.zeros((1, 256), dtype=np.float32)
        row[0, i] = c
        y, bad = oracle.rotate_rows(_bf16_from_f32_exact(row))
        assert bad == 0
        assert list(y[0, :4]) == yv
        q, s = oracle.rotate_quantize(_bf16_from_f32_exact(row))
        assert list(q[0, :4]) == qv
        assert s[0] == np.float32(np.float32(abs(c) / 16.0) / np.float32(127.0))


def test_rotation_closed_forms_in_second_group():
    rng = np.random.default_rng(5)
    H = scipy.linalg.hadamard(256)
    for _ in range(20):
        i = int(rng.integers(256))
        c = np.float32(rng.choice([1.0, -2.0, 0.375, 96.0]))
        row = np.zeros((1, 512), dtype=np.float32)
        row[0, 256 + i] = c
        y, _ = oracle.rotate_rows(_bf16_from_f32_exact(row))
        assert np.all(y[0, :256] == 0)
        assert np.array_equal(y[0, 256:], (c * H[i] / 16.0).astype(np.float32))
    # constant group -> (16c, 0, ..., 0)
    row = np.full((1, 256), 0.75, dtype=np.float32)
    y, _ = oracle.rotate_rows(_bf16_from_f32_exact(row))
    assert y[0, 0] == np.float32(12.0) and np.all(y[0, 1:] == 0)


def test_rotation_involution_and_parseval():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((3, 768))
    y = oracle.rotate_rows_f64(x)
    assert np.allclose(oracle.rotate_rows_f64(y), x, rtol=0, atol=1e-12)
    for g in range(3):
        sl = slice(256 * g, 256 * (g + 1))
        assert np.allclose(np.linalg.norm(y[:, sl], axis=1),
                           np.linalg.norm(x[:, sl], axis=1), rtol=1e-13)


def test_rotation_preserves_the_layer():
    # (X R)(W R)^T = X W^T, FP64, to 1e-5 relative
    lin = synth.tiny()[0]
    x = oracle.bf16_bits_to_f64(lin.x_np())
    w = oracle.bf16_bits_to_f64(lin.w_np())
    lhs = oracle.rotate_rows_f64(x) @ oracle.rotate_rows_f64(w).T
    rhs = x @ w.T
    assert np.max(np.abs(lhs - rhs)) <= 1e-5 * np.max(np.abs(rhs))


def test_rotation_counts_inexact_groups():
    row = np.zeros((1, 512), dtype=np.float32)
    row[0, 0] = 2.0 ** 10
    row[0, 1] = 2.0 ** -30      # 41 binades apart inside group 0
    row[0, 256] = 1.0
    row[0, 257] = 2.0 ** -20    # 21 binades apart inside group 1: fine
    _, bad = oracle.rotate_rows(_bf16_from_f32_exact(row))
    assert bad == 1
    with pytest.raises(oracle.OracleError):
        oracle.rotate_quantize(_bf16_from_f32_exact(row))


def test_rotation_rejects_bad_group():
    x = np.zeros((1, 384), dtype=np.uint16)
    with pytest.raises(oracle.OracleError):
        oracle.rotate_rows(x, 256)       # 384 is not a multiple of 256
    with pytest.raises(oracle.OracleError):
        oracle.rotate_rows(np.zeros((1, 288), np.uint16), 96)   # not a power of 2


# ---------------------------------------------------------------------------
# tensor-wise simple INT8 (embedding table) and the lookup
# ---------------------------------------------------------------------------
def test_tensor_quant_closed_forms():
    f2b = synth.f32_to_bf16_bits
    p = -3
    # the largest magnitude 127 * 2^p sets s = 2^p exactly; y / s are then
    # exact, ties go to even, and one scale serves every row
    x = np.array([[127.0, 2.5, 3.5, -0.5, 1.0], [0.25, -4.5, 6.5, 0.0, -127.0]], np.float32) * 2.0 ** p
    q, sc, ties = oracle.quantize_tensor(f2b(x))
    assert sc == np.float32(2.0 ** p) and ties == 5
    assert np.array_equal(q, np.array([[127, 2, 4, 0, 1], [0, -4, 6, 0, -127]], np.int8))
    # per-row scales would differ (row 1's own maximum is the same here, so
    # use a table whose rows have different maxima)
    y = np.array([[127.0, 1.0], [1.0, 0.5]], np.float32)
    qt, st, _ = oracle.quantize_tensor(f2b(y))
    qr, sr, _ = oracle.quantize_rows(y)
    assert st == sr[0] and np.array_equal(qt[0], qr[0]) and not np.array_equal(qt[1], qr[1])
    assert list(qt[1]) == [1, 0]                     # 0.5 / 1 = 0.5 -> 0 (ties to even)
    # all-zero table
    q0, s0, _ = oracle.quantize_tensor(np.zeros((3, 4), np.uint16))
    assert s0 == 0 and not q0.any()


def test_embed_lookup_closed_forms():
    rng = np.random.default_rng(11)
    q = rng.integers(-127, 128, (50, 32)).astype(np.int8)
    s = np.float32(2.0 ** -5)
    tokens = np.array([3, 49, 0, 3, -1, 50], np.int32)
    out = oracle.embed_lookup(tokens, q, s)
    want = q[[3, 49, 0, 3]].astype(np.float32) * np.float32(2.0 ** -5)     # exact in BF16
    assert np.array_equal(synth.bf16_bits_to_f32(out[:4]), want)
    assert not out[4:].any()                                                # out of range -> zero rows
    # a scale that is not a power of two rounds each product once to BF16
    s2 = np.float32(0.0123)
    out2 = oracle.embed_lookup(np.array([7], np.int32), q, s2)
    assert np.array_equal(out2[0], _f32_to_bf16_torch(q[7].astype(np.float32) * s2))


# ---------------------------------------------------------------------------
# INT4 weights (W4A8)
# ---------------------------------------------------------------------------
def test_int4_quant_closed_forms():
    p = 4
    y = np.array([[7.0, 2.5, 3.5, -0.5, 6.5, -1.5, -7.0, 0.25]], np.float32) * 2.0 ** p
    q, s, ties = oracle.quantize_rows4(y)
    assert s[0] == np.float32(2.0 ** p) and ties == 5
    assert list(q[0]) == [7, 2, 4, 0, 6, -2, -7, 0]
    q0, s0, _ = oracle.quantize_rows4(np.zeros((1, 16), np.float32))
    assert s0[0] == 0 and not q0.any()
    rng = np.random.default_rng(12)
    yr = (rng.standard_normal((4, 512)) * rng.uniform(0.1, 10, (4, 1))).astype(np.float32)
    qr, sr, _ = oracle.quantize_rows4(yr)
    assert np.all(np.abs(yr - sr[:, None] * qr) <= sr[:, None] / 2 * (1 + 1e-6))
    assert np.array_equal(np.abs(qr).max(axis=1), np.full(4, 7))
    want = np.clip(np.rint(yr / (np.abs(yr).max(axis=1) / np.float32(7))[:, None]), -7, 7)
    assert np.array_equal(qr, want.astype(np.int8))


def test_int4_pack_golden_and_round_trip():
    lines = [l.split() for l in open(os.path.join(GOLDEN, "int4_pack.txt")) if l.strip() and not l.startswith("#")]
    codes = np.array([int(v) for v in lines[0]], np.int8).reshape(1, 16)
    want = np.array([int(v, 16) for v in lines[1]], np.uint8).reshape(1, 8)
    assert np.array_equal(oracle.pack_int4(codes), want)
    assert np.array_equal(oracle.unpack_int4(want), codes)
    rng = np.random.default_rng(13)
    q = rng.integers(-8, 8, (5, 96)).astype(np.int8)
    assert np.array_equal(oracle.unpack_int4(oracle.pack_int4(q)), q)
    # every code at every position of a chunk
    allq = np.array([[(v + j) % 16 - 8 for j in range(16)] for v in range(16)], np.int8)
    assert np.array_equal(oracle.unpack_int4(oracle.pack_int4(allq)), allq)


def test_w4a8_linear_composes():
    lin = synth.tiny()[0]
    x, w = lin.x_np(), lin.w_np()
    packed, sw = oracle.rotate_quantize4(w)
    y_rot, _ = oracle.rotate_rows(w)
    q4, s4, _ = oracle.quantize_rows4(y_rot)
    assert np.array_equal(oracle.unpack_int4(packed), q4) and np.array_equal(sw, s4)
    out = oracle.linear_w4a8(x, packed, sw)
    xq, sx = oracle.rotate_quantize(x)
    acc = xq.astype(np.int64) @ q4.astype(np.int64).T
    assert np.array_equal(out["acc"], acc)
    assert np.array_equal(out["y"], oracle.dequant_bf16(acc.astype(np.int32), sx, sw))
    # the 4-bit layer still approximates X W^T (coarser than INT8)
    ref = oracle.bf16_bits_to_f64(x) @ oracle.bf16_bits_to_f64(w).T
    err = np.max(np.abs(oracle.bf16_bits_to_f64(out["y"]) - ref)) / np.max(np.abs(ref))
    assert err < 0.3


# ---------------------------------------------------------------------------
# 2-D convolution as the layer on its im2col matrix
# ---------------------------------------------------------------------------
def _conv_direct_f64(x, w, stride, pad, dil):
    """Plain loops: out[b, oy, ox, o] = sum_{c, ky, kx} x[b, iy, ix, c] * w[o, c, ky, kx]."""
    n, h, wd, c = x.shape
    o, _, kh, kw = w.shape
    oh, ow = oracle.conv_out_size(h, kh, stride, pad, dil), oracle.conv_out_size(wd, kw, stride, pad, dil)
    out = np.zeros((n, oh, ow, o))
    for b in range(n):
        for oy in range(oh):
            for ox in range(ow):
                for ky in range(kh):
                    for kx in range(kw):
                        iy, ix = oy * stride - pad + ky * dil, ox * stride - pad + kx * dil
                        if 0 <= iy < h and 0 <= ix < wd:
                            out[b, oy, ox] += w[:, :, ky, kx] @ x[b, iy, ix]
    return out


@pytest.mark.parametrize("stride,pad,dil,kh", [(1, 1, 1, 3), (2, 1, 1, 3), (1, 2, 2, 3), (1, 0, 1, 1), (2, 0, 1, 2)])
def test_im2col_matches_direct_conv_and_torch(stride, pad, dil, kh):
    rng = np.random.default_rng(stride * 10 + pad + kh)
    xf = rng.standard_normal((2, 7, 6, 32)).astype(np.float32)
    wf = rng.standard_normal((5, 32, kh, kh)).astype(np.float32)
    xb, wb = synth.f32_to_bf16_bits(xf), synth.f32_to_bf16_bits(wf)
    x64, w64 = synth.bf16_bits_to_f32(xb).astype(np.float64), synth.bf16_bits_to_f32(wb).astype(np.float64)
    cols = synth.bf16_bits_to_f32(oracle.im2col_nhwc(xb, kh, kh, stride, pad, dil)).astype(np.float64)
    rows = synth.bf16_bits_to_f32(oracle.conv_weight_rows(wb)).astype(np.float64)
    got = cols @ rows.T
    direct = _conv_direct_f64(x64, w64, stride, pad, dil)
    assert np.allclose(got, direct.reshape(got.shape), rtol=1e-12, atol=1e-12)
    ref = torch.nn.functional.conv2d(torch.from_numpy(x64).permute(0, 3, 1, 2), torch.from_numpy(w64),
                                     stride=stride, padding=pad, dilation=dil).permute(0, 2, 3, 1).numpy()
    assert np.allclose(got, ref.reshape(got.shape), rtol=1e-10, atol=1e-10)


def test_rotation_preserves_the_convolution_and_int8_approximates_it():
    # groups lie inside a tap's channels, so rotating both sides keeps the product
    rng = np.random.default_rng(31)
    xf = rng.standard_normal((1, 6, 6, 256)).astype(np.float32)
    xf[..., 7] *= 40.0                                   # an outlier channel
    wf = (rng.standard_normal((16, 256, 3, 3)) * 0.02).astype(np.float32)
    xb, wb = synth.f32_to_bf16_bits(xf), synth.f32_to_bf16_bits(wf)
    cols = synth.bf16_bits_to_f32(oracle.im2col_nhwc(xb, 3, 3, 1, 1, 1)).astype(np.float64)
    rows = synth.bf16_bits_to_f32(oracle.conv_weight_rows(wb)).astype(np.float64)
    rot = oracle.rotate_rows_f64(cols, 256) @ oracle.rotate_rows_f64(rows, 256).T
    assert np.max(np.abs(rot - cols @ rows.T)) <= 1e-9 * np.max(np.abs(cols @ rows.T))
    out = oracle.conv2d_int8(xb, wb, 1, 1, 1)
    ref = (cols @ rows.T).reshape(out["y"].shape)
    y = oracle.bf16_bits_to_f64(out["y"])
    assert np.max(np.abs(y - ref)) / np.max(np.abs(ref)) < 0.05


# ---------------------------------------------------------------------------
# --dynamic-convrot: smaller power-of-two groups
# ---------------------------------------------------------------------------
def test_dynamic_group_choice():
    # the pages' own case: in_features 5376 = 21 x 256 keeps the full group
    assert oracle.dynamic_group(5376) == 256
    assert oracle.dynamic_group(640) == 128 and oracle.dynamic_group(5440) == 64
    assert oracle.dynamic_group(48) == 16 and oracle.dynamic_group(1024, 64) == 64
    # brute force: the largest power of two <= cap dividing k
    for cap in (256, 128, 100):
        for k in range(1, 3000):
            best = max(g for g in (1, 2, 4, 8, 16, 32, 64, 128, 256) if g <= cap and k % g == 0)
            assert oracle.dynamic_group(k, cap) == best, (k, cap)


@pytest.mark.parametrize("group", [16, 32, 64, 128])
def test_small_group_rotation_matches_scipy(group):
    # S exact in FP64 (any summation order), then S / sqrt(G) correctly
    # rounded in FP64, then rounded to FP32: numpy with scipy's Hadamard
    # computes the same value bit for bit
    rng = np.random.default_rng(group)
    x = synth.f32_to_bf16_bits(rng.standard_normal((5, 4 * group)).astype(np.float32))
    y, bad = oracle.rotate_rows(x, group)
    assert bad == 0
    xf = synth.bf16_bits_to_f32(x).astype(np.float64).reshape(5, 4, group)
    ref = (xf @ scipy.linalg.hadamard(group).astype(np.float64)) / np.sqrt(np.float64(group))
    assert np.array_equal(y, ref.reshape(5, 4 * group).astype(np.float32))


def test_small_group_closed_forms():
    # one-hot c * e_i in a group of 128 -> +-c / sqrt(128) everywhere in it,
    # zero in the other groups; orthonormal: applying it twice returns x
    c = 3.0
    x = np.zeros((1, 256), np.float32)
    x[0, 128 + 5] = c
    y, _ = oracle.rotate_rows(synth.f32_to_bf16_bits(x), 128)
    assert np.all(y[0, :128] == 0)
    assert np.array_equal(np.abs(y[0, 128:]), np.full(128, np.float32(c / np.sqrt(128.0))))
    h = scipy.linalg.hadamard(128)
    assert np.array_equal(np.sign(y[0, 128:]), h[5].astype(np.float32))
    rng = np.random.default_rng(9)
    xf = rng.standard_normal((3, 384))
    twice = oracle.rotate_rows_f64(oracle.rotate_rows_f64(xf, 128), 128)
    assert np.max(np.abs(twice - xf)) < 1e-12
    assert np.allclose(np.sum(oracle.rotate_rows_f64(xf, 32) ** 2, axis=1), np.sum(xf ** 2, axis=1), rtol=1e-12)


# ---------------------------------------------------------------------------
# quantisation
# ---------------------------------------------------------------------------
def test_quantize_golden_ties():
    for line in _golden_rows("quant_ties.txt"):
        p, ys, qs, away = [v.strip() for v in line.split("|")]
        p = int(p)
        y = (np.array([float(v) for v in ys.split()]) * 2.0 ** p).astype(np.float32)[None, :]
        q, s, ties = oracle.quantize_rows(y)
        assert s[0] == np.float32(2.0 ** p)
        assert list(q[0]) == [int(v) for v in qs.split()]
        assert list(q[0]) != [int(v) for v in away.split()]
        assert ties == sum(1 for v in ys.split() if float(v) % 1 == 0.5)


def test_quantize_subnormal_scale_matches_numpy_definition():
    # rows whose scale a / 127 is subnormal in FP32 (a < 127 * 2^-126): numpy's
    # FP32 division (IEEE, gradual underflow) gives s and y / s; the codes
    # stay in [-127, 127] and the row maximum still maps to +-127
    rng = np.random.default_rng(11)
    y = (rng.standard_normal((6, 256)) * np.float32(2.0 ** -126)).astype(np.float32)
    y *= np.array([1, 4, 16, 0.25, 8, 0.03], dtype=np.float32)[:, None]
    q, s, _ = oracle.quantize_rows(y)
    a = np.max(np.abs(y), axis=1)
    s_ref = (a / np.float32(127.0)).astype(np.float32)
    assert np.all(s_ref < np.float32(1.17549435e-38)) and np.all(s_ref > 0)
    assert np.array_equal(s.view(np.uint32), s_ref.view(np.uint32))
    t = (y / s_ref[:, None]).astype(np.float32)
    q_ref = np.clip(np.rint(t), -127, 127).astype(np.int8)
    assert np.array_equal(q, q_ref)
    assert np.all(np.abs(q[np.arange(6), np.argmax(np.abs(y), axis=1)]) == 127)


def test_quantize_matches_numpy_definition():
    rng = np.random.default_rng(2)
    y = (rng.standard_normal((16, 1024)) * rng.uniform(0.01, 100, (16, 1))).astype(np.float32)
    y[3] *= 0  # an all-zero row
    q, s, _ = oracle.quantize_rows(y)
    a = np.max(np.abs(y), axis=1)
    s_ref = (a / np.float32(127.0)).astype(np.float32)
    assert np.array_equal(s, s_ref)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (y / s_ref[:, None]).astype(np.float32)
    q_ref = np.where(a[:, None] == 0, 0, np.clip(np.rint(t), -127, 127)).astype(np.int8)
    assert np.array_equal(q, q_ref)
    assert np.all(q[3] == 0) and s[3] == 0
    # error bound |y - s q| <= s / 2 (plus the rounding of y / s)
    err = np.abs(y.astype(np.float64) - s[:, None].astype(np.float64) * q)
    assert np.all(err <= s[:, None] * (0.5 + 1e-6))
    # the row maximum maps to +-127
    amax = np.argmax(np.abs(y), axis=1)
    for r in range(16):
        if r != 3:
            assert abs(int(q[r, amax[r]])) == 127


def test_exhaustive_bf16_one_hot():
    # every finite BF16 c whose scale stays a normal FP32, one-hot at a
    # position that cycles over the group: q = 127 sign(c) H[i, :]
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = synth.bf16_bits_to_f32(bits)
    keep = np.isfinite(vals) & (np.abs(vals) >= 2.0 ** -120)
    bits, vals = bits[keep], vals[keep]
    pos = np.arange(len(bits)) % 256
    rows = np.zeros((len(bits), 256), dtype=np.uint16)
    rows[np.arange(len(bits)), pos] = bits
    q, s = oracle.rotate_quantize(rows)
    H = scipy.linalg.hadamard(256)
    expect = (127 * np.sign(vals)[:, None] * H[pos]).astype(np.int8)
    assert np.array_equal(q, expect)
    s_ref = ((np.abs(vals) / np.float32(16.0)).astype(np.float32) / np.float32(127.0)).astype(np.float32)
    assert np.array_equal(s, s_ref)


# ---------------------------------------------------------------------------
# INT8 GEMM
# ---------------------------------------------------------------------------
def test_gemm_brute_force_tiny():
    rng = np.random.default_rng(3)
    xq = rng.integers(-127, 128, (3, 64), dtype=np.int8)
    wq = rng.integers(-127, 128, (5, 64), dtype=np.int8)
    acc = oracle.gemm_i32(xq, wq)
    for i in range(3):
        for j in range(5):
            assert acc[i, j] == sum(int(xq[i, t]) * int(wq[j, t]) for t in range(64))


def test_gemm_matches_numpy_int64():
    rng = np.random.default_rng(4)
    xq = rng.integers(-127, 128, (7, 1024), dtype=np.int8)
    wq = rng.integers(-127, 128, (33, 1024), dtype=np.int8)
    ref = xq.astype(np.int64) @ wq.astype(np.int64).T
    assert np.array_equal(oracle.gemm_i32(xq, wq), ref.astype(np.int32))
    # asymmetric operands catch a transposed index
    assert not np.array_equal(oracle.gemm_i32(xq, wq)[:, :7], ref[:7, :7].T)


def test_gemm_extremes_and_overflow():
    k = 25600
    ones = np.full((1, k), 127, dtype=np.int8)
    assert oracle.gemm_i32(ones, -ones)[0, 0] == -k * 127 * 127
    k_over = 140000   # 140000 * 127^2 > 2^31 - 1
    with pytest.raises(oracle.OracleError):
        oracle.gemm_i32(np.full((1, k_over), 127, np.int8), np.full((1, k_over), 127, np.int8))


# ---------------------------------------------------------------------------
# dequantisation
# ---------------------------------------------------------------------------
def test_float_to_bf16_matches_torch():
    rng = np.random.default_rng(6)
    u = rng.integers(0, 2 ** 32, 200000, dtype=np.uint64).astype(np.uint32)
    f = u.view(np.float32)
    f = f[np.isfinite(f) & (np.abs(f) < 3.0e38)]
    # add exact ties and values right next to them
    base = synth.bf16_bits_to_f32(rng.integers(0, 0x7F00, 2000).astype(np.uint16))
    ties = (base.view(np.uint32) + np.uint32(0x8000)).view(np.float32)
    f = np.concatenate([f, ties, -ties, np.nextafter(ties, np.float32(np.inf))])
    mine = np.array([oracle.float_to_bf16(float(v)) for v in f[:40000]], dtype=np.uint16)
    assert np.array_equal(mine, _f32_to_bf16_torch(f[:40000]))
    mine_t = np.array([oracle.float_to_bf16(float(v)) for v in f[-6000:]], dtype=np.uint16)
    assert np.array_equal(mine_t, _f32_to_bf16_torch(f[-6000:]))


def test_dequant_matches_definition():
    rng = np.random.default_rng(7)
    acc = rng.integers(-400_000_000, 400_000_000, (6, 50)).astype(np.int32)
    sx = rng.uniform(1e-3, 1, 6).astype(np.float32)
    sw = rng.uniform(1e-5, 1e-3, 50).astype(np.float32)
    y = oracle.dequant_bf16(acc, sx, sw)
    v = (acc.astype(np.float32) * sx[:, None]).astype(np.float32) * sw[None, :]
    assert np.array_equal(y, _f32_to_bf16_torch(v.astype(np.float32)))
    # a scale applied along the wrong axis is caught
    y_bad = oracle.dequant_bf16(acc[:, :6].copy(), sw[:6].copy(), sx)
    assert not np.array_equal(y[:, :6], y_bad)


def test_dequant_bias_closed_forms():
    f2b = synth.f32_to_bf16_bits
    # acc = 0: the output is the bias itself, bit for bit
    bias = f2b(np.array([1.5, -3.25, 0.0, 2.0 ** -20, -65504.0], np.float32))
    y = oracle.dequant_bf16(np.zeros((2, 5), np.int32), np.ones(2, np.float32), np.ones(5, np.float32), bias)
    assert np.array_equal(y, np.stack([bias, bias]))
    # a zero bias changes nothing; None means no bias
    rng = np.random.default_rng(8)
    acc = rng.integers(-10 ** 6, 10 ** 6, (3, 7)).astype(np.int32)
    sx, sw = rng.uniform(0.1, 1, 3).astype(np.float32), rng.uniform(0.1, 1, 7).astype(np.float32)
    assert np.array_equal(oracle.dequant_bf16(acc, sx, sw, np.zeros(7, np.uint16)), oracle.dequant_bf16(acc, sx, sw))
    # 3 * 0.5 * 2 + 1.5 = 4.5 exactly
    y = oracle.dequant_bf16(np.array([[3]], np.int32), np.array([0.5], np.float32), np.array([2.0], np.float32),
                            f2b(np.array([1.5], np.float32)))
    assert synth.bf16_bits_to_f32(y)[0, 0] == 4.5
    # the bias joins the FP32 product before the one rounding to BF16:
    # 513 * 2^-9 + 2^-8 = 1 + 3 * 2^-9 rounds up to 1 + 2^-7, while rounding
    # the product first (to 1.0) and then adding would give a tie -> 1.0
    y = oracle.dequant_bf16(np.array([[513]], np.int32), np.array([2.0 ** -9], np.float32),
                            np.array([1.0], np.float32), f2b(np.array([2.0 ** -8], np.float32)))
    assert synth.bf16_bits_to_f32(y)[0, 0] == np.float32(1 + 2.0 ** -7)
    # the bias is indexed by the output column
    b = f2b(np.arange(7, dtype=np.float32))
    y = oracle.dequant_bf16(np.zeros((3, 7), np.int32), sx, sw, b)
    assert np.array_equal(synth.bf16_bits_to_f32(y), np.tile(np.arange(7, dtype=np.float32), (3, 1)))


# ---------------------------------------------------------------------------
# whole layer
# ---------------------------------------------------------------------------
def test_linear_composes_steps_and_approximates_fp64():
    lin = synth.tiny()[0]
    x, w = lin.x_np(), lin.w_np()
    wq, sw = oracle.rotate_quantize(w)
    out = oracle.linear_int8(x, wq, sw)
    xq, sx = oracle.rotate_quantize(x)
    assert np.array_equal(out["xq"], xq) and np.array_equal(out["sx"], sx)
    acc = xq.astype(np.int64) @ wq.astype(np.int64).T
    assert np.array_equal(out["acc"], acc)
    assert np.array_equal(out["y"], oracle.dequant_bf16(acc.astype(np.int32), sx, sw))
    # the quantised layer approximates the FP64 layer X W^T
    ref = oracle.bf16_bits_to_f64(x) @ oracle.bf16_bits_to_f64(w).T
    y = oracle.bf16_bits_to_f64(out["y"])
    assert np.max(np.abs(y - ref)) / np.max(np.abs(ref)) < 0.05


def test_rotation_spreads_outliers():
    # the method's purpose: with outlier channels, rotating before row INT8
    # quantisation lowers the quantisation error of the activations
    lin = synth.tiny()[0]
    x = lin.x_np()
    x64 = oracle.bf16_bits_to_f64(x)
    q_rot, s_rot = oracle.rotate_quantize(x)
    deq_rot = oracle.rotate_rows_f64(q_rot.astype(np.float64) * s_rot[:, None].astype(np.float64))
    q_plain, s_plain, _ = oracle.quantize_rows(x64.astype(np.float32))
    deq_plain = q_plain.astype(np.float64) * s_plain[:, None]
    err_rot = np.linalg.norm(deq_rot - x64)
    err_plain = np.linalg.norm(deq_plain - x64)
    assert err_rot < 0.5 * err_plain


def test_matmul_f64_matches_numpy():
    rng = np.random.default_rng(8)
    a = rng.standard_normal((4, 37))
    b = rng.standard_normal((6, 37))
    assert np.allclose(oracle.matmul_nt_f64(a, b), a @ b.T, rtol=1e-13, atol=1e-13)


def test_openmp_build_equals_single_threaded_build():
    # the all-cores CPU baseline runs the same C source built with -fopenmp
    # (rows split over threads); every output must equal the single-threaded
    # oracle's bit for bit, inexact-group counts and ties included
    import os
    import synth
    lin = synth.qwen_layer(37)[1]
    x = lin.x_np()
    w_bits = lin.w_rows_np(np.arange(300))
    y_in = np.random.default_rng(11).standard_normal((40, 768)).astype(np.float32)
    y_in[3, :] = np.float32(2.5)                        # s = 1: a row of exact ties
    y_in[3, 0] = np.float32(127.0)
    tiny = np.zeros((3, 512), np.uint16)
    tiny[0, 0] = 0x3F80                                 # 1.0 and 2^-60 in one group: inexact
    tiny[0, 1] = synth.f32_to_bf16_bits(np.array([2.0 ** -60], np.float32))[0]
    results = []
    old = os.environ.get("OMP_NUM_THREADS")
    os.environ["OMP_NUM_THREADS"] = "4"
    try:
        for par in (False, True):
            oracle.set_parallel(par)
            wq, sw = oracle.rotate_quantize(w_bits)
            ref = oracle.linear_int8(x, wq, sw)
            y, bad = oracle.rotate_rows(tiny)
            q, s, ties = oracle.quantize_rows(y_in)
            results.append([wq, sw, ref["y"], ref["acc"], ref["xq"], y, q, s, bad, ties])
    finally:
        oracle.set_parallel(False)
        if old is None:
            del os.environ["OMP_NUM_THREADS"]
        else:
            os.environ["OMP_NUM_THREADS"] = old
    a, b = results
    for u, v in zip(a[:8], b[:8]):
        assert np.array_equal(u, v)
    assert a[8] == b[8] == 1
    assert a[9] == b[9] > 0
