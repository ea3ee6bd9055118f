"""The tiled im2col gather's launch plan (host arithmetic, no GPU): for the
library's chosen tile shapes, a model of the kernel's index arithmetic stays
inside its buffers and writes every code of every im2col row exactly once.

The model restates, in plain Python, what conv_gather_tile_kernel addresses:
one bulk copy per in-image region row into the region buffer, the pixel
maxima (zero outside the image), and per output row the 16-value chunks
base + lane read from the region (or its zero pixel) with the float4 parts
in the swizzled order and stored as 16 bytes at row * K + 16 * chunk.
"""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

SMEM_TWO_BUFFERS = 226 * 1024
SMS = 148


def out_size(size, k, stride, pad, dil):
    return (size + 2 * pad - dil * (k - 1) - 1) // stride + 1


def check_plan(n, h, w, c, k, stride, pad, dil, plan, full=True, tile_sample=None):
    oh, ow = out_size(h, k, stride, pad, dil), out_size(w, k, stride, pad, dil)
    th, tw, rh, rw = plan.th, plan.tw, plan.rh, plan.rw
    assert rh == (th - 1) * stride + (k - 1) * dil + 1 and rw == (tw - 1) * stride + (k - 1) * dil + 1
    ty_n, tx_n = -(-oh // th), -(-ow // tw)
    assert plan.tiles == n * ty_n * tx_n
    region = rh * rw * c * 4
    assert region + c * 4 + rh * rw * 4 <= plan.buf_bytes and plan.buf_bytes % 16 == 0
    assert 2 * plan.buf_bytes <= SMEM_TWO_BUFFERS
    taps, cc = k * k, c // 16
    kc = taps * cc                       # 16-value chunks per row
    kbytes = taps * c
    zero_pixel = rh * rw * (c // 4)      # float4 offset of the zero pixel
    written = set()
    tiles = range(plan.tiles) if tile_sample is None else tile_sample
    for tile in tiles:
        b, r = divmod(tile, ty_n * tx_n)
        ty0, tx0 = divmod(r, tx_n)
        oy0, ox0 = ty0 * th, tx0 * tw
        iy0, ix0 = oy0 * stride - pad, ox0 * stride - pad
        cx0, cx1 = max(ix0, 0), min(ix0 + rw, w)
        loaded = set()
        for rr in range(rh):
            iy = iy0 + rr
            if not 0 <= iy < h or cx1 <= cx0:
                continue
            nbytes = (cx1 - cx0) * c * 4
            dst = (rr * rw + (cx0 - ix0)) * c * 4
            src = ((b * h + iy) * w + cx0) * c * 4
            assert dst % 16 == 0 and src % 16 == 0 and nbytes % 16 == 0
            assert 0 <= dst and dst + nbytes <= region
            assert 0 <= src and src + nbytes <= n * h * w * c * 4
            loaded.update((rr, x - ix0) for x in range(cx0, cx1))
        for q in range(th * tw):
            ty, tx = divmod(q, tw)
            oy, ox = oy0 + ty, ox0 + tx
            if oy >= oh or ox >= ow:
                continue
            row = (b * oh + oy) * ow + ox
            off = [zero_pixel] * 32
            for t in range(taps):
                ky, kx = divmod(t, k)
                ry, rx = ty * stride + ky * dil, tx * stride + kx * dil
                assert 0 <= ry < rh and 0 <= rx < rw
                if 0 <= iy0 + ry < h and 0 <= ix0 + rx < w:
                    assert (ry, rx) in loaded
                    off[t] = (ry * rw + rx) * (c // 4)
            if not full:
                continue
            for chunk in range(kc):
                t, ci = divmod(chunk, cc)
                base4 = off[t] + 4 * ci
                for j in range(4):
                    pos = base4 + (j ^ ((ci >> 1) & 3))
                    assert 0 <= pos < (rh * rw + 1) * (c // 4)
                    if off[t] != zero_pixel:
                        pix, part = divmod(pos, c // 4)
                        assert part // 4 == ci and (part % 4) ^ ((ci >> 1) & 3) == j
                store = row * kbytes + 16 * chunk
                assert 0 <= store and store + 16 <= n * oh * ow * kbytes
                assert (row, chunk) not in written
                written.add((row, chunk))
    if full and tile_sample is None:
        assert len(written) == n * oh * ow * kc


CASES = [(1, 8, 8, 256, 3, 1, 1, 1), (2, 9, 7, 128, 3, 2, 1, 1), (1, 10, 10, 64, 3, 1, 2, 2),
         (1, 12, 12, 96, 3, 1, 1, 1), (1, 3, 3, 256, 3, 1, 0, 1), (2, 20, 13, 16, 3, 1, 1, 1),
         (1, 9, 9, 48, 5, 1, 2, 1), (1, 7, 7, 32, 3, 3, 3, 2), (1, 40, 40, 256, 3, 1, 1, 1),
         (1, 36, 36, 512, 3, 1, 1, 1)]


@pytest.mark.parametrize("n,h,w,c,k,stride,pad,dil", CASES)
def test_tiled_gather_plan_covers_every_code_once(n, h, w, c, k, stride, pad, dil):
    import rotated_int8_quantized_b200 as cr
    plan = cr.conv2d_gather_plan((n, h, w, c), k, k, stride, pad, dil, SMS)
    assert plan.tiled == 1
    check_plan(n, h, w, c, k, stride, pad, dil, plan)


@pytest.mark.parametrize("h,c", [(128, 512), (256, 256), (512, 128)])
def test_tiled_gather_plan_vae_shapes(h, c):
    import rotated_int8_quantized_b200 as cr
    plan = cr.conv2d_gather_plan((1, h, h, c), 3, 3, 1, 1, 1, SMS)
    assert plan.tiled == 1 and plan.tiles >= SMS
    # whole rows per warp (16 quantising warps) at these sizes
    assert (plan.th * plan.tw) % 16 == 0
    check_plan(1, h, h, c, 3, 1, 1, 1, plan, full=False)
    tx_n = -(-h // plan.tw)
    check_plan(1, h, h, c, 3, 1, 1, 1, plan, tile_sample=[0, 1, tx_n - 1, tx_n, plan.tiles // 2, plan.tiles - 1])


def test_untiled_and_rejected_plans():
    import rotated_int8_quantized_b200 as cr
    assert cr.conv2d_gather_plan((1, 12, 12, 32), 7, 7, 1, 3, 1).tiled == 0      # 49 taps > 32 lanes
    with pytest.raises(cr.ConvrotError):
        cr.conv2d_gather_plan((1, 16, 16, 64), 1, 1)                              # 1x1: one-step gather
    with pytest.raises(cr.ConvrotError):
        cr.conv2d_gather_plan((1, 16, 16, 64), 3, 3, sms=0)


def test_random_geometries_stay_in_bounds():
    # seeded sweep: small images (so every code is modelled) over channel
    # counts, kernel sizes, strides, paddings and dilations
    import rotated_int8_quantized_b200 as cr
    rng = np.random.default_rng(7)
    tried = 0
    while tried < 60:
        k = int(rng.choice([2, 3, 4, 5]))
        stride, dil = int(rng.integers(1, 3)), int(rng.integers(1, 3))
        pad = int(rng.integers(0, k))
        n, h, w = int(rng.integers(1, 3)), int(rng.integers(k, 14)), int(rng.integers(k, 14))
        c = int(rng.choice([16, 32, 48, 64, 128, 256, 512]))
        if out_size(h, k, stride, pad, dil) < 1 or out_size(w, k, stride, pad, dil) < 1:
            continue
        plan = cr.conv2d_gather_plan((n, h, w, c), k, k, stride, pad, dil, int(rng.choice([1, 8, 148])))
        if plan.tiled == 0:
            # only when not even one output pixel's region fits a buffer
            r1 = (k - 1) * dil + 1
            assert (r1 * r1 + 1) * c * 4 + r1 * r1 * 4 > SMEM_TWO_BUFFERS // 2
            continue
        check_plan(n, h, w, c, k, stride, pad, dil, plan)
        tried += 1
