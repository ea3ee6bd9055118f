"""The GEMM launch plan (host arithmetic, no GPU): every (job, tile, K block)
of a product is processed by exactly one CTA, and each plan fits the SM.

The coverage model restates, in plain Python, the order in which a CTA takes
its work (as the header documents for convrot_gemm_plan): whole tiles in
full waves, a piece of the split tail, then a contiguous range of stream-K
units.
"""
import collections
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

SMS = 148
SMEM_PER_CTA = 227 * 1024


def covered_units(p):
    """(job, tile, kb) -> how many CTAs process it."""
    seen = collections.Counter()
    for c in range(p.grid):
        wave = 0
        while wave < p.full_waves and wave * p.grid + c < p.full_tiles:
            tile = wave * p.grid + c
            for kb in range(p.kbpt[0]):
                seen[(0, tile, kb)] += 1
            wave += 1
        if p.split_ways > 1 and c < p.split_pieces:
            slot, piece = divmod(c, p.split_ways)
            kbpt = p.kbpt[0]
            for kb in range(piece * kbpt // p.split_ways, (piece + 1) * kbpt // p.split_ways):
                seen[(0, p.full_tiles + slot, kb)] += 1
        rep = p.rep
        q, r = divmod(c, rep)
        groups = p.grid // rep
        u, u_end = p.tail_units * q // groups, p.tail_units * (q + 1) // groups
        j = 0
        while u < u_end:
            while j + 1 < p.njobs and u >= p.unit0[j + 1]:
                j += 1
            lu = u - p.unit0[j]
            t, kb0 = divmod(lu, p.kbpt[j])
            kb1 = min(kb0 + (u_end - u), p.kbpt[j])
            tile = p.tile_base[j] + t * rep + r
            for kb in range(kb0, kb1):
                seen[(j, tile, kb)] += 1
            u += kb1 - kb0
    return seen


def check(p, m, ns, ks):
    assert p.njobs == len(ns)
    assert p.grid >= 1 and p.grid <= SMS and p.grid % p.rep == 0
    assert 2 <= p.stages <= 8 and p.smem_bytes <= SMEM_PER_CTA
    assert p.tmem_cols <= 512 and p.tmem_cols & (p.tmem_cols - 1) == 0 and p.tmem_cols >= 2 * p.bn
    want = set()
    for j, (n, k) in enumerate(zip(ns, ks)):
        rows_a, rows_b = (n, m) if p.swap else (m, n)
        assert p.tiles_a[j] == -(-rows_a // 128) and p.tiles_b[j] == -(-rows_b // p.bn)
        assert p.kbpt[j] == -(-k // 128)
        for tile in range(p.tiles_a[j] * p.tiles_b[j]):
            for kb in range(p.kbpt[j]):
                want.add((j, tile, kb))
    seen = covered_units(p)
    assert set(seen) == want
    assert max(seen.values()) == 1


QWEN_N = [8192, 1024, 1024, 5120, 25600, 25600, 5120]
QWEN_K = [5120, 5120, 5120, 8192, 5120, 5120, 25600]


@pytest.mark.parametrize("m,n,k", [
    (4, 256, 512), (12, 8192, 5120), (12, 1024, 5120), (17, 5120, 25600), (256, 768, 1024),
    (300, 768, 1024), (400, 5120, 5120), (512, 25600, 5120),                  # a few hundred rows
    (4096, 8192, 5120), (4096, 1024, 5120), (4096, 25600, 5120), (4096, 5120, 25600),
    (8192, 16128, 5376), (32768, 16128, 5376),                                  # A in groups of 16 tiles
    (65536, 256, 2304), (65536, 200, 1024), (10112, 1000, 5376),                # narrow B, ragged
])
def test_single_product_covers_every_block_once(m, n, k):
    import rotated_int8_quantized_b200 as cr
    p = cr.gemm_plan(m, [n], [k], sms=SMS)
    check(p, m, [n], [k])
    if m <= 256:
        assert p.swap == 1
    if m > 512:
        assert p.swap == 0 and p.rep == 1


@pytest.mark.parametrize("m", [1, 12, 100, 256, 257, 400, 512])
def test_batched_layer_covers_every_block_once(m):
    import rotated_int8_quantized_b200 as cr
    p = cr.gemm_plan(m, QWEN_N, QWEN_K, sms=SMS)
    check(p, m, QWEN_N, QWEN_K)
    assert p.full_waves == 0 and p.tail_units == sum(
        (p.tiles_a[j] if p.swap else p.tiles_b[j]) * p.kbpt[j] for j in range(7))


def test_int4_batch_and_other_gpu_sizes():
    import rotated_int8_quantized_b200 as cr
    p = cr.gemm_plan(12, QWEN_N, QWEN_K, w4=True, sms=SMS)
    check(p, 12, QWEN_N, QWEN_K)
    # INT4 weights at any m: the batched stream-K plan up to 512 rows, whole
    # tiles (weights the 256-row B operand) for single products beyond
    for m in (300, 512):
        check(cr.gemm_plan(m, QWEN_N, QWEN_K, w4=True, sms=SMS), m, QWEN_N, QWEN_K)
    for (m, n, k) in ((4096, 8192, 5120), (4096, 5120, 25600), (700, 1000, 1536)):
        p = cr.gemm_plan(m, [n], [k], w4=True, sms=SMS)
        assert p.swap == 0 and p.bn == 256 and p.stages >= 3
        check(p, m, [n], [k])
    for sms in (1, 7, 64, 132):
        for (m, n, k) in ((12, 5120, 8192), (4096, 8192, 5120), (400, 5120, 5120)):
            check(cr.gemm_plan(m, [n], [k], sms=sms), m, [n], [k])


def test_plan_rejections():
    import rotated_int8_quantized_b200 as cr
    with pytest.raises(cr.ConvrotError):
        cr.gemm_plan(600, [1024, 1024], [512, 512])      # batches are for m <= 512
    with pytest.raises(cr.ConvrotError):
        cr.gemm_plan(12, [1024], [512], sms=0)


def test_random_shapes_cover_every_block_once():
    # seeded sweep over shapes and SM counts (single products and batches),
    # sized so the coverage model stays quick
    import numpy as np
    import rotated_int8_quantized_b200 as cr
    rng = np.random.default_rng(2024)
    for _ in range(150):
        sms = int(rng.choice([1, 3, 8, 37, 132, 148]))
        if rng.random() < 0.5:
            m = int(rng.choice([1, 5, 12, 100, 256, 257, 300, 511, 512, 513, 1000, 3000, 9000]))
            n = int(rng.integers(1, 40)) * 16 * int(rng.choice([1, 4, 16]))
            k = int(rng.integers(1, 64)) * 16 * int(rng.choice([1, 2, 8]))
            check(cr.gemm_plan(m, [n], [k], w4=bool(rng.random() < 0.3), sms=sms), m, [n], [k])
        else:
            m = int(rng.choice([1, 7, 12, 64, 200, 256, 300, 512]))
            count = int(rng.integers(2, 9))
            ns = [int(rng.integers(1, 50)) * 64 for _ in range(count)]
            ks = [int(rng.integers(1, 40)) * 128 for _ in range(count)]
            w4 = bool(rng.random() < 0.3)
            check(cr.gemm_plan(m, ns, ks, w4=w4, sms=sms), m, ns, ks)
