"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bit-exact: the rotated INT8 codes and FP32 scales of weights and
activations, and the INT32 accumulators.  The BF16 output must be within
max|Y - Y_oracle| / max|Y_oracle| <= 1e-2; since both sides evaluate
((float)acc * sx) * sw and round once to BF16, it is in fact compared
bit for bit as well.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

TOL = 1e-2


@pytest.fixture(scope="module")
def cr():
    from rotated_int8_quantized_b200 import build
    build.build()
    import rotated_int8_quantized_b200 as m
    m.load_library()
    return m


def to_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def rel_err(y_bits, ref_bits):
    y = oracle.bf16_bits_to_f64(y_bits)
    r = oracle.bf16_bits_to_f64(ref_bits)
    return float(np.max(np.abs(y - r)) / max(np.max(np.abs(r)), 1e-30))


def gpu_quantize(cr, a_bits):
    """Rotate+quantise rows on the GPU with the weight entry point."""
    w = cr.quantize_weight(from_bits(a_bits))
    torch.cuda.synchronize()
    return w, w.q.cpu().numpy(), w.scale.cpu().numpy()


# ---------------------------------------------------------------- K3 / K1
def test_weight_quant_tiny_bit_exact(cr):
    lin = synth.tiny()[0]
    w_bits = lin.w_np()
    _, q, s = gpu_quantize(cr, w_bits)
    q_ref, s_ref = oracle.rotate_quantize(w_bits)
    assert np.array_equal(q, q_ref)
    assert np.array_equal(s.view(np.uint32), s_ref.view(np.uint32))


# m and k span every launch shape of the kernel: rows split over a cluster of
# up to 8 CTAs (few rows, or rows of more than 32 groups), one CTA per row
# (>= 148 rows), one or several groups per slot and a ragged last slot, and
# the longest rows the API accepts; short rows of a tall matrix packed 16 or 8
# to a CTA (a ragged last CTA included); tall matrices of 16 to 128 groups
@pytest.mark.parametrize("m,k", [(1, 256), (4, 512), (3, 768), (17, 5120), (2, 8448), (3, 16384),
                                 (2, 24576), (5, 25600), (2, 38912), (2, 40960), (2, 65536),
                                 (150, 512), (160, 8448), (148, 25600), (149, 40960), (200, 65536),
                                 (3, 133120), (150, 133120), (1200, 256), (1187, 256), (1190, 512),
                                 (2048, 512),
                                 # tall matrices of long rows: persistent CTAs walking the rows
                                 (300, 4096), (597, 5120), (1000, 8192), (320, 6144), (400, 25600),
                                 (350, 32768)])
def test_act_quant_bit_exact(cr, m, k):
    cs = synth.outlier_scale_fraction(synth.stream_key(m * 7 + k, 2), k, 0.01, 30.0)
    x_bits = synth.draw_np(synth.stream_key(m * 7 + k, 0), m, k, 1.0, cs)
    xq = torch.empty((m, k), dtype=torch.int8, device="cuda")
    sx = torch.empty((m,), dtype=torch.float32, device="cuda")
    cr.convrot_quantize_act(from_bits(x_bits), xq, sx)
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.rotate_quantize(x_bits)
    assert np.array_equal(xq.cpu().numpy(), q_ref)
    assert np.array_equal(sx.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


def test_act_quant_zero_row_and_one_hot(cr):
    x = np.zeros((3, 512), dtype=np.float32)
    x[1, 7] = -3.0
    x[2, :] = 0.25
    bits = synth.f32_to_bf16_bits(x)
    xq = torch.empty((3, 512), dtype=torch.int8, device="cuda")
    sx = torch.empty((3,), dtype=torch.float32, device="cuda")
    cr.convrot_quantize_act(from_bits(bits), xq, sx)
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.rotate_quantize(bits)
    assert np.array_equal(xq.cpu().numpy(), q_ref)
    assert np.array_equal(sx.cpu().numpy(), s_ref)
    assert sx[0].item() == 0 and int(xq[0].abs().max()) == 0


def test_act_quant_exact_ties(cr):
    # rows whose rotated values fall exactly on half-integers of y / s: group 0
    # is the constant 127 * 2^(p-4) (rotates to (127 * 2^p, 0, ...), so
    # s = 2^p exactly), groups 1.. are constants c * 2^(p-4) (rotating to
    # (c * 2^p, 0, ...)), so y / s = c exactly; ties must go to even
    ties = [2.5, 3.5, -4.5, 0.5, -126.5, 1.5, -0.5, 6.5]
    rows = []
    for p in (0, -3, 5, -10):
        row = np.zeros(256 * (1 + len(ties)), dtype=np.float32)
        row[:256] = 127.0 * 2.0 ** (p - 4)
        for g, c in enumerate(ties):
            row[256 * (g + 1): 256 * (g + 2)] = c * 2.0 ** (p - 4)
        rows.append(row)
    x = np.stack(rows)
    bits = synth.f32_to_bf16_bits(x)
    assert np.array_equal(synth.bf16_bits_to_f32(bits), x)
    m, k = x.shape
    xq = torch.empty((m, k), dtype=torch.int8, device="cuda")
    sx = torch.empty((m,), dtype=torch.float32, device="cuda")
    cr.convrot_quantize_act(from_bits(bits), xq, sx)
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.rotate_quantize(bits)
    got = xq.cpu().numpy()
    assert np.array_equal(got, q_ref)
    assert np.array_equal(sx.cpu().numpy(), s_ref)
    assert list(got[0, 256::256]) == [2, 4, -4, 0, -126, 2, 0, 6]


def test_act_quant_subnormal_scale(cr):
    # rows so small that s = amax / 127 is subnormal in FP32 (amax < 127 * 2^-126):
    # the codes still follow q = clamp(rne(fl(y / s))) exactly
    m, k = 6, 512
    x = np.random.default_rng(5).standard_normal((m, k)).astype(np.float32)
    x *= np.float32(2.0 ** -125) * np.array([1, 2, 4, 0.5, 8, 16], dtype=np.float32)[:, None]
    bits = synth.f32_to_bf16_bits(x)
    xq = torch.empty((m, k), dtype=torch.int8, device="cuda")
    sx = torch.empty((m,), dtype=torch.float32, device="cuda")
    cr.convrot_quantize_act(from_bits(bits), xq, sx)
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.rotate_quantize(bits)
    assert np.all(s_ref < np.float32(1.17549435e-38)) and np.all(s_ref > 0)
    assert np.array_equal(xq.cpu().numpy(), q_ref)
    assert np.array_equal(sx.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


# ---------------------------------------------------------------- K2
def _gemm_case(cr, m, n, k, seed):
    cs = synth.outlier_scale_fraction(synth.stream_key(seed, 2), k, 0.01, 30.0)
    x_bits = synth.draw_np(synth.stream_key(seed, 0), m, k, 1.0, cs)
    w_bits = synth.draw_np(synth.stream_key(seed, 1), n, k, synth.W_SIGMA)
    wq_ref, sw_ref = oracle.rotate_quantize(w_bits)
    ref = oracle.linear_int8(x_bits, wq_ref, sw_ref)
    w, wq, sw = gpu_quantize(cr, w_bits)
    assert np.array_equal(wq, wq_ref) and np.array_equal(sw, sw_ref)
    return x_bits, w, ref


GEMM_SHAPES = [
    (4, 256, 512),      # tiny: swap path, one 16-row activation tile, 2 weight tiles
    (1, 384, 256),      # single token, one K block pair
    (12, 1024, 5120),   # decode shape, stream-K across many CTAs
    (17, 1000, 1280),   # ragged weight tile, activation tile of 32
    (100, 640, 2560),   # swap with bn = 112
    (256, 512, 768),    # largest swap case, bn = 256
    (257, 512, 512),    # stream-K with activations = A: 3 tiles, the last of 1 row
    (400, 640, 5120),   # stream-K, 4 x 3 tiles, many K blocks per CTA
    (512, 1000, 2560),  # stream-K, 4 full activation tiles, ragged weight tile
    (513, 512, 512),    # smallest large-M case, ragged activation tile
    (640, 1000, 1536),  # non-swap, ragged weight tile (1000 % 256), one partial wave
    (9500, 500, 1024),  # 150 tiles: one full wave, 2 tail tiles split in 2 K ranges
    (5083, 1000, 4096), # 160 tiles: 12 tail tiles split in 6 K ranges, ragged both ways
]


@pytest.mark.parametrize("m,n,k", GEMM_SHAPES)
def test_gemm_acc_and_y_bit_exact(cr, m, n, k):
    x_bits, w, ref = _gemm_case(cr, m, n, k, seed=m * 131 + n * 7 + k)
    xq = torch.from_numpy(ref["xq"]).cuda()
    sx = torch.from_numpy(ref["sx"]).cuda()
    acc = torch.empty((m, n), dtype=torch.int32, device="cuda")
    y = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    ws = cr.make_workspace(m, w, linear=False)
    cr.convrot_gemm_i8(xq, sx, w, y, acc, ws)
    cr.convrot_device_status()
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    yb = to_bits(y)
    assert rel_err(yb, ref["y"]) <= TOL
    assert np.array_equal(yb, ref["y"])
    assert int(ws.count_nonzero()) == 0      # workspace returned to zero


@pytest.mark.parametrize("m,n,k", [(32, 1024, 5120), (64, 512, 768), (400, 640, 5120), (4096, 1024, 5120)])
def test_int32_accumulators_match_a_vendor_int8_gemm(cr, m, n, k):
    # a second opinion, run not read: a library INT8 GEMM (torch._int_mm,
    # cuBLASLt) on the same INT8 operands; both INT32 products are exact
    if not hasattr(torch, "_int_mm"):
        pytest.skip("torch._int_mm unavailable")
    gen = torch.Generator(device="cuda").manual_seed(m * 7 + n * 3 + k)
    xq = torch.randint(-127, 128, (m, k), generator=gen, device="cuda", dtype=torch.int32).to(torch.int8)
    wq = torch.randint(-127, 128, (n, k), generator=gen, device="cuda", dtype=torch.int32).to(torch.int8)
    sx = torch.ones(m, dtype=torch.float32, device="cuda")
    sw = torch.ones(n, dtype=torch.float32, device="cuda")
    w = cr.convrot_weight_init(wq, sw)
    acc = torch.empty((m, n), dtype=torch.int32, device="cuda")
    ws = cr.make_workspace(m, w, linear=False)
    cr.convrot_gemm_i8(xq, sx, w, None, acc, ws)
    cr.convrot_device_status()
    try:
        ref = torch._int_mm(xq, wq.t())
    except RuntimeError as e:
        pytest.skip("torch._int_mm does not take this shape here: %s" % e)
    torch.cuda.synchronize()
    assert torch.equal(acc, ref)


@pytest.mark.parametrize("m,n,k", [(4, 256, 512), (12, 1024, 5120), (300, 768, 1024)])
def test_linear_end_to_end(cr, m, n, k):
    x_bits, w, ref = _gemm_case(cr, m, n, k, seed=m + n + k)
    ws = cr.make_workspace(m, w)
    x = from_bits(x_bits)
    y1 = cr.linear_int8(x, w, ws)
    y2 = cr.linear_int8(x, w, ws)     # second call reuses the self-cleaned workspace
    cr.convrot_device_status()
    assert rel_err(to_bits(y1), ref["y"]) <= TOL
    assert np.array_equal(to_bits(y1), ref["y"])
    assert np.array_equal(to_bits(y2), ref["y"])


def test_tiny_config_layer(cr):
    lin = synth.tiny()[0]
    x_bits, w_bits = lin.x_np(), lin.w_np()
    wq_ref, sw_ref = oracle.rotate_quantize(w_bits)
    ref = oracle.linear_int8(x_bits, wq_ref, sw_ref)
    w = cr.quantize_weight(from_bits(w_bits))
    y = cr.linear_int8(from_bits(x_bits), w, cr.make_workspace(lin.m, w))
    cr.convrot_device_status()
    assert np.array_equal(to_bits(y), ref["y"])


def test_errors_are_statuses(cr):
    w = cr.quantize_weight(torch.zeros((256, 512), dtype=torch.bfloat16, device="cuda"))
    x = torch.zeros((4, 512), dtype=torch.bfloat16, device="cuda")
    small = torch.zeros(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(cr.ConvrotError) as e:
        cr.linear_int8(x, w, small)
    assert e.value.status == 5
    with pytest.raises(cr.ConvrotError) as e:
        cr.convrot_quantize_act(torch.zeros((4, 300), dtype=torch.bfloat16, device="cuda"),
                                torch.empty((4, 300), dtype=torch.int8, device="cuda"),
                                torch.empty(4, dtype=torch.float32, device="cuda"))
    assert e.value.status == 3
    cr.convrot_device_status()


# ---------------------------------------------------------------- full sizes, sampled
def _sampled_layer_check(cr, lin, rows_w, rows_x=None):
    """Whole-size weights drawn on the GPU, quantised there; the oracle
    recomputes the sampled weight rows (and activation rows) from the
    counter-based generator and checks codes, scales and outputs."""
    dev = "cuda"
    w_bf = lin.w_torch(dev)
    w = cr.quantize_weight(w_bf)
    x = lin.x_torch(dev)
    ws = cr.make_workspace(lin.m, w)
    y = cr.linear_int8(x, w, ws)
    acc = torch.empty((lin.m, lin.n), dtype=torch.int32, device=dev)
    xq = torch.empty((lin.m, lin.k), dtype=torch.int8, device=dev)
    sx = torch.empty((lin.m,), dtype=torch.float32, device=dev)
    cr.convrot_quantize_act(x, xq, sx)
    cr.convrot_gemm_i8(xq, sx, w, None, acc, cr.make_workspace(lin.m, w, linear=False))
    cr.convrot_device_status()
    del w_bf
    w_rows = lin.w_rows_np(rows_w)
    assert np.array_equal(to_bits(lin.w_torch(dev)[torch.as_tensor(rows_w, device=dev)]), w_rows)
    wq_ref, sw_ref = oracle.rotate_quantize(w_rows)
    assert np.array_equal(w.q[torch.as_tensor(rows_w, device=dev)].cpu().numpy(), wq_ref)
    assert np.array_equal(w.scale[torch.as_tensor(rows_w, device=dev)].cpu().numpy(), sw_ref)
    rows_x = np.arange(lin.m) if rows_x is None else np.asarray(rows_x)
    x_rows = lin.x_rows_np(rows_x)
    ref = oracle.linear_int8(x_rows, wq_ref, sw_ref)
    rx = torch.as_tensor(rows_x, device=dev)
    assert np.array_equal(xq[rx].cpu().numpy(), ref["xq"])
    assert np.array_equal(sx[rx].cpu().numpy(), ref["sx"])
    rw = torch.as_tensor(rows_w, device=dev)
    assert np.array_equal(acc[rx][:, rw].cpu().numpy(), ref["acc"])
    yb = to_bits(y[rx][:, rw])
    assert rel_err(yb, ref["y"]) <= TOL
    assert np.array_equal(yb, ref["y"])


@pytest.mark.parametrize("idx", range(7))
def test_qwen_decode_full_size_sampled(cr, idx):
    lin = synth.qwen_layer(12)[idx]
    rng = np.random.default_rng(idx)
    rows = np.unique(np.concatenate([[0, lin.n - 1], rng.integers(0, lin.n, 30)]))
    _sampled_layer_check(cr, lin, rows)


@pytest.mark.parametrize("idx", [0, 6])
def test_qwen_prefill_full_size_sampled(cr, idx):
    lin = synth.qwen_layer(4096)[idx]
    rng = np.random.default_rng(100 + idx)
    rows_w = np.unique(np.concatenate([[0, lin.n - 1], rng.integers(0, lin.n, 14)]))
    rows_x = np.unique(np.concatenate([[0, lin.m - 1], rng.integers(0, lin.m, 14)]))
    _sampled_layer_check(cr, lin, rows_w, rows_x)


def test_minimax_qkv_sampled(cr):
    lin = synth.minimax_qkv(8192)[0]
    rng = np.random.default_rng(4)
    rows_w = np.unique(np.concatenate([[0, lin.n - 1], rng.integers(0, lin.n, 14)]))
    rows_x = np.unique(np.concatenate([[0, lin.m - 1], rng.integers(0, lin.m, 14)]))
    _sampled_layer_check(cr, lin, rows_w, rows_x)


def test_minimax_qkv_m32768_sampled(cr):
    # 176 MB of INT8 activations: tiles are taken in groups of 16 A tiles
    lin = synth.minimax_qkv(32768)[0]
    rng = np.random.default_rng(5)
    rows_w = np.unique(np.concatenate([[0, lin.n - 1], rng.integers(0, lin.n, 10)]))
    rows_x = np.unique(np.concatenate([[0, 2047, 2048, lin.m - 1], rng.integers(0, lin.m, 10)]))
    _sampled_layer_check(cr, lin, rows_w, rows_x)


@pytest.mark.parametrize("n", [256, 200])
def test_narrow_n_large_m_sampled(cr, n):
    # 64 MB of INT8 activations against at most 256 weight rows: 128-row B
    # tiles (two per A tile, the second ragged for n = 200), A in groups of 16
    lin = synth.Linear("narrow", 65536, 1024, n, 31 + n)
    rng = np.random.default_rng(n)
    rows_w = np.unique(np.concatenate([[0, 127, 128, n - 1], rng.integers(0, n, 8)]))
    rows_x = np.unique(np.concatenate([[0, 127, 128, 2047, 2048, lin.m - 1], rng.integers(0, lin.m, 10)]))
    _sampled_layer_check(cr, lin, rows_w, rows_x)


def test_grouped_tile_order_ragged_sampled(cr):
    # 79 A tiles = 4 groups of 16 + a ragged group of 15, 4 B tiles (the last
    # ragged), 316 tiles = 2 full waves + 20 tail tiles split along K
    k = 5376
    lin = synth.Linear("grouped", 10000, k, 1000, 77, synth.student_t3_scale(synth.stream_key(77, 2), k))
    rng = np.random.default_rng(77)
    rows_w = np.unique(np.concatenate([[0, 255, 256, 767, 768, lin.n - 1], rng.integers(0, lin.n, 8)]))
    rows_x = np.unique(np.concatenate([[0, 2047, 2048, 8191, 8192, 9983, 9984, lin.m - 1],
                                       rng.integers(0, lin.m, 8)]))
    _sampled_layer_check(cr, lin, rows_w, rows_x)


# ---------------------------------------------------------------- batched layer entry point
# (m, [(k, n), ...]): fewer K blocks than SMs (grid < 148), ragged N, many
# jobs, long rows split over a cluster of up to 8 CTAs in the prologue, many
# K blocks per SM, and m > 256, where the GEMMs run one after another
BATCH_CASES = [
    (1, [(512, 256), (768, 384), (256, 1000)]),
    (5, [(1280, 640), (512, 128), (2560, 1024), (768, 130)]),
    (3, [(5120, 2048), (2560, 1024)]),
    (5, [(5120, 8192), (2560, 512)]),       # many K blocks per SM
    (17, [(1024, 384), (1024, 384)]),
    (32, [(1024, 2048), (3072, 512), (256, 1280)]),
    (24, [(25600, 1024)]),
    (100, [(512, 512), (1536, 256), (256, 640)]),
    (64, [(25600, 640)]),
    (300, [(768, 512), (512, 1000)]),
    (512, [(5120, 1024), (2560, 640), (512, 384)]),
    (600, [(768, 512), (512, 1000)]),
    # several inputs of the same row length rotated by one persistent launch
    (400, [(4096, 640), (4096, 384), (5120, 512), (4096, 256)]),
    (700, [(4096, 256), (4096, 384)]),
]


@pytest.mark.parametrize("m,shapes", BATCH_CASES)
def test_batch_matches_oracle_and_single_calls(cr, m, shapes):
    xs, ws_, ys, refs, singles = [], [], [], [], []
    for idx, (k, n) in enumerate(shapes):
        x_bits, w, ref = _gemm_case(cr, m, n, k, seed=1000 + 37 * idx + m)
        x = from_bits(x_bits)
        xs.append(x)
        ws_.append(w)
        ys.append(torch.empty((m, n), dtype=torch.bfloat16, device="cuda"))
        refs.append(ref)
        singles.append(cr.linear_int8(x, w, cr.make_workspace(m, w)))
    batch = cr.LinearBatch(xs, ws_, ys)
    batch()
    cr.convrot_device_status()
    for y, ref, single in zip(ys, refs, singles):
        assert np.array_equal(to_bits(y), ref["y"])
        assert np.array_equal(to_bits(y), to_bits(single))
    for y in ys:
        y.zero_()
    batch()                            # the workspace returned to zero: same result again
    cr.convrot_device_status()
    for y, ref in zip(ys, refs):
        assert np.array_equal(to_bits(y), ref["y"])
    if m <= 256:
        # the batched GEMM alone, INT32 accumulators out
        xqs = [torch.from_numpy(r["xq"]).cuda() for r in refs]
        sxs = [torch.from_numpy(r["sx"]).cuda() for r in refs]
        accs = [torch.empty((m, w.n), dtype=torch.int32, device="cuda") for w in ws_]
        yg = [torch.empty((m, w.n), dtype=torch.bfloat16, device="cuda") for w in ws_]
        gb = cr.GemmBatch(xqs, sxs, ws_, yg, accs)
        gb()
        cr.convrot_device_status()
        for acc, y, ref in zip(accs, yg, refs):
            assert np.array_equal(acc.cpu().numpy(), ref["acc"])
            assert np.array_equal(to_bits(y), ref["y"])
        assert int(gb.ws.count_nonzero()) == 0


def test_batch_rejects_output_overlapping_an_input(cr):
    w = cr.quantize_weight(torch.zeros((256, 512), dtype=torch.bfloat16, device="cuda"))
    buf = torch.zeros((4, 512), dtype=torch.bfloat16, device="cuda")
    y_alias = buf.view(-1)[: 4 * 256].view(4, 256)      # output inside the input's memory
    ws = torch.zeros(1 << 22, dtype=torch.uint8, device="cuda")
    with pytest.raises(cr.ConvrotError) as e:
        cr.convrot_linear_int8_batch([buf], [w], [y_alias], ws)
    assert e.value.status == 1


def test_batch_qwen_decode_layer_full_size(cr):
    lins = synth.qwen_layer(12)
    dev = "cuda"
    weights, xs, ys, singles = [], [], [], []
    for lin in lins:
        w_bf = lin.w_torch(dev)
        w = cr.quantize_weight(w_bf)
        del w_bf
        x = lin.x_torch(dev)
        weights.append(w)
        xs.append(x)
        ys.append(torch.empty((lin.m, lin.n), dtype=torch.bfloat16, device=dev))
        singles.append(cr.linear_int8(x, w, cr.make_workspace(lin.m, w)))
    batch = cr.LinearBatch(xs, weights, ys)
    batch()
    batch()
    cr.convrot_device_status()
    for lin, w, y, single in zip(lins, weights, ys, singles):
        assert torch.equal(y.view(torch.int16), single.view(torch.int16))
        rows = np.array([0, 1, lin.n // 2, lin.n - 1])
        wq_ref, sw_ref = oracle.rotate_quantize(lin.w_rows_np(rows))
        ref = oracle.linear_int8(lin.x_np(), wq_ref, sw_ref)
        assert np.array_equal(to_bits(y[:, torch.as_tensor(rows, device=dev)]), ref["y"])


# ---------------------------------------------------------------- bias, shared inputs
# (m, [(k, n), ...]): jobs with equal k read the same input tensor (one
# prologue for them); every other job has a BF16 bias.  Decode orientation,
# the stream-K large-M orientation (m <= 512), and per-job launches (m > 512)
BIAS_CASES = [
    (12, [(5120, 1024), (5120, 768), (2560, 512)]),
    (300, [(768, 512), (768, 1000), (512, 384)]),
    (700, [(512, 640), (512, 384), (1024, 256)]),
]


def _bias_bits(seed, n):
    return synth.draw_np(synth.stream_key(seed, 5), 1, n, 1.0).reshape(n)


@pytest.mark.parametrize("m,shapes", BIAS_CASES)
def test_batch_bias_and_shared_inputs(cr, m, shapes):
    x_by_k, xs, ws_, ys, biases, refs = {}, [], [], [], [], []
    for idx, (k, n) in enumerate(shapes):
        seed = 4000 + 17 * idx + m
        if k not in x_by_k:
            cs = synth.outlier_scale_fraction(synth.stream_key(seed, 2), k, 0.01, 30.0)
            x_by_k[k] = synth.draw_np(synth.stream_key(seed, 0), m, k, 1.0, cs)
        x_bits = x_by_k[k]
        w_bits = synth.draw_np(synth.stream_key(seed, 1), n, k, synth.W_SIGMA)
        wq_ref, sw_ref = oracle.rotate_quantize(w_bits)
        b_bits = _bias_bits(seed, n) if idx % 2 == 0 else None
        refs.append(oracle.linear_int8(x_bits, wq_ref, sw_ref, bias=b_bits))
        ws_.append(cr.quantize_weight(from_bits(w_bits)))
        ys.append(torch.empty((m, n), dtype=torch.bfloat16, device="cuda"))
        biases.append(None if b_bits is None else from_bits(b_bits))
    x_dev = {k: from_bits(v) for k, v in x_by_k.items()}
    xs = [x_dev[k] for k, _ in shapes]
    batch = cr.LinearBatch(xs, ws_, ys, biases=biases)
    batch()
    batch()                      # the workspace is left reusable
    cr.convrot_device_status()
    for y, ref in zip(ys, refs):
        yb = to_bits(y)
        assert rel_err(yb, ref["y"]) <= TOL
        assert np.array_equal(yb, ref["y"])


@pytest.mark.parametrize("m", [12, 400])
def test_gemm_batch_bias(cr, m):
    shapes = [(1024, 640), (2048, 256)]
    xqs, sxs, ws_, ys, biases, refs = [], [], [], [], [], []
    for idx, (k, n) in enumerate(shapes):
        x_bits, w, ref = _gemm_case(cr, m, n, k, seed=5000 + idx + m)
        b_bits = _bias_bits(5000 + idx, n)
        xqs.append(torch.from_numpy(ref["xq"]).cuda())
        sxs.append(torch.from_numpy(ref["sx"]).cuda())
        ws_.append(w)
        ys.append(torch.empty((m, n), dtype=torch.bfloat16, device="cuda"))
        biases.append(from_bits(b_bits))
        refs.append(oracle.dequant_bf16(ref["acc"], ref["sx"], w.scale.cpu().numpy(), b_bits))
    gb = cr.GemmBatch(xqs, sxs, ws_, ys, biases=biases)
    gb()
    cr.convrot_device_status()
    for y, ref in zip(ys, refs):
        assert np.array_equal(to_bits(y), ref)


# ---------------------------------------------------------------- --dynamic-convrot groups
# (m, k, group): groups below 256, rows that end in a partial 256-element
# chunk, rows shorter than 256, decode-sized launches (rows over a cluster)
# and one-CTA-per-row launches, the FP64 division by sqrt(G) for G = 32, 128
DYN_ACT = [(3, 640, 128), (150, 640, 128), (4, 48, 16), (160, 48, 16), (2, 5440, 64), (150, 5440, 64),
           (5, 1376, 32), (149, 1376, 32), (3, 1024, 128), (2, 25600, 128), (148, 8192, 32),
           (1300, 384, 128), (1250, 48, 16), (1203, 160, 32)]


@pytest.mark.parametrize("m,k,group", DYN_ACT)
def test_act_quant_dynamic_group_bit_exact(cr, m, k, group):
    assert cr.convrot_dynamic_group(k) == group or k % 256 == 0
    cs = synth.outlier_scale_fraction(synth.stream_key(m + k + group, 2), k, 0.01, 30.0)
    x_bits = synth.draw_np(synth.stream_key(m + k + group, 0), m, k, 1.0, cs)
    xq = torch.empty((m, k), dtype=torch.int8, device="cuda")
    sx = torch.empty((m,), dtype=torch.float32, device="cuda")
    cr.convrot_quantize_act(from_bits(x_bits), xq, sx, group=group)
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.rotate_quantize(x_bits, group)
    assert np.array_equal(xq.cpu().numpy(), q_ref)
    assert np.array_equal(sx.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


# (m, n, k): K not a multiple of the 128-byte K block (the last block reads
# zeros past k), through both GEMM orientations and the batched layer
DYN_LINEAR = [(12, 384, 640), (4, 256, 48), (300, 512, 640), (700, 640, 5440), (12, 1000, 1376)]


@pytest.mark.parametrize("m,n,k", DYN_LINEAR)
def test_linear_dynamic_group(cr, m, n, k):
    group = cr.convrot_dynamic_group(k)
    seed = 7000 + m + n + k
    cs = synth.outlier_scale_fraction(synth.stream_key(seed, 2), k, 0.01, 30.0)
    x_bits = synth.draw_np(synth.stream_key(seed, 0), m, k, 1.0, cs)
    w_bits = synth.draw_np(synth.stream_key(seed, 1), n, k, synth.W_SIGMA)
    wq_ref, sw_ref = oracle.rotate_quantize(w_bits, group)
    ref = oracle.linear_int8(x_bits, wq_ref, sw_ref, group=group)
    w = cr.quantize_weight(from_bits(w_bits), dynamic=True)
    assert w.group == group
    assert np.array_equal(w.q.cpu().numpy(), wq_ref) and np.array_equal(w.scale.cpu().numpy(), sw_ref)
    y = cr.linear_int8(from_bits(x_bits), w, cr.make_workspace(m, w))
    acc = torch.empty((m, n), dtype=torch.int32, device="cuda")
    cr.convrot_gemm_i8(torch.from_numpy(ref["xq"]).cuda(), torch.from_numpy(ref["sx"]).cuda(), w, None, acc,
                       cr.make_workspace(m, w, linear=False))
    ys = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    cr.LinearBatch([from_bits(x_bits)], [w], [ys])()
    cr.convrot_device_status()
    assert np.array_equal(acc.cpu().numpy(), ref["acc"])
    assert np.array_equal(to_bits(y), ref["y"])
    assert np.array_equal(to_bits(ys), ref["y"])


# ---------------------------------------------------------------- tensor-wise INT8 (embedding table)
@pytest.mark.parametrize("vocab,dim", [(4096, 5120), (3, 16), (1000, 48)])
def test_tensor_quant_bit_exact(cr, vocab, dim):
    w_bits = synth.draw_np(synth.stream_key(vocab + dim, 7), vocab, dim, 0.05, None)
    q = torch.empty((vocab, dim), dtype=torch.int8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    cr.convrot_quantize_tensor(from_bits(w_bits), q, s)
    torch.cuda.synchronize()
    q_ref, s_ref, _ = oracle.quantize_tensor(w_bits)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert s.cpu().numpy().view(np.uint32)[0] == np.float32(s_ref).view(np.uint32)


def test_tensor_quant_ties_and_zero(cr):
    p = -6
    row = np.array([127.0, 2.5, -3.5, 0.5, -126.5, 1.5, 6.5, -0.5] * 4, np.float32) * 2.0 ** p
    bits = synth.f32_to_bf16_bits(np.tile(row, (3, 1)))
    q = torch.empty((3, 32), dtype=torch.int8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    cr.convrot_quantize_tensor(from_bits(bits), q, s)
    torch.cuda.synchronize()
    q_ref, s_ref, ties = oracle.quantize_tensor(bits)
    assert ties > 0 and np.array_equal(q.cpu().numpy(), q_ref) and s.item() == s_ref == 2.0 ** p
    qz = torch.full((2, 16), 5, dtype=torch.int8, device="cuda")
    cr.convrot_quantize_tensor(torch.zeros((2, 16), dtype=torch.bfloat16, device="cuda"), qz, s)
    torch.cuda.synchronize()
    assert s.item() == 0 and int(qz.abs().max()) == 0


def test_embed_lookup_matches_oracle(cr):
    vocab, dim = 2000, 1024
    w_bits = synth.draw_np(synth.stream_key(99, 7), vocab, dim, 0.05, None)
    q = torch.empty((vocab, dim), dtype=torch.int8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    cr.convrot_quantize_tensor(from_bits(w_bits), q, s)
    rng = np.random.default_rng(3)
    tokens = np.concatenate([[0, vocab - 1, 5, 5], rng.integers(0, vocab, 60)]).astype(np.int32)
    out = torch.empty((tokens.size, dim), dtype=torch.bfloat16, device="cuda")
    cr.convrot_embed_lookup(torch.from_numpy(tokens).cuda(), q, s, out)
    cr.convrot_device_status()
    q_ref, s_ref, _ = oracle.quantize_tensor(w_bits)
    assert np.array_equal(to_bits(out), oracle.embed_lookup(tokens, q_ref, s_ref))
    # an id outside the table: zero row, reported by the status word
    bad = torch.tensor([1, vocab, -3], dtype=torch.int32, device="cuda")
    out2 = torch.full((3, dim), 1.0, dtype=torch.bfloat16, device="cuda")
    cr.convrot_embed_lookup(bad, q, s, out2)
    with pytest.raises(cr.ConvrotError) as e:
        cr.convrot_device_status()
    assert e.value.status == 1
    cr.convrot_device_status()           # cleared by the read
    assert np.array_equal(to_bits(out2[:1]), oracle.embed_lookup(np.array([1], np.int32), q_ref, s_ref))
    assert not to_bits(out2[1:]).any()



# ---------------------------------------------------------------- INT4 weights (W4A8)
@pytest.mark.parametrize("n,k,dyn", [(256, 512, False), (1000, 5120, False), (300, 640, True), (150, 25600, False)])
def test_weight4_quant_bit_exact(cr, n, k, dyn):
    w_bits = synth.draw_np(synth.stream_key(n + k, 1), n, k, synth.W_SIGMA)
    w4 = cr.quantize_weight4(from_bits(w_bits), dynamic=dyn)
    torch.cuda.synchronize()
    packed_ref, s_ref = oracle.rotate_quantize4(w_bits, w4.group)
    assert np.array_equal(w4.q.cpu().numpy(), packed_ref)
    assert np.array_equal(w4.scale.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


# (m, [(k, n), ...]): decode sizes, several weights in one launch, a shared
# input, a bias, a ragged weight tile, K not a multiple of 128 (dynamic group)
W4_CASES = [
    (1, [(512, 256)]),
    (12, [(5120, 1024), (5120, 768), (2560, 512)]),
    (4, [(640, 384)]),
    (100, [(1536, 640), (512, 1000)]),
    (256, [(1024, 512)]),
    # activations = A, the INT4 weight unpacked into the 256-row B operand:
    # replicated stream-K (m <= 512), whole tiles with a split tail, ragged
    # tiles both ways, a K not a multiple of 128 (dynamic group)
    (300, [(1024, 512), (768, 384)]),
    (512, [(2560, 640), (2560, 1000)]),
    (700, [(1536, 640), (512, 1000)]),
    (1200, [(5120, 1000), (640, 384)]),
    (9500, [(1024, 500)]),
]


@pytest.mark.parametrize("m,shapes", W4_CASES)
def test_w4a8_linear_bit_exact(cr, m, shapes):
    x_by_k, ws4, ys, biases, refs = {}, [], [], [], []
    for idx, (k, n) in enumerate(shapes):
        seed = 9000 + 13 * idx + m
        group = cr.convrot_dynamic_group(k)
        if k not in x_by_k:
            cs = synth.outlier_scale_fraction(synth.stream_key(seed, 2), k, 0.01, 30.0)
            x_by_k[k] = synth.draw_np(synth.stream_key(seed, 0), m, k, 1.0, cs)
        w_bits = synth.draw_np(synth.stream_key(seed, 1), n, k, synth.W_SIGMA)
        packed, sw = oracle.rotate_quantize4(w_bits, group)
        b_bits = _bias_bits(seed, n) if idx == 1 else None
        refs.append(oracle.linear_w4a8(x_by_k[k], packed, sw, group=group, bias=b_bits))
        ws4.append(cr.quantize_weight4(from_bits(w_bits), dynamic=True))
        ys.append(torch.empty((m, n), dtype=torch.bfloat16, device="cuda"))
        biases.append(None if b_bits is None else from_bits(b_bits))
    x_dev = {k: from_bits(v) for k, v in x_by_k.items()}
    batch = cr.LinearBatchW4([x_dev[k] for k, _ in shapes], ws4, ys, biases=biases)
    batch()
    batch()                      # the GEMM scratch is left reusable
    cr.convrot_device_status()
    for y, ref in zip(ys, refs):
        yb = to_bits(y)
        assert rel_err(yb, ref["y"]) <= TOL
        assert np.array_equal(yb, ref["y"])


@pytest.mark.parametrize("m", [12, 300, 1200])
def test_w4a8_largest_sums_at_max_k(cr, m):
    """The largest products the W4A8 path can accumulate, at the largest K
    the API accepts: one unit spike per 256-group rotates to a constant
    group (the first Hadamard row is all ones), so every activation code is
    127 and every weight code +7 or -7, and each output sums K products of
    +-889.  The GEMM's tensor cores see the unpacked weights as 16 x code,
    so their INT32 sums reach 16 * 889 * 133120 = 1.89e9 (< 2^31) before the
    epilogue divides by 16.  Decode (weights as A), 256 < M <= 512 (weights
    as B) and larger M (the weight unpacked to INT8 first) are covered; all
    rows of x are equal, so the oracle runs on one."""
    k, n = 133120, 256
    x_bits = np.zeros((1, k), dtype=np.uint16)
    x_bits[0, ::256] = 0x3F80                        # 1.0 at the start of every group
    w_bits = np.zeros((n, k), dtype=np.uint16)
    w_bits[: n // 2, ::256] = 0x3F80                 # rows of +7 codes
    w_bits[n // 2:, ::256] = 0xBF80                  # rows of -7 codes
    packed_ref, s_ref = oracle.rotate_quantize4(w_bits)
    assert np.array_equal(oracle.unpack_int4(packed_ref[:1]), np.full((1, k), 7, dtype=np.int8))
    ref = oracle.linear_w4a8(x_bits, packed_ref, s_ref)
    assert int(ref["acc"][0, 0]) == 889 * k and int(ref["acc"][0, n - 1]) == -889 * k
    w4 = cr.quantize_weight4(from_bits(w_bits))
    assert np.array_equal(w4.q.cpu().numpy(), packed_ref)
    x = from_bits(x_bits).expand(m, k).contiguous()
    y = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    cr.LinearBatchW4([x], [w4], [y])()
    cr.convrot_device_status()
    yb = to_bits(y)
    assert np.array_equal(yb, np.broadcast_to(ref["y"], (m, n)))


def test_w4a8_qwen_decode_layer_sampled(cr):
    lins = synth.qwen_layer(12)
    xs, ws4, ys = [], [], []
    for lin in lins:
        w_bf = lin.w_torch("cuda")
        ws4.append(cr.quantize_weight4(w_bf))
        del w_bf
        xs.append(lin.x_torch("cuda"))
        ys.append(torch.empty((lin.m, lin.n), dtype=torch.bfloat16, device="cuda"))
    cr.LinearBatchW4(xs, ws4, ys)()
    cr.convrot_device_status()
    rng = np.random.default_rng(21)
    for lin, w4, y in zip(lins, ws4, ys):
        rows = np.unique(np.concatenate([[0, lin.n - 1], rng.integers(0, lin.n, 12)]))
        packed_ref, s_ref = oracle.rotate_quantize4(lin.w_rows_np(rows))
        rw = torch.as_tensor(rows, device="cuda")
        assert np.array_equal(w4.q[rw].cpu().numpy(), packed_ref)
        ref = oracle.linear_w4a8(lin.x_np(), packed_ref, s_ref)
        assert np.array_equal(to_bits(y[:, rw]), ref["y"])



# ---------------------------------------------------------------- convolutions (int8_convrot)
# (n, h, w, c, o, k, stride, pad, dil): 3x3 with padding, stride 2, dilation,
# a 1x1, channels below 256 (dynamic group), a ragged last chunk, enough rows
# for the large-M GEMM path, and a few rows (stream-K path)
CONV_CASES = [
    (1, 8, 8, 256, 64, 3, 1, 1, 1),
    (2, 9, 7, 128, 96, 3, 2, 1, 1),
    (1, 10, 10, 64, 32, 3, 1, 2, 2),
    (1, 16, 16, 512, 256, 1, 1, 0, 1),
    (1, 12, 12, 96, 48, 3, 1, 1, 1),
    (1, 32, 32, 128, 128, 3, 1, 1, 1),
    (1, 3, 3, 256, 64, 3, 1, 0, 1),
    # enough pixels that the pixel rotation packs 16 / 8 / 16 rows to a CTA
    (1, 40, 40, 256, 64, 3, 1, 1, 1),
    (1, 36, 36, 512, 64, 3, 1, 1, 1),
    (1, 48, 48, 128, 64, 3, 1, 1, 1),
    (2, 20, 13, 16, 32, 3, 1, 1, 1),
    (1, 9, 9, 48, 32, 5, 1, 2, 1),
    # 49 taps: more than a warp's lanes, so the untiled gather
    (1, 12, 12, 32, 16, 7, 1, 3, 1),
    # 1x1 with enough pixels that the one-step gather packs 16 rows to a CTA, and strided
    (1, 40, 40, 256, 64, 1, 1, 0, 1),
    (2, 50, 50, 128, 32, 1, 2, 0, 1),
]


@pytest.mark.parametrize("n,h,w,c,o,k,stride,pad,dil", CONV_CASES)
def test_conv2d_int8_bit_exact(cr, n, h, w, c, o, k, stride, pad, dil):
    seed = n * 1000 + h * 10 + c + o + k
    cs = synth.outlier_scale_fraction(synth.stream_key(seed, 2), c, 0.02, 30.0)
    x_bits = synth.draw_np(synth.stream_key(seed, 0), n * h * w, c, 1.0, cs).reshape(n, h, w, c)
    w_bits = synth.draw_np(synth.stream_key(seed, 1), o, c * k * k, synth.W_SIGMA).reshape(o, c, k, k)
    group = cr.convrot_dynamic_group(c)
    ref = oracle.conv2d_int8(x_bits, w_bits, stride, pad, dil, group=group)
    wq = cr.quantize_conv_weight(from_bits(w_bits))
    torch.cuda.synchronize()
    assert np.array_equal(wq.q.cpu().numpy(), ref["wq"]) and np.array_equal(wq.scale.cpu().numpy(), ref["sw"])
    y = cr.conv2d_int8(from_bits(x_bits), wq, k, k, stride, pad, dil)
    cr.convrot_device_status()
    yb = to_bits(y)
    assert yb.shape == ref["y"].shape
    assert rel_err(yb, ref["y"]) <= TOL
    assert np.array_equal(yb, ref["y"])


# ---------------------------------------------------------------- benchmarked configurations at full size
def _sampled_batch_check(cr, lins, rows_w, rows_x, dev="cuda"):
    """The layer's linears in one LinearBatch call (the bench's entry point),
    whole-size weights quantised on the GPU; the oracle recomputes the
    sampled weight rows and token rows of every linear from the counter-based
    generator and checks weight codes and scales and the BF16 outputs bit for
    bit."""
    weights, xs, ys = [], [], []
    for lin in lins:
        w_bf = lin.w_torch(dev)
        weights.append(cr.quantize_weight(w_bf))
        del w_bf
        xs.append(lin.x_torch(dev))
        ys.append(torch.empty((lin.m, lin.n), dtype=torch.bfloat16, device=dev))
    batch = cr.LinearBatch(xs, weights, ys)
    batch()
    batch()                      # the batched workspace is left reusable
    cr.convrot_device_status()
    for j, (lin, w, y) in enumerate(zip(lins, weights, ys)):
        rw = np.asarray(rows_w[j])
        rx = np.asarray(rows_x)
        wq_ref, sw_ref = oracle.rotate_quantize(lin.w_rows_np(rw))
        rwt = torch.as_tensor(rw, device=dev)
        assert np.array_equal(w.q[rwt].cpu().numpy(), wq_ref), lin.name
        assert np.array_equal(w.scale[rwt].cpu().numpy(), sw_ref), lin.name
        ref = oracle.linear_int8(lin.x_rows_np(rx), wq_ref, sw_ref)
        yb = to_bits(y[torch.as_tensor(rx, device=dev)][:, rwt])
        assert rel_err(yb, ref["y"]) <= TOL, lin.name
        assert np.array_equal(yb, ref["y"]), lin.name
    del batch, weights, xs, ys
    torch.cuda.empty_cache()


def _edge_rows(n, rng, count, tile=256):
    # first and last rows, both sides of the first tile boundary, random others
    picks = [0, n - 1, min(tile - 1, n - 1), min(tile, n - 1)]
    return np.unique(np.concatenate([picks, rng.integers(0, n, count)]))


def test_stack_layer_m512_batch_sampled(cr):
    # one layer of the 50-layer stack at M = 512 exactly as the bench runs it:
    # seven Qwen-shaped weights in one batched GEMM launch (activations = A,
    # four 128-row tiles replicated over CTA groups, stream-K over the K
    # blocks of the 256-row weight tiles of all seven weights)
    lins = synth.qwen_stack(512, layers=1)
    plan = cr.gemm_plan(512, [l.n for l in lins], [l.k for l in lins])
    assert plan.swap == 0 and plan.rep == 4 and plan.njobs == 7
    rng = np.random.default_rng(512)
    rows_w = [_edge_rows(lin.n, rng, 12) for lin in lins]
    rows_x = np.unique(np.concatenate([[0, 127, 128, 255, 256, 383, 384, 511], rng.integers(0, 512, 8)]))
    _sampled_batch_check(cr, lins, rows_w, rows_x)


def test_qwen_prefill_layer_batch_sampled(cr):
    # the prefill layer as the bench runs it: all seven linears at M = 4096
    # through LinearBatch (one GEMM launch per linear, whole 128 x 256 tiles
    # in full waves; gate and up have 3200 tiles = 21 waves + a 92-tile tail)
    lins = synth.qwen_layer(4096)
    rng = np.random.default_rng(4096)
    rows_w = [_edge_rows(lin.n, rng, 10) for lin in lins]
    rows_x = np.unique(np.concatenate([[0, 127, 128, 2047, 2048, 4095], rng.integers(0, 4096, 8)]))
    _sampled_batch_check(cr, lins, rows_w, rows_x)


def _conv_rows_oracle(x_rows_fn, h, w, c, pixels):
    """im2col rows (3x3, stride 1, pad 1) of the sampled output pixels, each
    from its 3 x 3 input window (zeros outside the image) through the
    oracle's own im2col."""
    out = []
    for (oy, ox) in pixels:
        win = np.zeros((1, 3, 3, c), dtype=np.uint16)
        for dy in range(3):
            for dx in range(3):
                iy, ix = oy - 1 + dy, ox - 1 + dx
                if 0 <= iy < h and 0 <= ix < w:
                    win[0, dy, dx] = x_rows_fn([iy * w + ix])[0]
        out.append(oracle.im2col_nhwc(win, 3, 3, 1, 0, 1)[0])
    return np.stack(out)


@pytest.mark.parametrize("h,c", [(128, 512), (256, 256)])
def test_vae_conv_bench_shapes_sampled(cr, h, c):
    # the two VAE-decoder-shaped 3x3 convolutions the bench times, drawn as
    # the bench draws them, through the same entry point and tile plan
    seed = 77 + c
    xl = synth.Linear("conv_x", h * h, c, 1, seed, None)
    wl = synth.Linear("conv_w", 1, 9 * c, c, seed, None)
    x = xl.x_torch("cuda").view(1, h, h, c)
    w_oihw = wl.w_torch("cuda").view(c, c, 3, 3)
    plan = cr.conv2d_gather_plan(tuple(x.shape), 3, 3, 1, 1, 1)
    assert plan.tiled == 1
    wq = cr.quantize_conv_weight(w_oihw)
    y = cr.conv2d_int8(x, wq, 3, 3, 1, 1, 1)
    y2 = cr.conv2d_int8(x, wq, 3, 3, 1, 1, 1)
    cr.convrot_device_status()
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    rng = np.random.default_rng(h + c)
    chans = np.unique(np.concatenate([[0, c - 1], rng.integers(0, c, 10)]))
    w_rows = oracle.conv_weight_rows(wl.w_rows_np(chans).reshape(len(chans), c, 3, 3))
    wq_ref, sw_ref = oracle.rotate_quantize(w_rows)
    ct = torch.as_tensor(chans, device="cuda")
    assert np.array_equal(wq.q[ct].cpu().numpy(), wq_ref)
    assert np.array_equal(wq.scale[ct].cpu().numpy(), sw_ref)
    pix = [(0, 0), (0, h - 1), (h - 1, 0), (h - 1, h - 1), (1, 1), (h // 2, 0)]
    pix += [tuple(p) for p in rng.integers(0, h, (10, 2))]
    rows = _conv_rows_oracle(xl.x_rows_np, h, h, c, pix)
    ref = oracle.linear_int8(rows, wq_ref, sw_ref)
    got = np.stack([to_bits(y[0, oy, ox][ct]) for (oy, ox) in pix])
    assert rel_err(got, ref["y"]) <= TOL
    assert np.array_equal(got, ref["y"])


# ---------------------------------------------------------------- exactness domain of the rotation
def _plant_wide_group(x_bits, row, group):
    # 1.0 and 2^-60 in one group: its nonzero magnitudes span 61 binades
    x = x_bits.copy()
    x[row, 256 * group] = 0x3F80
    x[row, 256 * group + 1] = synth.f32_to_bf16_bits(np.array([2.0 ** -60], np.float32))[0]
    return x


def _status_after(cr, fn):
    fn()
    try:
        cr.convrot_device_status()
    except cr.ConvrotError as e:
        return e.status
    return 0


@pytest.mark.parametrize("m,k", [(300, 4096), (3, 512), (400, 25600), (5, 25600), (310, 12288)])
def test_inexact_domain_is_reported(cr, m, k):
    # the lean prefill kernel (register and staged rows), the row kernel
    # (few rows, clusters), through the activation and the weight entry points
    x_bits = synth.draw_np(synth.stream_key(m + k, 0), m, k, 1.0)
    assert oracle.rotate_rows(x_bits)[1] == 0
    xq = torch.empty((m, k), dtype=torch.int8, device="cuda")
    sx = torch.empty((m,), dtype=torch.float32, device="cuda")
    assert _status_after(cr, lambda: cr.convrot_quantize_act(from_bits(x_bits), xq, sx)) == 0
    planted = _plant_wide_group(x_bits, m // 2, (k // 256) // 2)
    assert oracle.rotate_rows(planted)[1] == 1
    assert _status_after(cr, lambda: cr.convrot_quantize_act(from_bits(planted), xq, sx)) == 8
    assert _status_after(cr, lambda: cr.quantize_weight(from_bits(planted))) == 8
    assert _status_after(cr, lambda: cr.quantize_weight(from_bits(x_bits))) == 0


def test_inexact_domain_warning_is_conservative(cr):
    # every group exact on its own (one group of ~1, one of ~2^-40), but the
    # row's scale cannot tell them apart: the warning is raised although the
    # oracle finds no inexact group, and the codes are still bit-exact
    m, k = 300, 4096
    x = synth.bf16_bits_to_f32(synth.draw_np(synth.stream_key(9, 0), m, k, 1.0))
    x[7, 256:512] *= np.float32(2.0 ** -40)
    bits = synth.f32_to_bf16_bits(x)
    assert oracle.rotate_rows(bits)[1] == 0
    xq = torch.empty((m, k), dtype=torch.int8, device="cuda")
    sx = torch.empty((m,), dtype=torch.float32, device="cuda")
    assert _status_after(cr, lambda: cr.convrot_quantize_act(from_bits(bits), xq, sx)) == 8
    q_ref, s_ref = oracle.rotate_quantize(bits)
    assert np.array_equal(xq.cpu().numpy(), q_ref)
    assert np.array_equal(sx.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


def test_inexact_domain_reported_by_convolution_pixels(cr):
    # 3x3 convolution: every input pixel is rotated once; a pixel holding a
    # 61-binade group raises the warning
    n, h, w, c, o = 1, 20, 20, 256, 64
    x_bits = synth.draw_np(synth.stream_key(21, 0), n * h * w, c, 1.0)
    w_bits = synth.draw_np(synth.stream_key(21, 1), o, c * 9, synth.W_SIGMA).reshape(o, c, 3, 3)
    wq = cr.quantize_conv_weight(from_bits(w_bits))
    xd = from_bits(x_bits.reshape(n, h, w, c))
    assert _status_after(cr, lambda: cr.conv2d_int8(xd, wq, 3, 3, 1, 1, 1)) == 0
    planted = _plant_wide_group(x_bits, 123, 0).reshape(n, h, w, c)
    assert _status_after(cr, lambda: cr.conv2d_int8(from_bits(planted), wq, 3, 3, 1, 1, 1)) == 8


def test_w4a8_qwen_prefill_layer_sampled(cr):
    # INT4 weights at prefill size: every linear of the layer at M = 4096
    # through LinearBatchW4 (one whole-tile GEMM launch per linear)
    lins = synth.qwen_layer(4096)
    xs, ws4, ys = [], [], []
    for lin in lins:
        w_bf = lin.w_torch("cuda")
        ws4.append(cr.quantize_weight4(w_bf))
        del w_bf
        xs.append(lin.x_torch("cuda"))
        ys.append(torch.empty((lin.m, lin.n), dtype=torch.bfloat16, device="cuda"))
    batch = cr.LinearBatchW4(xs, ws4, ys)
    batch()
    batch()
    cr.convrot_device_status()
    rng = np.random.default_rng(4094)
    rows_x = np.unique(np.concatenate([[0, 127, 128, 4095], rng.integers(0, 4096, 8)]))
    for lin, w4, y in zip(lins, ws4, ys):
        rows = _edge_rows(lin.n, rng, 8)
        packed_ref, s_ref = oracle.rotate_quantize4(lin.w_rows_np(rows))
        rw = torch.as_tensor(rows, device="cuda")
        assert np.array_equal(w4.q[rw].cpu().numpy(), packed_ref), lin.name
        ref = oracle.linear_w4a8(lin.x_rows_np(rows_x), packed_ref, s_ref)
        yb = to_bits(y[torch.as_tensor(rows_x, device="cuda")][:, rw])
        assert rel_err(yb, ref["y"]) <= TOL, lin.name
        assert np.array_equal(yb, ref["y"]), lin.name
    del batch, ws4, xs, ys
    torch.cuda.empty_cache()
