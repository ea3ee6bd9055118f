"""convrot_gemm_i8_noalloc: the GEMM entry point for callers that cannot pass
a device workspace (for example a plugin whose host engine owns all device
memory and forbids outside allocations).  It keeps its scratch in an array
built into the library.  Checked through the C ABI, on two calls in a row (so
the second call sees the array the first one left behind), against the
oracle and against convrot_gemm_i8 (which uses a caller workspace): the same
plan and kernel, so the INT32 accumulators and the BF16 outputs must be
bit-identical.  The shapes take the stream-K paths, where the scratch is
actually used.

This file is named to be collected last, so that a run stopping at the
first failure has already run every other test.
"""
import ctypes

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


def _rel_err(y, ref):
    y = y.float().double().cpu().numpy()
    r = ref.float().double().cpu().numpy()
    return float(np.max(np.abs(y - r)) / max(np.max(np.abs(r)), 1e-30))


def _noalloc(cr, xq, sx, w, y, acc):
    lib = cr.load_library()
    P = ctypes.c_void_p
    return lib.convrot_gemm_i8_noalloc(P(xq.data_ptr()), P(sx.data_ptr()), xq.shape[0], ctypes.byref(w.handle),
                                       P(y.data_ptr()), P(acc.data_ptr()),
                                       P(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("m,n,k", [(12, 1024, 5120), (4, 256, 512), (300, 512, 768)])
def test_noalloc_matches_workspace_entry_point(cr, m, n, k):
    dev = "cuda"
    seed = 7 * m + n + k
    x = synth.draw_torch(synth.stream_key(seed, 0), m, k, device=dev)
    w_bits = synth.draw_np(synth.stream_key(seed, 1), n, k, synth.W_SIGMA)
    w = cr.quantize_weight(torch.from_numpy(w_bits.view(np.int16)).view(torch.bfloat16).to(dev))
    wq_ref, sw_ref = oracle.rotate_quantize(w_bits)
    ref = oracle.linear_int8(synth.draw_np(synth.stream_key(seed, 0), m, k), wq_ref, sw_ref)
    xq = torch.empty((m, k), dtype=torch.int8, device=dev)
    sx = torch.empty((m,), dtype=torch.float32, device=dev)
    cr.convrot_quantize_act(x, xq, sx)
    y_ref = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
    acc_ref = torch.empty((m, n), dtype=torch.int32, device=dev)
    cr.convrot_gemm_i8(xq, sx, w, y_ref, acc_ref, cr.make_workspace(m, w, linear=False))
    for call in range(2):
        y = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device=dev)
        acc = torch.zeros((m, n), dtype=torch.int32, device=dev)
        assert _noalloc(cr, xq, sx, w, y, acc) == 0, "call %d" % call
        cr.convrot_device_status()
        assert _rel_err(y, y_ref) <= TOL, "call %d" % call
        assert torch.equal(acc, acc_ref), "call %d" % call
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), "call %d" % call
        assert np.array_equal(acc.cpu().numpy(), ref["acc"]), "call %d" % call
        assert np.array_equal(y.cpu().view(torch.int16).numpy().view(np.uint16), ref["y"]), "call %d" % call


def test_noalloc_rejects_problems_beyond_its_scratch(cr):
    # 256 tokens against 147 weight tiles: every tile is split along K and
    # needs a 128 KB INT32 partial tile -- far more than the built-in 8 MiB
    m, n, k = 256, 147 * 128, 512
    dev = "cuda"
    w = cr.convrot_weight_init(torch.zeros((n, k), dtype=torch.int8, device=dev),
                               torch.zeros((n,), dtype=torch.float32, device=dev))
    xq = torch.zeros((m, k), dtype=torch.int8, device=dev)
    sx = torch.zeros((m,), dtype=torch.float32, device=dev)
    y = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
    acc = torch.empty((m, n), dtype=torch.int32, device=dev)
    assert _noalloc(cr, xq, sx, w, y, acc) == 5      # CONVROT_ERR_WORKSPACE
    assert b"8 MiB" in cr.load_library().convrot_last_error_string()
