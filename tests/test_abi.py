"""The C ABI without a GPU: the library loads, exports every entry point
that include/convrot.h declares, and rejects bad arguments on the host
before touching a device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "convrot.h")


@pytest.fixture(scope="module")
def lib():
    from rotated_int8_quantized_b200 import build
    build.build()
    import rotated_int8_quantized_b200 as cr
    return cr.load_library()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(convrot_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("convrot_quantize_weight", "convrot_quantize_act", "convrot_gemm_i8",
                     "convrot_linear_int8", "convrot_weight_init"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    import rotated_int8_quantized_b200 as cr
    for name in _declared_functions():
        assert hasattr(lib, name), name
        assert name in cr.SIGNATURES, name


def test_status_strings(lib):
    import rotated_int8_quantized_b200 as cr
    for code, name in cr._STATUS.items():
        assert cr.convrot_status_string(code) == name
    assert cr.convrot_version() >= 100


def _init(lib, q, s, n, k, g):
    import rotated_int8_quantized_b200 as cr
    h = cr.convrot_weight_t()
    return lib.convrot_weight_init(ctypes.byref(h), ctypes.c_void_p(q), ctypes.c_void_p(s), n, k, g), h


def test_weight_init_validation(lib):
    ok, h = _init(lib, 0x10000, 0x20000, 256, 512, 256)
    assert ok == 0 and h.n == 256 and h.k == 512 and h.group == 256
    assert _init(lib, 0, 0x20000, 256, 512, 256)[0] == 1          # null q
    assert _init(lib, 0x10000, 0x20000, 0, 512, 256)[0] == 1      # n = 0
    assert _init(lib, 0x10000, 0x20000, 8, 300, 256)[0] == 3      # k % 256
    assert _init(lib, 0x10000, 0x20000, 8, 512, 128)[0] == 0      # a smaller power-of-two group
    assert _init(lib, 0x10000, 0x20000, 8, 640, 128)[0] == 0      # ... need not divide 256
    assert _init(lib, 0x10000, 0x20000, 8, 512, 96)[0] == 3       # not a power of two
    assert _init(lib, 0x10000, 0x20000, 8, 512, 8)[0] == 3        # below 16
    assert _init(lib, 0x10000, 0x20000, 8, 512, 512)[0] == 3      # above 256
    assert _init(lib, 0x10000, 0x20000, 8, 640, 256)[0] == 3      # k % group
    assert _init(lib, 0x10000, 0x20000, 8, 133376, 256)[0] == 3   # INT32 accumulation bound
    assert _init(lib, 0x10001, 0x20000, 8, 512, 256)[0] == 2      # misaligned q
    assert _init(lib, 0x10000, 0x20004, 8, 512, 256)[0] == 2      # misaligned scale


def test_calls_reject_bad_arguments_before_any_device_work(lib):
    P = ctypes.c_void_p
    assert lib.convrot_quantize_act(P(0), 4, 512, 256, P(0x100), P(0x200), P(0)) == 1
    assert lib.convrot_quantize_act(P(0x100), 4, 500, 256, P(0x100), P(0x200), P(0)) == 3
    assert lib.convrot_quantize_act(P(0x101), 4, 512, 256, P(0x100), P(0x200), P(0)) == 2
    _, h = _init(lib, 0x10000, 0x20000, 256, 512, 256)
    assert lib.convrot_gemm_i8(P(0x100), P(0x200), 4, ctypes.byref(h), P(0), P(0), P(0), 0, P(0)) == 1
    assert lib.convrot_linear_int8(P(0x100), 4, ctypes.byref(h), P(0x300), P(0), 0, P(0)) == 1
    assert lib.convrot_linear_int8(P(0x100), 0, ctypes.byref(h), P(0x300), P(0x400), 1 << 20, P(0)) == 1


def test_workspace_sizes_follow_the_tiling(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("sizes below assume the 148-SM default used without a device")
    # decode: weight is the 128-row operand, 12 tokens pad to one 16-row
    # tile; 64 weight tiles < 148 SMs, so the K blocks are dealt out over all
    # 148 CTAs (stream-K) and a tile shared by several CTAs sums in the slot
    # of one of them: 148 counters (768 B) + 148 INT32 partial tiles of
    # 16 x 128 x 4 B
    assert lib.convrot_gemm_workspace_bytes(12, 8192, 5120) == 768 + 148 * 16 * 128 * 4
    # 512 rows: four 128-row activation tiles x 20 weight tiles of 256 rows,
    # stream-K again (128 x 256 INT32 partial tiles)
    assert lib.convrot_gemm_workspace_bytes(512, 5120, 5120) == 768 + 148 * 256 * 128 * 4
    # prefill: 32 x 100 tiles of 128 x 256, whole tiles only (22 waves over
    # 148 SMs, the last one partial): no scratch at all
    assert lib.convrot_gemm_workspace_bytes(4096, 25600, 5120) == 0
    # prefill down projection: 32 x 20 = 640 tiles, 4 full waves; the 48 tail
    # tiles are split into 148 // 48 = 3 K ranges with private 128 KB INT32
    # partial tiles
    assert lib.convrot_gemm_workspace_bytes(4096, 5120, 25600) == 256 + 48 * 3 * 256 * 128 * 4
    lw = lib.convrot_linear_workspace_bytes(12, 8192, 5120)
    assert lw == lib.convrot_gemm_workspace_bytes(12, 8192, 5120) + 61440 + 256


def test_binding_structs_match_the_header(tmp_path):
    """The ctypes mirrors of the job structs have the C layout: a C program
    compiled against include/convrot.h prints sizes and offsets."""
    import subprocess
    import rotated_int8_quantized_b200 as cr
    src = tmp_path / "layout.c"
    src.write_text(r'''
#include <stdio.h>
#include "convrot.h"
#define F(T, f) printf(#T "." #f " %zu\n", offsetof(T, f));
int main(void) {
    printf("convrot_weight_t %zu\n", sizeof(convrot_weight_t));
    printf("convrot_gemm_job_t %zu\n", sizeof(convrot_gemm_job_t));
    printf("convrot_linear_job_t %zu\n", sizeof(convrot_linear_job_t));
    F(convrot_weight_t, group) F(convrot_gemm_job_t, acc) F(convrot_gemm_job_t, bias_bf16)
    F(convrot_linear_job_t, y_bf16) F(convrot_linear_job_t, bias_bf16)
    printf("convrot_weight4_t %zu\n", sizeof(convrot_weight4_t));
    printf("convrot_linear4_job_t %zu\n", sizeof(convrot_linear4_job_t));
    F(convrot_weight4_t, group) F(convrot_linear4_job_t, bias_bf16)
    printf("convrot_conv2d_t %zu\n", sizeof(convrot_conv2d_t));
    printf("convrot_conv2d_plan_t %zu\n", sizeof(convrot_conv2d_plan_t));
    F(convrot_conv2d_t, dilation) F(convrot_conv2d_plan_t, tiles) F(convrot_conv2d_plan_t, buf_bytes)
    return 0;
}
''')
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    got = dict(line.split() for line in subprocess.check_output([str(exe)], text=True).splitlines())
    want = {
        "convrot_weight_t": ctypes.sizeof(cr.convrot_weight_t),
        "convrot_gemm_job_t": ctypes.sizeof(cr.convrot_gemm_job_t),
        "convrot_linear_job_t": ctypes.sizeof(cr.convrot_linear_job_t),
        "convrot_weight_t.group": cr.convrot_weight_t.group.offset,
        "convrot_gemm_job_t.acc": cr.convrot_gemm_job_t.acc.offset,
        "convrot_gemm_job_t.bias_bf16": cr.convrot_gemm_job_t.bias_bf16.offset,
        "convrot_linear_job_t.y_bf16": cr.convrot_linear_job_t.y_bf16.offset,
        "convrot_linear_job_t.bias_bf16": cr.convrot_linear_job_t.bias_bf16.offset,
        "convrot_weight4_t": ctypes.sizeof(cr.convrot_weight4_t),
        "convrot_linear4_job_t": ctypes.sizeof(cr.convrot_linear4_job_t),
        "convrot_weight4_t.group": cr.convrot_weight4_t.group.offset,
        "convrot_linear4_job_t.bias_bf16": cr.convrot_linear4_job_t.bias_bf16.offset,
        "convrot_conv2d_t": ctypes.sizeof(cr.convrot_conv2d_t),
        "convrot_conv2d_plan_t": ctypes.sizeof(cr.convrot_conv2d_plan_t),
        "convrot_conv2d_t.dilation": cr.convrot_conv2d_t.dilation.offset,
        "convrot_conv2d_plan_t.tiles": cr.convrot_conv2d_plan_t.tiles.offset,
        "convrot_conv2d_plan_t.buf_bytes": cr.convrot_conv2d_plan_t.buf_bytes.offset,
    }
    assert {k: int(v) for k, v in got.items()} == want


def test_dynamic_group(lib):
    # the largest power of two <= the cap dividing k; 0 below 16
    assert lib.convrot_dynamic_group(5376, 256) == 256
    assert lib.convrot_dynamic_group(640, 256) == 128
    assert lib.convrot_dynamic_group(5440, 256) == 64
    assert lib.convrot_dynamic_group(1024, 64) == 64
    assert lib.convrot_dynamic_group(40, 256) == 0
    for k in range(16, 4000, 16):
        g = lib.convrot_dynamic_group(k, 256)
        assert g >= 16 and g <= 256 and k % g == 0 and (g == 256 or k % (2 * g) != 0)


def test_weight4_validation(lib):
    import rotated_int8_quantized_b200 as cr
    h = cr.convrot_weight4_t()
    P = ctypes.c_void_p
    assert lib.convrot_weight4_init(ctypes.byref(h), P(0x10000), P(0x20000), 8, 512, 256) == 0
    assert h.k == 512 and h.group == 256
    assert lib.convrot_weight4_init(ctypes.byref(h), P(0x10000), P(0x20000), 8, 48, 16) == 3   # k % 32
    assert lib.convrot_weight4_init(ctypes.byref(h), P(0x10001), P(0x20000), 8, 512, 256) == 2
    # the GEMM accumulates INT4 weights as 16 x code, exact while
    # 16 * 7 * 127 * k < 2^31: the largest accepted k keeps that, the next one
    # is refused when the handle is made
    kmax = 133120
    assert 16 * 7 * 127 * kmax < 2 ** 31
    assert lib.convrot_weight4_init(ctypes.byref(h), P(0x10000), P(0x20000), 8, kmax, 256) == 0
    assert lib.convrot_weight4_init(ctypes.byref(h), P(0x10000), P(0x20000), 8, kmax + 256, 256) == 3
    assert lib.convrot_weight4_init(ctypes.byref(h), P(0x10000), P(0x20000), 8, 512, 256) == 0
    job = (cr.convrot_linear4_job_t * 1)()
    job[0].x_bf16, job[0].w, job[0].y_bf16 = P(0x100000), ctypes.pointer(h), P(0x200000)
    assert lib.convrot_linear_w4a8(0, 1, job, P(0x300000), 1 << 30, P(0)) == 1
    assert lib.convrot_linear_w4a8_workspace_bytes(12, 1, job) > 0
    # any token count: prefill sizes take per-job GEMM launches
    assert lib.convrot_linear_w4a8_workspace_bytes(300, 1, job) > 0
    job[0].y_bf16 = P(0x10000000)        # clear of the 4 MB input at m = 4096
    assert lib.convrot_linear_w4a8_workspace_bytes(4096, 1, job) > 0


def test_conv2d_shape_and_validation(lib):
    import rotated_int8_quantized_b200 as cr
    g = cr.convrot_conv2d_t(1, 64, 64, 512, 3, 3, 1, 1, 1)
    oh, ow = ctypes.c_int32(), ctypes.c_int32()
    assert lib.convrot_conv2d_shape(ctypes.byref(g), ctypes.byref(oh), ctypes.byref(ow)) == 0
    assert (oh.value, ow.value) == (64, 64)
    g2 = cr.convrot_conv2d_t(2, 9, 7, 128, 3, 3, 2, 1, 1)
    assert lib.convrot_conv2d_shape(ctypes.byref(g2), ctypes.byref(oh), ctypes.byref(ow)) == 0
    assert (oh.value, ow.value) == (5, 4)
    bad = cr.convrot_conv2d_t(1, 8, 8, 24, 3, 3, 1, 1, 1)      # channels not a multiple of 16
    assert lib.convrot_conv2d_shape(ctypes.byref(bad), None, None) == 3
    h = cr.convrot_weight_t()
    P = ctypes.c_void_p
    assert lib.convrot_weight_init(ctypes.byref(h), P(0x10000), P(0x20000), 64, 3 * 3 * 512, 256) == 0
    assert lib.convrot_conv2d_workspace_bytes(ctypes.byref(g), ctypes.byref(h)) > 64 * 64 * 4608
    assert lib.convrot_weight_init(ctypes.byref(h), P(0x10000), P(0x20000), 64, 3 * 3 * 96, 32) == 0
    g3 = cr.convrot_conv2d_t(1, 8, 8, 96, 3, 3, 1, 1, 1)
    assert lib.convrot_conv2d_workspace_bytes(ctypes.byref(g3), ctypes.byref(h)) > 0
    g4 = cr.convrot_conv2d_t(1, 8, 8, 96, 1, 1, 1, 0, 1)         # k mismatch
    assert lib.convrot_conv2d_workspace_bytes(ctypes.byref(g4), ctypes.byref(h)) == 0


def test_plain_c_program_uses_the_library(tmp_path):
    """The C ABI needs no Python: a C99 program compiled against
    include/convrot.h and linked with libconvrot.so calls the host-only
    entry points (version, status strings, argument checks, dynamic group,
    plan queries) and checks their answers."""
    import subprocess
    import rotated_int8_quantized_b200 as cr
    lib_dir = os.path.dirname(cr.LIB_PATH)
    src = tmp_path / "use.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "convrot.h"
#define CHECK(c) do { if (!(c)) { printf("FAIL %s:%d %s\n", __FILE__, __LINE__, #c); return 1; } } while (0)
int main(void) {
    CHECK(convrot_version() >= 100);
    CHECK(strcmp(convrot_status_string(CONVROT_OK), "CONVROT_OK") == 0);
    CHECK(convrot_dynamic_group(5376, 256) == 256 && convrot_dynamic_group(640, 256) == 128);
    convrot_weight_t w;
    CHECK(convrot_weight_init(&w, NULL, NULL, 256, 512, 256) != CONVROT_OK);      /* null storage */
    int64_t n[7] = {8192, 1024, 1024, 5120, 25600, 25600, 5120};
    int64_t k[7] = {5120, 5120, 5120, 8192, 5120, 5120, 25600};
    convrot_gemm_plan_t p;
    CHECK(convrot_gemm_plan(12, 7, n, k, 0, 148, &p) == CONVROT_OK);
    CHECK(p.njobs == 7 && p.swap == 1 && p.bn == 16 && p.grid == 148);
    CHECK(p.tail_units == 29760 && p.full_waves == 0);
    CHECK(convrot_gemm_plan(600, 2, n, k, 0, 148, &p) == CONVROT_ERR_UNSUPPORTED_SHAPE);
    convrot_conv2d_t g = {1, 256, 256, 256, 3, 3, 1, 1, 1};
    int32_t oh = 0, ow = 0;
    CHECK(convrot_conv2d_shape(&g, &oh, &ow) == CONVROT_OK && oh == 256 && ow == 256);
    convrot_conv2d_plan_t cp;
    CHECK(convrot_conv2d_gather_plan(&g, 148, &cp) == CONVROT_OK && cp.tiled == 1);
    CHECK(cp.tiles == (int64_t)(256 / cp.th + (256 % cp.th != 0)) * (256 / cp.tw + (256 % cp.tw != 0)));
    printf("ok\n");
    return 0;
}
''')
    exe = tmp_path / "use"
    subprocess.check_call(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                           "-L", lib_dir, "-l:libconvrot.so", "-Wl,-rpath," + lib_dir])
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr
