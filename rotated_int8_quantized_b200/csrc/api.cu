// api.cu -- the C ABI of libconvrot (declared in include/convrot.h):
// argument checks on the host, workspace layout, and the launches of the
// rotation/quantisation kernel and the tcgen05 INT8 GEMM.
#include <cstdint>
#include <cstring>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/convrot.h"
#include "common.cuh"
#include "gemm_i8.h"
#include "rotate_quant.h"

// Hash of the sources and flags this library was compiled from (set by the
// build script; a build without it says so).
#ifndef CONVROT_BUILD_ID
#define CONVROT_BUILD_ID "unknown"
#endif

namespace {

constexpr int64_t kGroup = 256;         // the pages' group; also the largest
constexpr int64_t kMinGroup = 16;       // INT8 rows must be 16-byte multiples (TMA row stride)
// |acc| <= k * 127^2 must fit in INT32: k <= 133144; largest multiple of 256.
constexpr int64_t kMaxK = 133120;
constexpr int64_t kMaxRows = 0x7FFFFFFF;
constexpr int kDefaultSms = 148;
constexpr int kMaxBatch = convrot::kMaxJobs;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round256(size_t v) { return (v + 255) / 256 * 256; }

struct DeviceInfo {
    bool valid = false;
    bool arch_ok = false;
    int num_sms = 0;
};

// Current device: compute capability 10.0 check and SM count, cached.
convrot_status_t current_device(DeviceInfo *out) {
    static DeviceInfo cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return CONVROT_ERR_CUDA;
    }
    DeviceInfo tmp;
    DeviceInfo &d = (dev >= 0 && dev < 64) ? cache[dev] : tmp;
    if (!d.valid) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return CONVROT_ERR_CUDA;
        }
        d.arch_ok = (major == 10 && minor == 0);
        d.num_sms = sms;
        d.valid = true;
    }
    *out = d;
    return d.arch_ok ? CONVROT_OK : CONVROT_ERR_UNSUPPORTED_ARCH;
}

// SM count for workspace sizing; the B200's 148 when no device answers.
int sms_for_sizing() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0)
        return sms;
    cudaGetLastError();
    return kDefaultSms;
}

bool is_pow2(int64_t g) { return g > 0 && (g & (g - 1)) == 0; }

convrot_status_t check_shape(int64_t rows, int64_t k, int64_t group) {
    if (rows < 1 || k < 1) return CONVROT_ERR_INVALID_ARG;
    if (!is_pow2(group) || group < kMinGroup || group > kGroup) return CONVROT_ERR_UNSUPPORTED_SHAPE;
    if (k % group != 0 || k > kMaxK || rows > kMaxRows) return CONVROT_ERR_UNSUPPORTED_SHAPE;
    return CONVROT_OK;
}

convrot_status_t check_weight(const convrot_weight_t *w) {
    if (!w || !w->q || !w->scale) return CONVROT_ERR_INVALID_ARG;
    convrot_status_t s = check_shape(w->n, w->k, w->group);
    if (s != CONVROT_OK) return s;
    if (!aligned16(w->q) || !aligned16(w->scale)) return CONVROT_ERR_ALIGNMENT;
    return CONVROT_OK;
}

// INT4 rows are k/2 bytes: a multiple of 16 (TMA row stride) needs k % 32 == 0.
convrot_status_t check_weight4(const convrot_weight4_t *w) {
    if (!w || !w->q || !w->scale) return CONVROT_ERR_INVALID_ARG;
    convrot_status_t s = check_shape(w->n, w->k, w->group);
    if (s != CONVROT_OK) return s;
    if (w->k % 32 != 0) return CONVROT_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(w->q) || !aligned16(w->scale)) return CONVROT_ERR_ALIGNMENT;
    return CONVROT_OK;
}

thread_local const char *t_last_error = "no error";

convrot_status_t from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return CONVROT_OK;
    t_last_error = cudaGetErrorString(e);
    cudaGetLastError();
    return CONVROT_ERR_CUDA;
}

}  // namespace

#pragma GCC visibility push(default)
extern "C" {

const char *convrot_status_string(convrot_status_t s) {
    switch (s) {
        case CONVROT_OK: return "CONVROT_OK";
        case CONVROT_ERR_INVALID_ARG: return "CONVROT_ERR_INVALID_ARG";
        case CONVROT_ERR_ALIGNMENT: return "CONVROT_ERR_ALIGNMENT";
        case CONVROT_ERR_UNSUPPORTED_SHAPE: return "CONVROT_ERR_UNSUPPORTED_SHAPE";
        case CONVROT_ERR_UNSUPPORTED_ARCH: return "CONVROT_ERR_UNSUPPORTED_ARCH";
        case CONVROT_ERR_WORKSPACE: return "CONVROT_ERR_WORKSPACE";
        case CONVROT_ERR_CUDA: return "CONVROT_ERR_CUDA";
        case CONVROT_ERR_DEVICE_TIMEOUT: return "CONVROT_ERR_DEVICE_TIMEOUT";
        case CONVROT_WARN_INEXACT_DOMAIN: return "CONVROT_WARN_INEXACT_DOMAIN";
    }
    return "CONVROT_ERR_UNKNOWN";
}

int convrot_version(void) { return 100; }

const char *convrot_build_id(void) { return CONVROT_BUILD_ID; }

int32_t convrot_dynamic_group(int64_t k, int32_t max_group) {
    if (k < 1 || max_group < 1) return 0;
    int64_t g = 1;
    while (g * 2 <= max_group && g * 2 <= kGroup) g *= 2;
    while (g > 1 && k % g != 0) g /= 2;
    return g >= kMinGroup ? (int32_t)g : 0;
}

const char *convrot_last_error_string(void) { return t_last_error; }

convrot_status_t convrot_weight_init(convrot_weight_t *w, int8_t *q, float *scale, int64_t n, int64_t k,
                                     int32_t group) {
    if (!w) return CONVROT_ERR_INVALID_ARG;
    convrot_weight_t t;
    t.q = q;
    t.scale = scale;
    t.n = n;
    t.k = k;
    t.group = group;
    convrot_status_t s = check_weight(&t);
    if (s != CONVROT_OK) return s;
    *w = t;
    return CONVROT_OK;
}

convrot_status_t convrot_quantize_weight(const void *w_bf16, const convrot_weight_t *out, void *stream) {
    if (!w_bf16) return CONVROT_ERR_INVALID_ARG;
    convrot_status_t s = check_weight(out);
    if (s != CONVROT_OK) return s;
    if (!aligned16(w_bf16)) return CONVROT_ERR_ALIGNMENT;
    DeviceInfo dev;
    if ((s = current_device(&dev)) != CONVROT_OK) return s;
    convrot::RQProblem prob = {w_bf16, out->k, out->group, out->q, out->scale};
    return from_cuda(convrot::launch_rotate_quant(1, out->n, &prob, static_cast<cudaStream_t>(stream), false));
}

convrot_status_t convrot_quantize_act(const void *x_bf16, int64_t m, int64_t k, int32_t group, int8_t *xq,
                                      float *sx, void *stream) {
    if (!x_bf16 || !xq || !sx) return CONVROT_ERR_INVALID_ARG;
    convrot_status_t s = check_shape(m, k, group);
    if (s != CONVROT_OK) return s;
    if (!aligned16(x_bf16) || !aligned16(xq) || !aligned16(sx)) return CONVROT_ERR_ALIGNMENT;
    DeviceInfo dev;
    if ((s = current_device(&dev)) != CONVROT_OK) return s;
    convrot::RQProblem prob = {x_bf16, k, (int)group, xq, sx};
    return from_cuda(convrot::launch_rotate_quant(1, m, &prob, static_cast<cudaStream_t>(stream), false));
}

size_t convrot_gemm_workspace_bytes(int64_t m, int64_t n, int64_t k) {
    if (m < 1 || n < 1 || k < kMinGroup || k % kMinGroup != 0 || k > kMaxK) return 0;
    convrot::GemmPlan p;
    convrot::plan_gemm(m, n, k, sms_for_sizing(), &p);
    return round256(p.ws_bytes);
}


convrot_status_t convrot_gemm_plan(int64_t m, int32_t count, const int64_t *n, const int64_t *k, int32_t w4,
                                   int32_t sms, convrot_gemm_plan_t *out) {
    if (!out || !n || !k || count < 1 || count > kMaxBatch || m < 1 || sms < 1) return CONVROT_ERR_INVALID_ARG;
    for (int j = 0; j < count; ++j)
        if (n[j] < 1 || k[j] < 1) return CONVROT_ERR_INVALID_ARG;
    if (count > 1 && m > convrot::kMaxSwapM) return CONVROT_ERR_UNSUPPORTED_SHAPE;
    convrot::GemmPlan p;
    if (count == 1)
        convrot::plan_gemm(m, n[0], k[0], sms, &p, w4 != 0);
    else
        convrot::plan_gemm_batch(m, count, n, k, sms, &p, w4 != 0);
    *out = convrot_gemm_plan_t{};
    out->njobs = p.njobs;
    out->swap = p.swap;
    out->bn = p.bn;
    out->grid = p.grid;
    out->full_waves = p.full_waves;
    out->full_tiles = p.full_tiles;
    out->split_ways = p.split_ways;
    out->split_pieces = p.split_pieces;
    out->rep = p.rep > 0 ? p.rep : 1;   // as the launch passes it
    out->stages = p.stages;
    out->tmem_cols = p.tmem_cols;
    out->slots = p.slots;
    out->tail_units = p.tail_units;
    out->smem_bytes = p.smem_bytes;
    out->ws_bytes = (int64_t)p.ws_bytes;
    for (int j = 0; j < p.njobs; ++j) {
        out->tiles_a[j] = p.tiles_a[j];
        out->tiles_b[j] = p.tiles_b[j];
        out->group_a[j] = p.group_a[j];
        out->kbpt[j] = p.kbpt[j];
        out->tile_base[j] = p.tile_base[j];
        out->unit0[j] = p.unit0[j];
    }
    return CONVROT_OK;
}

convrot_status_t convrot_workspace_init(void *ws, size_t ws_bytes, void *stream) {
    if (!ws && ws_bytes) return CONVROT_ERR_INVALID_ARG;
    if (!ws_bytes) return CONVROT_OK;
    return from_cuda(cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)));
}

convrot_status_t convrot_gemm_i8(const int8_t *xq, const float *sx, int64_t m, const convrot_weight_t *w,
                                 void *y_bf16, int32_t *acc, void *ws, size_t ws_bytes, void *stream) {
    if (!xq || !sx || (!y_bf16 && !acc)) return CONVROT_ERR_INVALID_ARG;
    convrot_status_t s = check_weight(w);
    if (s != CONVROT_OK) return s;
    if ((s = check_shape(m, w->k, w->group)) != CONVROT_OK) return s;
    if (!aligned16(xq) || !aligned16(sx) || (y_bf16 && !aligned16(y_bf16)) || (acc && !aligned16(acc)) ||
        (ws && !aligned16(ws)))
        return CONVROT_ERR_ALIGNMENT;
    DeviceInfo dev;
    if ((s = current_device(&dev)) != CONVROT_OK) return s;
    convrot::GemmPlan p;
    convrot::plan_gemm(m, w->n, w->k, dev.num_sms, &p);
    if (p.ws_bytes > 0 && (!ws || ws_bytes < p.ws_bytes)) return CONVROT_ERR_WORKSPACE;
    convrot::GemmProblem prob = {m, w->n, w->k, xq, sx, w->q, w->scale, static_cast<__nv_bfloat16 *>(y_bf16), acc};
    return from_cuda(convrot::launch_gemm_i8(p, &prob, ws, static_cast<cudaStream_t>(stream), false, false));
}

namespace {

bool ranges_overlap(const void *a, size_t an, const void *b, size_t bn) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + bn && b0 < a0 + an;
}

// One linear as the layer entry points see it (INT8 or packed INT4 weight).
struct LinJob {
    const void *x;
    const int8_t *wq;       // int8 [n, k], or INT4 codes [n, k/2] bytes
    const float *sw;
    int64_t n, k;
    int32_t group;
    void *y;
    const void *bias;
};

LinJob lin_job(const convrot_linear_job_t &J) {
    return {J.x_bf16, J.w->q, J.w->scale, J.w->n, J.w->k, J.w->group, J.y_bf16, J.bias_bf16};
}

// Checks common to the layer entry points, after the weights' own checks.
convrot_status_t check_lin_jobs(int64_t m, int count, const LinJob *jobs) {
    for (int j = 0; j < count; ++j) {
        const LinJob &J = jobs[j];
        if (!J.x || !J.y) return CONVROT_ERR_INVALID_ARG;
        convrot_status_t s = check_shape(m, J.k, J.group);
        if (s != CONVROT_OK) return s;
        if (!aligned16(J.x) || !aligned16(J.y) || (J.bias && !aligned16(J.bias))) return CONVROT_ERR_ALIGNMENT;
    }
    // no output may overlap any input or another output: the jobs run as
    // one launch pair, so an output cannot feed a later job
    for (int j = 0; j < count; ++j) {
        const size_t ybytes = (size_t)m * (size_t)jobs[j].n * 2;
        for (int i = 0; i < count; ++i) {
            if (ranges_overlap(jobs[j].y, ybytes, jobs[i].x, (size_t)m * (size_t)jobs[i].k * 2))
                return CONVROT_ERR_INVALID_ARG;
            if (jobs[i].bias && ranges_overlap(jobs[j].y, ybytes, jobs[i].bias, (size_t)jobs[i].n * 2))
                return CONVROT_ERR_INVALID_ARG;
            if (i != j && ranges_overlap(jobs[j].y, ybytes, jobs[i].y, (size_t)m * (size_t)jobs[i].n * 2))
                return CONVROT_ERR_INVALID_ARG;
        }
    }
    return CONVROT_OK;
}

// INT8 jobs -> LinJob array (and the weights' checks).
convrot_status_t collect_jobs(int64_t m, int count, const convrot_linear_job_t *jobs, LinJob *out) {
    if (!jobs || count < 1 || count > kMaxBatch) return CONVROT_ERR_INVALID_ARG;
    for (int j = 0; j < count; ++j) {
        convrot_status_t s = check_weight(jobs[j].w);
        if (s != CONVROT_OK) return s;
        out[j] = lin_job(jobs[j]);
    }
    return check_lin_jobs(m, count, out);
}

convrot_status_t collect_jobs4(int64_t m, int count, const convrot_linear4_job_t *jobs, LinJob *out) {
    if (!jobs || count < 1 || count > kMaxBatch || m < 1) return CONVROT_ERR_INVALID_ARG;
    for (int j = 0; j < count; ++j) {
        const convrot_linear4_job_t &J = jobs[j];
        convrot_status_t s = check_weight4(J.w);
        if (s != CONVROT_OK) return s;
        out[j] = {J.x_bf16, reinterpret_cast<const int8_t *>(J.w->q), J.w->scale, J.w->n, J.w->k, J.w->group,
                  J.y_bf16, J.bias_bf16};
    }
    return check_lin_jobs(m, count, out);
}

// Workspace layout of the layer entry points: [GEMM scratch][xq_0][sx_0][xq_1][sx_1]...
// and, for INT4 weights with per-job GEMMs, [one weight unpacked to INT8].
struct LinearLayout {
    bool batched_gemm;
    convrot::GemmPlan batch;       // when batched_gemm
    size_t gemm_bytes;
    size_t unpack_off, unpack_bytes;
    size_t total;
};

void linear_layout(int64_t m, int count, const LinJob *jobs, bool w4, int sms, LinearLayout *L) {
    L->batched_gemm = m <= convrot::kMaxSwapM;
    size_t g = 0;
    if (L->batched_gemm) {
        int64_t n[kMaxBatch], k[kMaxBatch];
        for (int j = 0; j < count; ++j) {
            n[j] = jobs[j].n;
            k[j] = jobs[j].k;
        }
        convrot::plan_gemm_batch(m, count, n, k, sms, &L->batch, w4);
        g = L->batch.ws_bytes;
    } else {
        for (int j = 0; j < count; ++j) {
            convrot::GemmPlan p;
            convrot::plan_gemm(m, jobs[j].n, jobs[j].k, sms, &p);    // INT4 weights: unpacked first (below)
            g = p.ws_bytes > g ? p.ws_bytes : g;
        }
    }
    L->gemm_bytes = round256(g);
    size_t t = L->gemm_bytes;
    for (int j = 0; j < count; ++j) t += round256((size_t)m * (size_t)jobs[j].k) + round256((size_t)m * 4);
    // INT4 weights beyond the batched sizes: each weight is unpacked to INT8
    // once per call (one HBM pass) and multiplied by the INT8 GEMM, instead
    // of every CTA unpacking every weight tile it reads (shared-memory-bound)
    L->unpack_off = t;
    L->unpack_bytes = 0;
    if (w4 && !L->batched_gemm) {
        size_t mx = 0;
        for (int j = 0; j < count; ++j) {
            const size_t b = (size_t)jobs[j].n * (size_t)jobs[j].k;
            mx = b > mx ? b : mx;
        }
        L->unpack_bytes = round256(mx);
    }
    L->total = t + L->unpack_bytes;
}

convrot_status_t run_linear(int64_t m, int count, const LinJob *jobs, bool w4, void *ws, size_t ws_bytes,
                            cudaStream_t st) {
    if (!ws) return CONVROT_ERR_WORKSPACE;
    if (!aligned16(ws)) return CONVROT_ERR_ALIGNMENT;
    DeviceInfo dev;
    convrot_status_t s = current_device(&dev);
    if (s != CONVROT_OK) return s;
    LinearLayout L;
    linear_layout(m, count, jobs, w4, dev.num_sms, &L);
    if (ws_bytes < L.total) return CONVROT_ERR_WORKSPACE;
    uint8_t *base = static_cast<uint8_t *>(ws);
    convrot::RQProblem rq[kMaxBatch];
    convrot::GemmProblem gp[kMaxBatch];
    size_t off = L.gemm_bytes;
    int nrq = 0;
    for (int j = 0; j < count; ++j) {
        int8_t *xq = reinterpret_cast<int8_t *>(base + off);
        off += round256((size_t)m * (size_t)jobs[j].k);
        float *sx = reinterpret_cast<float *>(base + off);
        off += round256((size_t)m * 4);
        // a job whose input an earlier job already rotates reuses its codes
        int same = -1;
        for (int i = 0; i < j && same < 0; ++i)
            if (jobs[i].x == jobs[j].x && jobs[i].k == jobs[j].k && jobs[i].group == jobs[j].group) same = i;
        if (same >= 0) {
            xq = const_cast<int8_t *>(gp[same].xq);
            sx = const_cast<float *>(gp[same].sx);
        } else {
            rq[nrq++] = {jobs[j].x, jobs[j].k, jobs[j].group, xq, sx, 0};
        }
        gp[j] = {m, jobs[j].n, jobs[j].k, xq, sx, jobs[j].wq, jobs[j].sw, static_cast<__nv_bfloat16 *>(jobs[j].y),
                 nullptr, static_cast<const __nv_bfloat16 *>(jobs[j].bias)};
    }
    cudaError_t e = convrot::launch_rotate_quant(nrq, m, rq, st, true);
    if (e != cudaSuccess) return from_cuda(e);
    if (L.batched_gemm) return from_cuda(convrot::launch_gemm_i8(L.batch, gp, base, st, true, true));
    for (int j = 0; j < count; ++j) {
        convrot::GemmPlan p;
        if (w4) {
            // the unpacked weight is written by the launch just before the
            // GEMM (which waits for it: no weight prefetch ahead of the wait);
            // the unpack itself waits for the previous GEMM, which read the
            // same buffer
            int8_t *wq8 = reinterpret_cast<int8_t *>(base + L.unpack_off);
            e = convrot::launch_unpack_int4(reinterpret_cast<const uint8_t *>(jobs[j].wq), jobs[j].n, jobs[j].k, wq8,
                                            st, true);
            if (e != cudaSuccess) return from_cuda(e);
            gp[j].wq = wq8;
            convrot::plan_gemm(m, jobs[j].n, jobs[j].k, dev.num_sms, &p);
            e = convrot::launch_gemm_i8(p, &gp[j], base, st, true, false);
        } else {
            convrot::plan_gemm(m, jobs[j].n, jobs[j].k, dev.num_sms, &p);
            // the first product may prefetch weights under the prologue; later
            // ones follow another GEMM that could still be reading the scratch
            e = convrot::launch_gemm_i8(p, &gp[j], base, st, true, j == 0);
        }
        if (e != cudaSuccess) return from_cuda(e);
    }
    return CONVROT_OK;
}

}  // namespace

namespace {

convrot_status_t check_gemm_jobs(int64_t m, int count, const convrot_gemm_job_t *jobs) {
    if (!jobs || count < 1 || count > kMaxBatch || m < 1 || m > convrot::kMaxSwapM) return CONVROT_ERR_INVALID_ARG;
    for (int j = 0; j < count; ++j) {
        const convrot_gemm_job_t &J = jobs[j];
        if (!J.xq || !J.sx || (!J.y_bf16 && !J.acc)) return CONVROT_ERR_INVALID_ARG;
        convrot_status_t s = check_weight(J.w);
        if (s != CONVROT_OK) return s;
        if ((s = check_shape(m, J.w->k, J.w->group)) != CONVROT_OK) return s;
        if (!aligned16(J.xq) || !aligned16(J.sx) || (J.y_bf16 && !aligned16(J.y_bf16)) ||
            (J.acc && !aligned16(J.acc)) || (J.bias_bf16 && !aligned16(J.bias_bf16)))
            return CONVROT_ERR_ALIGNMENT;
    }
    return CONVROT_OK;
}

void gemm_batch_plan(int64_t m, int count, const convrot_gemm_job_t *jobs, int sms, convrot::GemmPlan *p) {
    int64_t n[kMaxBatch], k[kMaxBatch];
    for (int j = 0; j < count; ++j) {
        n[j] = jobs[j].w->n;
        k[j] = jobs[j].w->k;
    }
    convrot::plan_gemm_batch(m, count, n, k, sms, p);
}

}  // namespace

size_t convrot_gemm_batch_workspace_bytes(int64_t m, int count, const convrot_gemm_job_t *jobs) {
    if (check_gemm_jobs(m, count, jobs) != CONVROT_OK) return 0;
    convrot::GemmPlan p;
    gemm_batch_plan(m, count, jobs, sms_for_sizing(), &p);
    return round256(p.ws_bytes);
}

convrot_status_t convrot_gemm_i8_batch(int64_t m, int count, const convrot_gemm_job_t *jobs, void *ws,
                                       size_t ws_bytes, void *stream) {
    convrot_status_t s = check_gemm_jobs(m, count, jobs);
    if (s != CONVROT_OK) return s;
    if (ws && !aligned16(ws)) return CONVROT_ERR_ALIGNMENT;
    DeviceInfo dev;
    if ((s = current_device(&dev)) != CONVROT_OK) return s;
    convrot::GemmPlan p;
    gemm_batch_plan(m, count, jobs, dev.num_sms, &p);
    if (!ws || ws_bytes < p.ws_bytes) return CONVROT_ERR_WORKSPACE;
    convrot::GemmProblem gp[kMaxBatch];
    for (int j = 0; j < count; ++j)
        gp[j] = {m, jobs[j].w->n, jobs[j].w->k, jobs[j].xq, jobs[j].sx, jobs[j].w->q, jobs[j].w->scale,
                 static_cast<__nv_bfloat16 *>(jobs[j].y_bf16), jobs[j].acc,
                 static_cast<const __nv_bfloat16 *>(jobs[j].bias_bf16)};
    return from_cuda(convrot::launch_gemm_i8(p, gp, ws, static_cast<cudaStream_t>(stream), false, false));
}

size_t convrot_linear_workspace_bytes(int64_t m, int64_t n, int64_t k) {
    if (m < 1 || n < 1 || k < kMinGroup || k % kMinGroup != 0 || k > kMaxK) return 0;
    LinJob job = {nullptr, nullptr, nullptr, n, k, (int32_t)kGroup, nullptr, nullptr};
    LinearLayout L;
    linear_layout(m, 1, &job, false, sms_for_sizing(), &L);
    return L.total;
}

convrot_status_t convrot_linear_int8(const void *x_bf16, int64_t m, const convrot_weight_t *w, void *y_bf16,
                                     void *ws, size_t ws_bytes, void *stream) {
    convrot_linear_job_t job = {x_bf16, w, y_bf16, nullptr};
    LinJob lj[1];
    convrot_status_t s = collect_jobs(m, 1, &job, lj);
    if (s != CONVROT_OK) return s;
    return run_linear(m, 1, lj, false, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

size_t convrot_linear_batch_workspace_bytes(int64_t m, int count, const convrot_linear_job_t *jobs) {
    LinJob lj[kMaxBatch];
    if (collect_jobs(m, count, jobs, lj) != CONVROT_OK) return 0;
    LinearLayout L;
    linear_layout(m, count, lj, false, sms_for_sizing(), &L);
    return L.total;
}

convrot_status_t convrot_linear_int8_batch(int64_t m, int count, const convrot_linear_job_t *jobs, void *ws,
                                           size_t ws_bytes, void *stream) {
    LinJob lj[kMaxBatch];
    convrot_status_t s = collect_jobs(m, count, jobs, lj);
    if (s != CONVROT_OK) return s;
    return run_linear(m, count, lj, false, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------- INT4 weights (W4A8)
convrot_status_t convrot_weight4_init(convrot_weight4_t *w, uint8_t *q, float *scale, int64_t n, int64_t k,
                                      int32_t group) {
    if (!w) return CONVROT_ERR_INVALID_ARG;
    convrot_weight4_t t = {q, scale, n, k, group};
    convrot_status_t s = check_weight4(&t);
    if (s != CONVROT_OK) return s;
    *w = t;
    return CONVROT_OK;
}

convrot_status_t convrot_quantize_weight4(const void *w_bf16, const convrot_weight4_t *out, void *stream) {
    if (!w_bf16) return CONVROT_ERR_INVALID_ARG;
    convrot_status_t s = check_weight4(out);
    if (s != CONVROT_OK) return s;
    if (!aligned16(w_bf16)) return CONVROT_ERR_ALIGNMENT;
    DeviceInfo dev;
    if ((s = current_device(&dev)) != CONVROT_OK) return s;
    convrot::RQProblem prob = {w_bf16, out->k, out->group, reinterpret_cast<int8_t *>(out->q), out->scale, 1};
    return from_cuda(convrot::launch_rotate_quant(1, out->n, &prob, static_cast<cudaStream_t>(stream), false));
}


size_t convrot_linear_w4a8_workspace_bytes(int64_t m, int count, const convrot_linear4_job_t *jobs) {
    LinJob lj[kMaxBatch];
    if (collect_jobs4(m, count, jobs, lj) != CONVROT_OK) return 0;
    LinearLayout L;
    linear_layout(m, count, lj, true, sms_for_sizing(), &L);
    return L.total;
}

convrot_status_t convrot_linear_w4a8(int64_t m, int count, const convrot_linear4_job_t *jobs, void *ws,
                                     size_t ws_bytes, void *stream) {
    LinJob lj[kMaxBatch];
    convrot_status_t s = collect_jobs4(m, count, jobs, lj);
    if (s != CONVROT_OK) return s;
    return run_linear(m, count, lj, true, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------- convolutions
namespace {
convrot_status_t conv_geom(const convrot_conv2d_t *g, convrot::ConvGeom *cg) {
    if (!g || g->n < 1 || g->h < 1 || g->w < 1 || g->c < 1 || g->kh < 1 || g->kw < 1 || g->stride < 1 ||
        g->pad < 0 || g->dilation < 1)
        return CONVROT_ERR_INVALID_ARG;
    if (g->c % 16 != 0) return CONVROT_ERR_UNSUPPORTED_SHAPE;
    const int64_t oh = ((int64_t)g->h + 2 * g->pad - (int64_t)g->dilation * (g->kh - 1) - 1) / g->stride + 1;
    const int64_t ow = ((int64_t)g->w + 2 * g->pad - (int64_t)g->dilation * (g->kw - 1) - 1) / g->stride + 1;
    if (oh < 1 || ow < 1) return CONVROT_ERR_UNSUPPORTED_SHAPE;
    if ((int64_t)g->n * oh * ow > 0x7FFFFFFF || (int64_t)g->kh * g->kw * g->c > kMaxK ||
        (int64_t)g->n * g->h * g->w * g->c > ((int64_t)1 << 40))
        return CONVROT_ERR_UNSUPPORTED_SHAPE;
    *cg = {0, g->n, g->h, g->w, g->c, g->kh, g->kw, g->stride, g->pad, g->dilation, (int)oh, (int)ow};
    return CONVROT_OK;
}

convrot_status_t check_conv_weight(const convrot_conv2d_t *g, const convrot_weight_t *w, convrot::ConvGeom *cg) {
    convrot_status_t s = conv_geom(g, cg);
    if (s != CONVROT_OK) return s;
    if ((s = check_weight(w)) != CONVROT_OK) return s;
    if (w->k != (int64_t)g->kh * g->kw * g->c || g->c % w->group != 0) return CONVROT_ERR_UNSUPPORTED_SHAPE;
    return CONVROT_OK;
}
}  // namespace

convrot_status_t convrot_conv2d_shape(const convrot_conv2d_t *g, int32_t *oh, int32_t *ow) {
    convrot::ConvGeom cg;
    convrot_status_t s = conv_geom(g, &cg);
    if (s != CONVROT_OK) return s;
    if (oh) *oh = cg.oh;
    if (ow) *ow = cg.ow;
    return CONVROT_OK;
}

convrot_status_t convrot_conv2d_gather_plan(const convrot_conv2d_t *g, int32_t sms, convrot_conv2d_plan_t *out) {
    if (!out || sms < 1) return CONVROT_ERR_INVALID_ARG;
    convrot::ConvGeom cg;
    convrot_status_t s = conv_geom(g, &cg);
    if (s != CONVROT_OK) return s;
    if (cg.kh * cg.kw == 1) return CONVROT_ERR_UNSUPPORTED_SHAPE;
    *out = convrot_conv2d_plan_t{};
    int th, tw, rh, rw;
    int64_t tiles, bytes;
    if (convrot::conv_gather_tile_plan(cg, sms, &th, &tw, &rh, &rw, &tiles, &bytes)) {
        out->tiled = 1;
        out->th = th;
        out->tw = tw;
        out->rh = rh;
        out->rw = rw;
        out->tiles = tiles;
        out->buf_bytes = bytes;
    }
    return CONVROT_OK;
}

convrot_status_t convrot_quantize_conv_weight(const void *w_oihw_bf16, const convrot_conv2d_t *g,
                                              const convrot_weight_t *out, void *stream) {
    if (!w_oihw_bf16) return CONVROT_ERR_INVALID_ARG;
    convrot::ConvGeom cg;
    convrot_status_t s = check_conv_weight(g, out, &cg);
    if (s != CONVROT_OK) return s;
    if ((reinterpret_cast<uintptr_t>(w_oihw_bf16) & 1u) != 0) return CONVROT_ERR_ALIGNMENT;
    DeviceInfo dev;
    if ((s = current_device(&dev)) != CONVROT_OK) return s;
    cg.mode = 4;
    convrot::RQProblem prob = {w_oihw_bf16, out->k, out->group, out->q, out->scale, 0};
    return from_cuda(convrot::launch_rotate_quant(1, out->n, &prob, static_cast<cudaStream_t>(stream), false, &cg));
}

namespace {
// Workspace: [GEMM scratch][xq M x K][sx M] and, for kernels larger than
// 1x1, [every pixel rotated once: FP32 n*h*w x c][the pixels' maxima].
bool conv_two_pass(const convrot::ConvGeom &cg) { return cg.kh * cg.kw > 1; }

size_t conv_layout(const convrot::ConvGeom &cg, const convrot_weight_t *w, int sms, convrot::GemmPlan *p,
                   size_t *gemm_bytes) {
    const int64_t m = (int64_t)cg.n * cg.oh * cg.ow;
    convrot::plan_gemm(m, w->n, w->k, sms, p);
    *gemm_bytes = round256(p->ws_bytes);
    size_t t = *gemm_bytes + round256((size_t)m * (size_t)w->k) + round256((size_t)m * 4);
    if (conv_two_pass(cg)) {
        const size_t pix = (size_t)cg.n * cg.h * cg.w;
        t += round256(pix * (size_t)cg.c * 4) + round256(pix * 4);
    }
    return t;
}
}  // namespace

size_t convrot_conv2d_workspace_bytes(const convrot_conv2d_t *g, const convrot_weight_t *w) {
    convrot::ConvGeom cg;
    if (check_conv_weight(g, w, &cg) != CONVROT_OK) return 0;
    convrot::GemmPlan p;
    size_t gb;
    return conv_layout(cg, w, sms_for_sizing(), &p, &gb);
}

convrot_status_t convrot_conv2d_int8(const void *x_nhwc_bf16, const convrot_conv2d_t *g, const convrot_weight_t *w,
                                     void *y_nhwc_bf16, void *ws, size_t ws_bytes, void *stream) {
    if (!x_nhwc_bf16 || !y_nhwc_bf16) return CONVROT_ERR_INVALID_ARG;
    convrot::ConvGeom cg;
    convrot_status_t s = check_conv_weight(g, w, &cg);
    if (s != CONVROT_OK) return s;
    if (!aligned16(x_nhwc_bf16) || !aligned16(y_nhwc_bf16)) return CONVROT_ERR_ALIGNMENT;
    if (!ws) return CONVROT_ERR_WORKSPACE;
    if (!aligned16(ws)) return CONVROT_ERR_ALIGNMENT;
    const int64_t m = (int64_t)cg.n * cg.oh * cg.ow;
    if (ranges_overlap(y_nhwc_bf16, (size_t)m * (size_t)w->n * 2, x_nhwc_bf16,
                       (size_t)g->n * g->h * g->w * g->c * 2))
        return CONVROT_ERR_INVALID_ARG;
    DeviceInfo dev;
    if ((s = current_device(&dev)) != CONVROT_OK) return s;
    convrot::GemmPlan p;
    size_t gb;
    if (ws_bytes < conv_layout(cg, w, dev.num_sms, &p, &gb)) return CONVROT_ERR_WORKSPACE;
    uint8_t *base = static_cast<uint8_t *>(ws);
    int8_t *xq = reinterpret_cast<int8_t *>(base + gb);
    float *sx = reinterpret_cast<float *>(base + gb + round256((size_t)m * (size_t)w->k));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (conv_two_pass(cg)) {
        // every input pixel rotated once (its C channels, FP32) with its
        // maximum; then the im2col rows gathered from them and quantised
        const size_t pix = (size_t)cg.n * cg.h * cg.w;
        float *yrot = reinterpret_cast<float *>(base + gb + round256((size_t)m * (size_t)w->k) + round256((size_t)m * 4));
        float *pmax = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(yrot) + round256(pix * (size_t)cg.c * 4));
        cg.mode = 5;
        convrot::RQProblem rq = {x_nhwc_bf16, g->c, w->group, reinterpret_cast<int8_t *>(yrot), pmax, 0};
        e = convrot::launch_rotate_quant(1, (int64_t)pix, &rq, st, true, &cg);
        if (e != cudaSuccess) return from_cuda(e);
        e = convrot::launch_conv_gather_quant(yrot, pmax, cg, m, xq, sx, st);
        if (e != cudaSuccess) return from_cuda(e);
    } else {
        cg.mode = 3;
        convrot::RQProblem rq = {x_nhwc_bf16, w->k, w->group, xq, sx, 0};
        e = convrot::launch_rotate_quant(1, m, &rq, st, true, &cg);
        if (e != cudaSuccess) return from_cuda(e);
    }
    convrot::GemmProblem gp = {m, w->n, w->k, xq, sx, w->q, w->scale, static_cast<__nv_bfloat16 *>(y_nhwc_bf16),
                               nullptr, nullptr};
    return from_cuda(convrot::launch_gemm_i8(p, &gp, base, st, true, true));
}

convrot_status_t convrot_quantize_tensor(const void *w_bf16, int64_t count, int8_t *q, float *scale,
                                         void *stream) {
    if (!w_bf16 || !q || !scale || count < 16) return CONVROT_ERR_INVALID_ARG;
    if (count % 16 != 0) return CONVROT_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(w_bf16) || !aligned16(q) || (reinterpret_cast<uintptr_t>(scale) & 3u) != 0)
        return CONVROT_ERR_ALIGNMENT;
    if (ranges_overlap(scale, 4, w_bf16, (size_t)count * 2) || ranges_overlap(scale, 4, q, (size_t)count))
        return CONVROT_ERR_INVALID_ARG;
    DeviceInfo dev;
    convrot_status_t s = current_device(&dev);
    if (s != CONVROT_OK) return s;
    return from_cuda(convrot::launch_quantize_tensor(w_bf16, count, q, scale, static_cast<cudaStream_t>(stream)));
}

convrot_status_t convrot_embed_lookup(const int32_t *tokens, int64_t t, const int8_t *q, const float *scale,
                                      int64_t vocab, int64_t dim, void *out_bf16, void *stream) {
    if (!tokens || !q || !scale || !out_bf16 || t < 1 || vocab < 1 || dim < 16) return CONVROT_ERR_INVALID_ARG;
    if (dim % 16 != 0) return CONVROT_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(q) || !aligned16(out_bf16) || (reinterpret_cast<uintptr_t>(tokens) & 3u) != 0 ||
        (reinterpret_cast<uintptr_t>(scale) & 3u) != 0)
        return CONVROT_ERR_ALIGNMENT;
    DeviceInfo dev;
    convrot_status_t s = current_device(&dev);
    if (s != CONVROT_OK) return s;
    return from_cuda(convrot::launch_embed_lookup(tokens, t, q, scale, vocab, dim, out_bf16,
                                                  static_cast<cudaStream_t>(stream)));
}

convrot_status_t convrot_device_status(void *stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) {
        cudaGetLastError();
        return CONVROT_ERR_CUDA;
    }
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, convrot::g_device_status, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return CONVROT_ERR_CUDA;
    }
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(convrot::g_device_status, &zero, sizeof(int)) != cudaSuccess) {
            cudaGetLastError();
            return CONVROT_ERR_CUDA;
        }
        return static_cast<convrot_status_t>(v);
    }
    return CONVROT_OK;
}

}  // extern "C"
#pragma GCC visibility pop
