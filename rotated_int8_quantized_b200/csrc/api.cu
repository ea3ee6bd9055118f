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

namespace {

constexpr int64_t kGroup = 256;
// |acc| <= k * 127^2 must fit in INT32: k <= 133144; largest multiple of 256.
constexpr int64_t kMaxK = 133120;
constexpr int64_t kMaxRows = 0x7FFFFFFF;
constexpr int kDefaultSms = 148;

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

convrot_status_t check_shape(int64_t rows, int64_t k, int64_t group) {
    if (rows < 1 || k < 1) return CONVROT_ERR_INVALID_ARG;
    if (group != kGroup) return CONVROT_ERR_UNSUPPORTED_SHAPE;
    if (k % kGroup != 0 || k > kMaxK || rows > kMaxRows) return CONVROT_ERR_UNSUPPORTED_SHAPE;
    return CONVROT_OK;
}

convrot_status_t check_weight(const convrot_weight_t *w) {
    if (!w || !w->q || !w->scale) return CONVROT_ERR_INVALID_ARG;
    convrot_status_t s = check_shape(w->n, w->k, w->group);
    if (s != CONVROT_OK) return s;
    if (!aligned16(w->q) || !aligned16(w->scale)) return CONVROT_ERR_ALIGNMENT;
    return CONVROT_OK;
}

convrot_status_t from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return CONVROT_OK;
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
    }
    return "CONVROT_ERR_UNKNOWN";
}

int convrot_version(void) { return 100; }

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
    return from_cuda(convrot::launch_rotate_quant(w_bf16, out->n, out->k, out->q, out->scale,
                                                  static_cast<cudaStream_t>(stream), false));
}

convrot_status_t convrot_quantize_act(const void *x_bf16, int64_t m, int64_t k, int32_t group, int8_t *xq,
                                      float *sx, void *stream) {
    if (!x_bf16 || !xq || !sx) return CONVROT_ERR_INVALID_ARG;
    convrot_status_t s = check_shape(m, k, group);
    if (s != CONVROT_OK) return s;
    if (!aligned16(x_bf16) || !aligned16(xq) || !aligned16(sx)) return CONVROT_ERR_ALIGNMENT;
    DeviceInfo dev;
    if ((s = current_device(&dev)) != CONVROT_OK) return s;
    return from_cuda(convrot::launch_rotate_quant(x_bf16, m, k, xq, sx, static_cast<cudaStream_t>(stream), false));
}

size_t convrot_gemm_workspace_bytes(int64_t m, int64_t n, int64_t k) {
    if (m < 1 || n < 1 || k < kGroup) return 0;
    convrot::GemmPlan p;
    convrot::plan_gemm(m, n, k, sms_for_sizing(), &p);
    return round256(p.ws_bytes);
}

size_t convrot_linear_workspace_bytes(int64_t m, int64_t n, int64_t k) {
    if (m < 1 || n < 1 || k < kGroup) return 0;
    return convrot_gemm_workspace_bytes(m, n, k) + round256((size_t)m * (size_t)k) + round256((size_t)m * 4);
}

convrot_status_t convrot_workspace_init(void *ws, size_t ws_bytes, void *stream) {
    if (!ws && ws_bytes) return CONVROT_ERR_INVALID_ARG;
    if (!ws_bytes) return CONVROT_OK;
    return from_cuda(cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)));
}

static convrot_status_t gemm_impl(const int8_t *xq, const float *sx, int64_t m, const convrot_weight_t *w,
                                  void *y, int32_t *acc, void *ws, size_t ws_bytes, cudaStream_t stream,
                                  bool pdl, bool w_prefetch) {
    DeviceInfo dev;
    convrot_status_t s = current_device(&dev);
    if (s != CONVROT_OK) return s;
    convrot::GemmPlan p;
    convrot::plan_gemm(m, w->n, w->k, dev.num_sms, &p);
    if (p.ws_bytes > 0 && (!ws || ws_bytes < p.ws_bytes)) return CONVROT_ERR_WORKSPACE;
    return from_cuda(convrot::launch_gemm_i8(p, xq, sx, m, w->q, w->scale, w->n, w->k,
                                             static_cast<__nv_bfloat16 *>(y), acc, ws, stream, pdl, w_prefetch));
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
    return gemm_impl(xq, sx, m, w, y_bf16, acc, ws, ws_bytes, static_cast<cudaStream_t>(stream), false, false);
}

convrot_status_t convrot_linear_int8(const void *x_bf16, int64_t m, const convrot_weight_t *w, void *y_bf16,
                                     void *ws, size_t ws_bytes, void *stream) {
    if (!x_bf16 || !y_bf16 || !ws) return CONVROT_ERR_INVALID_ARG;
    convrot_status_t s = check_weight(w);
    if (s != CONVROT_OK) return s;
    if ((s = check_shape(m, w->k, w->group)) != CONVROT_OK) return s;
    if (!aligned16(x_bf16) || !aligned16(y_bf16) || !aligned16(ws)) return CONVROT_ERR_ALIGNMENT;
    const size_t need = convrot_linear_workspace_bytes(m, w->n, w->k);
    DeviceInfo dev;
    if ((s = current_device(&dev)) != CONVROT_OK) return s;
    convrot::GemmPlan p;
    convrot::plan_gemm(m, w->n, w->k, dev.num_sms, &p);
    const size_t gemm_ws = round256(p.ws_bytes);
    const size_t need_here = gemm_ws + round256((size_t)m * (size_t)w->k) + round256((size_t)m * 4);
    if (ws_bytes < need_here || ws_bytes < need) return CONVROT_ERR_WORKSPACE;
    uint8_t *base = static_cast<uint8_t *>(ws);
    int8_t *xq = reinterpret_cast<int8_t *>(base + gemm_ws);
    float *sx = reinterpret_cast<float *>(base + gemm_ws + round256((size_t)m * (size_t)w->k));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = convrot::launch_rotate_quant(x_bf16, m, w->k, xq, sx, st, true);
    if (e != cudaSuccess) return from_cuda(e);
    return from_cuda(convrot::launch_gemm_i8(p, xq, sx, m, w->q, w->scale, w->n, w->k,
                                             static_cast<__nv_bfloat16 *>(y_bf16), nullptr, base, st, true, true));
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
