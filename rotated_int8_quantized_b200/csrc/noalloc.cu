// noalloc.cu -- convrot_gemm_i8_noalloc: the INT8 GEMM for callers that
// cannot hand the library a device workspace.
//
// Some callers cannot allocate device memory at the point where they run
// the layer: a plugin inside an engine that owns every byte of device memory
// through its own pool and forbids outside cudaMalloc calls, or code on a
// latency-critical path that must not risk cudaMalloc's implicit device
// synchronisation.  For them this entry point keeps the GEMM's scratch (the
// stream-K ticket counters and INT32 partial tiles) in a fixed array that
// lives in the library's own device memory, so the call needs only its
// inputs and outputs.
//
// The array holds kStaticScratchBytes (8 MiB) on every GPU that loads the
// library, until the process exits.  Problems whose scratch would not fit
// are rejected with CONVROT_ERR_WORKSPACE before anything is launched.
// Every call on a device uses the same array, so calls whose GPU work
// overlaps (different streams, or host threads racing) corrupt each other.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

namespace {

constexpr size_t kStaticScratchBytes = 8u << 20;

// The scratch itself.  Host code cannot use this name as a device address;
// the address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the array on the current device, looked up once per
// device (with that device current) and cached.
convrot_status_t static_scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return CONVROT_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess || !p) return from_cuda(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return CONVROT_OK;
}

}  // namespace

#pragma GCC visibility push(default)
extern "C" {

convrot_status_t convrot_gemm_i8_noalloc(const int8_t *xq, const float *sx, int64_t m, const convrot_weight_t *w,
                                         void *y_bf16, int32_t *acc, void *stream) {
    if (!xq || !sx || (!y_bf16 && !acc)) return CONVROT_ERR_INVALID_ARG;
    convrot_status_t s = check_weight(w);
    if (s != CONVROT_OK) return s;
    if ((s = check_shape(m, w->k, w->group)) != CONVROT_OK) return s;
    if (!aligned16(xq) || !aligned16(sx) || (y_bf16 && !aligned16(y_bf16)) || (acc && !aligned16(acc)))
        return CONVROT_ERR_ALIGNMENT;
    DeviceInfo dev;
    if ((s = current_device(&dev)) != CONVROT_OK) return s;
    convrot::GemmPlan p;
    convrot::plan_gemm(m, w->n, w->k, dev.num_sms, &p);
    if (p.ws_bytes > kStaticScratchBytes) {
        t_last_error = "the problem needs more scratch than the 8 MiB built into convrot_gemm_i8_noalloc";
        return CONVROT_ERR_WORKSPACE;
    }
    void *scratch = nullptr;
    if ((s = static_scratch_address(&scratch)) != CONVROT_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the counters and partial tiles must start at zero; the previous call
    // left them zero unless it failed, so clear them every time
    if (p.ws_bytes > 0) {
        cudaError_t e = cudaMemsetAsync(scratch, 0, p.ws_bytes, st);
        if (e != cudaSuccess) return from_cuda(e);
    }
    convrot::GemmProblem prob = {m, w->n, w->k, xq, sx, w->q, w->scale, static_cast<__nv_bfloat16 *>(y_bf16), acc};
    return from_cuda(convrot::launch_gemm_i8(p, &prob, scratch, st, false, false));
}

}  // extern "C"
#pragma GCC visibility pop
