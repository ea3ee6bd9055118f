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
// library's module, until the process exits -- also in processes that
// never call this entry point, since the array is part of the library's one
// module.  Problems whose scratch would not fit are rejected with
// CONVROT_ERR_WORKSPACE before anything is launched.  Every call on a
// device uses the same array, so calls whose GPU work overlaps (different
// streams, or host threads racing) corrupt each other.
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

namespace {

constexpr size_t kStaticScratchBytes = 8u << 20;

// The scratch itself.  Host code cannot use this name as a device address;
// the address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

// The array's address belongs to the module loaded in one CUDA context: a
// cudaDeviceReset (or any teardown of the primary context) unloads the
// module, and the next context may place the array elsewhere.  So the
// cached address is keyed on the current context's unique id, not on the
// device index, and is looked up again whenever the id changes.
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

struct ScratchEntry {
    unsigned long long ctx_id;   // 0: empty
    void *addr;
};
constexpr int kScratchEntries = 64;
std::mutex g_scratch_mutex;
ScratchEntry g_scratch_cache[kScratchEntries] = {};

// Unique id of the current context, 0 if none is current or the driver
// entry points are unavailable.
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static bool looked_up = false;
    if (!looked_up) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
        cudaGetLastError();
        looked_up = true;
    }
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of the array in the current context.  The first call in
// a context looks it up with cudaGetSymbolAddress (which may load the
// library's module into that context); later calls in the same context
// reuse it.  Without a context id (no driver entry points) every call looks
// it up.
convrot_status_t static_scratch_address(void **out) {
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    unsigned long long id = current_context_id();
    if (id != 0) {
        for (int i = 0; i < kScratchEntries; ++i) {
            if (g_scratch_cache[i].ctx_id == id) {
                *out = g_scratch_cache[i].addr;
                return CONVROT_OK;
            }
        }
    }
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || !p) return from_cuda(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
    // the lookup makes the context current if none was: take its id now
    if (id == 0) id = current_context_id();
    if (id != 0) {
        int slot = (int)(id % kScratchEntries);     // table full: overwrite one entry
        for (int i = 0; i < kScratchEntries; ++i) {
            if (g_scratch_cache[i].ctx_id == 0) {
                slot = i;
                break;
            }
        }
        g_scratch_cache[slot] = {id, p};
    }
    *out = p;
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
