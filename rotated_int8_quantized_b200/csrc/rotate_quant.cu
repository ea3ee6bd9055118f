// rotate_quant.cu -- grouped Hadamard rotation fused with row-wise INT8
// round-to-nearest quantisation, for activations (per call) and weights
// (offline).  Both are the same operation on the rows of a BF16 matrix:
//
//   y[r, g*256 + j] = fp32( (sum_i a[r, g*256 + i] * H[i][j]) / 16 )
//   s[r] = max_j |y[r, j]| / 127;   q[r, j] = clamp(rne(y / s), -127, 127)
//
// [0539edu.com "minimax-h3-nvfp4-convrot", section 4 "INT8 ConvRot":
//  Hadamard pre-rotation in fixed groups of 256 before quantisation;
//  section 5: activations and weights both rotated, "--simple" RTN;
//  zskr.cn "Qwen3-VL-32B ... INT8-ConvRot": "--int8 --scaling_mode row"]
//
// Design (B200): one warp rotates one 256-wide group.  Each lane loads 8
// consecutive BF16 values with one 16-byte load (the warp reads the group's
// 512 bytes fully coalesced), widens them to FP64 and runs the fast
// Walsh-Hadamard transform: three butterfly stages inside the lane (index
// bits 0-2) and five across lanes with xor-shuffles (index bits 3-7).  Every
// partial sum of +-BF16 values is exact in FP64, so the butterfly order
// gives the same exact sum as the explicit matrix product, and one rounding
// to FP32 follows.  The row's rotated FP32 values wait in shared memory
// while the CTA reduces the row maximum; then each thread packs 16 INT8
// codes into one 16-byte store.  Rows too long for shared memory take a
// two-pass variant that recomputes the (cheap, L2-resident) rotation.
#include <cstdint>
#include <cstring>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "gemm_i8.h"

namespace convrot {

constexpr int kRQThreads = 256;
constexpr int kRQWarps = kRQThreads / 32;

// In-place unnormalised Walsh-Hadamard transform of one 256-group held as
// 8 values per lane (lane L holds elements 8L .. 8L+7).  Natural (Sylvester)
// order: y_j = sum_i x_i * (-1)^popcount(i & j).
__device__ __forceinline__ void fwht256_warp(double (&v)[8], int lane) {
#pragma unroll
    for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if ((e & h) == 0) {
                double a = v[e], b = v[e + h];
                v[e] = a + b;
                v[e + h] = a - b;
            }
        }
    }
#pragma unroll
    for (int lm = 1; lm < 32; lm <<= 1) {
        const bool upper = (lane & lm) != 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            double p = __shfl_xor_sync(0xffffffffu, v[e], lm);
            v[e] = upper ? (p - v[e]) : (v[e] + p);
        }
    }
}

// Load 8 BF16 (one 16-byte vector) and widen to FP64 (exact).
__device__ __forceinline__ void load8_bf16_as_f64(const __nv_bfloat16 *p, double (&v)[8]) {
    uint4 raw = __ldg(reinterpret_cast<const uint4 *>(p));
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = (double)__uint_as_float(w[i] << 16);
        v[2 * i + 1] = (double)__uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// Rotate one group: returns the 8 FP32 outputs of this lane.
__device__ __forceinline__ void rotate_group(const __nv_bfloat16 *grp, int lane, float (&y)[8]) {
    double v[8];
    load8_bf16_as_f64(grp + lane * 8, v);
    fwht256_warp(v, lane);
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] = __double2float_rn(v[e] * 0.0625);   // / sqrt(256), exact
}

__device__ __forceinline__ float block_max(float v, float *red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float r = red[0];
#pragma unroll
    for (int w = 1; w < kRQWarps; ++w) r = fmaxf(r, red[w]);
    return r;
}

__device__ __forceinline__ int8_t quant1(float y, float s, bool zero_row) {
    if (zero_row) return 0;
    int q = __float2int_rn(__fdiv_rn(y, s));
    q = q > 127 ? 127 : (q < -127 ? -127 : q);
    return (int8_t)q;
}

// One CTA per row, no staging: pass 1 finds the row maximum, pass 2
// recomputes the rotation (the row is L2-resident) and quantises.
__global__ void __launch_bounds__(kRQThreads) rotate_quant_rows_twopass(
    const __nv_bfloat16 *__restrict__ a, int k, int8_t *__restrict__ q, float *__restrict__ s) {
    __shared__ float red[kRQWarps];
    pdl_wait();
    pdl_launch_dependents();
    const int row = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const __nv_bfloat16 *arow = a + (size_t)row * k;
    const int groups = k >> 8;
    float amax = 0.f;
    for (int g = warp; g < groups; g += kRQWarps) {
        float y[8];
        rotate_group(arow + g * 256, lane, y);
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(y[e]));
    }
    amax = block_max(amax, red);
    const float sc = __fdiv_rn(amax, 127.0f);
    const bool zero_row = (amax == 0.0f);
    int8_t *qrow = q + (size_t)row * k;
    for (int g = warp; g < groups; g += kRQWarps) {
        float y[8];
        rotate_group(arow + g * 256, lane, y);
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) lo |= (uint32_t)(uint8_t)quant1(y[e], sc, zero_row) << (8 * e);
#pragma unroll
        for (int e = 0; e < 4; ++e) hi |= (uint32_t)(uint8_t)quant1(y[4 + e], sc, zero_row) << (8 * e);
        *reinterpret_cast<uint2 *>(qrow + g * 256 + lane * 8) = make_uint2(lo, hi);
    }
    if (threadIdx.x == 0) s[row] = sc;
}

// ---------------------------------------------------------------------------
// Main variant: 16 threads ("a slot") per 256-group, H_256 = H_16 (x) H_16.
// Thread t of a slot loads elements 16t .. 16t+15 (32 contiguous bytes; the
// slot reads the group's 512 bytes coalesced), transforms index bits 0-3 in
// registers, exchanges through a padded shared-memory transpose (stride 17
// doubles: conflict-free both ways), transforms index bits 4-7 in registers
// and so ends up holding outputs t, t+16, ..., t+240.  Every group of a row
// is in flight at once (up to 32 slots per CTA, several groups per slot for
// long rows), so a decode-sized matrix of a few rows costs one load latency.
// ---------------------------------------------------------------------------
constexpr int kMaxSlots = 32;          // 512 threads
constexpr int kXchStride = 16 * 17;    // doubles per slot exchange buffer
constexpr int kSlotsSmemMax = 226 * 1024;   // dynamic shared memory per CTA (227 KB minus the static part)

__device__ __forceinline__ void fwht16_regs(double (&v)[16]) {
#pragma unroll
    for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            if ((e & h) == 0) {
                double a = v[e], b = v[e + h];
                v[e] = a + b;
                v[e + h] = a - b;
            }
        }
    }
}

__device__ __forceinline__ void bf16x2_to_f64(uint32_t w, double &lo, double &hi) {
    lo = (double)__uint_as_float(w << 16);
    hi = (double)__uint_as_float(w & 0xFFFF0000u);
}

struct RQJobDev {
    const __nv_bfloat16 *a;
    int8_t *q;
    float *s;
    int k, gps, slots;
};
struct RQArgs {
    int njobs, rows;
    RQJobDev job[kMaxJobs];
};

// Groups per slot and slots for a row of k elements.
static void rq_shape(int64_t k, int *gps, int *slots) {
    const int groups = (int)(k >> 8);
    int g = (groups + kMaxSlots - 1) / kMaxSlots;
    if (g == 5) g = 6;
    *gps = g;
    *slots = (groups + g - 1) / g;
}

template <int GPS>
__global__ void __launch_bounds__(kMaxSlots * 16, 1) rotate_quant_rows_slots(const __grid_constant__ RQArgs args) {
    extern __shared__ __align__(16) uint8_t rq_smem[];
    __shared__ float red[kMaxSlots / 2];
    pdl_wait();
    pdl_launch_dependents();

    const int jb = blockIdx.x / args.rows;
    const int row = blockIdx.x - jb * args.rows;
    const RQJobDev &J = args.job[jb];
    const int k = J.k, gps = J.gps, slots = J.slots;
    double *xch = reinterpret_cast<double *>(rq_smem);                    // slots * 272 doubles
    float *ybuf = reinterpret_cast<float *>(rq_smem + (size_t)(blockDim.x >> 4) * kXchStride * 8);  // k floats

    const int tid = threadIdx.x;
    const int slot = tid >> 4, t = tid & 15;
    const int groups = k >> 8;
    const unsigned half_mask = 0xFFFFu << (16 * (slot & 1));
    const __nv_bfloat16 *arow = J.a + (size_t)row * k;

    // issue every load of this thread first
    uint4 raw[GPS][2];
#pragma unroll
    for (int gi = 0; gi < GPS; ++gi) {
        const int g = slot + gi * slots;
        if (gi < gps && slot < slots && g < groups) {
            const uint4 *src = reinterpret_cast<const uint4 *>(arow + (size_t)g * 256 + t * 16);
            raw[gi][0] = __ldg(src);
            raw[gi][1] = __ldg(src + 1);
        }
    }

    double *xb = xch + slot * kXchStride;
    float amax = 0.f;
#pragma unroll
    for (int gi = 0; gi < GPS; ++gi) {
        const int g = slot + gi * slots;
        if (gi < gps && slot < slots && g < groups) {
            double v[16];
            const uint32_t w[8] = {raw[gi][0].x, raw[gi][0].y, raw[gi][0].z, raw[gi][0].w,
                                   raw[gi][1].x, raw[gi][1].y, raw[gi][1].z, raw[gi][1].w};
#pragma unroll
            for (int i = 0; i < 8; ++i) bf16x2_to_f64(w[i], v[2 * i], v[2 * i + 1]);
            fwht16_regs(v);                                  // index bits 0-3
#pragma unroll
            for (int i = 0; i < 16; ++i) xb[17 * t + i] = v[i];
            __syncwarp(half_mask);
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = xb[t + 17 * i];
            __syncwarp(half_mask);
            fwht16_regs(v);                                  // index bits 4-7
            float *yg = ybuf + (size_t)g * 256 + t;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float y = __double2float_rn(v[i] * 0.0625);   // / sqrt(256), exact
                yg[16 * i] = y;
                amax = fmaxf(amax, fabsf(y));
            }
        }
    }

    // row maximum
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const int warp = tid >> 5, lane = tid & 31, nwarps = (blockDim.x + 31) >> 5;
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    float rmax = red[0];
    for (int w = 1; w < nwarps; ++w) rmax = fmaxf(rmax, red[w]);
    const float sc = __fdiv_rn(rmax, 127.0f);
    const bool zero_row = (rmax == 0.0f);

    // quantise 16 consecutive outputs per thread, one 16-byte store
    int8_t *qrow = J.q + (size_t)row * k;
    for (int c = tid; c < (k >> 4); c += blockDim.x) {
        const float4 *src = reinterpret_cast<const float4 *>(ybuf + c * 16);
        uint32_t packed[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float4 f = src[i];
            uint32_t b0 = (uint8_t)quant1(f.x, sc, zero_row);
            uint32_t b1 = (uint8_t)quant1(f.y, sc, zero_row);
            uint32_t b2 = (uint8_t)quant1(f.z, sc, zero_row);
            uint32_t b3 = (uint8_t)quant1(f.w, sc, zero_row);
            packed[i] = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
        }
        *reinterpret_cast<uint4 *>(qrow + c * 16) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
    if (tid == 0) J.s[row] = sc;
}

template <int GPS>
static cudaError_t launch_slots(cudaLaunchConfig_t &cfg, const RQArgs &args, int max_slots, int64_t max_k) {
    cfg.blockDim = dim3(max_slots * 16);
    cfg.dynamicSmemBytes = (size_t)max_slots * kXchStride * 8 + (size_t)max_k * 4;
    static bool configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !configured[dev]) {
        e = cudaFuncSetAttribute(rotate_quant_rows_slots<GPS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSlotsSmemMax);
        if (e != cudaSuccess) return e;
        if (dev < 64) configured[dev] = true;
    }
    return cudaLaunchKernelEx(&cfg, rotate_quant_rows_slots<GPS>, args);
}

// Shared-memory bytes one CTA of a batched launch needs.
static size_t rq_smem_bytes(int njobs, const RQProblem *probs, int *max_slots, int *max_gps, int64_t *max_k) {
    int ms = 0, mg = 0;
    int64_t mk = 0;
    for (int j = 0; j < njobs; ++j) {
        int g, sl;
        rq_shape(probs[j].k, &g, &sl);
        ms = sl > ms ? sl : ms;
        mg = g > mg ? g : mg;
        mk = probs[j].k > mk ? probs[j].k : mk;
    }
    *max_slots = ms;
    *max_gps = mg;
    *max_k = mk;
    return (size_t)ms * kXchStride * 8 + (size_t)mk * 4;
}

bool rotate_quant_batchable(int njobs, const RQProblem *probs) {
    int ms, mg;
    int64_t mk;
    return njobs <= kMaxJobs && rq_smem_bytes(njobs, probs, &ms, &mg, &mk) <= (size_t)kSlotsSmemMax;
}

cudaError_t launch_rotate_quant(int njobs, int64_t rows, const RQProblem *probs, cudaStream_t stream, bool pdl) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)(rows * njobs));
    cfg.blockDim = dim3(kRQThreads);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    int max_slots, max_gps;
    int64_t max_k;
    if (njobs <= kMaxJobs && rq_smem_bytes(njobs, probs, &max_slots, &max_gps, &max_k) <= (size_t)kSlotsSmemMax) {
        RQArgs args;
        memset(&args, 0, sizeof(args));
        args.njobs = njobs;
        args.rows = (int)rows;
        for (int j = 0; j < njobs; ++j) {
            RQJobDev &J = args.job[j];
            J.a = static_cast<const __nv_bfloat16 *>(probs[j].a);
            J.q = probs[j].q;
            J.s = probs[j].s;
            J.k = (int)probs[j].k;
            rq_shape(probs[j].k, &J.gps, &J.slots);
        }
        switch (max_gps) {
            case 1: return launch_slots<1>(cfg, args, max_slots, max_k);
            case 2: return launch_slots<2>(cfg, args, max_slots, max_k);
            case 3: return launch_slots<3>(cfg, args, max_slots, max_k);
            case 4: return launch_slots<4>(cfg, args, max_slots, max_k);
            default: return launch_slots<6>(cfg, args, max_slots, max_k);
        }
    }
    // rows too long to stage: one launch per matrix, rotation recomputed in a second pass
    cfg.dynamicSmemBytes = 0;
    cfg.gridDim = dim3((unsigned)rows);
    for (int j = 0; j < njobs; ++j) {
        cudaError_t e = cudaLaunchKernelEx(&cfg, rotate_quant_rows_twopass,
                                           static_cast<const __nv_bfloat16 *>(probs[j].a), (int)probs[j].k,
                                           probs[j].q, probs[j].s);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace convrot
