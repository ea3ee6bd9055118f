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
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"

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

// One CTA per row; the rotated row is staged in shared memory (k floats).
__global__ void __launch_bounds__(kRQThreads) rotate_quant_rows_smem(
    const __nv_bfloat16 *__restrict__ a, int k, int8_t *__restrict__ q, float *__restrict__ s) {
    extern __shared__ float ybuf[];
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
        float4 *dst = reinterpret_cast<float4 *>(ybuf + g * 256 + lane * 8);
        dst[0] = make_float4(y[0], y[1], y[2], y[3]);
        dst[1] = make_float4(y[4], y[5], y[6], y[7]);
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(y[e]));
    }
    amax = block_max(amax, red);   // contains __syncthreads: ybuf complete
    const float sc = __fdiv_rn(amax, 127.0f);
    const bool zero_row = (amax == 0.0f);
    int8_t *qrow = q + (size_t)row * k;
    for (int c = threadIdx.x; c < (k >> 4); c += kRQThreads) {
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
    if (threadIdx.x == 0) s[row] = sc;
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

// Largest row (in elements) the shared-memory variant stages.
constexpr int kRQSmemMaxK = 48 * 1024;

cudaError_t launch_rotate_quant(const void *a, int64_t rows, int64_t k, int8_t *q, float *s,
                                cudaStream_t stream, bool pdl) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)rows);
    cfg.blockDim = dim3(kRQThreads);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    const __nv_bfloat16 *ab = static_cast<const __nv_bfloat16 *>(a);
    if (k <= kRQSmemMaxK) {
        static bool configured[64] = {};
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev >= 64 || !configured[dev]) {
            e = cudaFuncSetAttribute(rotate_quant_rows_smem,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kRQSmemMaxK * 4);
            if (e != cudaSuccess) return e;
            if (dev < 64) configured[dev] = true;
        }
        cfg.dynamicSmemBytes = (size_t)k * 4;
        return cudaLaunchKernelEx(&cfg, rotate_quant_rows_smem, ab, (int)k, q, s);
    }
    cfg.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&cfg, rotate_quant_rows_twopass, ab, (int)k, q, s);
}

}  // namespace convrot
