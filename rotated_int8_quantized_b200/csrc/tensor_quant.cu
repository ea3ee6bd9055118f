// tensor_quant.cu -- tensor-wise "simple" INT8 for the word-embedding table
// and the lookup from it.
//
// The converter keeps the embedding table out of ConvRot: no rotation, one
// FP32 scale for the whole tensor, round-to-nearest [zskr.cn "Qwen3-VL-32B
// ... INT8-ConvRot", quantisation configuration: word embedding "simple
// tensor-wise INT8"; conversion command: --custom-layers embed_tokens
// --custom-type int8 --custom-scaling-mode tensor --custom-simple].
//
//   a = max |x| over the tensor;  s = fl(a / 127);  q = clamp(rne(fl(x / s)))
//   lookup: out[i, :] = bf16(fl((float)q[tokens[i], :] * s))
//
// Three stream-ordered launches quantise: the absolute maximum of the
// tensor (atomicMax on the bit pattern of a non-negative float, into the
// caller's scale word, zeroed first), the codes (every thread derives s from
// that maximum with the row quantiser of rotate_quant.cu), and one thread
// that turns the maximum into s.  All loads and stores are 16 bytes wide.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "gemm_i8.h"
#include "rotate_quant.h"

namespace convrot {

constexpr int kTqThreads = 256;

__device__ __forceinline__ void bf16x16_to_f32(const uint4 &lo, const uint4 &hi, float (&y)[16]) {
    const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        y[2 * i] = __uint_as_float(w[i] << 16);
        y[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// max |x| over units of 16 BF16 values, into *amax_bits (zero on entry).
__global__ void __launch_bounds__(kTqThreads) tensor_absmax_kernel(const uint4 *a, int64_t units,
                                                                 unsigned *amax_bits) {
    __shared__ float red[kTqThreads / 32];
    float m = 0.f;
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < units; u += (int64_t)gridDim.x * blockDim.x) {
        float y[16];
        bf16x16_to_f32(__ldg(a + 2 * u), __ldg(a + 2 * u + 1), y);
#pragma unroll
        for (int e = 0; e < 16; ++e) m = fmaxf(m, fabsf(y[e]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kTqThreads / 32; ++w) m = fmaxf(m, red[w]);
        atomicMax(amax_bits, __float_as_uint(m));     // non-negative floats order as their bits
    }
}

// q = clamp(rne(x / s)) with s = fl(amax / 127), 16 codes per unit.
__global__ void __launch_bounds__(kTqThreads) tensor_quant_kernel(const uint4 *a, int64_t units,
                                                                const unsigned *amax_bits, uint4 *q) {
    const RowScale rs = make_row_scale(__uint_as_float(*amax_bits));
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t u0 = (int64_t)blockIdx.x * blockDim.x; u0 < units; u0 += stride) {
        const int64_t u = u0 + threadIdx.x;
        const unsigned mask = __ballot_sync(0xffffffffu, u < units);
        if (u < units) {
            float y[16];
            bf16x16_to_f32(__ldg(a + 2 * u), __ldg(a + 2 * u + 1), y);
            q[u] = quant16(y, rs, mask);
        }
    }
}

__global__ void tensor_scale_kernel(float *scale) {
    *scale = __fdiv_rn(__uint_as_float(*reinterpret_cast<unsigned *>(scale)), 127.0f);
}

// out[i, :] = bf16(q[tokens[i], :] * s): 16 columns per thread.  A token
// outside [0, vocab) gives a zero row and records CONVROT_ERR_INVALID_ARG
// in the device status word.
__global__ void __launch_bounds__(kTqThreads) embed_lookup_kernel(const int32_t *tokens, int64_t t,
                                                                const int8_t *q, const float *scale,
                                                                int64_t vocab, int64_t dim, __nv_bfloat16 *out) {
    const float s = *scale;
    const int64_t per_row = dim / 16;
    const int64_t total = t * per_row;
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < total; u += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = u / per_row, c = u - i * per_row;
        const int64_t tok = tokens[i];
        uint32_t pk[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        if (tok >= 0 && tok < vocab) {
            const uint4 w = __ldg(reinterpret_cast<const uint4 *>(q + tok * dim) + c);
            const uint32_t b[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
                const float f0 = __fmul_rn((float)(int8_t)(b[e >> 2] >> (8 * (e & 3))), s);
                const float f1 = __fmul_rn((float)(int8_t)(b[(e + 1) >> 2] >> (8 * ((e + 1) & 3))), s);
                __nv_bfloat162 h = __halves2bfloat162(__float2bfloat16_rn(f0), __float2bfloat16_rn(f1));
                pk[e >> 1] = *reinterpret_cast<uint32_t *>(&h);
            }
        } else if (c == 0) {
            // an error replaces a recorded warning, never a recorded error
            if (atomicCAS(&g_device_status, 0, 1 /* CONVROT_ERR_INVALID_ARG */) == 8)
                atomicCAS(&g_device_status, 8, 1);
        }
        uint4 *dst = reinterpret_cast<uint4 *>(out + i * dim) + 2 * c;
        dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
}

// Sign-extend the low nibble of each byte of v (bytes 0..15) to int8: bit 3
// of a byte times 30 is 0xF0, which lands in its empty high nibble.
__device__ __forceinline__ uint32_t sext_nibbles4(uint32_t v) {
    return (v & 0x08080808u) * 30u + v;
}

static int tq_grid(int64_t work) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t blocks = (work + kTqThreads - 1) / kTqThreads;
    const int64_t cap = (int64_t)sms * 8;
    return (int)(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

cudaError_t launch_quantize_tensor(const void *a, int64_t count, int8_t *q, float *scale, cudaStream_t stream) {
    const int64_t units = count / 16;
    cudaError_t e = cudaMemsetAsync(scale, 0, sizeof(float), stream);
    if (e != cudaSuccess) return e;
    unsigned *amax = reinterpret_cast<unsigned *>(scale);
    const int g = tq_grid(units);
    tensor_absmax_kernel<<<g, kTqThreads, 0, stream>>>(static_cast<const uint4 *>(a), units, amax);
    tensor_quant_kernel<<<g, kTqThreads, 0, stream>>>(static_cast<const uint4 *>(a), units, amax,
                                                       reinterpret_cast<uint4 *>(q));
    tensor_scale_kernel<<<1, 1, 0, stream>>>(scale);
    return cudaGetLastError();
}

// INT4 weight codes (this library's packing: within each 16-code chunk, byte
// j holds code j in its low nibble and code 8 + j in its high nibble) to
// INT8 codes in their natural order, two chunks (16 packed bytes -> 32 code
// bytes) per thread and step.  HBM-bound; used before an INT8 GEMM at
// prefill sizes, where unpacking every weight tile inside each CTA that
// reads it would cost far more shared-memory bandwidth than one pass here.
__global__ void __launch_bounds__(kTqThreads) unpack_int4_kernel(const uint4 *packed, int64_t pairs, uint4 *out) {
    pdl_wait();
    pdl_launch_dependents();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < pairs; i += stride) {
        const uint4 w = __ldg(packed + i);
        const uint32_t h[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const uint32_t lo = h[2 * c], hi = h[2 * c + 1];     // the chunk's 8 packed bytes
            uint4 o;
            o.x = sext_nibbles4(lo & 0x0F0F0F0Fu);               // codes 0-3
            o.y = sext_nibbles4(hi & 0x0F0F0F0Fu);               // codes 4-7
            o.z = sext_nibbles4((lo >> 4) & 0x0F0F0F0Fu);        // codes 8-11
            o.w = sext_nibbles4((hi >> 4) & 0x0F0F0F0Fu);        // codes 12-15
            out[2 * i + c] = o;
        }
    }
}

cudaError_t launch_unpack_int4(const uint8_t *packed, int64_t n, int64_t k, int8_t *out, cudaStream_t stream, bool pdl) {
    const int64_t pairs = n * k / 32;          // k % 32 == 0 for INT4 weights
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)tq_grid(pairs));
    cfg.blockDim = dim3(kTqThreads);
    cfg.stream = stream;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, unpack_int4_kernel, reinterpret_cast<const uint4 *>(packed), pairs,
                              reinterpret_cast<uint4 *>(out));
}

cudaError_t launch_embed_lookup(const int32_t *tokens, int64_t t, const int8_t *q, const float *scale,
                                int64_t vocab, int64_t dim, void *out, cudaStream_t stream) {
    embed_lookup_kernel<<<tq_grid(t * (dim / 16)), kTqThreads, 0, stream>>>(tokens, t, q, scale, vocab, dim,
                                                                            static_cast<__nv_bfloat16 *>(out));
    return cudaGetLastError();
}

}  // namespace convrot
