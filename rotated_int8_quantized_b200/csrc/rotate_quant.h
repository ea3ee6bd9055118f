// rotate_quant.h -- internal interface of the libconvrot prologue kernels
// (rotation + quantisation, the convolution gathers, tensor-wise INT8); not
// part of the public C ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "gemm_i8.h"

namespace convrot {

// ------------------------------------------------------------------ rotation + quantisation
struct RQProblem {
    const void *a;      // BF16 [rows, k]
    int64_t k;
    int group;          // rotation group (power of two, 16 .. 256)
    int8_t *q;          // int8 [rows, k], or packed INT4 [rows, k/2] (int4)
    float *s;           // fp32 [rows]
    int int4;           // 1: INT4 weight codes (levels -7..7), packed
};

// Geometry of a convolution whose im2col rows (mode 3) or OIHW weight rows
// (mode 4) the rotation kernel gathers.
struct ConvGeom {
    int mode;           // 3: activations (NHWC input), 4: weights (OIHW), 5: pixels rotated once
    int n, h, w, c;     // input batch, height, width, channels
    int kh, kw, stride, pad, dil;
    int oh, ow;         // output height and width
};

// Rotate and quantise `rows` rows of each of `njobs` matrices (same row
// count) in one launch; `conv`: the rows are gathered from a convolution.
cudaError_t launch_rotate_quant(int njobs, int64_t rows, const RQProblem *probs, cudaStream_t stream, bool pdl,
                                const ConvGeom *conv = nullptr);

// The tiled gather's shape for a geometry (false: the untiled gather runs).
bool conv_gather_tile_plan(const ConvGeom &g, int sms, int *th, int *tw, int *rh, int *rw, int64_t *tiles,
                           int64_t *buf_bytes);

// Convolution im2col codes from pixels rotated once (yrot FP32 [n*h*w, c],
// pmax [n*h*w]): codes xq [rows, kh*kw*c] and scales sx [rows].
cudaError_t launch_conv_gather_quant(const float *yrot, const float *pmax, const ConvGeom &g, int64_t rows,
                                     int8_t *xq, float *sx, cudaStream_t stream);

// ------------------------------------------------------------------ tensor-wise INT8 (embedding table)
cudaError_t launch_quantize_tensor(const void *a, int64_t count, int8_t *q, float *scale, cudaStream_t stream);
// Packed INT4 weight [n, k/2] -> INT8 codes [n, k] (natural order).
cudaError_t launch_unpack_int4(const uint8_t *packed, int64_t n, int64_t k, int8_t *out, cudaStream_t stream, bool pdl);
cudaError_t launch_embed_lookup(const int32_t *tokens, int64_t t, const int8_t *q, const float *scale,
                                int64_t vocab, int64_t dim, void *out, cudaStream_t stream);

}  // namespace convrot
