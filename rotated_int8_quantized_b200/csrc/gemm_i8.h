// gemm_i8.h -- internal interface of the tcgen05 INT8 GEMM (not part of the
// public C ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace convrot {

constexpr int kMaxStages = 8;

// Kernel arguments (passed by value).
struct GemmArgs {
    int m, n, k;
    int bn;            // UMMA N: rows of a B tile
    int swap;          // 1: A = weights, B = activations; 0: A = activations, B = weights
    int tiles_a;       // 128-row tiles of A
    int kbpt;          // 128-byte K blocks per tile
    int full_waves;    // data-parallel waves of whole tiles
    int tail_tile0;    // first tile of the stream-K tail
    long long tail_units;  // K blocks in the tail
    int stages;
    int acc_cols;      // TMEM columns per accumulator buffer
    int tmem_cols;     // TMEM columns allocated (power of two >= 32)
    int w_prefetch;    // load weight tiles before the grid-dependency wait
    const float *sx;
    const float *sw;
    __nv_bfloat16 *y;
    int32_t *acc;
    int32_t *partial;  // [tail tiles][bn][128] INT32, zero on entry and exit
    int32_t *counters; // [tail tiles], zero on entry and exit
};

// Host-side tiling of one problem.
struct GemmPlan {
    int swap, bn;
    int64_t rows_a, rows_b;
    int tiles_a, tiles_b, kbpt, num_tiles;
    int grid, full_waves, tail_tile0, tail_tiles;
    long long tail_units;
    int stages, acc_cols, tmem_cols, smem_bytes;
    size_t ws_counters_off, ws_partial_off, ws_bytes;
};

void plan_gemm(int64_t m, int64_t n, int64_t k, int num_sms, GemmPlan *p);

cudaError_t launch_gemm_i8(const GemmPlan &p, const int8_t *xq, const float *sx, int64_t m,
                           const int8_t *wq, const float *sw, int64_t n, int64_t k, __nv_bfloat16 *y,
                           int32_t *acc, void *ws, cudaStream_t stream, bool pdl, bool w_prefetch);

cudaError_t launch_rotate_quant(const void *a, int64_t rows, int64_t k, int8_t *q, float *s,
                                cudaStream_t stream, bool pdl);

}  // namespace convrot
