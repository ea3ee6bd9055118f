// gemm_i8.h -- internal interface of the libconvrot kernels (not part of the
// public C ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace convrot {

constexpr int kMaxStages = 8;
constexpr int kMaxJobs = 8;      // linears in one batched launch
constexpr int kMaxSwapM = 512;   // rows up to which the weights are the A operand (stream-K)

// ------------------------------------------------------------------ GEMM
// One product of a (batched) launch, as the kernel sees it.
struct GemmJob {
    int m, n, k;
    int tiles_a;        // 128-row tiles of the A operand
    int n_tiles_b;      // tiles of the B operand
    int group_a;        // tile order: groups of group_a A tiles, B tiles outer within a group
    int kbpt;           // 128-byte K blocks per tile
    int tile_base;      // first tile of this job handled by stream-K
    long long unit0;    // first stream-K unit (K block) of this job
    const float *sx;
    const float *sw;
    __nv_bfloat16 *y;
    int32_t *acc;
    const __nv_bfloat16 *bias;   // [n] or null
};

struct GemmArgs {
    int njobs;
    int bn;             // UMMA N: rows of a B tile (same for every job)
    int swap;           // 1: A = weights, B = activations; 0: A = activations, B = weights
    int full_waves;     // data-parallel waves of whole tiles (single job only)
    int full_tiles;     // tiles those waves cover (the last wave may be partial)
    // split tail (large M): the tiles after the full waves are each split into
    // split_ways K ranges, one per CTA; every piece stores its INT32 partial
    // tile privately and the last piece of a tile (ticket counter) sums them
    int split_ways;     // 0: no split tail
    int split_pieces;   // tail tiles x split_ways (CTAs 0 .. pieces-1 take one each)
    long long tail_units;   // K blocks dealt out by stream-K
    int rep;            // stream-K CTAs per group sharing a weight tile (one per A tile), 1: none
    int stages;
    int acc_cols;       // TMEM columns per accumulator buffer
    int tmem_cols;      // TMEM columns allocated (power of two >= 32)
    int w_prefetch;     // load weight tiles before the grid-dependency wait
    int32_t *partial;   // [slots][bn][128] INT32, zero on entry and exit
    int32_t *counters;  // [slots], zero on entry and exit
    GemmJob job[kMaxJobs];
};

struct GemmMaps {
    CUtensorMap a[kMaxJobs];
    CUtensorMap b[kMaxJobs];
};

// One problem as the host describes it.
struct GemmProblem {
    int64_t m, n, k;
    const int8_t *xq;
    const float *sx;
    const int8_t *wq;
    const float *sw;
    __nv_bfloat16 *y;
    int32_t *acc;
    const __nv_bfloat16 *bias;   // [n] or null
};

// Host-side tiling of a launch.
struct GemmPlan {
    int njobs, swap, bn;
    int grid, full_waves, full_tiles, split_ways, split_pieces, stages, acc_cols, tmem_cols, smem_bytes, rep;
    int w4;             // INT4 weights (packed), unpacked in shared memory
    long long tail_units;
    int tiles_a[kMaxJobs], tiles_b[kMaxJobs], group_a[kMaxJobs], kbpt[kMaxJobs], tile_base[kMaxJobs];
    long long unit0[kMaxJobs];
    int64_t rows_a[kMaxJobs], rows_b[kMaxJobs];
    int slots;
    size_t ws_counters_off, ws_partial_off, ws_bytes;
};

// Single product: whole tiles dealt round-robin in full waves, the last
// partial wave split along K (stream-K).  w4: INT4 weights (packed two
// codes per byte), unpacked in shared memory.
void plan_gemm(int64_t m, int64_t n, int64_t k, int num_sms, GemmPlan *p, bool w4 = false);
// Several products with the same m <= kMaxSwapM in one launch: every K
// block of every (weight tile, activation tile) pair dealt out evenly by
// stream-K.
// w4: INT4 weights (packed two codes per byte).
void plan_gemm_batch(int64_t m, int njobs, const int64_t *n, const int64_t *k, int num_sms, GemmPlan *p,
                     bool w4 = false);

cudaError_t launch_gemm_i8(const GemmPlan &p, const GemmProblem *probs, void *ws, cudaStream_t stream,
                           bool pdl, bool w_prefetch);

}  // namespace convrot
