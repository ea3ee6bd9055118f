// gemm_i8.cu -- INT8 x INT8 -> INT32 GEMM on the sm_100a tcgen05 tensor
// cores with the ConvRot dequantisation fused into the epilogue:
//
//   acc[m, n] = sum_k xq[m, k] * wq[n, k];   y[m, n] = bf16(acc * sx[m] * sw[n])
//
// [0539edu.com "minimax-h3-nvfp4-convrot", section 4 "INT8 ConvRot": the
//  rotated INT8 layer runs on INT8 tensor cores; "INT8 row-scale" per
//  weight row; zskr.cn "Qwen3-VL-32B ... INT8-ConvRot": the tail LM head is
//  computed row-wise in chunks so that no dequantised weight is ever
//  materialised -- here the GEMM consumes INT8 directly, always.]
//
// One kernel serves both regimes of the layer:
//   * decode-sized M (M <= 256): the weight is the 128-row UMMA "A" operand
//     and the few token rows are the N = roundup16(M) "B" operand, so every
//     weight byte is streamed from HBM exactly once through a deep TMA
//     pipeline; the K loop is split across all SMs (stream-K) because the
//     weight has too few 128-row tiles to fill 148 SMs.
//   * large M: activations are A (128-row tiles), weights are B (256-row
//     tiles); whole tiles are dealt round-robin to a persistent grid of one
//     CTA per SM, and the last partial wave is split along K (stream-K).
//
// Both operands are K-major INT8, loaded by TMA with 128-byte swizzle into a
// multi-stage shared-memory ring; one thread issues tcgen05.mma kind::i8
// (M = 128, N = bn, K = 32 per instruction) into an INT32 accumulator in
// tensor memory; four epilogue warps drain the accumulator with tcgen05.ld
// while the next tile accumulates into the second TMEM buffer.
//
// A K-range that covers only part of a tile (stream-K) adds its INT32
// partial sums into a caller-provided workspace with integer atomics (exact
// and order-free); the CTA that completes the tile's K range (found with a
// per-tile ticket counter, no spin-waiting) reads the total, applies the
// epilogue and returns the workspace tile and the counter to zero.
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "gemm_i8.h"

namespace convrot {

constexpr int kThreads = 192;          // warp 0: TMA, warp 1: MMA + TMEM, warps 2-5: epilogue
constexpr int kTileA = 128;            // UMMA M
constexpr int kBlockK = 128;           // bytes of K per stage (one 128-byte swizzle row)
constexpr int kUmmaK = 32;             // K per tcgen05.mma kind::i8
constexpr int kATileBytes = kTileA * kBlockK;

__device__ __forceinline__ void named_bar_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Work of one CTA: a list of segments (tile, kb0, kb1), first the whole
// tiles of the data-parallel waves, then its contiguous share of the
// stream-K tail.
struct SegmentIter {
    int wave;
    long long u, u_end;
    __device__ __forceinline__ void init(const GemmArgs &a) {
        wave = 0;
        const long long c = blockIdx.x, G = gridDim.x;
        u = a.tail_units * c / G;
        u_end = a.tail_units * (c + 1) / G;
    }
    __device__ __forceinline__ bool next(const GemmArgs &a, int &tile, int &kb0, int &kb1) {
        if (wave < a.full_waves) {
            tile = wave * (int)gridDim.x + (int)blockIdx.x;
            kb0 = 0;
            kb1 = a.kbpt;
            ++wave;
            return true;
        }
        if (u < u_end) {
            const long long t = u / a.kbpt;
            tile = a.tail_tile0 + (int)t;
            kb0 = (int)(u - t * a.kbpt);
            long long rem = u_end - u;
            kb1 = (int)((long long)kb0 + rem < a.kbpt ? kb0 + rem : a.kbpt);
            u += kb1 - kb0;
            return true;
        }
        return false;
    }
};

// Dequantise and store 16 consecutive B-rows (j0 .. j0+15) of one A-row i.
__device__ __forceinline__ void emit16(const GemmArgs &a, int i, int j0, const int32_t (&v)[16]) {
    if (!a.swap) {
        const int m = i;
        if (m >= a.m) return;
        const float sxm = a.sx[m];
        const bool full = (j0 + 16 <= a.n) && ((a.n & 7) == 0);
        if (a.acc) {
            int32_t *dst = a.acc + (size_t)m * a.n + j0;
            if (full && (a.n & 3) == 0) {
#pragma unroll
                for (int e = 0; e < 16; e += 4)
                    *reinterpret_cast<int4 *>(dst + e) = make_int4(v[e], v[e + 1], v[e + 2], v[e + 3]);
            } else {
                for (int e = 0; e < 16 && j0 + e < a.n; ++e) dst[e] = v[e];
            }
        }
        if (a.y) {
            __nv_bfloat16 *dst = a.y + (size_t)m * a.n + j0;
            if (full) {
                uint32_t pk[8];
#pragma unroll
                for (int e = 0; e < 16; e += 2) {
                    float f0 = __fmul_rn(__fmul_rn(__int2float_rn(v[e]), sxm), __ldg(a.sw + j0 + e));
                    float f1 = __fmul_rn(__fmul_rn(__int2float_rn(v[e + 1]), sxm), __ldg(a.sw + j0 + e + 1));
                    __nv_bfloat162 h = __halves2bfloat162(__float2bfloat16_rn(f0), __float2bfloat16_rn(f1));
                    pk[e >> 1] = *reinterpret_cast<uint32_t *>(&h);
                }
                reinterpret_cast<uint4 *>(dst)[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                reinterpret_cast<uint4 *>(dst)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            } else {
                for (int e = 0; e < 16 && j0 + e < a.n; ++e) {
                    float f = __fmul_rn(__fmul_rn(__int2float_rn(v[e]), sxm), __ldg(a.sw + j0 + e));
                    dst[e] = __float2bfloat16_rn(f);
                }
            }
        }
    } else {
        const int n = i;
        if (n >= a.n) return;
        const float swn = a.sw[n];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int m = j0 + e;
            if (m < a.m) {
                if (a.acc) a.acc[(size_t)m * a.n + n] = v[e];
                if (a.y) {
                    float f = __fmul_rn(__fmul_rn(__int2float_rn(v[e]), __ldg(a.sx + m)), swn);
                    a.y[(size_t)m * a.n + n] = __float2bfloat16_rn(f);
                }
            }
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_i8_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const GemmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment for the 128-byte-swizzled operand tiles
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw);

    const int S = a.stages;
    const uint32_t b_bytes = (uint32_t)a.bn * kBlockK;
    const uint32_t a_off = 0;
    const uint32_t b_off = (uint32_t)S * kATileBytes;
    const uint32_t bar_off = b_off + (uint32_t)S * b_bytes;
    // barriers: full[S], empty[S], tfull[2], tempty[2], drain
    const uint32_t full_bar = base + bar_off;
    const uint32_t empty_bar = full_bar + 8u * S;
    const uint32_t tfull_bar = empty_bar + 8u * S;
    const uint32_t tempty_bar = tfull_bar + 16u;
    const uint32_t drain_bar = tempty_bar + 16u;
    uint8_t *misc = smem + bar_off + 8u * (2 * S + 5);
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(misc);
    volatile int *ticket = reinterpret_cast<volatile int *>(misc + 4);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 8);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar + 8u * s, 1);
            mbar_init(empty_bar + 8u * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar + 8u * b, 1);
            mbar_init(tempty_bar + 8u * b, 4);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        *ticket = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(smem_addr((const void *)tmem_slot), (uint32_t)a.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint32_t tx = (uint32_t)kATileBytes + b_bytes;
            int stage = 0;
            uint32_t phase = 0;
            bool waited = !a.w_prefetch;
            if (waited) pdl_wait();
            // activation loads held back until the grid dependency resolves
            int pend_n = 0;
            int pend_stage[kMaxStages], pend_x[kMaxStages], pend_y[kMaxStages];
            uint32_t issued_mask = 0, issued_par = 0;
            const CUtensorMap *tmW = a.swap ? &tmA : &tmB;
            const CUtensorMap *tmX = a.swap ? &tmB : &tmA;
            SegmentIter it;
            it.init(a);
            int tile, kb0, kb1;
            bool ok = true;
            while (ok && it.next(a, tile, kb0, kb1)) {
                const int ta = tile % a.tiles_a, tb = tile / a.tiles_a;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait_bounded(empty_bar + 8u * stage, phase ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = full_bar + 8u * stage;
                    mbar_arrive_expect_tx(fb, tx);
                    const uint32_t sa = base + a_off + (uint32_t)stage * kATileBytes;
                    const uint32_t sb = base + b_off + (uint32_t)stage * b_bytes;
                    const int kx = kb * kBlockK;
                    const uint32_t sW = a.swap ? sa : sb, sX = a.swap ? sb : sa;
                    const int rowW = a.swap ? ta * kTileA : tb * a.bn;
                    const int rowX = a.swap ? tb * a.bn : ta * kTileA;
                    tma_load_2d(sW, tmW, fb, kx, rowW);
                    if (waited) {
                        tma_load_2d(sX, tmX, fb, kx, rowX);
                    } else {
                        pend_stage[pend_n] = stage;
                        pend_x[pend_n] = kx;
                        pend_y[pend_n] = rowX;
                        if (++pend_n == S) {
                            pdl_wait();
                            waited = true;
                            for (int p = 0; p < pend_n; ++p) {
                                const int st = pend_stage[p];
                                const uint32_t sxa = a.swap ? base + b_off + (uint32_t)st * b_bytes
                                                            : base + a_off + (uint32_t)st * kATileBytes;
                                tma_load_2d(sxa, tmX, full_bar + 8u * st, pend_x[p], pend_y[p]);
                            }
                            pend_n = 0;
                        }
                    }
                    issued_mask |= 1u << stage;
                    issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!waited) {
                pdl_wait();
                for (int p = 0; p < pend_n; ++p) {
                    const int st = pend_stage[p];
                    const uint32_t sxa = a.swap ? base + b_off + (uint32_t)st * b_bytes
                                                : base + a_off + (uint32_t)st * kATileBytes;
                    tma_load_2d(sxa, tmX, full_bar + 8u * st, pend_x[p], pend_y[p]);
                }
            }
            if (!ok) {
                // let every copy this thread started land before the CTA exits
                volatile int no_abort = 0;
                for (int s = 0; s < S; ++s)
                    if (issued_mask & (1u << s))
                        mbar_wait_bounded(full_bar + 8u * s, (issued_par >> s) & 1u, &no_abort);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            pdl_wait();
            const uint32_t idesc = idesc_i8(kTileA, (uint32_t)a.bn);
            int stage = 0;
            uint32_t phase = 0;
            int seg = 0;
            SegmentIter it;
            it.init(a);
            int tile, kb0, kb1;
            bool ok = true;
            while (ok && it.next(a, tile, kb0, kb1)) {
                const int buf = seg & 1;
                const uint32_t use = (uint32_t)(seg >> 1);
                if (!mbar_wait_bounded(tempty_bar + 8u * buf, (use & 1u) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)(buf * a.acc_cols);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait_bounded(full_bar + 8u * stage, phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t da = smem_desc_k_sw128(base + a_off + (uint32_t)stage * kATileBytes);
                    const uint64_t db = smem_desc_k_sw128(base + b_off + (uint32_t)stage * b_bytes);
#pragma unroll
                    for (int kk = 0; kk < kBlockK / kUmmaK; ++kk) {
                        // advance the start address by 32 bytes (2 x 16 B) along K
                        umma_i8(d, da + 2u * kk, db + 2u * kk, idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(empty_bar + 8u * stage);
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(tfull_bar + 8u * buf);
                ++seg;
            }
            if (!ok) {
                volatile int no_abort = 0;
                umma_commit(drain_bar);
                mbar_wait_bounded(drain_bar, 0, &no_abort);
            }
        }
    } else {
        // ------------------------------------------------ epilogue (4 warps)
        pdl_wait();
        const int quarter = warp & 3;              // TMEM lanes 32*quarter .. +31
        const int row = quarter * 32 + lane;       // row of the A tile
        const int ew = warp - 2;
        int seg = 0;
        SegmentIter it;
        it.init(a);
        int tile, kb0, kb1;
        while (it.next(a, tile, kb0, kb1)) {
            const int ta = tile % a.tiles_a, tb = tile / a.tiles_a;
            const int buf = seg & 1;
            const uint32_t use = (uint32_t)(seg >> 1);
            if (!mbar_wait_bounded(tfull_bar + 8u * buf, use & 1u, abort_flag)) break;
            tc_fence_after();
            const int i = ta * kTileA + row;
            const bool whole = (kb0 == 0 && kb1 == a.kbpt);
            const int slot = tile - a.tail_tile0;
            const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * a.acc_cols);
            for (int c = 0; c < a.bn / 16; ++c) {
                uint32_t r[16];
                __syncwarp();
                tmem_ld_32x32b_x16(tbase + (uint32_t)(c * 16), r);
                tmem_ld_wait();
                int32_t v[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] = (int32_t)r[e];
                if (whole) {
                    emit16(a, i, tb * a.bn + c * 16, v);
                } else {
                    int32_t *p = a.partial + ((size_t)slot * a.bn + c * 16) * kTileA + row;
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        if (v[e] != 0) atomicAdd(p + (size_t)e * kTileA, v[e]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty_bar + 8u * buf);
            if (!whole) {
                __threadfence();
                named_bar_sync(1, 128);
                if (ew == 0 && lane == 0) {
                    const int mine = kb1 - kb0;
                    const int old = atomicAdd(a.counters + slot, mine);
                    *ticket = (old + mine == a.kbpt) ? 1 : 0;
                }
                named_bar_sync(1, 128);
                const bool last = (*ticket != 0);
                if (last) {
                    __threadfence();
                    for (int c = 0; c < a.bn / 16; ++c) {
                        int32_t *p = a.partial + ((size_t)slot * a.bn + c * 16) * kTileA + row;
                        int32_t v[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = __ldcg(p + (size_t)e * kTileA);
#pragma unroll
                        for (int e = 0; e < 16; ++e) __stcg(p + (size_t)e * kTileA, 0);
                        emit16(a, i, tb * a.bn + c * 16, v);
                    }
                    if (ew == 0 && lane == 0) a.counters[slot] = 0;
                }
                named_bar_sync(1, 128);
            }
            ++seg;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, (uint32_t)a.tmem_cols);
    }
}

// ---------------------------------------------------------------- host side

void plan_gemm(int64_t m, int64_t n, int64_t k, int num_sms, GemmPlan *p) {
    p->swap = (m <= 256) ? 1 : 0;
    p->bn = p->swap ? (int)((m + 15) / 16 * 16) : 256;
    p->rows_a = p->swap ? n : m;
    p->rows_b = p->swap ? m : n;
    p->tiles_a = (int)((p->rows_a + kTileA - 1) / kTileA);
    p->tiles_b = (int)((p->rows_b + p->bn - 1) / p->bn);
    p->kbpt = (int)(k / kBlockK);
    p->num_tiles = p->tiles_a * p->tiles_b;
    const long long units = (long long)p->num_tiles * p->kbpt;
    p->grid = (int)(units < num_sms ? units : num_sms);
    p->full_waves = p->num_tiles / p->grid;
    p->tail_tile0 = p->full_waves * p->grid;
    p->tail_tiles = p->num_tiles - p->tail_tile0;
    p->tail_units = (long long)p->tail_tiles * p->kbpt;
    const int stage_bytes = kATileBytes + p->bn * kBlockK;
    int stages = (200 * 1024) / stage_bytes;
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages < 2) stages = 2;
    p->stages = stages;
    p->acc_cols = p->bn;
    int cols = 32;
    while (cols < 2 * p->bn) cols <<= 1;
    p->tmem_cols = cols;
    p->smem_bytes = 1024 + stages * stage_bytes + 8 * (2 * stages + 5) + 16;
    // workspace: counters, then INT32 partial tiles [tail_tiles][bn][128]
    const size_t cnt = ((size_t)p->tail_tiles * 4 + 255) / 256 * 256;
    p->ws_counters_off = 0;
    p->ws_partial_off = cnt;
    p->ws_bytes = cnt + (size_t)p->tail_tiles * p->bn * kTileA * 4;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// K-major INT8 matrix [rows, k] -> tensor map with a (128 bytes x box_rows)
// box and 128-byte swizzle.
static bool make_tmap(CUtensorMap *map, const void *ptr, int64_t rows, int64_t k, int box_rows) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)k, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)k};
    cuuint32_t box[2] = {(cuuint32_t)kBlockK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

cudaError_t launch_gemm_i8(const GemmPlan &p, const int8_t *xq, const float *sx, int64_t m,
                           const int8_t *wq, const float *sw, int64_t n, int64_t k, __nv_bfloat16 *y,
                           int32_t *acc, void *ws, cudaStream_t stream, bool pdl, bool w_prefetch) {
    CUtensorMap tmA, tmB;
    const int8_t *A = p.swap ? wq : xq;
    const int8_t *B = p.swap ? xq : wq;
    if (!make_tmap(&tmA, A, p.rows_a, k, kTileA)) return cudaErrorInvalidValue;
    if (!make_tmap(&tmB, B, p.rows_b, k, p.bn)) return cudaErrorInvalidValue;

    GemmArgs a = {};
    a.m = (int)m;
    a.n = (int)n;
    a.k = (int)k;
    a.bn = p.bn;
    a.swap = p.swap;
    a.tiles_a = p.tiles_a;
    a.kbpt = p.kbpt;
    a.full_waves = p.full_waves;
    a.tail_tile0 = p.tail_tile0;
    a.tail_units = p.tail_units;
    a.stages = p.stages;
    a.acc_cols = p.acc_cols;
    a.tmem_cols = p.tmem_cols;
    a.w_prefetch = w_prefetch ? 1 : 0;
    a.sx = sx;
    a.sw = sw;
    a.y = y;
    a.acc = acc;
    a.counters = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + p.ws_counters_off);
    a.partial = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + p.ws_partial_off);

    static bool configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !configured[dev]) {
        e = cudaFuncSetAttribute(gemm_i8_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        if (dev < 64) configured[dev] = true;
    }

    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)p.grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)p.smem_bytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, gemm_i8_tc_kernel, tmA, tmB, a);
}

}  // namespace convrot
