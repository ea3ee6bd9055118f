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
#include <cstring>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "gemm_i8.h"

namespace convrot {

constexpr int kThreads = 192;          // warp 0: TMA, warp 1: MMA + TMEM, warps 2-5: epilogue
constexpr int kW4Warps = 8;            // INT4 weights: warps 6.. unpack the packed weight tiles
constexpr int kMaxRing = kMaxStages;
constexpr int kThreadsW4 = kThreads + 32 * kW4Warps;
constexpr int kTileA = 128;            // UMMA M
constexpr int kBlockK = 128;           // bytes of K per stage (one 128-byte swizzle row)
constexpr int kUmmaK = 32;             // K per tcgen05.mma kind::i8
constexpr int kATileBytes = kTileA * kBlockK;
constexpr uint32_t kPackedRowBytes = kBlockK / 2;   // INT4 codes of one 128-byte K block of a weight row
constexpr int kL2PrefetchBlocks = 16;  // weight K blocks pulled into L2 ahead of the grid-dependency wait
constexpr int kMaxSplitWays = 6;       // K ranges per split tail tile (large M)
constexpr long long kGroupABytes = 48ll << 20;   // INT8 A operand above this is taken in tile groups
constexpr int kBiasStage = 256;        // offset of the staged bias after the staged scales of a tile
constexpr int kExtraBars = 7;          // tfull[2], tempty[2], drain, red[2]
// The split-tail reduction double-buffers at least 32 columns of every other
// piece's partial in the operand ring of a bn = 256 launch.
static_assert(2 * (kMaxSplitWays - 1) * 32 * kTileA * 4 <=
                  (200 * 1024 / (kATileBytes + 256 * kBlockK)) * (kATileBytes + 256 * kBlockK),
              "split-tail reduction buffers exceed the operand ring");

__device__ __forceinline__ void named_bar_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Barrier over `n` threads that also returns the AND of their predicates, so
// that all of them take the same branch after a bounded wait.
__device__ __forceinline__ bool named_bar_and(int id, int n, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

// Work of one CTA: a list of segments (job, tile, kb0, kb1), first the
// whole tiles of the data-parallel waves (single-job launches), then its
// contiguous share of the stream-K units.  A stream-K segment never crosses
// a tile or a job boundary.
struct Segment {
    int job, tile, kb0, kb1, slot;
    int split;          // >= 0: a piece of a split tail tile (private partial)
};

// The stream-K CTA whose unit range [total*c/G, total*(c+1)/G) holds unit u.
__device__ __forceinline__ int stream_k_cta(long long u, long long total, int G) {
    int c = (int)((u * G) / total);
    while (c + 1 < G && (total * (c + 1)) / G <= u) ++c;
    while (c > 0 && (total * c) / G > u) --c;
    return c;
}

// Stream-K with replication R = a.rep: the grid is Q = G / R groups of R
// consecutive CTAs; group q takes a contiguous share of the units (K blocks
// of B tiles when R > 1, of whole tiles when R = 1) and CTA r of the group
// computes A tile r for them, so the R CTAs of a group read the same weight
// blocks at about the same time and share them in L2.
struct SegmentIter {
    int wave, j, r;
    bool piece_done;
    long long u, u_end;
    __device__ __forceinline__ void init(const GemmArgs &a) {
        wave = 0;
        j = 0;
        piece_done = false;
        const int R = a.rep;
        const long long q = blockIdx.x / R, Q = gridDim.x / R;
        r = (int)blockIdx.x - (int)q * R;
        u = a.tail_units * q / Q;
        u_end = a.tail_units * (q + 1) / Q;
    }
    // want_slot: also find the workspace slot of a shared (partial) tile;
    // only the epilogue needs it
    __device__ __forceinline__ bool next(const GemmArgs &a, Segment &s, bool want_slot = false) {
        if (wave < a.full_waves && wave * (int)gridDim.x + (int)blockIdx.x < a.full_tiles) {
            s.job = 0;
            s.tile = wave * (int)gridDim.x + (int)blockIdx.x;
            s.kb0 = 0;
            s.kb1 = a.job[0].kbpt;
            s.slot = -1;
            s.split = -1;
            ++wave;
            return true;
        }
        if (a.split_ways > 1 && !piece_done) {
            piece_done = true;
            const int c = (int)blockIdx.x;
            if (c < a.split_pieces) {
                const int kbpt = a.job[0].kbpt;
                s.job = 0;
                s.slot = c / a.split_ways;
                s.split = c - s.slot * a.split_ways;
                s.tile = a.full_tiles + s.slot;
                s.kb0 = s.split * kbpt / a.split_ways;
                s.kb1 = (s.split + 1) * kbpt / a.split_ways;
                return true;
            }
        }
        if (u < u_end) {
            while (j + 1 < a.njobs && u >= a.job[j + 1].unit0) ++j;
            const GemmJob &J = a.job[j];
            const int lu = (int)(u - J.unit0);           // < tiles x kbpt of one job
            const int t = lu / J.kbpt;
            s.job = j;
            s.tile = J.tile_base + t * a.rep + r;
            s.kb0 = lu - t * J.kbpt;
            const long long rem = u_end - u;
            s.kb1 = (int)((long long)s.kb0 + rem < J.kbpt ? s.kb0 + rem : J.kbpt);
            s.split = -1;
            s.slot = -1;
            // a tile shared by several CTAs sums in the workspace slot of the
            // last of them (its range starts inside this tile, so no other
            // shared tile maps to the same slot)
            if (want_slot && (s.kb0 != 0 || s.kb1 != J.kbpt))
                s.slot = stream_k_cta(J.unit0 + (long long)(t + 1) * J.kbpt - 1, a.tail_units,
                                      (int)gridDim.x / a.rep) * a.rep + r;
            u += s.kb1 - s.kb0;
            return true;
        }
        return false;
    }
};

// Tile index -> (A tile, B tile).  Tiles run in groups of group_a A tiles;
// inside a group the A tile varies fastest, so the CTAs of one wave share a
// few B tiles and a group's A rows stay in L2 while the group sweeps B.
__device__ __forceinline__ void tile_coords(const GemmJob &J, int tile, int &ta, int &tb) {
    if (J.n_tiles_b == 1) {         // one B tile (decode): no division
        ta = tile;
        tb = 0;
        return;
    }
    const int per_group = J.group_a * (J.n_tiles_b);
    const int g = tile / per_group;
    const int w = tile - g * per_group;
    const int a0 = g * J.group_a;
    const int ga = (J.tiles_a - a0 < J.group_a) ? J.tiles_a - a0 : J.group_a;
    tb = w / ga;
    ta = a0 + (w - tb * ga);
}

// Large-M orientation: dequantise and store columns j0 .. j0+15 of output
// row m, with the row scale sxm in a register and the tile's weight scales
// staged in shared memory (sws[e] = sw[j0 + e]; with a bias, the bias
// values follow kBiasStage floats later: sws[kBiasStage + e] = bias[j0 + e]).
__device__ __forceinline__ float dq_row(int32_t acc, float sxm, const float *sws, int e, bool bias) {
    const float f = __fmul_rn(__fmul_rn(__int2float_rn(acc), sxm), sws[e]);
    return bias ? __fadd_rn(f, sws[kBiasStage + e]) : f;
}

// sh: the accumulators are 2^sh times the products' sums (INT4 weights are
// unpacked as 16 x code); the exact sum is v >> sh.
__device__ __forceinline__ void emit_row16(const GemmJob &J, int m, int j0, const int32_t (&v_in)[16], float sxm,
                                           const float *sws, int sh) {
    if (m >= J.m) return;
    int32_t v[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = v_in[e] >> sh;
    const bool full = (j0 + 16 <= J.n) && ((J.n & 7) == 0);
    if (J.acc) {
        int32_t *dst = J.acc + (size_t)m * J.n + j0;
        if (full) {
#pragma unroll
            for (int e = 0; e < 16; e += 4)
                *reinterpret_cast<int4 *>(dst + e) = make_int4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        } else {
            for (int e = 0; e < 16 && j0 + e < J.n; ++e) dst[e] = v[e];
        }
    }
    if (J.y) {
        __nv_bfloat16 *dst = J.y + (size_t)m * J.n + j0;
        if (full) {
            uint32_t pk[8];
            const bool bias = J.bias != nullptr;
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
                const float f0 = dq_row(v[e], sxm, sws, e, bias);
                const float f1 = dq_row(v[e + 1], sxm, sws, e + 1, bias);
                __nv_bfloat162 h = __halves2bfloat162(__float2bfloat16_rn(f0), __float2bfloat16_rn(f1));
                pk[e >> 1] = *reinterpret_cast<uint32_t *>(&h);
            }
            reinterpret_cast<uint4 *>(dst)[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            reinterpret_cast<uint4 *>(dst)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        } else {
            for (int e = 0; e < 16 && j0 + e < J.n; ++e) dst[e] = __float2bfloat16_rn(dq_row(v[e], sxm, sws, e, J.bias));
        }
    }
}

// Swapped orientation (A = weight rows n, B = activation rows m): the 16
// accumulators of weight row n = a0 + row for activation rows j0 .. j0+15.
// The BF16 results are transposed through `stg` ([16][128], this chunk's
// buffer) so that each output row leaves as 16-byte segments instead of
// 2-byte scatters.  Called by all 128 epilogue threads (it holds a barrier).
__device__ __forceinline__ void emit_swap16(const GemmJob &J, int a0, int row, int tid, int j0,
                                            const int32_t (&v_in)[16], float srow, float brow, const float *scol,
                                            __nv_bfloat16 *stg, int sh) {
    const int n = a0 + row;
    int32_t v[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = v_in[e] >> sh;
    if (J.acc && n < J.n) {
#pragma unroll
        for (int e = 0; e < 16; ++e)
            if (j0 + e < J.m) J.acc[(size_t)(j0 + e) * J.n + n] = v[e];
    }
    if (!J.y) return;
    const bool bias = J.bias != nullptr;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        const float f = __fmul_rn(__fmul_rn(__int2float_rn(v[e]), scol[e]), srow);
        stg[e * kTileA + row] = __float2bfloat16_rn(bias ? __fadd_rn(f, brow) : f);
    }
    named_bar_sync(1, 128);
    const bool vec = (J.n & 7) == 0;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const int idx = tid + q * 128;          // 16 rows x 16 segments of 8 columns
        const int ml = idx >> 4, seg8 = idx & 15;
        const int m = j0 + ml, nb = a0 + seg8 * 8;
        if (m >= J.m || nb >= J.n) continue;
        const __nv_bfloat16 *src = stg + ml * kTileA + seg8 * 8;
        __nv_bfloat16 *dst = J.y + (size_t)m * J.n + nb;
        if (vec && nb + 8 <= J.n) {
            *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(src);
        } else {
            for (int e = 0; e < 8 && nb + e < J.n; ++e) dst[e] = src[e];
        }
    }
}

// Dequantise and store the 16 accumulators of A-row a0 + row and B-rows
// j0 .. j0+15 in either orientation.  srow is the scale of the A row and
// scol[e] the scale of B-row j0 + e (both staged by the caller): sx[m] and
// sw[n] for large M, sw[n] and sx[m] for the swapped (weights = A)
// orientation.  Both compute bf16(((float)acc * sx[m]) * sw[n]).  Called by
// all 128 epilogue threads; `chunk` counts the calls (it picks the transpose
// buffer of the swapped orientation).  sh: see emit_row16.
__device__ __forceinline__ void emit16s(const GemmJob &J, int swap, int a0, int row, int tid, int j0,
                                        const int32_t (&v)[16], float srow, float brow, const float *scol,
                                        __nv_bfloat16 *y_stage, int &chunk, int sh) {
    if (!swap) {
        emit_row16(J, a0 + row, j0, v, srow, scol, sh);
        return;
    }
    emit_swap16(J, a0, row, tid, j0, v, srow, brow, scol, y_stage + (chunk & 1) * 16 * kTileA, sh);
    ++chunk;
}

// Two TMEM loads of 16 columns each, one wait.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, int32_t (&v0)[16], int32_t (&v1)[16]) {
    uint32_t r0[16], r1[16];
    tmem_ld_32x32b_x16(taddr, r0);
    tmem_ld_32x32b_x16(taddr + 16u, r1);
    tmem_ld_wait();
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        v0[e] = (int32_t)r0[e];
        v1[e] = (int32_t)r1[e];
    }
}

// W4: the weight arrives as packed INT4 codes (wrows x 64 bytes per K
// block: the A tile of 128 rows in the swapped orientation, the B tile of bn
// rows otherwise); warps 6-13 unpack it into the wrows x 128-byte
// 128B-swizzled INT8 tile the MMA reads.
// WO: where INT4 weights go -- 0: INT8 weights (no unpacking), 1: the A
// operand (weight-streaming, a 128-row tile), 2: the B operand (bn rows).
template <int WO>
__global__ void __launch_bounds__(WO ? kThreadsW4 : kThreads, 1)
    gemm_i8_tc_kernel(const __grid_constant__ GemmMaps maps, const __grid_constant__ GemmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment for the 128-byte-swizzled operand tiles
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw);

    const int S = a.stages;
    const uint32_t b_bytes = (uint32_t)a.bn * kBlockK;
    const uint32_t a_off = 0;
    const uint32_t b_off = (uint32_t)S * kATileBytes;
    // W4: a staging slot per stage where the packed weight tile lands
    constexpr bool W4 = WO != 0;
    // W4: the unpacked weight bytes are 16 x code, so the accumulators are
    // 16 x the sums (exact: |16 * 7 * 127 * k| < 2^31 for every accepted k)
    constexpr int kAccShift = W4 ? 4 : 0;
    const int wrows = WO == 1 ? kTileA : a.bn;          // rows of the weight tile
    const uint32_t packed_bytes = (uint32_t)wrows * kPackedRowBytes;
    const uint32_t p_off = b_off + (uint32_t)S * b_bytes;
    const uint32_t bar_off = p_off + (W4 ? (uint32_t)S * packed_bytes : 0u);
    // barriers: full[S], empty[S], tfull[2], tempty[2], drain, red[2], W4: pfull[S]
    const uint32_t full_bar = base + bar_off;
    const uint32_t empty_bar = full_bar + 8u * S;
    const uint32_t tfull_bar = empty_bar + 8u * S;
    const uint32_t tempty_bar = tfull_bar + 16u;
    const uint32_t drain_bar = tempty_bar + 16u;
    const uint32_t red_bar = drain_bar + 8u;
    const uint32_t pfull_bar = red_bar + 16u;
    // W4: TMA copies land on pfull; the unpacking warps then arrive on full
    const uint32_t land_bar = W4 ? pfull_bar : full_bar;
    uint8_t *misc = smem + ((bar_off + 8u * (2 * S + kExtraBars + (W4 ? S : 0)) + 15u) & ~15u);
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(misc);
    volatile int *ticket = reinterpret_cast<volatile int *>(misc + 4);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 8);
    volatile int *red_ok = reinterpret_cast<volatile int *>(misc + 12);
    // [2][2 * kBiasStage]: B-row scales of a tile, then (large M, with a
    // bias) the bias of its columns
    float *sw_stage = reinterpret_cast<float *>(misc + 16);
    // [2][16][128] BF16: swapped-orientation output chunks, transposed so
    // that they leave as 16-byte row segments
    __nv_bfloat16 *y_stage = reinterpret_cast<__nv_bfloat16 *>(misc + 16 + 2 * 2 * kBiasStage * 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar + 8u * s, W4 ? kW4Warps : 1);
            mbar_init(empty_bar + 8u * s, 1);
            if (W4) mbar_init(pfull_bar + 8u * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar + 8u * b, 1);
            mbar_init(tempty_bar + 8u * b, 4);
        }
        mbar_init(drain_bar, 1);
        mbar_init(red_bar, 1);
        mbar_init(red_bar + 8u, 1);
        *abort_flag = 0;
        *ticket = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane < a.njobs) {
        tma_prefetch_desc(&maps.a[lane]);
        tma_prefetch_desc(&maps.b[lane]);
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
            // W4: the packed weight tile lands in the stage's staging slot
            // (unpacked into its operand slot by the unpacking warps)
            const uint32_t tx = W4 ? packed_bytes + (WO == 1 ? b_bytes : (uint32_t)kATileBytes)
                                   : (uint32_t)kATileBytes + b_bytes;
            const int RS = S;
            const uint32_t free_bar = empty_bar;
            int stage = 0;
            uint32_t phase = 0;
            bool waited = !a.w_prefetch;
            if (waited) pdl_wait();
            // activation loads held back until the grid dependency resolves
            int pend_n = 0;
            int pend_stage[kMaxRing], pend_x[kMaxRing], pend_y[kMaxRing], pend_job[kMaxRing];
            uint32_t issued_mask = 0, issued_par = 0;
            SegmentIter it;
            it.init(a);
            Segment sg;
            bool ok = true;
            while (ok && it.next(a, sg)) {
                const GemmJob &J = a.job[sg.job];
                int ta, tb;
                tile_coords(J, sg.tile, ta, tb);
                const CUtensorMap *tmW = a.swap ? &maps.a[sg.job] : &maps.b[sg.job];
                const CUtensorMap *tmX = a.swap ? &maps.b[sg.job] : &maps.a[sg.job];
                const int rowW = a.swap ? ta * kTileA : tb * a.bn;
                const int rowX = a.swap ? tb * a.bn : ta * kTileA;
                for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
                    if (!mbar_wait_bounded(free_bar + 8u * stage, phase ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t lb = land_bar + 8u * stage;
                    mbar_arrive_expect_tx(lb, tx);
                    const uint32_t sa = base + a_off + (uint32_t)stage * kATileBytes;
                    const uint32_t sb = base + b_off + (uint32_t)stage * b_bytes;
                    const int kx = kb * kBlockK;
                    const uint32_t sp = base + p_off + (uint32_t)stage * packed_bytes;   // W4 staging
                    const uint32_t sW = W4 ? sp : (a.swap ? sa : sb);
                    const uint32_t sX = a.swap ? sb : sa;
                    tma_load_2d(sW, tmW, lb, W4 ? kx / 2 : kx, rowW);
                    if (waited) {
                        tma_load_2d(sX, tmX, lb, kx, rowX);
                    } else {
                        pend_stage[pend_n] = stage;
                        pend_x[pend_n] = kx;
                        pend_y[pend_n] = rowX;
                        pend_job[pend_n] = sg.job;
                        if (++pend_n == RS) {
                            // while the prologue is still running, pull the
                            // next weight tiles of this CTA into L2 as well
                            SegmentIter it2 = it;
                            Segment s2 = sg;
                            int kb2 = kb + 1;
                            for (int pf = 0; pf < kL2PrefetchBlocks;) {
                                if (kb2 >= s2.kb1) {
                                    if (!it2.next(a, s2)) break;
                                    kb2 = s2.kb0;
                                    continue;
                                }
                                const GemmJob &J2 = a.job[s2.job];
                                int ta2, tb2;
                                tile_coords(J2, s2.tile, ta2, tb2);
                                const CUtensorMap *tw2 = a.swap ? &maps.a[s2.job] : &maps.b[s2.job];
                                tma_prefetch_l2_2d(tw2, kb2 * (W4 ? kBlockK / 2 : kBlockK),
                                                   a.swap ? ta2 * kTileA : tb2 * a.bn);
                                ++kb2;
                                ++pf;
                            }
                            pdl_wait();
                            waited = true;
                            for (int p = 0; p < pend_n; ++p) {
                                const int st = pend_stage[p];
                                const uint32_t sxa = a.swap ? base + b_off + (uint32_t)st * b_bytes
                                                            : base + a_off + (uint32_t)st * kATileBytes;
                                const CUtensorMap *tp = a.swap ? &maps.b[pend_job[p]] : &maps.a[pend_job[p]];
                                tma_load_2d(sxa, tp, land_bar + 8u * st, pend_x[p], pend_y[p]);
                            }
                            pend_n = 0;
                        }
                    }
                    issued_mask |= 1u << stage;
                    issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == RS) {
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
                    const CUtensorMap *tp = a.swap ? &maps.b[pend_job[p]] : &maps.a[pend_job[p]];
                    tma_load_2d(sxa, tp, land_bar + 8u * st, pend_x[p], pend_y[p]);
                }
            }
            if (!ok) {
                // let every copy this thread started land before the CTA exits
                volatile int no_abort = 0;
                for (int s = 0; s < RS; ++s)
                    if (issued_mask & (1u << s))
                        mbar_wait_bounded(land_bar + 8u * s, (issued_par >> s) & 1u, &no_abort);
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
            Segment sg;
            bool ok = true;
            while (ok && it.next(a, sg)) {
                const int buf = seg & 1;
                const uint32_t use = (uint32_t)(seg >> 1);
                if (!mbar_wait_bounded(tempty_bar + 8u * buf, (use & 1u) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)(buf * a.acc_cols);
                for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
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
                        umma_i8(d, da + 2u * kk, db + 2u * kk, idesc, (kb > sg.kb0 || kk > 0) ? 1u : 0u);
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
    } else if (W4 && warp >= 6) {
        // ------------------------------------------------ INT4 unpacking (kW4Warps warps)
        // All unpacking warps walk every K block in ring order (so no wait
        // runs ahead of a phase) and each unpacks its share of the stage:
        // wrows rows x 8 chunks of 16 codes, 8 B of nibbles -> 16 B of INT8
        // at the chunk's swizzled position (chunk c of row r sits at
        // 16 * (c ^ (r & 7)) in the row's 128 bytes) in the weight operand's
        // slot (A when swapped, else B); then full[stage].
        const int ct = (int)threadIdx.x - kThreads;
        constexpr int kCT = 32 * kW4Warps;
        int stage = 0;
        uint32_t phase = 0;
        SegmentIter it;
        it.init(a);
        Segment sg;
        bool ok = true;
        while (ok && it.next(a, sg)) {
            for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
                if (!mbar_wait_bounded(pfull_bar + 8u * stage, phase, abort_flag)) {
                    ok = false;
                    break;
                }
                const uint8_t *src = smem + p_off + (uint32_t)stage * packed_bytes;
                uint8_t *dst = WO == 1 ? smem + a_off + (uint32_t)stage * kATileBytes
                                       : smem + b_off + (uint32_t)stage * b_bytes;
                auto unpack = [&](int item) {
                    const int r = item >> 3, c = item & 7;
                    const uint2 w = *reinterpret_cast<const uint2 *>(src + r * 64 + c * 8);
                    // a two's-complement nibble in the high half of a byte,
                    // low half zero, is the int8 value 16 x code: no sign
                    // extension (the epilogue divides the exact sums by 16)
                    uint4 o;
                    o.x = (w.x << 4) & 0xF0F0F0F0u;     // codes 0-3 of the chunk
                    o.y = (w.y << 4) & 0xF0F0F0F0u;     // codes 4-7
                    o.z = w.x & 0xF0F0F0F0u;            // codes 8-11
                    o.w = w.y & 0xF0F0F0F0u;            // codes 12-15
                    *reinterpret_cast<uint4 *>(dst + r * 128 + ((c ^ (r & 7)) << 4)) = o;
                };
                if (WO == 1) {
                    // weight-streaming: a 128-row tile, a fixed trip count (fully unrolled)
#pragma unroll
                    for (int i = 0; i < kTileA * 8 / kCT; ++i) unpack(ct + kCT * i);
                } else {
#pragma unroll 4
                    for (int item = ct; item < wrows * 8; item += kCT) unpack(item);
                }
                fence_proxy_async_shared();      // the tensor core reads these stores
                __syncwarp();
                if (lane == 0) mbar_arrive(full_bar + 8u * stage);
                if (++stage == S) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else {
        // ------------------------------------------------ epilogue (4 warps)
        pdl_wait();
        const int quarter = warp & 3;              // TMEM lanes 32*quarter .. +31
        const int row = quarter * 32 + lane;       // row of the A tile
        const int ew = warp - 2;
        const int tid = ew * 32 + lane;
        int ychunk = 0;
        int seg = 0;
        SegmentIter it;
        it.init(a);
        Segment sg;
        while (it.next(a, sg, true)) {
            const GemmJob &J = a.job[sg.job];
            int ta, tb;
            tile_coords(J, sg.tile, ta, tb);
            const int buf = seg & 1;
            const uint32_t use = (uint32_t)(seg >> 1);
            const int i = ta * kTileA + row;
            // the scales of the tile's B rows go to shared memory and the
            // scale of this thread's A row to a register while the
            // accumulator is still being computed (double-buffered by
            // segment parity; the barrier below publishes them)
            float *scol = sw_stage + (seg & 1) * 2 * kBiasStage;
            float srow = 0.f, brow = 0.f;
            {
                const float *cs = a.swap ? J.sx : J.sw;
                const int clim = a.swap ? J.m : J.n;
                for (int cidx = tid; cidx < a.bn; cidx += 128) {
                    const int col = tb * a.bn + cidx;
                    scol[cidx] = col < clim ? __ldg(cs + col) : 0.f;
                    if (!a.swap && J.bias) scol[kBiasStage + cidx] = col < clim ? __bfloat162float(J.bias[col]) : 0.f;
                }
                if (a.swap && J.bias && i < J.n) brow = __bfloat162float(J.bias[i]);
                const float *rs = a.swap ? J.sw : J.sx;
                if (i < (a.swap ? J.n : J.m)) srow = __ldg(rs + i);
            }
            const bool full = mbar_wait_bounded(tfull_bar + 8u * buf, use & 1u, abort_flag);
            if (!named_bar_and(1, 128, full)) break;
            tc_fence_after();
            const bool whole = (sg.kb0 == 0 && sg.kb1 == J.kbpt);
            const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * a.acc_cols);
            if (sg.split < 0 && whole && !a.swap) {
                for (int c = 0; c < a.bn; c += 32) {
                    int32_t v0[16], v1[16];
                    __syncwarp();
                    tmem_ld32(tbase + (uint32_t)c, v0, v1);
                    const int j0 = tb * a.bn + c;
                    emit_row16(J, i, j0, v0, srow, scol + c, kAccShift);
                    emit_row16(J, i, j0 + 16, v1, srow, scol + c + 16, kAccShift);
                }
            } else if (sg.split < 0) {
                for (int c = 0; c < a.bn / 16; ++c) {
                    uint32_t r[16];
                    __syncwarp();
                    tmem_ld_32x32b_x16(tbase + (uint32_t)(c * 16), r);
                    tmem_ld_wait();
                    int32_t v[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] = (int32_t)r[e];
                    if (whole) {
                        emit16s(J, a.swap, ta * kTileA, row, tid, tb * a.bn + c * 16, v, srow, brow, scol + c * 16,
                                y_stage, ychunk, kAccShift);
                    } else {
                        int32_t *p = a.partial + ((size_t)sg.slot * a.bn + c * 16) * kTileA + row;
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            if (v[e] != 0) atomicAdd(p + (size_t)e * kTileA, v[e]);
                    }
                }
            } else {
                // A piece of a split tail tile.  The tile's counter holds the
                // pieces that finished their K range (low 16 bits) and the
                // pieces whose partial is stored (high bits).  Every piece
                // but the last to finish stores its INT32 partial in its own
                // region; the last one waits for those stores (the pieces it
                // waits on are already running), pulls the partials into
                // shared memory with bulk copies (the operand ring is idle:
                // this is the CTA's last segment and its MMAs are complete),
                // adds them to its accumulator in TMEM and writes the tile.
                const int ways = a.split_ways;
                named_bar_sync(1, 128);
                if (ew == 0 && lane == 0) {
                    const int old = atomicAdd(a.counters + sg.slot, 1);
                    *ticket = ((old & 0xFFFF) == ways - 1) ? 1 : 0;
                }
                named_bar_sync(1, 128);
                if (*ticket == 0) {
                    int32_t *pbase = a.partial + ((size_t)sg.slot * ways + sg.split) * a.bn * kTileA + row;
                    for (int c = 0; c < a.bn; c += 32) {
                        int32_t v0[16], v1[16];
                        __syncwarp();
                        tmem_ld32(tbase + (uint32_t)c, v0, v1);
                        int32_t *p = pbase + (size_t)c * kTileA;
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            __stcg(p + (size_t)e * kTileA, v0[e]);
                            __stcg(p + (size_t)(e + 16) * kTileA, v1[e]);
                        }
                    }
                    __threadfence();
                    named_bar_sync(1, 128);
                    if (ew == 0 && lane == 0) atomicAdd(a.counters + sg.slot, 1 << 16);
                } else {
                    const int others = ways - 1;
                    // column rounds, double-buffered in the operand ring
                    // (W4: the packed staging slots follow the operand slots and are idle too)
                    const uint32_t ring = (uint32_t)S * ((uint32_t)kATileBytes + b_bytes + (W4 ? packed_bytes : 0u));
                    int cols = (int)(ring / (2u * (uint32_t)others * kTileA * 4u)) / 32 * 32;
                    if (cols > a.bn) cols = a.bn;
                    const int rounds = (a.bn + cols - 1) / cols;
                    const uint32_t buf_bytes = (uint32_t)others * (uint32_t)cols * kTileA * 4u;
                    const int32_t *tile_parts = a.partial + (size_t)sg.slot * ways * a.bn * kTileA;
                    auto issue = [&](int r) {
                        const int col0 = r * cols;
                        const int nc = (a.bn - col0 < cols) ? a.bn - col0 : cols;
                        const uint32_t bytes = (uint32_t)nc * kTileA * 4u;
                        const uint32_t bar = red_bar + 8u * (uint32_t)(r & 1);
                        const uint32_t dst = base + (uint32_t)(r & 1) * buf_bytes;
                        mbar_arrive_expect_tx(bar, bytes * (uint32_t)others);
                        int o = 0;
                        for (int sp = 0; sp < ways; ++sp) {
                            if (sp == sg.split) continue;
                            bulk_load_1d(dst + (uint32_t)o * bytes,
                                         tile_parts + ((size_t)sp * a.bn + col0) * kTileA, bytes, bar);
                            ++o;
                        }
                    };
                    if (ew == 0 && lane == 0) {
                        int ok_wait = 1;
                        if ((ld_acquire_gpu(a.counters + sg.slot) >> 16) < others) {
                            const unsigned long long t0 = global_timer_ns();
                            for (uint32_t it_w = 1;; ++it_w) {
                                if ((ld_acquire_gpu(a.counters + sg.slot) >> 16) >= others) break;
                                if ((it_w & 63u) == 0 && global_timer_ns() - t0 > kWaitLimitNs) {
                                    atomicExch(&g_device_status, 7 /* CONVROT_ERR_DEVICE_TIMEOUT */);
                                    ok_wait = 0;
                                    break;
                                }
                            }
                        }
                        if (ok_wait) {
                            fence_proxy_async();
                            issue(0);
                            if (rounds > 1) issue(1);
                        }
                        *red_ok = ok_wait;
                    }
                    named_bar_sync(1, 128);
                    bool ok_red = *red_ok != 0;
                    int r = 0;
                    for (; r < rounds && ok_red; ++r) {
                        const int col0 = r * cols;
                        const int nc = (a.bn - col0 < cols) ? a.bn - col0 : cols;
                        const bool landed =
                            mbar_wait_bounded(red_bar + 8u * (uint32_t)(r & 1), (uint32_t)((r >> 1) & 1), abort_flag);
                        ok_red = named_bar_and(1, 128, landed);
                        if (!ok_red) break;
                        const int32_t *sbuf =
                            reinterpret_cast<const int32_t *>(smem + (size_t)(r & 1) * buf_bytes) + row;
                        for (int cc = 0; cc < nc; cc += 32) {
                            int32_t v0[16], v1[16];
                            __syncwarp();
                            tmem_ld32(tbase + (uint32_t)(col0 + cc), v0, v1);
                            for (int o = 0; o < others; ++o) {
                                const int32_t *q = sbuf + ((size_t)o * nc + cc) * kTileA;
#pragma unroll
                                for (int e = 0; e < 16; ++e) {
                                    v0[e] += q[(size_t)e * kTileA];
                                    v1[e] += q[(size_t)(e + 16) * kTileA];
                                }
                            }
                            const int j0 = tb * a.bn + col0 + cc;
                            emit_row16(J, i, j0, v0, srow, scol + col0 + cc, kAccShift);
                            emit_row16(J, i, j0 + 16, v1, srow, scol + col0 + cc + 16, kAccShift);
                        }
                        named_bar_sync(1, 128);     // buffer (r & 1) is read by everyone
                        if (r + 2 < rounds && ew == 0 && lane == 0) {
                            fence_proxy_async();
                            issue(r + 2);
                        }
                    }
                    if (ok_red) {
                        // leave the other pieces' regions zero again (the
                        // workspace is zero between calls), then the counter
                        const int4 z = make_int4(0, 0, 0, 0);
                        const size_t n4 = (size_t)a.bn * kTileA / 4;
                        for (int sp = 0; sp < ways; ++sp) {
                            if (sp == sg.split) continue;
                            int4 *dst = reinterpret_cast<int4 *>(const_cast<int32_t *>(tile_parts) +
                                                                 (size_t)sp * a.bn * kTileA);
                            for (size_t x = (size_t)tid; x < n4; x += 128) __stcg(dst + x, z);
                        }
                        if (ew == 0 && lane == 0) a.counters[sg.slot] = 0;
                    } else if (ew == 0 && lane == 0 && *red_ok) {
                        // a wait gave up at round r: let the copies already
                        // started (rounds r and r + 1 at most) land first
                        volatile int no_abort = 0;
                        const int issued = rounds < r + 2 ? rounds : r + 2;
                        for (int q = r; q < issued; ++q)
                            mbar_wait_bounded(red_bar + 8u * (uint32_t)(q & 1), (uint32_t)((q >> 1) & 1), &no_abort);
                    }
                }
                named_bar_sync(1, 128);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty_bar + 8u * buf);
            if (!whole && sg.split < 0) {
                __threadfence();
                named_bar_sync(1, 128);
                if (ew == 0 && lane == 0) {
                    const int mine = sg.kb1 - sg.kb0;
                    const int old = atomicAdd(a.counters + sg.slot, mine);
                    *ticket = (old + mine == J.kbpt) ? 1 : 0;
                }
                named_bar_sync(1, 128);
                const bool last = (*ticket != 0);
                if (last) {
                    __threadfence();
                    const int chunks = a.bn / 16;
                    int c = 0;
                    // four 16-column chunks in flight at a time (wide tiles)
                    for (; c + 4 <= chunks; c += 4) {
                        int32_t *p = a.partial + ((size_t)sg.slot * a.bn + c * 16) * kTileA + row;
                        int32_t v[4][16];
#pragma unroll
                        for (int h = 0; h < 4; ++h)
#pragma unroll
                            for (int e = 0; e < 16; ++e) v[h][e] = __ldcg(p + (size_t)(h * 16 + e) * kTileA);
#pragma unroll
                        for (int e = 0; e < 64; ++e) __stcg(p + (size_t)e * kTileA, 0);
#pragma unroll
                        for (int h = 0; h < 4; ++h)
                            emit16s(J, a.swap, ta * kTileA, row, tid, tb * a.bn + (c + h) * 16, v[h], srow, brow,
                                    scol + (c + h) * 16, y_stage, ychunk, kAccShift);
                    }
                    for (; c < chunks; ++c) {
                        int32_t *p = a.partial + ((size_t)sg.slot * a.bn + c * 16) * kTileA + row;
                        int32_t v[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = __ldcg(p + (size_t)e * kTileA);
#pragma unroll
                        for (int e = 0; e < 16; ++e) __stcg(p + (size_t)e * kTileA, 0);
                        emit16s(J, a.swap, ta * kTileA, row, tid, tb * a.bn + c * 16, v, srow, brow, scol + c * 16,
                                y_stage, ychunk, kAccShift);
                    }
                    if (ew == 0 && lane == 0) a.counters[sg.slot] = 0;
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

static void plan_common(GemmPlan *p) {
    // W4: every stage also holds the packed weight tile it is unpacked from
    const int wrows = p->swap ? kTileA : p->bn;
    const int stage_bytes = kATileBytes + p->bn * kBlockK + (p->w4 ? wrows * (int)kPackedRowBytes : 0);
    int stages = (200 * 1024) / stage_bytes;
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages < 2) stages = 2;
    p->stages = stages;
    p->acc_cols = p->bn;
    int cols = 32;
    while (cols < 2 * p->bn) cols <<= 1;
    p->tmem_cols = cols;
    p->smem_bytes = 1024 + stages * stage_bytes + 8 * (2 * stages + kExtraBars + (p->w4 ? stages : 0)) + 16 + 16 +
                    2 * 2 * kBiasStage * 4 + 2 * 16 * kTileA * 2;
    // workspace: counters, then INT32 partial tiles [slots][bn][128]
    const size_t cnt = ((size_t)p->slots * 4 + 255) / 256 * 256;
    p->ws_counters_off = 0;
    p->ws_partial_off = cnt;
    const int per_slot = p->split_ways > 1 ? p->split_ways : 1;
    p->ws_bytes = cnt + (size_t)p->slots * per_slot * p->bn * kTileA * 4;
}

void plan_gemm(int64_t m, int64_t n, int64_t k, int num_sms, GemmPlan *p, bool w4) {
    if (m > 256 && m <= kMaxSwapM) {
        // a few hundred rows: too few 128 x 256 tiles for 148 SMs; stream-K
        // over all of them, as in a batched launch
        plan_gemm_batch(m, 1, &n, &k, num_sms, p, w4);
        return;
    }
    *p = GemmPlan{};
    p->w4 = w4 ? 1 : 0;
    p->njobs = 1;
    p->swap = (m <= 256) ? 1 : 0;
    // an A operand streamed once from HBM against a single B tile (a
    // convolution's im2col rows with few output channels): 128-row B tiles
    // halve the ring stage, so twice the stages keep A in flight; the two
    // B tiles of an A tile run in the same wave and share its rows in L2
    const bool narrow = !p->swap && n <= 256 && (long long)m * k > kGroupABytes;
    p->bn = p->swap ? (int)((m + 15) / 16 * 16) : (narrow ? 128 : 256);
    p->rows_a[0] = p->swap ? n : m;
    p->rows_b[0] = p->swap ? m : n;
    const int tiles_a = (int)((p->rows_a[0] + kTileA - 1) / kTileA);
    const int tiles_b = (int)((p->rows_b[0] + p->bn - 1) / p->bn);
    const int kbpt = (int)((k + kBlockK - 1) / kBlockK);   // a partial last block reads zeros past k
    const int num_tiles = tiles_a * tiles_b;
    const long long units = (long long)num_tiles * kbpt;
    int tail_tile0;
    if (p->swap) {
        // few weight tiles: whole tiles in full waves, the rest split along K
        // (the INT32 partial tiles are small: bn <= 256 columns x 128 rows)
        p->grid = (int)(units < num_sms ? units : num_sms);
        p->full_waves = num_tiles / p->grid;
        tail_tile0 = p->full_waves * p->grid;
        p->full_tiles = tail_tile0;
    } else {
        // large M: whole 128 x 256 tiles in full waves.  A last, partial wave
        // that would leave most SMs idle is split instead: each of its tiles
        // into `ways` K ranges, one CTA each, with private INT32 partial tiles
        // (plain stores) summed by the tile's last piece.  Atomic stream-K
        // partials would cost more than the idle SMs lose at 128 x 256.
        p->grid = num_tiles < num_sms ? num_tiles : num_sms;
        p->full_waves = num_tiles / p->grid;
        const int tail = num_tiles - p->full_waves * p->grid;
        int ways = tail > 0 ? p->grid / tail : 0;
        if (ways > kMaxSplitWays) ways = kMaxSplitWays;
        if (ways > kbpt / 4) ways = kbpt / 4;
        if (ways >= 2) {
            p->full_tiles = p->full_waves * p->grid;
            p->split_ways = ways;
            p->split_pieces = tail * ways;
            p->slots = tail;
        } else {
            p->full_waves += tail > 0 ? 1 : 0;
            p->full_tiles = num_tiles;
        }
        tail_tile0 = num_tiles;
    }
    if (p->swap) {
        // stream-K over the tiles after the full waves; a tile shared by
        // several CTAs sums in the slot of one of them (one slot per CTA)
        p->tail_units = (long long)(num_tiles - tail_tile0) * kbpt;
        p->slots = p->tail_units > 0 ? p->grid : 0;
    }
    p->tiles_a[0] = tiles_a;
    p->tiles_b[0] = tiles_b;
    // an A operand that would not stay in L2 while a wave sweeps it is
    // taken in groups of 16 tiles (2048 rows)
    p->group_a[0] = (!p->swap && (long long)p->rows_a[0] * k > kGroupABytes && tiles_a > 16) ? 16 : tiles_a;
    p->kbpt[0] = kbpt;
    p->tile_base[0] = tail_tile0;
    p->unit0[0] = 0;
    plan_common(p);
}

void plan_gemm_batch(int64_t m, int njobs, const int64_t *n, const int64_t *k, int num_sms, GemmPlan *p,
                     bool w4) {
    *p = GemmPlan{};
    p->w4 = w4 ? 1 : 0;         // INT4 weights, unpacked into whichever operand holds them
    p->njobs = njobs;
    // m <= 256: the weights are the 128-row A operand and the activations
    // one B tile of roundup16(m) rows.  256 < m <= 512: activations are A
    // (up to four 128-row tiles), weights B (256-row tiles), and the A tiles
    // vary fastest, so a CTA reuses a weight tile from L2 for every
    // activation tile
    p->swap = m <= 256 ? 1 : 0;
    p->bn = p->swap ? (int)((m + 15) / 16 * 16) : 256;
    // large-M orientation: the A tiles (<= 4) are replicated over groups of
    // CTAs, the units are the K blocks of the weight (B) tiles
    p->rep = p->swap ? 1 : (int)((m + kTileA - 1) / kTileA);
    long long units = 0;
    for (int j = 0; j < njobs; ++j) {
        p->rows_a[j] = p->swap ? n[j] : m;
        p->rows_b[j] = p->swap ? m : n[j];
        p->tiles_a[j] = (int)((p->rows_a[j] + kTileA - 1) / kTileA);
        p->tiles_b[j] = (int)((p->rows_b[j] + p->bn - 1) / p->bn);
        p->group_a[j] = p->tiles_a[j];
        p->kbpt[j] = (int)((k[j] + kBlockK - 1) / kBlockK);
        p->tile_base[j] = 0;
        p->unit0[j] = units;
        units += (long long)(p->swap ? p->tiles_a[j] : p->tiles_b[j]) * p->kbpt[j];
    }
    // (at least one group: a GPU with fewer SMs than replicas still runs)
    const long long groups = num_sms >= p->rep ? num_sms / p->rep : 1;
    p->grid = (int)(units < groups ? units : groups) * p->rep;
    p->full_waves = 0;
    p->slots = p->grid;
    p->tail_units = units;
    plan_common(p);
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

// Byte matrix [rows, cols] -> tensor map with a (box_cols bytes x box_rows)
// box, no swizzle (packed INT4 weight tiles, unpacked in shared memory).
static bool make_tmap_plain(CUtensorMap *map, const void *ptr, int64_t rows, int64_t cols, int box_rows,
                            int box_cols) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
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

cudaError_t launch_gemm_i8(const GemmPlan &p, const GemmProblem *probs, void *ws, cudaStream_t stream,
                           bool pdl, bool w_prefetch) {
    GemmMaps maps;
    memset(&maps, 0, sizeof(maps));
    GemmArgs a;
    memset(&a, 0, sizeof(a));
    a.njobs = p.njobs;
    a.bn = p.bn;
    a.swap = p.swap;
    a.full_waves = p.full_waves;
    a.full_tiles = p.full_tiles;
    a.split_ways = p.split_ways;
    a.split_pieces = p.split_pieces;
    a.rep = p.rep > 0 ? p.rep : 1;

    a.tail_units = p.tail_units;
    a.stages = p.stages;
    a.acc_cols = p.acc_cols;
    a.tmem_cols = p.tmem_cols;
    a.w_prefetch = w_prefetch ? 1 : 0;
    a.counters = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + p.ws_counters_off);
    a.partial = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + p.ws_partial_off);
    for (int j = 0; j < p.njobs; ++j) {
        const GemmProblem &q = probs[j];
        const int8_t *A = p.swap ? q.wq : q.xq;
        const int8_t *B = p.swap ? q.xq : q.wq;
        // the weight's map: packed INT4 [n, k/2] bytes in plain (unswizzled)
        // 64-byte boxes, or INT8 [n, k] in 128-byte swizzled boxes
        const bool a_w4 = p.w4 && p.swap, b_w4 = p.w4 && !p.swap;
        if (a_w4 ? !make_tmap_plain(&maps.a[j], A, p.rows_a[j], q.k / 2, kTileA, (int)kPackedRowBytes)
                 : !make_tmap(&maps.a[j], A, p.rows_a[j], q.k, kTileA))
            return cudaErrorInvalidValue;
        if (b_w4 ? !make_tmap_plain(&maps.b[j], B, p.rows_b[j], q.k / 2, p.bn, (int)kPackedRowBytes)
                 : !make_tmap(&maps.b[j], B, p.rows_b[j], q.k, p.bn))
            return cudaErrorInvalidValue;
        GemmJob &J = a.job[j];
        J.m = (int)q.m;
        J.n = (int)q.n;
        J.k = (int)q.k;
        J.tiles_a = p.tiles_a[j];
        J.n_tiles_b = p.tiles_b[j];
        J.group_a = p.group_a[j];
        J.kbpt = p.kbpt[j];
        J.tile_base = p.tile_base[j];
        J.unit0 = p.unit0[j];
        J.sx = q.sx;
        J.sw = q.sw;
        J.y = q.y;
        J.acc = q.acc;
        J.bias = q.bias;
    }

    static bool configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !configured[dev]) {
        e = cudaFuncSetAttribute(gemm_i8_tc_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(gemm_i8_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(gemm_i8_tc_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        if (dev < 64) configured[dev] = true;
    }

    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)p.grid);
    cfg.blockDim = dim3(p.w4 ? kThreadsW4 : kThreads);
    cfg.dynamicSmemBytes = (size_t)p.smem_bytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    if (p.w4) return cudaLaunchKernelEx(&cfg, p.swap ? gemm_i8_tc_kernel<1> : gemm_i8_tc_kernel<2>, maps, a);
    return cudaLaunchKernelEx(&cfg, gemm_i8_tc_kernel<0>, maps, a);
}

}  // namespace convrot
