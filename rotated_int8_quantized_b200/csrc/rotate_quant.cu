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
// Design (B200): the main kernel (rotate_quant_rows_slots, below) gives 16
// threads to each 256-wide group and splits H_256 = H_16 (x) H_16; rows are
// split over a thread-block cluster when there are too few to fill the GPU.
// Every partial sum of +-BF16 values is exact in FP64, so any butterfly order
// gives the exact sum of the explicit matrix product, and one rounding to
// FP32 follows.  The row's rotated FP32 values wait in shared memory while
// the row maximum is reduced; then each thread packs 16 INT8 codes into one
// 16-byte store.  Long rows are split over a cluster too (at most one group
// per slot), so every row the API accepts (k <= 133120) stages in shared
// memory.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "gemm_i8.h"
#include "rotate_quant.h"

namespace convrot {

// Row quantisation helper: everything quant16 needs about a row's scale s.
struct RowScale {
    float s;        // s = fl(amax / 127)
    float r;        // fl(1 / s), correctly rounded
    bool zero;      // all-zero row: every code is 0
    bool fast;      // r is finite, so the rounding test below applies
};

__device__ __forceinline__ RowScale make_row_scale_levels(float amax, float levels) {
    RowScale rs;
    rs.s = __fdiv_rn(amax, levels);
    rs.zero = (amax == 0.0f);
    rs.r = rs.zero ? 0.0f : __frcp_rn(rs.s);
    rs.fast = !rs.zero && isfinite(rs.r);
    return rs;
}

__device__ __forceinline__ RowScale make_row_scale(float amax) {
    RowScale rs;
    rs.s = __fdiv_rn(amax, 127.0f);
    rs.zero = (amax == 0.0f);
    rs.r = rs.zero ? 0.0f : __frcp_rn(rs.s);
    // a subnormal s carries less than 24 bits, so the bound below needs a
    // normal one; rows that small take the division
    rs.fast = !rs.zero && isfinite(rs.r) && rs.s >= 1.17549435e-38f;
    return rs;
}

// The low bytes of a, b, c, d as one word (a in byte 0).
__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// q = clamp(rne(fl(y / s)), -127, 127) for 16 consecutive values y: the
// integer nearest to the correctly rounded FP32 quotient, ties to even,
// packed into one 16-byte word.
//
// Evaluated with Ziv's rounding test (A. Ziv, "Fast evaluation of elementary
// mathematical functions with correctly rounded last bit", ACM TOMS 17(3),
// 1991): a cheap approximation with a proven error bound decides the
// rounding whenever it lies far enough from a rounding boundary, and the
// exact evaluation runs only otherwise.  Here t = fl(y * r) with
// r = fl(1/s) satisfies |t - y/s| <= |y/s| (2^-23 + 2^-48) and
// |fl(y/s) - y/s| <= |y/s| 2^-24; since |y/s| <= 127 (1 + 2^-23),
// |t - fl(y/s)| < 2.3e-5.  When t is more than 3e-5 away from every
// half-integer, fl(y/s) rounds to the same integer as t; otherwise (about
// 6e-5 of the elements) the IEEE division is evaluated.
// Rounding to the nearest integer, ties to even, on the FP32 pipe instead of
// the conversion unit: for |t| < 2^22 the sum fl(t + 1.5 * 2^23) has an ulp
// of 1, so the addition itself rounds t to an integer (round-to-nearest-even
// is the FP32 mode), and the sum's low byte is that integer's two's
// complement byte (1.5 * 2^23 has a zero low byte).  With a normal s,
// |t| <= 127 (1 + 3 * 2^-24), so the fast path needs no clamp.
// The fast path is straight-line code over the 16 values (independent work
// for the scheduler), with one predicate accumulating "near a half-integer
// (or NaN)"; the division runs only where some thread of the warp needs
// it.  Every thread of `mask` (the active threads) must call it.
constexpr float kRoundMagic = 12582912.0f;          // 1.5 * 2^23
constexpr int kRoundMagicBits = 0x4B400000;         // its bit pattern

__device__ __forceinline__ uint4 quant16(const float (&y)[16], const RowScale &rs, unsigned mask) {
    uint32_t b[16];
    bool near = false;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        const float t = __fmul_rn(y[e], rs.r);
        const float big = __fadd_rn(t, kRoundMagic);
        b[e] = __float_as_uint(big);                                 // low byte: rne(t)
        near |= !(fabsf(__fsub_rn(t, __fsub_rn(big, kRoundMagic))) < 0.49997f);   // NaN too
    }
    const bool slow = near || !rs.fast;      // zero rows too (their codes are set below)
    if (__any_sync(mask, slow) && slow) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const float t = __fmul_rn(y[e], rs.r);
            const float f = __fsub_rn(__fadd_rn(t, kRoundMagic), kRoundMagic);
            if (!rs.fast || !(fabsf(__fsub_rn(t, f)) < 0.49997f)) {
                const int c = __float_as_int(__fadd_rn(__fdiv_rn(y[e], rs.s), kRoundMagic)) - kRoundMagicBits;
                b[e] = (uint32_t)min(max(c, -127), 127);
            }
        }
    }
    if (rs.zero) return make_uint4(0u, 0u, 0u, 0u);
    return make_uint4(pack_low_bytes(b[0], b[1], b[2], b[3]), pack_low_bytes(b[4], b[5], b[6], b[7]),
                      pack_low_bytes(b[8], b[9], b[10], b[11]), pack_low_bytes(b[12], b[13], b[14], b[15]));
}


// The same codes with the FP32 pair instructions of sm_100 (two values per
// instruction) and fused multiply-adds: e = fl(y r + 1.5 * 2^23) rounds the
// exact product y r to the nearest integer (ties to even; the sum's ulp is
// 1), and d = fl(y r - (e - 1.5 * 2^23)) is the exact residual rounded once
// (|d| <= 0.5, error <= 2^-25).  With |y r - y/s| <= |y/s| 2^-24 and
// |fl(y/s) - y/s| <= |y/s| 2^-24, |y/s| <= 127 (1 + 2^-23), a residual
// below 0.49997 puts fl(y/s) within 0.49999 of the same integer, so e's low
// byte is rne(fl(y/s)) there; elsewhere the division decides, as in
// quant16.  The largest |d| of the 16 values comes from 3-input maxima of
// magnitudes.  Inputs are finite (non-finite values give unspecified codes).
// max(|a|, |b|, |c|) in one instruction (sm_100).
__device__ __forceinline__ float max3abs(float a, float b, float c) {
    float d;
    asm("max.abs.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
__device__ __forceinline__ uint32_t min_s16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("min.s16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t sub_f32x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t pack_f32x2(float a, float b) {
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(a), "f"(b));
    return d;
}
__device__ __forceinline__ void unpack_f32x2(uint64_t d, float &a, float &b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(d));
}

__device__ __forceinline__ uint4 quant16x2(const float (&y)[16], const RowScale &rs, unsigned mask) {
    uint32_t b[16];
    float dmax = 0.f;
    const uint64_t r2 = pack_f32x2(rs.r, rs.r), m2 = pack_f32x2(kRoundMagic, kRoundMagic);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint64_t y2 = pack_f32x2(y[2 * i], y[2 * i + 1]);
        const uint64_t e2 = fma_f32x2(y2, r2, m2);                   // rne(y r) in the low byte
        const uint64_t d2 = fma_f32x2(y2, r2, sub_f32x2(m2, e2));    // y r - rne(y r), rounded once
        float d0, d1, e0, e1;
        unpack_f32x2(d2, d0, d1);
        unpack_f32x2(e2, e0, e1);
        b[2 * i] = __float_as_uint(e0);
        b[2 * i + 1] = __float_as_uint(e1);
        dmax = max3abs(d0, d1, dmax);
    }
    const bool slow = !(dmax < 0.49997f) || !rs.fast;   // zero rows too (codes set below)
    if (__any_sync(mask, slow) && slow) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const float ei = __fmaf_rn(y[e], rs.r, kRoundMagic);
            const float di = __fmaf_rn(y[e], rs.r, __fsub_rn(kRoundMagic, ei));
            if (!rs.fast || !(fabsf(di) < 0.49997f)) {
                const int c = __float_as_int(__fadd_rn(__fdiv_rn(y[e], rs.s), kRoundMagic)) - kRoundMagicBits;
                b[e] = (uint32_t)min(max(c, -127), 127);
            }
        }
    }
    if (rs.zero) return make_uint4(0u, 0u, 0u, 0u);
    return make_uint4(pack_low_bytes(b[0], b[1], b[2], b[3]), pack_low_bytes(b[4], b[5], b[6], b[7]),
                      pack_low_bytes(b[8], b[9], b[10], b[11]), pack_low_bytes(b[12], b[13], b[14], b[15]));
}


// INT4 weight codes (W4A8): q = clamp(rne(fl(y / s)), -7, 7) with s = a / 7,
// the same rounding test as quant16 (|y/s| <= 7 here, so the bound holds with
// room to spare), packed two per byte: byte j of the 8 holds code j in its
// low nibble and code 8 + j in its high nibble.
__device__ __forceinline__ uint2 quant16_int4(const float (&y)[16], const RowScale &rs, unsigned mask) {
    int code[16];
    bool slow = false;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        const float t = __fmul_rn(y[e], rs.r);
        const float big = __fadd_rn(t, kRoundMagic);
        code[e] = __float_as_int(big) - kRoundMagicBits;
        slow |= !(fabsf(__fsub_rn(t, __fsub_rn(big, kRoundMagic))) < 0.49997f);
    }
    slow = slow || !rs.fast;
    if (__any_sync(mask, slow) && slow) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const float t = __fmul_rn(y[e], rs.r);
            const float f = __fsub_rn(__fadd_rn(t, kRoundMagic), kRoundMagic);
            if (!rs.fast || !(fabsf(__fsub_rn(t, f)) < 0.49997f))
                code[e] = __float_as_int(__fadd_rn(__fdiv_rn(y[e], rs.s), kRoundMagic)) - kRoundMagicBits;
        }
    }
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int lo = rs.zero ? 0 : min(max(code[j], -7), 7);
        const int hi = rs.zero ? 0 : min(max(code[8 + j], -7), 7);
        w[j >> 2] |= (uint32_t)((lo & 0xF) | ((hi & 0xF) << 4)) << (8 * (j & 3));
    }
    return make_uint2(w[0], w[1]);
}

// ---------------------------------------------------------------------------
// Main variant: 16 threads ("a slot") per 256-group, H_256 = H_16 (x) H_16.
// Thread t of a slot loads elements 16t .. 16t+15 (32 contiguous bytes; the
// slot reads the group's 512 bytes coalesced), transforms index bits 0-3 in
// registers, exchanges through a padded shared-memory transpose, transforms
// index bits 4-7 in registers and so ends up holding outputs t, t+16, ...,
// t+240.  Every group of a row is in flight at once (up to 32 slots per CTA,
// several groups per slot for long rows), so a decode-sized matrix of a few
// rows costs one load latency.
// ---------------------------------------------------------------------------
constexpr int kMaxSlots = 32;          // 512 threads
constexpr int kXchFull = 16 * 17;     // doubles per slot: whole 16 x 16 transpose, padded
constexpr int kXchHalf = 16 * 9;      // doubles per slot: half of it at a time, padded
constexpr int kMaxParts = 8;           // CTAs per row (portable cluster size)
// FP32 staging of a rotated group: 256 values padded to 272 so that the two
// slots of a warp write different banks; inside, 16-value chunks whose four
// float4 parts are XOR-swizzled so that the quantiser's 16-byte reads of
// consecutive chunks are conflict-free.  Decode-sized launches (HALF) keep
// the plain layout: a few rows are latency-bound, not bank-bound, and the
// extra address arithmetic raised the decode variant above 96 registers,
// which cost a co-resident GEMM CTA during the programmatic-launch overlap
// (2 us per decode step).
constexpr int kYGroupStride = 272;
__host__ __device__ constexpr int y_group_stride(bool half) { return half ? 256 : kYGroupStride; }
constexpr int kSlotsSmemMax = 226 * 1024;   // dynamic shared memory per CTA (227 KB minus the static part)

// Butterflies of strides h < hmax only (hmax a power of two <= 16): the
// transform of groups smaller than 16 along these index bits.
__device__ __forceinline__ void fwht16_regs_upto(double (&v)[16], int hmax) {
#pragma unroll
    for (int h = 1; h < 16; h <<= 1) {
        if (h < hmax) {
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
}

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
    int k, gps, slots;      // gps / slots for the 256-element chunks of ONE part of a row
    int group;              // rotation group G (power of two, 16 .. 256; 256 unless DYN)
    int exact_scale;        // G a power of four: 1/sqrt(G) is a power of two
    double scale;           // 1/sqrt(G) when exact_scale
    double root;            // fl64(sqrt(G)) otherwise (the quotient is rounded once in FP64)
};
struct RQArgs {
    int njobs, rows;
    int parts;              // CTAs (a thread-block cluster) per row
    int rpc;                // rows per CTA: 1, or several short rows (parts == 1, at most 2 slots a row)
    ConvGeom conv;          // MODE 3 / 4: the convolution the rows come from
    RQJobDev job[kMaxJobs];
};

// Groups per slot and slots for `groups` groups.
static void rq_shape(int groups, int *gps, int *slots) {
    int g = (groups + kMaxSlots - 1) / kMaxSlots;
    if (g == 5) g = 6;
    if (g < 1) g = 1;
    *gps = g;
    *slots = (groups + g - 1) / g;
}

__device__ __forceinline__ uint32_t cluster_map(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t caddr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(caddr) : "memory");
    return v;
}
__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}


// Per 16-bit half of a word of two BF16 values: 0x7FFF + |x| for x != 0,
// and 0x7FFF for a zero, so that a signed 16-bit minimum ignores zeros and
// otherwise orders by magnitude (no carry crosses the halves: each half sum
// is at most 0xFFFE).
__device__ __forceinline__ uint32_t nonzero_mag_key(uint32_t w) {
    return (w & 0x7FFF7FFFu) + 0x7FFF7FFFu;
}
// The smallest nonzero BF16 magnitude (bits) a key minimum stands for, or
// 0x7FFF + 1 when every value was zero.
__device__ __forceinline__ int key_min_magnitude(uint32_t k) {
    const int lo = (int)(int16_t)(k & 0xFFFFu), hi = (int)(int16_t)(k >> 16);
    const int m = lo < hi ? lo : hi;
    return m == 0x7FFF ? 0x8000 : m + 0x8001;
}

// Exactness threshold of a row (BF16 magnitude bits): the FP64 sums of a
// group are exact while its nonzero inputs span at most 37 binades
// (frexp exponents e_max - e_min <= 37).  The group's largest input is at
// most max_j |S_j| = sqrt(G) max_j |y_j| <= 16 amax (Parseval), so
// e_max <= e(16 amax) <= e(amax) + 4; a row whose nonzero inputs are all at
// least 2^(e(amax) - 33) is inside the domain (one binade of slack).
// Returns the bits of 2^(e(amax) - 33) (0: no BF16 value is below it, or
// amax == 0); a nonzero input with smaller magnitude bits MAY be outside
// the domain.
__device__ __forceinline__ int exactness_threshold_bits(float amax) {
    // e(amax) from the FP32 exponent field (e = field - 126 for a normal
    // amax); a subnormal, zero or non-finite amax has no threshold that a
    // BF16 input could fall below except in the subnormal range: 0 there
    const int field = (int)((__float_as_uint(amax) >> 23) & 0xFFu);
    const int p = field - 159;                      // e(amax) - 33
    if (field == 0 || field == 0xFF) return 0;
    if (p >= -126) return (p + 127) << 7;
    if (p >= -133) return 1 << (p + 133);
    return 0;
}

// Record a possible exactness-domain violation (keeps an earlier status).
__device__ __forceinline__ void report_inexact_domain() {
    atomicCAS(&g_device_status, 0, 8 /* CONVROT_WARN_INEXACT_DOMAIN */);
}

// Layout of the rotated pixels (MODE 5 / 6, rotate_pixels_kernel): FP32
// [pixels, c], and inside each 16-value chunk ci of a pixel, float4 part j
// stored at position
// j ^ yrot_swizzle(ci), so that 8 lanes reading 8 consecutive chunks one
// float4 part at a time hit 8 different 16-byte bank groups.
__host__ __device__ __forceinline__ int yrot_swizzle(int ci) { return (ci >> 1) & 3; }

// One row per CTA (parts == 1) or per cluster of `parts` CTAs: CTA p of the
// cluster rotates groups [p*G/parts, (p+1)*G/parts) of the row, the row
// maximum is combined through distributed shared memory, then each CTA
// quantises its own groups.  Decode-sized matrices (a few rows) are spread
// over many SMs this way.
// HALF: transpose in two halves through a 16 x 9 buffer (half the shared
// memory, used for decode-sized launches whose CTAs should fit beside a
// GEMM CTA); otherwise in one pass through a 16 x 17 buffer and in place
// (fewer registers, for launches with a row per CTA).
// DYN: groups other than 256 (--dynamic-convrot): a 256-element chunk holds
// 256/G independent groups (butterflies of strides < G only), a row's last
// chunk may be partial (k % 256 != 0; k is a multiple of G), and the
// normalisation divides by sqrt(G) in FP64 when G is not a power of four.
// MODE 0: INT8 codes, groups of 256; 1: INT8, any group (DYN below); 2: INT4
// weight codes (levels -7..7, scale a/7), packed two per byte, any group;
// 3: INT8 codes of the im2col rows of a convolution, gathered from NHWC
// input; 4: INT8 codes of a convolution's OIHW weight in the im2col order;
// 5: the rotated FP32 rows themselves and their maxima (no quantisation):
// every input pixel of a convolution rotated once, for the im2col gather;
// 6: the same with groups of 256 and whole 256-chunks (no DYN paths).
template <int GPS, bool HALF, int MODE, bool MR = false>
__global__ void __launch_bounds__(kMaxSlots * 16, (GPS == 1 && !HALF) ? 2 : 1)
    rotate_quant_rows_slots(const __grid_constant__ RQArgs args) {
    constexpr bool ROT = MODE == 5 || MODE == 6;    // rotated values only
    constexpr bool DYN = MODE != 0 && MODE != 6;
    constexpr int kXchStride = HALF ? kXchHalf : kXchFull;
    extern __shared__ __align__(16) uint8_t rq_smem[];
    __shared__ float red[kMaxSlots / 2];
    __shared__ float part_max;
    pdl_wait();
    pdl_launch_dependents();

    const int C = args.parts;
    // several short rows per CTA: 16 or 32 threads a row, each row inside one warp
    const int R = MR ? args.rpc : 1;
    const int row_threads = (int)blockDim.x / R;
    const int rloc = R > 1 ? (int)threadIdx.x / row_threads : 0;
    const int part = R > 1 ? 0 : (int)(blockIdx.x % (unsigned)C);
    const int rowid = R > 1 ? (int)blockIdx.x * R + rloc : (int)(blockIdx.x / (unsigned)C);
    if (R > 1 && rowid >= args.rows * args.njobs) return;     // the last CTA's missing rows (whole warps or half-warps)
    const int jb = rowid / args.rows;
    const int row = rowid - jb * args.rows;
    const RQJobDev &J = args.job[jb];
    const int k = J.k, gps = J.gps, slots = J.slots;
    const int groups = DYN ? (k + 255) >> 8 : k >> 8;     // 256-element chunks
    const int g0 = part * groups / C, g1 = (part + 1) * groups / C;
    double *xch = reinterpret_cast<double *>(rq_smem);                    // slots * 272 doubles
    float *ybuf = reinterpret_cast<float *>(rq_smem + (size_t)(blockDim.x >> 4) * kXchStride * 8) +
                  (size_t)rloc * (g1 - g0) * y_group_stride(HALF);

    const int tid = (int)threadIdx.x - rloc * row_threads;     // thread within its row
    const int slot = tid >> 4, t = tid & 15;
    const int cta_slot = R > 1 ? (int)(threadIdx.x >> 4) : slot;      // half-warp within the CTA
    const unsigned half_mask = 0xFFFFu << (16 * (cta_slot & 1));
    const __nv_bfloat16 *arow = J.a + (size_t)row * k;

    // MODE 3: the row is output pixel (b, oy, ox) of the convolution
    int cb = 0, coy = 0, cox = 0;
    if (MODE == 3) {
        const int hw = args.conv.oh * args.conv.ow;
        cb = row / hw;
        coy = (row - cb * hw) / args.conv.ow;
        cox = row - cb * hw - coy * args.conv.ow;
    }

    // issue every load of this thread first
    uint4 raw[GPS][2];
#pragma unroll
    for (int gi = 0; gi < GPS; ++gi) {
        const int g = g0 + slot + gi * slots;
        if (gi < gps && slot < slots && g < g1) {
            const int kel = g * 256 + t * 16;            // first of this thread's 16 elements
            raw[gi][0] = make_uint4(0u, 0u, 0u, 0u);     // zeros past the row / outside the image
            raw[gi][1] = make_uint4(0u, 0u, 0u, 0u);
            if (MODE == 3) {
                // im2col gather from NHWC: tap (ky, kx), 16 channels from c0
                const ConvGeom &cg = args.conv;
                if (kel < k) {
                    const int tap = kel / cg.c, c0 = kel - tap * cg.c;
                    const int ky = tap / cg.kw, kx = tap - ky * cg.kw;
                    const int iy = coy * cg.stride - cg.pad + ky * cg.dil;
                    const int ix = cox * cg.stride - cg.pad + kx * cg.dil;
                    if (iy >= 0 && iy < cg.h && ix >= 0 && ix < cg.w) {
                        const uint4 *src = reinterpret_cast<const uint4 *>(
                            J.a + (((size_t)cb * cg.h + iy) * cg.w + ix) * cg.c + c0);
                        raw[gi][0] = __ldg(src);
                        raw[gi][1] = __ldg(src + 1);
                    }
                }
            } else if (MODE == 4) {
                // weight row o in the im2col order from OIHW: w[o, c0 + e, ky, kx]
                const ConvGeom &cg = args.conv;
                if (kel < k) {
                    const int tap = kel / cg.c, c0 = kel - tap * cg.c;
                    const int taps = cg.kh * cg.kw;
                    const unsigned short *w = reinterpret_cast<const unsigned short *>(J.a) +
                                              ((size_t)row * cg.c + c0) * taps + tap;
                    uint32_t v[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        v[e] = (uint32_t)__ldg(w + (size_t)(2 * e) * taps) |
                               ((uint32_t)__ldg(w + (size_t)(2 * e + 1) * taps) << 16);
                    raw[gi][0] = make_uint4(v[0], v[1], v[2], v[3]);
                    raw[gi][1] = make_uint4(v[4], v[5], v[6], v[7]);
                }
            } else if (!DYN || kel < k) {
                const uint4 *src = reinterpret_cast<const uint4 *>(arow + (size_t)g * 256 + t * 16);
                raw[gi][0] = __ldg(src);
                raw[gi][1] = __ldg(src + 1);
            }
        }
    }

    double *xb = xch + cta_slot * kXchStride;
    float amax = 0.f;
    uint32_t mkey = 0x7FFF7FFFu;       // smallest nonzero input magnitude (exactness domain)
#pragma unroll
    for (int gi = 0; gi < GPS; ++gi) {
        const int g = g0 + slot + gi * slots;
        if (gi < gps && slot < slots && g < g1) {
            double v[16];
            const uint32_t w[8] = {raw[gi][0].x, raw[gi][0].y, raw[gi][0].z, raw[gi][0].w,
                                   raw[gi][1].x, raw[gi][1].y, raw[gi][1].z, raw[gi][1].w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                mkey = min_s16x2(mkey, nonzero_mag_key(w[i]));
                bf16x2_to_f64(w[i], v[2 * i], v[2 * i + 1]);
            }
            if (DYN)
                fwht16_regs_upto(v, J.group < 16 ? J.group : 16);
            else
                fwht16_regs(v);                              // index bits 0-3
            // transpose across the slot's 16 threads: thread u needs element
            // 16*j + u of every thread j, i.e. v[u] of thread j (padded rows:
            // conflict-free both ways)
            double x[16];
            if (HALF) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) xb[9 * t + i] = v[8 * h + i];
                    __syncwarp(half_mask);
                    if ((t >> 3) == h) {
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj) x[jj] = xb[9 * jj + (t & 7)];
                    }
                    __syncwarp(half_mask);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) xb[17 * t + i] = v[i];
                __syncwarp(half_mask);
#pragma unroll
                for (int i = 0; i < 16; ++i) x[i] = xb[t + 17 * i];
                __syncwarp(half_mask);
            }
            if (DYN)
                fwht16_regs_upto(x, J.group >> 4);
            else
                fwht16_regs(x);                              // index bits 4-7
            // output 16*i + t of the group is element t of chunk i (its
            // float4 part XOR-swizzled in launches with a row per CTA)
            float *yg = ybuf + (size_t)(g - g0) * y_group_stride(HALF) + (HALF ? t : (t & 3));
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float y = DYN ? __double2float_rn(J.exact_scale ? x[i] * J.scale : __ddiv_rn(x[i], J.root))
                                    : __double2float_rn(x[i] * 0.0625);   // / sqrt(256), exact
                yg[16 * i + (HALF ? 0 : 4 * ((t >> 2) ^ ((i >> 1) & 3)))] = y;
                amax = fmaxf(amax, fabsf(y));
            }
        }
    }

    // maximum over this CTA's part of the row
    float rmax;
    if (R > 1) {
        const unsigned row_mask = row_threads == 32 ? 0xffffffffu : half_mask;
        for (int o = row_threads >> 1; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(row_mask, amax, o));
        rmax = amax;
    } else {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const int warp = tid >> 5, lane = tid & 31, nwarps = (blockDim.x + 31) >> 5;
        if (lane == 0) red[warp] = amax;
        __syncthreads();
        rmax = red[0];
        for (int w = 1; w < nwarps; ++w) rmax = fmaxf(rmax, red[w]);
    }
    if (C > 1) {
        // combine the parts of the row across the cluster
        if (tid == 0) part_max = rmax;
        cluster_arrive();
        cluster_wait();
        if (tid == 0) {
            const uint32_t local = smem_addr(&part_max);
            float m = 0.f;
            for (int r = 0; r < C; ++r) m = fmaxf(m, ld_cluster_f32(cluster_map(local, (uint32_t)r)));
            red[0] = m;
        }
        __syncthreads();
        rmax = red[0];
        cluster_arrive();   // this CTA no longer reads its peers; matched by the wait before exit
    }
    const RowScale rs = MODE == 2 ? make_row_scale_levels(rmax, 7.0f) : make_row_scale(rmax);
    {
        const unsigned all = __activemask();
        if (__any_sync(all, key_min_magnitude(mkey) < exactness_threshold_bits(rmax)) &&
            (threadIdx.x & 31) == (unsigned)(__ffs(all) - 1))
            report_inexact_domain();
    }

    // quantise 16 consecutive outputs per thread, one 16-byte store
    int8_t *qrow = J.q + (size_t)row * k + (size_t)g0 * 256;
    int chunks = (g1 - g0) * 16;
    if (DYN && g0 * 256 + chunks * 16 > k) chunks = (k - g0 * 256) / 16;     // partial last chunk
    for (int c0 = 0; c0 < chunks; c0 += (R > 1 ? (unsigned)row_threads : blockDim.x)) {
        const int c = c0 + tid;
        const unsigned mask = __ballot_sync(__activemask(), c < chunks);
        if (c < chunks) {
            const int ci = c & 15;     // chunk within its group
            const float4 *src = reinterpret_cast<const float4 *>(
                HALF ? ybuf + c * 16 : ybuf + (size_t)(c >> 4) * kYGroupStride + ci * 16);
            float y[16];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 f = src[HALF ? i : (i ^ ((ci >> 1) & 3))];
                y[4 * i] = f.x;
                y[4 * i + 1] = f.y;
                y[4 * i + 2] = f.z;
                y[4 * i + 3] = f.w;
            }
            if (ROT) {    // rotated values themselves (FP32 [rows, k], in J.q), float4 parts swizzled
                float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(J.q) + (size_t)row * k +
                                                         (size_t)g0 * 256 + c * 16);
                const int sw = yrot_swizzle(c);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dst[i ^ sw] = make_float4(y[4 * i], y[4 * i + 1], y[4 * i + 2], y[4 * i + 3]);
            } else if (MODE == 2) {     // packed INT4: row stride k/2 bytes
                *reinterpret_cast<uint2 *>(J.q + (size_t)row * (k / 2) + (size_t)g0 * 128 + c * 8) =
                    quant16_int4(y, rs, mask);
            } else {
                *reinterpret_cast<uint4 *>(qrow + c * 16) = HALF ? quant16(y, rs, mask) : quant16x2(y, rs, mask);
            }
        }
    }
    // MODE 5 / 6 keep the row maximum (the scale is a later, per-im2col-row step)
    if (tid == 0 && part == 0) J.s[row] = ROT ? rmax : rs.s;
    if (C > 1) {
        __syncwarp();
        cluster_wait();   // peers may still read part_max until they arrive
    }
}

template <int GPS, bool HALF, int MODE, bool MR = false>
static cudaError_t launch_slots(cudaLaunchConfig_t &cfg, const RQArgs &args, int max_slots, int max_local_groups) {
    cfg.blockDim = dim3(max_slots * 16 * args.rpc);
    cfg.dynamicSmemBytes = ((size_t)max_slots * (HALF ? kXchHalf : kXchFull) * 8 +
                            (size_t)max_local_groups * y_group_stride(HALF) * 4) * args.rpc;
    static bool configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !configured[dev]) {
        e = cudaFuncSetAttribute(rotate_quant_rows_slots<GPS, HALF, MODE, MR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSlotsSmemMax);
        if (e != cudaSuccess) return e;
        if (dev < 64) configured[dev] = true;
    }
    return cudaLaunchKernelEx(&cfg, rotate_quant_rows_slots<GPS, HALF, MODE, MR>, args);
}

template <int MODE>
static cudaError_t launch_gps(cudaLaunchConfig_t &cfg, const RQArgs &args, bool half, int max_gps, int max_slots,
                              int max_local) {
    if constexpr (MODE != 2 && MODE != 4) {
        if (args.rpc > 1) return launch_slots<1, false, MODE, true>(cfg, args, max_slots, max_local);
    }
    if constexpr (MODE < 2) {       // the half-size transpose: decode-sized activations only
        if (half) {
            switch (max_gps) {
                case 1: return launch_slots<1, true, MODE>(cfg, args, max_slots, max_local);
                case 2: return launch_slots<2, true, MODE>(cfg, args, max_slots, max_local);
                case 3: return launch_slots<3, true, MODE>(cfg, args, max_slots, max_local);
                case 4: return launch_slots<4, true, MODE>(cfg, args, max_slots, max_local);
                default: return launch_slots<6, true, MODE>(cfg, args, max_slots, max_local);
            }
        }
    }
    switch (max_gps) {
        case 1: return launch_slots<1, false, MODE>(cfg, args, max_slots, max_local);
        case 2: return launch_slots<2, false, MODE>(cfg, args, max_slots, max_local);
        case 3: return launch_slots<3, false, MODE>(cfg, args, max_slots, max_local);
        case 4: return launch_slots<4, false, MODE>(cfg, args, max_slots, max_local);
        default: return launch_slots<6, false, MODE>(cfg, args, max_slots, max_local);
    }
}

// CTAs per row (a thread-block cluster).  When the rows alone do not fill
// the GPU, enough to spread the work over the SMs while the whole grid stays
// within one wave (about two CTAs per SM), so every CTA starts at once and
// triggers the dependent GEMM's launch early.  Otherwise one, unless a row is
// too long to stage in one CTA's shared memory.
static size_t rq_smem_bytes(int njobs, const RQProblem *probs, int parts, bool half, int *max_slots,
                            int *max_gps, int *max_local);

static int rq_parts(int njobs, int64_t rows, const RQProblem *probs, int num_sms, bool half) {
    int parts = 1;
    int ms, mg, ml;
    while (parts < kMaxParts &&
           (rq_smem_bytes(njobs, probs, parts, half, &ms, &mg, &ml) > (size_t)kSlotsSmemMax || mg > 6))
        ++parts;
    const int64_t total_rows = rows * njobs;
    if (total_rows < num_sms) {
        int64_t spread = (2 * (int64_t)num_sms) / total_rows;
        if (spread > kMaxParts) spread = kMaxParts;
        if (spread > parts) parts = (int)spread;
    }
    return parts;
}

// Shared-memory bytes and shape of one CTA of a launch with `parts` CTAs per row.
static size_t rq_smem_bytes(int njobs, const RQProblem *probs, int parts, bool half, int *max_slots,
                            int *max_gps, int *max_local) {
    int ms = 0, mg = 0, ml = 0;
    for (int j = 0; j < njobs; ++j) {
        const int groups = (int)((probs[j].k + 255) >> 8);
        const int local = (groups + parts - 1) / parts;
        int g, sl;
        rq_shape(local, &g, &sl);
        ms = sl > ms ? sl : ms;
        mg = g > mg ? g : mg;
        ml = local > ml ? local : ml;
    }
    *max_slots = ms;
    *max_gps = mg;
    *max_local = ml;
    return (size_t)ms * (half ? kXchHalf : kXchFull) * 8 + (size_t)ml * y_group_stride(half) * 4;
}

// ---------------------------------------------------------------------------
// Every input pixel of a convolution rotated once, for pixels of CH = 1 or 2
// chunks of 256 channels (groups of 256): the same values and layout as
// rotate_quant_rows_slots MODE 6 with none of its row bookkeeping.  A half-
// warp per 256-chunk (two pixels per warp, or one pixel of two chunks),
// persistent warps striding over the pixels with the next pixel's 32 bytes
// per thread loaded while the current one is transformed; each thread stores
// its 16 rotated values straight to their swizzled places (a half-warp
// writes one 64-byte chunk per store) and the pixel maximum is reduced by
// shuffles.
// ---------------------------------------------------------------------------
constexpr int kPixThreads = 256;

template <int CH>
__global__ void __launch_bounds__(kPixThreads) rotate_pixels_kernel(const __nv_bfloat16 *x, int64_t pixels,
                                                                   float *yrot, float *pmax) {
    __shared__ double xch[kPixThreads / 16][kXchFull];
    pdl_wait();
    pdl_launch_dependents();
    constexpr int kPPW = 2 / CH;                         // pixels per warp
    constexpr int kC = 256 * CH;
    const int slot = threadIdx.x >> 4, t = threadIdx.x & 15, hw = slot & 1;
    const unsigned half_mask = 0xFFFFu << (16 * hw);
    const unsigned pix_mask = CH == 1 ? half_mask : 0xffffffffu;
    const int chunk = CH == 1 ? 0 : hw;                  // this half-warp's 256-chunk of the pixel
    const int64_t stride = (int64_t)gridDim.x * (kPixThreads / 32) * kPPW;
    int64_t p = ((int64_t)blockIdx.x * (kPixThreads / 32) + (threadIdx.x >> 5)) * kPPW + (CH == 1 ? hw : 0);
    double *xb = &xch[slot][0];
    uint4 r0 = make_uint4(0u, 0u, 0u, 0u), r1 = r0;
    if (p < pixels) {
        const uint4 *src = reinterpret_cast<const uint4 *>(x + p * kC + chunk * 256 + t * 16);
        r0 = __ldg(src);
        r1 = __ldg(src + 1);
    }
    for (; p < pixels; p += stride) {
        const int64_t pn = p + stride;
        uint4 n0 = make_uint4(0u, 0u, 0u, 0u), n1 = n0;
        if (pn < pixels) {                               // the next pixel's load overlaps this transform
            const uint4 *src = reinterpret_cast<const uint4 *>(x + pn * kC + chunk * 256 + t * 16);
            n0 = __ldg(src);
            n1 = __ldg(src + 1);
        }
        double v[16];
        const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
        uint32_t mkey = 0x7FFF7FFFu;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            mkey = min_s16x2(mkey, nonzero_mag_key(w[i]));
            bf16x2_to_f64(w[i], v[2 * i], v[2 * i + 1]);
        }
        fwht16_regs(v);                                  // index bits 0-3
#pragma unroll
        for (int i = 0; i < 16; ++i) xb[17 * t + i] = v[i];
        __syncwarp(half_mask);
        double xx[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) xx[i] = xb[t + 17 * i];
        __syncwarp(half_mask);
        fwht16_regs(xx);                                 // index bits 4-7: xx[i] is output 16 i + t
        float *dst = yrot + p * kC + chunk * 256 + (t & 3);
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float y = __double2float_rn(xx[i] * 0.0625);     // / sqrt(256), exact
            dst[16 * i + 4 * ((t >> 2) ^ yrot_swizzle(i))] = y;
            amax = fmaxf(amax, fabsf(y));
        }
#pragma unroll
        for (int o = 8 * CH; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(pix_mask, amax, o));
        if (t == 0 && chunk == 0) pmax[p] = amax;
        if (__any_sync(pix_mask, key_min_magnitude(mkey) < exactness_threshold_bits(amax)) &&
            (threadIdx.x & (CH == 1 ? 15 : 31)) == 0)
            report_inexact_domain();
        r0 = n0;
        r1 = n1;
    }
}

static cudaError_t launch_rotate_pixels(const void *x, int64_t pixels, int c, float *yrot, float *pmax,
                                        cudaStream_t stream, bool pdl) {
    int dev = 0, sms = 148, per_sm = 1;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const bool two = c == 512;
    cudaError_t e = two ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rotate_pixels_kernel<2>, kPixThreads, 0)
                        : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rotate_pixels_kernel<1>, kPixThreads, 0);
    if (e != cudaSuccess) return e;
    const int64_t per_cta = (kPixThreads / 32) * (two ? 1 : 2);
    const int64_t need = (pixels + per_cta - 1) / per_cta;
    const int64_t cap = (int64_t)sms * (per_sm > 0 ? per_sm : 1);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)(need < cap ? need : cap));
    cfg.blockDim = dim3(kPixThreads);
    cfg.stream = stream;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(x);
    return two ? cudaLaunchKernelEx(&cfg, rotate_pixels_kernel<2>, xb, pixels, yrot, pmax)
               : cudaLaunchKernelEx(&cfg, rotate_pixels_kernel<1>, xb, pixels, yrot, pmax);
}

// ---------------------------------------------------------------------------
// Many long rows with groups of 256 (activations at prefill, weights
// offline): persistent CTAs of S slots walk the rows (slot s takes groups
// s, s + S, ...; GPS groups per slot), each row's loads issued while the
// previous row is reduced and quantised.  Same values as
// rotate_quant_rows_slots MODE 0, with a leaner instruction and shared-
// memory budget (the kernel is issue- and shared-memory-bound, not HBM-bound):
//   * BF16 -> FP32 by a shift or mask, scaled by 1/16 there (exact: every
//     BF16 value times 2^-4 is an FP32 number), so the FP64 result only needs
//     one conversion to FP32 and no multiply;
//   * the 16 x 16 transpose between the two 16-point halves of the transform
//     writes 16-byte rows (8 x 128-bit stores, rows padded to 18 doubles) and
//     reads 8-byte columns;
//   * the row maximum is reduced by 3-input max instructions, then once per
//     CTA: warp 0 alone derives s, 1/s and the exactness threshold and hands
//     them out through shared memory (two barriers per row);
//   * REG (rows of at most 2 x 32 groups): a thread's 16 (32) rotated values
//     stay in registers until the row maximum is known; it quantises them
//     itself -- they are outputs 16 i + t of the group -- and a byte
//     transpose through the slot's transpose buffer turns them into one
//     16-byte store of 16 consecutive codes (no FP32 staging of the row);
//     otherwise the row is staged in shared memory as FP32 and quantised by
//     consecutive 16-value chunks;
//   * the quantiser tests the rounding with a fused multiply-add:
//     e = fl(y * (1/s) + 1.5 * 2^23) carries rne(y * (1/s)) in its low byte and
//     d = fl(y * (1/s) - rne) is the distance to that integer; |d| < 0.49997
//     proves that fl(y / s) rounds to the same integer (|y (1/s) - y / s|
//     <= 127 * 2^-24, |fl(y / s) - y / s| <= 127 * 2^-24, so fl(y / s) is
//     within 0.49997 + 1.6e-5 < 0.5 of it), else the IEEE division decides;
//     three FP32-pair instructions per two values and one 3-input max.
// Every row also reports, conservatively, whether it may lie outside the
// domain where the FP64 sums are exact (see exactness_threshold_bits).
// ---------------------------------------------------------------------------
constexpr int kLeanThreads = 512;
constexpr int kLeanMinGroups = 16;      // below this most slots would idle
constexpr int kLeanMaxGps = 4;
constexpr int kLeanXchStride = 18;      // doubles per transpose row: 16 + 2 (16-byte-aligned rows)
constexpr int kLeanXch = 16 * kLeanXchStride;
constexpr int kLeanRegMaxGps = 2;       // rows of more groups per slot stage the row in shared memory

// Warp maximum of non-negative floats in one instruction (their bit
// patterns order like unsigned integers).
__device__ __forceinline__ uint32_t warp_max_bits(uint32_t v) {
    uint32_t r;
    asm volatile("redux.sync.max.u32 %0, %1, 0xffffffff;" : "=r"(r) : "r"(v));
    return r;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// The row quantiser of the lean kernel.  s = fl(amax / 127) is the IEEE
// quotient (stored, and the divisor of the rare exact path); the rounding
// test multiplies by r = fl(127 * rcp.approx(amax)) instead of fl(1 / s), which
// needs no division on the row's critical path: rcp.approx is within 1 ulp
// (2^-23 relative) of 1/amax, so r is within 2^-23 + 2^-24 + 2^-24 (the
// product's and s's roundings) of 1/s, |y r - y/s| <= 127 * 2^-22 = 3.03e-5,
// and with |fl(y/s) - y/s| <= 7.6e-6 a distance |y r - rne(y r)| below
// 0.49995 still proves that fl(y/s) rounds to rne(y r).  Rows with a subnormal
// s (amax < 127 * 2^-126) or amax >= 2^125 (a subnormal 1/amax) take the
// division for every element.
constexpr float kLeanNear = 0.49995f;

// RCAP: register cap per thread (0: the 512-thread bound's 128), chosen per
// launch so that two or three CTAs of the row's width share an SM.
// The matrices of a lean launch: up to kMaxJobs with the same row count
// and row length; the launch walks all their rows as one sequence.
struct LeanJobs {
    const __nv_bfloat16 *a[kMaxJobs];
    int8_t *q[kMaxJobs];
    float *s[kMaxJobs];
};

template <int GPS, bool REG, int RCAP>
__global__ void __launch_bounds__(kLeanThreads, 1) __maxnreg__(RCAP ? RCAP : 128)
    rotate_quant_rows_lean(const __grid_constant__ LeanJobs jobs, int njobs, int64_t rows, int k) {
    extern __shared__ __align__(16) uint8_t lsm[];
    __shared__ uint32_t red[2][kLeanThreads / 32];    // per-warp maxima (bits), by row parity
    pdl_wait();
    pdl_launch_dependents();
    const int tid = threadIdx.x, slot = tid >> 4, t = tid & 15, lane = tid & 31, warp = tid >> 5;
    const int S = (int)blockDim.x >> 4;     // even: whole warps
    const int nwarps = (int)blockDim.x >> 5;
    const unsigned half_mask = 0xFFFFu << (16 * (slot & 1));
    const int groups = k >> 8, chunks = k >> 4;
    double *xb = reinterpret_cast<double *>(lsm) + slot * kLeanXch;
    // the slot's byte-transpose buffer (inside its transpose buffer; odd
    // slots 64 bytes in, so the two slots of a warp use different banks)
    uint8_t *xbytes = reinterpret_cast<uint8_t *>(xb) + (slot & 1) * 64;
    float *ybuf = reinterpret_cast<float *>(lsm + (size_t)S * kLeanXch * 8);   // !REG: the row in FP32
    const uint64_t sixteenth = pack_f32x2(0.0625f, 0.0625f);
    // rows are walked as one sequence over the jobs; (job, row) of the
    // current and of the prefetched row advance by gridDim.x without a
    // division (one job's rows subtracted per boundary crossed)
    const int64_t stride = gridDim.x;
    uint4 raw[GPS][2];
    auto advance = [&](int &jb, int64_t &r) {
        r += stride;
        while (r >= rows && jb < njobs) {
            r -= rows;
            ++jb;
        }
    };
    auto load = [&](int jb, int64_t r) {
        const __nv_bfloat16 *arow = jobs.a[jb] + r * k;
#pragma unroll
        for (int gi = 0; gi < GPS; ++gi) {
            const int g = slot + S * gi;
            if (g < groups) {
                const uint4 *src = reinterpret_cast<const uint4 *>(arow + g * 256 + t * 16);
                raw[gi][0] = __ldg(src);
                raw[gi][1] = __ldg(src + 1);
            }
        }
    };
    float yv[REG ? GPS : 1][16];
    int jb = 0, njb = 0;
    int64_t row = blockIdx.x, nrow = blockIdx.x;
    while (row >= rows && jb < njobs) {           // a grid larger than one job's rows
        row -= rows;
        ++jb;
    }
    njb = jb;
    nrow = row;
    if (jb < njobs) load(jb, row);
    int par = 0;
    for (; jb < njobs; par ^= 1) {
        float amax = 0.f;
        uint32_t mkey = 0x7FFF7FFFu;
#pragma unroll
        for (int gi = 0; gi < GPS; ++gi) {
            const int g = slot + S * gi;
            if (g < groups) {
                const uint32_t w[8] = {raw[gi][0].x, raw[gi][0].y, raw[gi][0].z, raw[gi][0].w,
                                       raw[gi][1].x, raw[gi][1].y, raw[gi][1].z, raw[gi][1].w};
                double v[16];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    mkey = min_s16x2(mkey, nonzero_mag_key(w[i]));
                    float lo, hi;
                    unpack_f32x2(mul_f32x2(pack_f32x2(__uint_as_float(w[i] << 16),
                                                      __uint_as_float(w[i] & 0xFFFF0000u)), sixteenth),
                                 lo, hi);
                    v[2 * i] = (double)lo;
                    v[2 * i + 1] = (double)hi;
                }
                fwht16_regs(v);                              // index bits 0-3
                double2 *row_t = reinterpret_cast<double2 *>(xb + kLeanXchStride * t);
#pragma unroll
                for (int i = 0; i < 8; ++i) row_t[i] = make_double2(v[2 * i], v[2 * i + 1]);
                __syncwarp(half_mask);
                double x[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) x[i] = xb[kLeanXchStride * i + t];
                __syncwarp(half_mask);
                fwht16_regs(x);                              // index bits 4-7: x[i] is output 16 i + t
                float y[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) y[i] = __double2float_rn(x[i]);
#pragma unroll
                for (int i = 0; i < 16; i += 2) amax = max3abs(y[i], y[i + 1], amax);
                if (REG) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) yv[REG ? gi : 0][i] = y[i];
                } else {
                    float *yg = ybuf + (size_t)g * kYGroupStride + (t & 3);
#pragma unroll
                    for (int i = 0; i < 16; ++i) yg[16 * i + 4 * ((t >> 2) ^ ((i >> 1) & 3))] = y[i];
                }
            }
        }
        advance(njb, nrow);
        if (njb < njobs) load(njb, nrow);     // in flight during this row's reduction and quantisation
        {
            const uint32_t wm = warp_max_bits(__float_as_uint(amax));
            if (lane == 0) red[par][warp] = wm;
        }
        // one barrier per row: afterwards every warp reads the per-warp maxima
        // of this row (red[par] is written again two rows later, after the
        // next row's barrier, by when every warp has read it)
        __syncthreads();
        const float rmax = __uint_as_float(warp_max_bits(lane < nwarps ? red[par][lane] : 0u));
        const bool zero = rmax == 0.f;
        const bool fast = rmax >= 127.0f * 1.17549435e-38f && rmax < 4.2535295865117308e37f;   // 2^125
        const float rr = __fmul_rn(127.0f, rcp_approx(rmax));
        if (key_min_magnitude(mkey) < exactness_threshold_bits(rmax)) report_inexact_domain();
        int8_t *qrow = jobs.q[jb] + row * k;
        if (REG) {
            const uint64_t r2 = pack_f32x2(rr, rr), m2 = pack_f32x2(kRoundMagic, kRoundMagic);
#pragma unroll
            for (int gi = 0; gi < GPS; ++gi) {
                const int g = slot + S * gi;
                const bool on = g < groups;
                const unsigned mask = __ballot_sync(0xffffffffu, on);
                if (on) {
                    const float(&y)[16] = yv[REG ? gi : 0];
                    uint32_t e[16];
                    float dmax = 0.f;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint64_t y2 = pack_f32x2(y[2 * i], y[2 * i + 1]);
                        const uint64_t e2 = fma_f32x2(y2, r2, m2);          // rne(y r) in the low byte
                        const uint64_t d2 = fma_f32x2(y2, r2, sub_f32x2(m2, e2));   // y r - rne(y r)
                        float d0, d1, e0, e1;
                        unpack_f32x2(d2, d0, d1);
                        unpack_f32x2(e2, e0, e1);
                        e[2 * i] = __float_as_uint(e0);
                        e[2 * i + 1] = __float_as_uint(e1);
                        dmax = max3abs(d0, d1, dmax);
                    }
                    const bool slow = !(dmax < kLeanNear) || !fast;   // zero rows too (codes set below)
                    if (__any_sync(mask, slow) && slow) {
                        const float sd = __fdiv_rn(rmax, 127.0f);
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float ei = __fmaf_rn(y[i], rr, kRoundMagic);
                            const float di = __fmaf_rn(y[i], rr, __fsub_rn(kRoundMagic, ei));
                            if (!fast || !(fabsf(di) < kLeanNear)) {
                                const int c =
                                    __float_as_int(__fadd_rn(__fdiv_rn(y[i], sd), kRoundMagic)) - kRoundMagicBits;
                                e[i] = (uint32_t)min(max(c, -127), 127);
                            }
                        }
                    }
                    if (zero) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) e[i] = 0u;
                    }
                    // codes of outputs 16 i + t -> bytes 16 i + t of the slot's buffer;
                    // then this thread stores outputs 16 t .. 16 t + 15
#pragma unroll
                    for (int i = 0; i < 16; ++i) xbytes[16 * i + t] = (uint8_t)e[i];
                    __syncwarp(mask & half_mask);
                    const uint4 pk = *reinterpret_cast<const uint4 *>(xbytes + 16 * t);
                    __syncwarp(mask & half_mask);
                    *reinterpret_cast<uint4 *>(qrow + g * 256 + 16 * t) = pk;
                }
            }
        } else {
            const RowScale rs = make_row_scale(rmax);
            for (int c0 = 0; c0 < chunks; c0 += (int)blockDim.x) {
                const int c = c0 + tid;
                const unsigned mask = __ballot_sync(0xffffffffu, c < chunks);
                if (c < chunks) {
                    const int ci = c & 15;
                    const float4 *src =
                        reinterpret_cast<const float4 *>(ybuf + (size_t)(c >> 4) * kYGroupStride + ci * 16);
                    float y[16];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float4 f = src[i ^ ((ci >> 1) & 3)];
                        y[4 * i] = f.x;
                        y[4 * i + 1] = f.y;
                        y[4 * i + 2] = f.z;
                        y[4 * i + 3] = f.w;
                    }
                    *reinterpret_cast<uint4 *>(qrow + c * 16) = quant16x2(y, rs, mask);
                }
            }
        }
        if (tid == 0) jobs.s[jb][row] = __fdiv_rn(rmax, 127.0f);
        if (!REG) __syncthreads();           // ybuf is written again by the next row
        jb = njb;
        row = nrow;
    }
}

// Shape of a lean launch for `groups` groups per row: GPS groups per slot,
// an even number of slots (whole warps), at most 32 (512 threads).  Rows of
// up to 64 groups keep their rotated values in registers (GPS <= 2); longer
// rows stage them in shared memory.
static void lean_shape(int groups, int *gps, int *slots, bool *reg) {
    // two groups per slot up to 64 groups when they pair up evenly
    // (measured: K = 4096, 5120 and 8192 at M = 4096 a few per cent faster
    // than one group per slot; K = 5376's 21 groups were not)
    const int g = (groups <= 64 && groups % 4 == 0) ? 2 : (groups + 31) / 32;
    const int sl = (groups + g - 1) / g;
    *gps = g;
    *slots = (sl + 1) & ~1;
    *reg = g <= kLeanRegMaxGps;
}

template <int GPS, bool REG, int RCAP>
static cudaError_t launch_lean(int njobs, const RQProblem *probs, int64_t rows, int sms, int slots, cudaStream_t stream,
                               bool pdl) {
    const RQProblem &pr = probs[0];
    const int groups = (int)(pr.k >> 8);
    const size_t smem = (size_t)slots * kLeanXch * 8 + (REG ? 0 : (size_t)groups * kYGroupStride * 4);
    static bool configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !configured[dev]) {
        e = cudaFuncSetAttribute(rotate_quant_rows_lean<GPS, REG, RCAP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSlotsSmemMax);
        if (e != cudaSuccess) return e;
        if (dev < 64) configured[dev] = true;
    }
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rotate_quant_rows_lean<GPS, REG, RCAP>, slots * 16, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int64_t cap = (int64_t)sms * per_sm;
    const int64_t total = rows * njobs;
    LeanJobs jobs;
    memset(&jobs, 0, sizeof(jobs));
    for (int j = 0; j < njobs; ++j) {
        jobs.a[j] = static_cast<const __nv_bfloat16 *>(probs[j].a);
        jobs.q[j] = probs[j].q;
        jobs.s[j] = probs[j].s;
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)(total < cap ? total : cap));
    cfg.blockDim = dim3(slots * 16);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, rotate_quant_rows_lean<GPS, REG, RCAP>, jobs, njobs, rows, (int)pr.k);
}

// The lean kernel takes INT8 codes of groups of 256 over rows of 16 to 128
// groups, when there are at least two rows per SM in the launch.
static bool lean_applies(const RQProblem &pr, int64_t total_rows, int num_sms) {
    if (pr.int4 || pr.group != 256 || (pr.k & 255) != 0 || total_rows < 2 * (int64_t)num_sms) return false;
    const int groups = (int)(pr.k >> 8);
    int gps, slots;
    bool reg;
    lean_shape(groups, &gps, &slots, &reg);
    return groups >= kLeanMinGroups && gps <= kLeanMaxGps;
}

// One lean launch over `nj` matrices of the same row length and row count.
static cudaError_t launch_lean_any(int nj, const RQProblem *probs, int64_t rows, int num_sms, cudaStream_t stream,
                                   bool pdl) {
    int gps, slots;
    bool reg;
    lean_shape((int)(probs[0].k >> 8), &gps, &slots, &reg);
    if (reg && gps == 1) {
        // one group per slot: a register cap that lets three (up to 336
        // threads) or two CTAs share an SM
        const int threads = slots * 16;
        if (threads <= 256) return launch_lean<1, true, 80>(nj, probs, rows, num_sms, slots, stream, pdl);
        if (threads <= 336) return launch_lean<1, true, 64>(nj, probs, rows, num_sms, slots, stream, pdl);
        if (threads <= 384) return launch_lean<1, true, 80>(nj, probs, rows, num_sms, slots, stream, pdl);
        return launch_lean<1, true, 64>(nj, probs, rows, num_sms, slots, stream, pdl);
    }
    if (reg) return launch_lean<2, true, 0>(nj, probs, rows, num_sms, slots, stream, pdl);
    if (gps == 3) return launch_lean<3, false, 0>(nj, probs, rows, num_sms, slots, stream, pdl);
    return launch_lean<4, false, 0>(nj, probs, rows, num_sms, slots, stream, pdl);
}

cudaError_t launch_rotate_quant(int njobs, int64_t rows, const RQProblem *probs, cudaStream_t stream, bool pdl,
                                const ConvGeom *conv) {
    int dev = 0, num_sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    const bool few_rows = rows * njobs < num_sms;
    if (!few_rows && njobs > 1) {
        // rows fill the GPU: one launch per row length (matrices of the same
        // row length walked together by the lean kernel, which then has
        // fewer tails), each with the CTA shape of its own row length (a
        // shared shape would size every CTA for the longest rows)
        bool done[kMaxJobs] = {};
        for (int jj = 0; jj < njobs; ++jj) {
            if (done[jj]) continue;
            RQProblem same[kMaxJobs];
            int ns = 0;
            for (int j2 = jj; j2 < njobs; ++j2) {
                if (!done[j2] && probs[j2].k == probs[jj].k && probs[j2].group == probs[jj].group &&
                    probs[j2].int4 == probs[jj].int4) {
                    same[ns++] = probs[j2];
                    done[j2] = true;
                }
            }
            cudaError_t e = cudaSuccess;
            if (!conv && lean_applies(same[0], rows * ns, num_sms)) {
                e = launch_lean_any(ns, same, rows, num_sms, stream, pdl);
            } else {
                for (int j2 = 0; j2 < ns && e == cudaSuccess; ++j2)
                    e = launch_rotate_quant(1, rows, same + j2, stream, pdl, conv);
            }
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    // decode-sized launches use the half-size transpose buffer, so that their
    // CTAs fit beside the GEMM's (INT4 weight conversion is offline: full)
    bool int4 = false;
    for (int j = 0; j < njobs; ++j) int4 = int4 || probs[j].int4;
    const int conv_mode = conv ? conv->mode : 0;
    if (conv_mode == 5 && njobs == 1 && probs[0].group == 256 && (probs[0].k == 256 || probs[0].k == 512))
        return launch_rotate_pixels(probs[0].a, rows, (int)probs[0].k, reinterpret_cast<float *>(probs[0].q),
                                    probs[0].s, stream, pdl);
    if (conv_mode == 0 && njobs == 1 && lean_applies(probs[0], rows, num_sms))
        return launch_lean_any(1, probs, rows, num_sms, stream, pdl);
    const bool half = few_rows && !int4 && conv_mode == 0;
    const int parts = rq_parts(njobs, rows, probs, num_sms, half);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    if (parts > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)parts;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = na;
    int max_slots, max_gps, max_local;
    if (njobs <= kMaxJobs &&
        rq_smem_bytes(njobs, probs, parts, half, &max_slots, &max_gps, &max_local) <= (size_t)kSlotsSmemMax) {
        RQArgs args;
        memset(&args, 0, sizeof(args));
        if (conv) args.conv = *conv;
        bool dyn = false;
        args.njobs = njobs;
        args.rows = (int)rows;
        args.parts = parts;
        // short rows (one or two 256-chunks) of a matrix that fills the GPU:
        // 256 threads per CTA, a row per half-warp or warp
        args.rpc = (!int4 && conv_mode != 4 && parts == 1 && njobs == 1 && !half && max_gps == 1 &&
                    max_slots <= 2 && rows >= 8 * (int64_t)num_sms) ? 16 / max_slots : 1;
        cfg.gridDim = dim3((unsigned)((rows * njobs * parts + args.rpc - 1) / args.rpc));
        for (int j = 0; j < njobs; ++j) {
            RQJobDev &J = args.job[j];
            J.a = static_cast<const __nv_bfloat16 *>(probs[j].a);
            J.q = probs[j].q;
            J.s = probs[j].s;
            J.k = (int)probs[j].k;
            J.group = probs[j].group;
            int lg = 0;
            while ((1 << lg) < J.group) ++lg;
            J.exact_scale = (lg % 2 == 0) ? 1 : 0;
            J.scale = 1.0 / (double)(1 << (lg / 2));
            J.root = sqrt((double)J.group);
            const int groups = (J.k + 255) >> 8;
            rq_shape((groups + parts - 1) / parts, &J.gps, &J.slots);
            dyn = dyn || J.group != 256 || (J.k & 255) != 0;
        }
        if (conv_mode == 5 && !dyn) return launch_gps<6>(cfg, args, false, max_gps, max_slots, max_local);
        if (conv_mode == 5) return launch_gps<5>(cfg, args, false, max_gps, max_slots, max_local);
        if (conv_mode == 3) return launch_gps<3>(cfg, args, false, max_gps, max_slots, max_local);
        if (conv_mode == 4) return launch_gps<4>(cfg, args, false, max_gps, max_slots, max_local);
        if (int4) return launch_gps<2>(cfg, args, half, max_gps, max_slots, max_local);
        if (dyn) return launch_gps<1>(cfg, args, half, max_gps, max_slots, max_local);
        return launch_gps<0>(cfg, args, half, max_gps, max_slots, max_local);
    }
    // unreachable within the shapes the API accepts (k <= 133120 stages in
    // at most 114 KB per CTA with 8 parts)
    return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------------------
// Convolutions, second pass: the INT8 codes of im2col row m from the pixels'
// rotated values (rotate_quant_rows_slots MODE 5).  A row's maximum is the
// maximum over its taps of the pixels' maxima (padding taps are zeros), so
// the scale and codes equal those of rotating and quantising the gathered
// row directly; each pixel is rotated once instead of kh * kw times.
// One warp per row (grid-stride over warps), 16 codes per lane per step.
// ---------------------------------------------------------------------------
constexpr int kGatherThreads = 256;

__global__ void __launch_bounds__(kGatherThreads) conv_gather_quant_kernel(const float *yrot, const float *pmax,
                                                                          const __grid_constant__ ConvGeom g,
                                                                          int64_t rows, int8_t *xq, float *sx) {
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int taps = g.kh * g.kw;
    const int k = taps * g.c;
    const int chunks = k / 16;
    const int hw = g.oh * g.ow;
    const int64_t nwarps = (int64_t)gridDim.x * (kGatherThreads / 32);
    for (int64_t row = (int64_t)blockIdx.x * (kGatherThreads / 32) + (threadIdx.x >> 5); row < rows; row += nwarps) {
        const int b = (int)(row / hw);
        const int oy = (int)(row - (int64_t)b * hw) / g.ow;
        const int ox = (int)(row - (int64_t)b * hw) - oy * g.ow;
        float m = 0.f;
        for (int t = lane; t < taps; t += 32) {
            const int ky = t / g.kw, kx = t - ky * g.kw;
            const int iy = oy * g.stride - g.pad + ky * g.dil, ix = ox * g.stride - g.pad + kx * g.dil;
            if (iy >= 0 && iy < g.h && ix >= 0 && ix < g.w)
                m = fmaxf(m, __ldg(pmax + ((size_t)b * g.h + iy) * g.w + ix));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const RowScale rs = make_row_scale(m);
        for (int c0 = 0; c0 < chunks; c0 += 32) {
            const int c = c0 + lane;
            const unsigned mask = __ballot_sync(0xffffffffu, c < chunks);
            if (c < chunks) {
                const int kel = c * 16;
                const int tap = kel / g.c, ch = kel - tap * g.c;
                const int ky = tap / g.kw, kx = tap - ky * g.kw;
                const int iy = oy * g.stride - g.pad + ky * g.dil, ix = ox * g.stride - g.pad + kx * g.dil;
                float y[16];
                if (iy >= 0 && iy < g.h && ix >= 0 && ix < g.w) {
                    const float4 *src =
                        reinterpret_cast<const float4 *>(yrot + (((size_t)b * g.h + iy) * g.w + ix) * g.c + ch);
                    const int sw = yrot_swizzle(ch >> 4);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float4 f = __ldg(src + (i ^ sw));
                        y[4 * i] = f.x;
                        y[4 * i + 1] = f.y;
                        y[4 * i + 2] = f.z;
                        y[4 * i + 3] = f.w;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) y[e] = 0.f;
                }
                *reinterpret_cast<uint4 *>(xq + row * (int64_t)k + kel) = quant16x2(y, rs, mask);
            }
        }
        if (lane == 0) sx[row] = rs.s;
    }
}

// ---------------------------------------------------------------------------
// Tiled variant of the same pass: a CTA takes a th x tw tile of output pixels
// of one image at a time.  A producer warp brings the rotated values of the
// input pixels the tile reads (its region, rh x rw pixels) into shared memory
// with one bulk copy per region row, and the pixels' maxima with 4-byte
// asynchronous copies, into one of two region buffers (full / empty
// mbarriers per buffer); the quantising warps take the tile's im2col rows from
// shared memory, each moving on to the next buffer as soon as its own rows
// are done.  A rotated pixel crosses from L2 once per tile that reads it
// instead of once per tap, and no warp waits on a global load between the
// row scale and its codes.
// One warp per row; lane l takes 16-value chunk base + l of the row (one
// 16-byte store of codes; a warp stores 512 contiguous bytes), reading its
// four float4 parts in the swizzled order of the rotated pixels, so that
// the warp's shared-memory reads are free of bank conflicts.
// ---------------------------------------------------------------------------
constexpr int kTileConsumers = 16;                    // quantising warps
constexpr int kTileThreads = 32 * kTileConsumers + 32;  // and one producer warp
constexpr int kTileMaxTaps = 32;                      // a row's taps, one per lane
constexpr size_t kTileSmemMax = 226 * 1024;           // both region buffers

struct ConvTileArgs {
    ConvGeom g;
    int th, tw, rh, rw;         // tile (output pixels) and its region (input pixels)
    int tiles_y, tiles_x;       // tiles per image
    int64_t ntiles;
    uint32_t buf_bytes;         // one buffer: rh*rw*c FP32 values, a zero pixel (c values), rh*rw maxima; 16-byte multiple
    int cc;                     // 16-value chunks per pixel (c / 16)
    int adv_t, adv_c;           // 32 chunks = adv_t pixels + adv_c chunks
};

struct TilePos {
    int b, oy0, ox0, iy0, ix0;
};

__device__ __forceinline__ TilePos tile_pos(const ConvTileArgs &A, int64_t tile) {
    const int per_img = A.tiles_y * A.tiles_x;
    TilePos p;
    p.b = (int)(tile / per_img);
    const int r = (int)(tile - (int64_t)p.b * per_img);
    const int ty = r / A.tiles_x;
    p.oy0 = ty * A.th;
    p.ox0 = (r - ty * A.tiles_x) * A.tw;
    p.iy0 = p.oy0 * A.g.stride - A.g.pad;
    p.ix0 = p.ox0 * A.g.stride - A.g.pad;
    return p;
}

__device__ __forceinline__ void cp_async_4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Start the copies of `tile`'s region into `buf` (the producer warp): lane
// 0 posts the byte count on `bar` and issues one bulk copy per region row;
// every lane copies its share of the maxima with 4-byte asynchronous copies
// (zero-filled outside the image) and arrives on `bar` when they complete.
__device__ __forceinline__ void cp_async_4_zfill(uint32_t dst, const void *src, bool valid) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(valid ? 4 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tile_issue(const ConvTileArgs &A, const float *yrot, const float *pmax,
                                           int64_t tile, uint8_t *buf, uint32_t bar, int lane) {
    const ConvGeom &g = A.g;
    const TilePos p = tile_pos(A, tile);
    const int cx0 = max(p.ix0, 0), cx1 = min(p.ix0 + A.rw, g.w);
    const uint32_t row_bytes = cx1 > cx0 ? (uint32_t)(cx1 - cx0) * (uint32_t)g.c * 4u : 0u;
    float *pm = reinterpret_cast<float *>(buf + (size_t)(A.rh * A.rw + 1) * g.c * 4);
    if (lane == 0) {
        uint32_t bytes = 0;
        for (int r = 0; r < A.rh; ++r) {
            const int iy = p.iy0 + r;
            if (iy >= 0 && iy < g.h) bytes += row_bytes;
        }
        fence_proxy_async_shared();      // the buffer's earlier reads (released through `empty`) first
        mbar_arrive_expect_tx(bar, bytes);
        if (row_bytes != 0) {
            for (int r = 0; r < A.rh; ++r) {
                const int iy = p.iy0 + r;
                if (iy < 0 || iy >= g.h) continue;
                bulk_load_1d(smem_addr(buf) + (uint32_t)(r * A.rw + (cx0 - p.ix0)) * (uint32_t)g.c * 4u,
                             yrot + (((size_t)p.b * g.h + iy) * g.w + cx0) * g.c, row_bytes, bar);
            }
        }
    }
    for (int i = lane; i < A.rh * A.rw; i += 32) {
        const int r = i / A.rw, cc = i - r * A.rw;
        const int iy = p.iy0 + r, ix = p.ix0 + cc;
        const bool in = iy >= 0 && iy < g.h && ix >= 0 && ix < g.w;     // padding: 0 in a row maximum
        cp_async_4_zfill(smem_addr(pm + i), in ? pmax + ((size_t)p.b * g.h + iy) * g.w + ix : pmax, in);
    }
    cp_async_arrive_noinc(bar);
}

// Quantise the im2col rows of `tile` from its region in `buf`.
__device__ __forceinline__ void tile_emit(const ConvTileArgs &A, int64_t tile, const uint8_t *buf, int8_t *xq,
                                          float *sx) {
    const ConvGeom &g = A.g;
    const TilePos p = tile_pos(A, tile);
    const float4 *reg4 = reinterpret_cast<const float4 *>(buf);
    const float *pm = reinterpret_cast<const float *>(buf + (size_t)(A.rh * A.rw + 1) * g.c * 4);
    const int zero_pixel = A.rh * A.rw * (g.c / 4);     // float4 offset of the buffer's zero pixel
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = kTileConsumers;
    const int taps = g.kh * g.kw;
    const int kc = taps * A.cc;                         // 16-value chunks per row
    const int64_t kbytes = (int64_t)taps * g.c;
    const int tky = lane < taps ? lane / g.kw : 0;      // this lane's tap, for the row's tap table
    const int tkx = lane < taps ? lane - tky * g.kw : 0;
    const int t0 = lane / A.cc, c0 = lane - t0 * A.cc;  // tap and chunk-in-pixel of chunk `lane`
    for (int q = warp; q < A.th * A.tw; q += nwarps) {
        const int ty = q / A.tw, tx = q - ty * A.tw;
        const int oy = p.oy0 + ty, ox = p.ox0 + tx;
        if (oy >= g.oh || ox >= g.ow) continue;        // ragged tile (warp-uniform)
        const int64_t row = ((int64_t)p.b * g.oh + oy) * g.ow + ox;
        // tap `lane` of the row: its pixel's first float4 in the region; the
        // zero pixel outside the image (and for lanes past the taps)
        int off = zero_pixel;
        float m = 0.f;
        if (lane < taps) {
            const int ry = ty * g.stride + tky * g.dil, rx = tx * g.stride + tkx * g.dil;
            const int iy = p.iy0 + ry, ix = p.ix0 + rx;
            if (iy >= 0 && iy < g.h && ix >= 0 && ix < g.w) {
                off = (ry * A.rw + rx) * (g.c / 4);
                m = pm[ry * A.rw + rx];
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const RowScale rs = make_row_scale(m);
        uint4 *qrow = reinterpret_cast<uint4 *>(xq + row * kbytes);
        int t = t0, ci = c0;                            // chunk base + lane: tap t, chunk ci of its pixel
        for (int base = 0; base < kc; base += 32) {
            // (past the row's end, t may name any lane: the values read are not stored)
            const int o = __shfl_sync(0xffffffffu, off, t & 31);
            const float4 *src = reg4 + o + 4 * ci;
            const int sw = yrot_swizzle(ci);
            float y[16];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float4 v = src[j ^ sw];
                y[4 * j] = v.x;
                y[4 * j + 1] = v.y;
                y[4 * j + 2] = v.z;
                y[4 * j + 3] = v.w;
            }
            const uint4 w = quant16x2(y, rs, 0xffffffffu);
            if (base + lane < kc) qrow[base + lane] = w;
            ci += A.adv_c;
            t += A.adv_t;
            if (ci >= A.cc) {
                ci -= A.cc;
                ++t;
            }
        }
        if (lane == 0) sx[row] = rs.s;
    }
}

__global__ void __launch_bounds__(kTileThreads, 1) conv_gather_tile_kernel(const float *yrot, const float *pmax,
                                                                          const __grid_constant__ ConvTileArgs A,
                                                                          int8_t *xq, float *sx) {
    extern __shared__ __align__(128) uint8_t tsmem[];
    __shared__ __align__(8) uint64_t full[2], empty[2];
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_addr(&full[b]), 1 + 32);           // byte count + the producer lanes' copies
            mbar_init(smem_addr(&empty[b]), kTileConsumers);  // one arrival per quantising warp
        }
        abort_flag = 0;
        fence_mbar_init();
    }
    for (int b = 0; b < 2; ++b) {
        float4 *zp = reinterpret_cast<float4 *>(tsmem + (size_t)b * A.buf_bytes + (size_t)A.rh * A.rw * A.g.c * 4);
        for (int i = threadIdx.x; i < A.g.c / 4; i += blockDim.x) zp[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    pdl_wait();
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t stride = gridDim.x;
    if (warp == kTileConsumers) {
        // producer: fill buffer it & 1 with tile `it` once its previous use is released
        int it = 0;
        int issued[2] = {0, 0};
        for (int64_t tile = blockIdx.x; tile < A.ntiles; tile += stride, ++it) {
            const int b = it & 1, use = it >> 1;
            if (use > 0 && !mbar_wait_bounded(smem_addr(&empty[b]), (uint32_t)((use - 1) & 1), &abort_flag)) break;
            tile_issue(A, yrot, pmax, tile, tsmem + (b ? A.buf_bytes : 0u), smem_addr(&full[b]), lane);
            ++issued[b];
        }
        cp_async_wait_all();
        // this warp keeps the CTA (and its shared memory) alive until every
        // copy it started has landed, even when the quantising warps gave up
        // early (a wait that ran out); normally these return at once
        volatile int no_abort = 0;
        for (int b = 0; b < 2; ++b)
            if (issued[b] > 0) mbar_wait_bounded(smem_addr(&full[b]), (uint32_t)((issued[b] - 1) & 1), &no_abort);
        return;
    }
    // quantising warps: no CTA-wide barrier, a warp that finishes its rows of
    // one tile goes on to the next tile's buffer
    int it = 0;
    for (int64_t tile = blockIdx.x; tile < A.ntiles; tile += stride, ++it) {
        const int b = it & 1, use = it >> 1;
        if (!mbar_wait_bounded(smem_addr(&full[b]), (uint32_t)(use & 1), &abort_flag)) break;
        tile_emit(A, tile, tsmem + (b ? A.buf_bytes : 0u), xq, sx);   // (not an indexed array: shared state space)
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&empty[b]));
    }
}

// Tile shape for the tiled pass, or false when no tile of at most 32 taps
// fits its two region buffers in shared memory.  Prefers a multiple of the
// warp count in rows, then the fewest region pixels copied per output pixel,
// with enough tiles for every SM.
static bool conv_tile_shape(const ConvGeom &g, int sms, ConvTileArgs *A) {
    const int taps = g.kh * g.kw;
    if (taps > kTileMaxTaps) return false;
    const size_t budget = kTileSmemMax / 2;
    double best = 0.0;
    bool found = false;
    for (int th = 1; th <= 64 && th <= g.oh; ++th) {
        for (int tw = 1; tw <= 128 && tw <= g.ow; ++tw) {
            const int64_t rh = (int64_t)(th - 1) * g.stride + (int64_t)(g.kh - 1) * g.dil + 1;
            const int64_t rw = (int64_t)(tw - 1) * g.stride + (int64_t)(g.kw - 1) * g.dil + 1;
            const size_t bytes = ((size_t)(rh * rw + 1) * g.c * 4 + (size_t)(rh * rw) * 4 + 15) / 16 * 16;
            if (bytes > budget) break;              // wider tiles only grow
            const int64_t ty = (g.oh + th - 1) / th, tx = (g.ow + tw - 1) / tw;
            const int64_t tiles = (int64_t)g.n * ty * tx;
            // quantising dominates: whole rows per warp first, then the
            // region pixels copied per row
            const int rows = th * tw, warps = kTileConsumers;
            double score = (double)((rows + warps - 1) / warps * warps) / rows *
                           (1.0 + 0.25 * ((double)(rh * rw) / rows - 1.0));
            if (tiles < sms) score *= (double)sms / (double)tiles;
            if (!found || score < best) {
                found = true;
                best = score;
                A->th = th;
                A->tw = tw;
                A->rh = (int)rh;
                A->rw = (int)rw;
                A->tiles_y = (int)ty;
                A->tiles_x = (int)tx;
                A->ntiles = tiles;
                A->buf_bytes = (uint32_t)bytes;
            }
        }
    }
    if (!found) return false;
    A->g = g;
    A->cc = g.c / 16;
    A->adv_t = 32 / A->cc;
    A->adv_c = 32 % A->cc;
    return true;
}

bool conv_gather_tile_plan(const ConvGeom &g, int sms, int *th, int *tw, int *rh, int *rw, int64_t *tiles,
                           int64_t *buf_bytes) {
    ConvTileArgs A;
    if (!conv_tile_shape(g, sms, &A)) return false;
    *th = A.th;
    *tw = A.tw;
    *rh = A.rh;
    *rw = A.rw;
    *tiles = A.ntiles;
    *buf_bytes = A.buf_bytes;
    return true;
}

cudaError_t launch_conv_gather_quant(const float *yrot, const float *pmax, const ConvGeom &g, int64_t rows,
                                     int8_t *xq, float *sx, cudaStream_t stream) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    ConvTileArgs A;
    if (conv_tile_shape(g, sms, &A)) {
        static bool configured[64] = {};
        if (dev >= 64 || !configured[dev]) {
            cudaError_t e = cudaFuncSetAttribute(conv_gather_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)kTileSmemMax);
            if (e != cudaSuccess) return e;
            if (dev < 64) configured[dev] = true;
        }
        cfg.gridDim = dim3((unsigned)(A.ntiles < sms ? A.ntiles : sms));
        cfg.blockDim = dim3(kTileThreads);
        cfg.dynamicSmemBytes = 2 * (size_t)A.buf_bytes;
        return cudaLaunchKernelEx(&cfg, conv_gather_tile_kernel, yrot, pmax, A, xq, sx);
    }
    const int64_t cap = (int64_t)sms * 8;
    const int64_t blocks = (rows + kGatherThreads / 32 - 1) / (kGatherThreads / 32);
    cfg.gridDim = dim3((unsigned)(blocks < cap ? blocks : cap));
    cfg.blockDim = dim3(kGatherThreads);
    return cudaLaunchKernelEx(&cfg, conv_gather_quant_kernel, yrot, pmax, g, rows, xq, sx);
}

}  // namespace convrot

