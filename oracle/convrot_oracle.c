/*
 * convrot_oracle.c -- CPU oracle for the INT8 ConvRot linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the package's smoke check and the CPU
 * baseline leg of the benchmark do.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * What it computes, written out plainly and slowly (no blocking, no fusion):
 *
 *   Grouped Hadamard pre-rotation ("ConvRot"):  the input dimension K is cut
 *   into groups of G = 256 consecutive channels and every group of every row
 *   is multiplied by the Sylvester Hadamard matrix H_G, normalised by
 *   1/sqrt(G) so that the rotation is orthogonal.
 *     [0539edu.com "minimax-h3-nvfp4-convrot", section 4 "INT8 ConvRot":
 *      Hadamard pre-rotation in fixed groups before quantisation, group 256;
 *      zskr.cn "Qwen3-VL-32B ... INT8-ConvRot", "INT8 ConvRot quantisation
 *      details": row-wise, group size 256; section 5 "INT4 W4A4 ConvRot":
 *      activations and weights are both rotated per group]
 *   Row-wise symmetric INT8 quantisation by round-to-nearest ("--simple"):
 *      s = max|y| / 127,  q = clamp(rne(y / s), -127, 127)
 *     [zskr.cn, conversion command: --int8 --scaling_mode row;
 *      0539edu.com section 4: "INT8 row-scale"; section 5: --simple = RTN]
 *   INT8 x INT8 -> INT32 GEMM and FP32 dequantisation to BF16:
 *      acc[m,n] = sum_k Xq[m,k] Wq[n,k];  Y[m,n] = bf16(acc * sx[m] * sw[n])
 *     [0539edu.com section 4: INT8 tensor-core throughput; summary item 3]
 *
 * Readings taken where the pages are silent (each one is listed in the
 * design notes):
 *   - H is the natural-order Sylvester matrix, H[i][j] = (-1)^popcount(i&j),
 *     built here by the recursion H_1 = [1], H_2n = [[H, H], [H, -H]].
 *   - The rotated value is the exact sum of products, evaluated in FP64
 *     (exact as long as the exponents in a group span at most 37 binades;
 *     the routine counts the groups that break this), divided by sqrt(G)
 *     (16 for G = 256, exact), then rounded once to FP32 (nearest-even).
 *   - The scale is one FP32 per row; s = a / 127 in FP32; q uses an FP32
 *     division y / s and round-half-to-even; an all-zero row has s = 0, q = 0.
 *   - INT8 range is symmetric [-127, 127].
 *   - Dequantisation is ((float)acc * sx[m]) * sw[n] in FP32, then rounded
 *     to BF16 nearest-even.  No bias.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -shared -fPIC -lm
 * (IEEE single and double arithmetic with round-to-nearest-even, no
 * contraction into fused multiply-adds).  The same file built with
 * -fopenmp splits independent rows (and output elements) over threads for
 * the timed all-cores CPU baseline; every value is computed by the same
 * operations in the same order either way.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

/* ------------------------------------------------------------------ */
/* BF16 and FP32 helpers                                               */
/* ------------------------------------------------------------------ */

/* A BF16 value is the upper 16 bits of an IEEE binary32; widening is exact. */
static float bf16_bits_to_float(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static uint32_t float_bits(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return u;
}

static float float_from_bits(uint32_t u)
{
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/*
 * Round a finite binary32 to the nearest BF16, ties to even, by comparing
 * the two neighbouring BF16 values: the one obtained by dropping the low 16
 * bits (toward zero) and the next one away from zero.  Distances are exact
 * in double.  Overflow past the largest BF16 gives infinity.
 */
uint16_t oracle_float_to_bf16(float f)
{
    uint32_t u = float_bits(f);
    uint32_t toward_zero = u & 0xFFFF0000u;
    float lo = float_from_bits(toward_zero);
    if ((u & 0xFFFFu) == 0)
        return (uint16_t)(toward_zero >> 16);
    /* next BF16 away from zero: add one unit in the last BF16 place */
    uint32_t away = toward_zero + 0x00010000u;
    float hi = float_from_bits(away);
    double d_lo = fabs((double)f - (double)lo);
    double d_hi = fabs((double)hi - (double)f);
    if ((away & 0x7F800000u) == 0x7F800000u) {
        /* the candidate away from zero is infinity: compare with the
           midpoint between the largest finite BF16 and 2^128 */
        double big = ldexp(1.0, 128);
        d_hi = big - fabs((double)f);
    }
    if (d_lo < d_hi) return (uint16_t)(toward_zero >> 16);
    if (d_hi < d_lo) return (uint16_t)(away >> 16);
    /* exact tie: keep the candidate whose last BF16 bit is zero */
    return (uint16_t)(((toward_zero >> 16) & 1u) ? (away >> 16) : (toward_zero >> 16));
}

/* Round a binary32 to the nearest integer, ties to even.  Work in FP64,
   where t - floor(t) is exact for every binary32 t. */
static float round_half_even(float t)
{
    double td = (double)t;
    double f = floor(td);
    double d = td - f;
    if (d > 0.5) return (float)(f + 1.0);
    if (d < 0.5) return (float)f;
    return (fmod(f, 2.0) == 0.0) ? (float)f : (float)(f + 1.0);
}

static int is_exact_half(float t)
{
    double td = (double)t;
    return td - floor(td) == 0.5;
}

/* ------------------------------------------------------------------ */
/* Hadamard matrix                                                     */
/* ------------------------------------------------------------------ */

/*
 * Sylvester's construction: H_1 = [1]; H_2n = [[H_n, H_n], [H_n, -H_n]].
 * n must be a power of two; H is n*n, row-major.  Returns 0 on success.
 */
int oracle_sylvester_hadamard(int n, int32_t *H)
{
    if (n < 1 || (n & (n - 1)) != 0) return -1;
    H[0] = 1;
    for (int size = 1; size < n; size *= 2) {
        for (int i = 0; i < size; ++i) {
            for (int j = 0; j < size; ++j) {
                int32_t h = H[i * n + j];
                H[i * n + (j + size)] = h;
                H[(i + size) * n + j] = h;
                H[(i + size) * n + (j + size)] = -h;
            }
        }
    }
    return 0;
}

static int is_power_of_two(int g)
{
    return g >= 1 && (g & (g - 1)) == 0;
}

/*
 * The rotation group --dynamic-convrot picks for a layer: the largest
 * compatible group size, i.e. the largest power of two that divides k and
 * does not exceed max_group (the --convrot-group-size cap, 256).
 * [0539edu.com "minimax-h3-nvfp4-convrot", section 4, item 3: the flag
 *  selects, per layer, the largest compatible group size.]
 * Counts down from max_group and tests divisibility (0 if max_group < 1).
 */
int oracle_dynamic_group(int64_t k, int max_group)
{
    int g = 1;
    while (g * 2 <= max_group) g *= 2;
    if (max_group < 1 || k < 1) return 0;
    while (g > 1 && k % g != 0) g /= 2;
    return g;
}

/* ------------------------------------------------------------------ */
/* Grouped Hadamard rotation                                           */
/* ------------------------------------------------------------------ */

/*
 * y[r, g*G + j] = fp32( ( sum_i a[r, g*G + i] * H[i][j] ) / sqrt(G) )
 *
 * a is BF16 bits [rows, k], row-major; y is FP32 [rows, k].  G must be a
 * power of two dividing k.  The sum S is accumulated in FP64 (exact, see
 * below).  When G is a power of four (256 and the other sizes the pages
 * use by default), sqrt(G) is a power of two and S / sqrt(G) is exact, so y
 * is S/sqrt(G) rounded once to FP32.  Otherwise (the smaller groups
 * --dynamic-convrot may pick, e.g. 128) S is divided by the FP64 square
 * root of G, both correctly rounded, and that quotient rounded to FP32.
 * *inexact counts the groups whose nonzero magnitudes span more than 37
 * binades, where an FP64 sum of 256 BF16 terms might not be exact.
 * Returns 0, or -1 on bad arguments.
 */
int oracle_rotate_rows(const uint16_t *a, int64_t rows, int64_t k, int group,
                       float *y, int64_t *inexact)
{
    if (!is_power_of_two(group) || k % group != 0) return -1;
    int32_t *H = (int32_t *)malloc(sizeof(int32_t) * group * group);
    if (!H) return -1;
    oracle_sylvester_hadamard(group, H);
    double root = sqrt((double)group);
    int64_t bad = 0;
    int nomem = 0;
    /* The rows are independent: an OpenMP build (the timed all-cores CPU
       baseline) splits them over threads; the arithmetic of a row is the
       same in either build. */
#ifdef _OPENMP
#pragma omp parallel reduction(+:bad, nomem)
#endif
    {
    double *x = (double *)malloc(sizeof(double) * group);
    if (!x) ++nomem;
#ifdef _OPENMP
#pragma omp for schedule(static)
#endif
    for (int64_t r = 0; r < rows; ++r) {
        if (!x) continue;
        for (int64_t g0 = 0; g0 < k; g0 += group) {
            int emin = 1000, emax = -1000;
            for (int i = 0; i < group; ++i) {
                x[i] = (double)bf16_bits_to_float(a[r * k + g0 + i]);
                if (x[i] != 0.0) {
                    int e;
                    frexp(x[i], &e);
                    if (e < emin) emin = e;
                    if (e > emax) emax = e;
                }
            }
            if (emax >= emin && emax - emin > 37) ++bad;
            for (int j = 0; j < group; ++j) {
                double s = 0.0;
                for (int i = 0; i < group; ++i)
                    s += x[i] * (double)H[i * group + j];
                y[r * k + g0 + j] = (float)(s / root);
            }
        }
    }
    free(x);
    }
    if (inexact) *inexact = bad;
    free(H);
    return nomem ? -1 : 0;
}

/*
 * The same rotation kept in FP64 (no rounding to FP32), for checking the
 * orthogonality identities of the rotation itself.  a is FP64 [rows, k].
 */
int oracle_rotate_rows_f64(const double *a, int64_t rows, int64_t k, int group,
                           double *y)
{
    if (!is_power_of_two(group) || k % group != 0) return -1;
    int32_t *H = (int32_t *)malloc(sizeof(int32_t) * group * group);
    if (!H) return -1;
    oracle_sylvester_hadamard(group, H);
    double root = sqrt((double)group);
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t g0 = 0; g0 < k; g0 += group)
            for (int j = 0; j < group; ++j) {
                double s = 0.0;
                for (int i = 0; i < group; ++i)
                    s += a[r * k + g0 + i] * (double)H[i * group + j];
                y[r * k + g0 + j] = s / root;
            }
    free(H);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Row-wise symmetric INT8 quantisation (round to nearest, ties even)  */
/* ------------------------------------------------------------------ */

/*
 * For every row r of y [rows, k] (FP32):
 *   a = max_k |y[r,k]|            (exact in FP32)
 *   s[r] = a / 127                (FP32 division, nearest-even)
 *   q[r,k] = 0 if a == 0, else clamp(rne(y[r,k] / s[r]), -127, 127)
 * Returns the number of exact .5 ties met (an FP64 check on y/s).
 */
int64_t oracle_quantize_rows(const float *y, int64_t rows, int64_t k,
                             int8_t *q, float *s)
{
    int64_t ties = 0;
#ifdef _OPENMP
#pragma omp parallel for reduction(+:ties) schedule(static)
#endif
    for (int64_t r = 0; r < rows; ++r) {
        float a = 0.0f;
        for (int64_t c = 0; c < k; ++c) {
            float v = fabsf(y[r * k + c]);
            if (v > a) a = v;
        }
        float scale = a / 127.0f;
        s[r] = scale;
        for (int64_t c = 0; c < k; ++c) {
            if (a == 0.0f) { q[r * k + c] = 0; continue; }
            float t = y[r * k + c] / scale;
            if (is_exact_half(t)) ++ties;
            float v = round_half_even(t);
            if (v > 127.0f) v = 127.0f;
            if (v < -127.0f) v = -127.0f;
            q[r * k + c] = (int8_t)v;
        }
    }
    return ties;
}

/* ------------------------------------------------------------------ */
/* Tensor-wise "simple" INT8 (the word-embedding table)                */
/* ------------------------------------------------------------------ */

/*
 * The converter treats the embedding table apart from the ConvRot matrices:
 * simple tensor-wise INT8, i.e. no rotation, ONE FP32 scale for the whole
 * tensor and round-to-nearest [zskr.cn "Qwen3-VL-32B ... INT8-ConvRot",
 * quantisation configuration: word embedding "simple tensor-wise INT8";
 * conversion command: --custom-layers embed_tokens --custom-type int8
 * --custom-scaling-mode tensor --custom-simple].  The scale and codes follow
 * the row rule above with the whole tensor as the row:
 *   a = max |x| over all elements,  s = a / 127,  q = clamp(rne(x / s)).
 * a is BF16 bits [count].  Returns the number of exact .5 ties met.
 */
int64_t oracle_quantize_tensor(const uint16_t *a, int64_t count, int8_t *q, float *s)
{
    float *x = (float *)malloc(sizeof(float) * (size_t)(count > 0 ? count : 1));
    if (!x) return -1;
    for (int64_t i = 0; i < count; ++i) x[i] = bf16_bits_to_float(a[i]);
    int64_t ties = oracle_quantize_rows(x, 1, count, q, s);
    free(x);
    return ties;
}

/*
 * Embedding lookup from the tensor-wise table q [vocab, dim] with scale s:
 *   out[i, d] = bf16_rne( (float)q[tokens[i], d] * s ).
 * A token outside [0, vocab) gives a zero row.  Returns the number of such
 * tokens.
 */
int64_t oracle_embed_lookup(const int32_t *tokens, int64_t t, const int8_t *q, float s,
                            int64_t vocab, int64_t dim, uint16_t *out)
{
    int64_t bad = 0;
    for (int64_t i = 0; i < t; ++i) {
        int64_t tok = tokens[i];
        int ok = tok >= 0 && tok < vocab;
        if (!ok) ++bad;
        for (int64_t d = 0; d < dim; ++d)
            out[i * dim + d] = ok ? oracle_float_to_bf16((float)q[tok * dim + d] * s) : 0;
    }
    return bad;
}

/* ------------------------------------------------------------------ */
/* INT4 ConvRot weights (W4A8)                                         */
/* ------------------------------------------------------------------ */

/*
 * The INT4 variants rotate weights (and activations) with the same grouped
 * Hadamard before a 4-bit round-to-nearest quantisation [0539edu.com
 * "minimax-h3-nvfp4-convrot", section 5 "INT4 W4A4 ConvRot": both operands
 * rotated per group, then 4-bit quantised; --simple = RTN].  On Blackwell the
 * W4A4 kernels take the INT8-activation path [same page, section 7], so the
 * product here is INT4 weights x INT8 activations (W4A8).
 *
 * Weight rows, after the rotation (same rule as the INT8 rows, levels 7):
 *   a = max_k |y[r,k]|;  s[r] = a / 7;  q = 0 if a == 0 else clamp(rne(y / s), -7, 7)
 * Returns the number of exact .5 ties met.
 */
int64_t oracle_quantize_rows4(const float *y, int64_t rows, int64_t k, int8_t *q, float *s)
{
    int64_t ties = 0;
#ifdef _OPENMP
#pragma omp parallel for reduction(+:ties) schedule(static)
#endif
    for (int64_t r = 0; r < rows; ++r) {
        float a = 0.0f;
        for (int64_t c = 0; c < k; ++c) {
            float v = fabsf(y[r * k + c]);
            if (v > a) a = v;
        }
        float scale = a / 7.0f;
        s[r] = scale;
        for (int64_t c = 0; c < k; ++c) {
            if (a == 0.0f) { q[r * k + c] = 0; continue; }
            float t = y[r * k + c] / scale;
            if (is_exact_half(t)) ++ties;
            float v = round_half_even(t);
            if (v > 7.0f) v = 7.0f;
            if (v < -7.0f) v = -7.0f;
            q[r * k + c] = (int8_t)v;
        }
    }
    return ties;
}

/*
 * Storage of INT4 codes (this library's format; the pages fix none): each
 * row of k codes (k % 16 == 0) is k/2 bytes; within every 16-code chunk c,
 * byte 8c + j holds code 16c + j in its low nibble and code 16c + 8 + j in
 * its high nibble (two's complement nibbles).
 */
void oracle_pack_int4(const int8_t *q, int64_t rows, int64_t k, uint8_t *packed)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < k / 16; ++c)
            for (int j = 0; j < 8; ++j) {
                uint8_t lo = (uint8_t)q[r * k + 16 * c + j] & 0x0F;
                uint8_t hi = (uint8_t)q[r * k + 16 * c + 8 + j] & 0x0F;
                packed[r * (k / 2) + 8 * c + j] = (uint8_t)(lo | (hi << 4));
            }
}

void oracle_unpack_int4(const uint8_t *packed, int64_t rows, int64_t k, int8_t *q)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < k / 16; ++c)
            for (int j = 0; j < 8; ++j) {
                uint8_t b = packed[r * (k / 2) + 8 * c + j];
                int lo = b & 0x0F, hi = b >> 4;
                q[r * k + 16 * c + j] = (int8_t)(lo >= 8 ? lo - 16 : lo);
                q[r * k + 16 * c + 8 + j] = (int8_t)(hi >= 8 ? hi - 16 : hi);
            }
}

/* Rotate, quantise to INT4 and pack the rows of a BF16 weight.  Returns the
   count of inexact rotation groups, or -1 on bad arguments. */
int64_t oracle_rotate_quantize4(const uint16_t *a, int64_t rows, int64_t k, int group,
                                uint8_t *packed, float *s)
{
    if (k % 16 != 0) return -1;
    float *y = (float *)malloc(sizeof(float) * (size_t)(rows * k > 0 ? rows * k : 1));
    int8_t *q = (int8_t *)malloc((size_t)(rows * k > 0 ? rows * k : 1));
    if (!y || !q) { free(y); free(q); return -1; }
    int64_t bad = 0;
    if (oracle_rotate_rows(a, rows, k, group, y, &bad) != 0) { free(y); free(q); return -1; }
    oracle_quantize_rows4(y, rows, k, q, s);
    oracle_pack_int4(q, rows, k, packed);
    free(y);
    free(q);
    return bad;
}

/* ------------------------------------------------------------------ */
/* ConvRot for 2-D convolutions (the VAE's int8_convrot)               */
/* ------------------------------------------------------------------ */

/*
 * The pages apply int8_convrot to the VAE's convolutions (a reported ~1.5x
 * decode speed-up) without describing it further [feinterview.poetries.top
 * "MiniMax-H3在ComfyUI的W4A8量化与VAE加速实战", the int8_convrot VAE
 * optimisation paragraph].  Reading: the convolution as the linear layer on its
 * im2col matrix.  Row (b, oy, ox) of the im2col matrix holds, tap by tap
 * (ky, kx row-major) and channel by channel inside a tap, the input
 * x[b, oy*stride - pad + ky*dil, ox*stride - pad + kx*dil, c] (NHWC), zero
 * outside the image; weight row o holds w[o, c, ky, kx] in the same order.
 * The rotation groups then lie inside one tap's channels (group | C), so
 * rotating both sides preserves the convolution tap by tap.
 *
 * x is BF16 bits [n, h, w, c]; out is BF16 bits [n*oh*ow, kh*kw*c].
 */
void oracle_im2col_nhwc(const uint16_t *x, int64_t n, int64_t h, int64_t w, int64_t c,
                        int kh, int kw, int stride, int pad, int dil, int64_t oh, int64_t ow,
                        uint16_t *out)
{
    int64_t k = (int64_t)kh * kw * c;
    for (int64_t b = 0; b < n; ++b)
        for (int64_t oy = 0; oy < oh; ++oy)
            for (int64_t ox = 0; ox < ow; ++ox) {
                int64_t row = (b * oh + oy) * ow + ox;
                for (int ky = 0; ky < kh; ++ky)
                    for (int kx = 0; kx < kw; ++kx) {
                        int64_t iy = oy * stride - pad + (int64_t)ky * dil;
                        int64_t ix = ox * stride - pad + (int64_t)kx * dil;
                        int inside = iy >= 0 && iy < h && ix >= 0 && ix < w;
                        for (int64_t ch = 0; ch < c; ++ch)
                            out[row * k + ((int64_t)ky * kw + kx) * c + ch] =
                                inside ? x[((b * h + iy) * w + ix) * c + ch] : 0;
                    }
            }
}

/* Weight w[o, c, ky, kx] (PyTorch OIHW, BF16 bits) -> rows [o, (ky, kx, c)]. */
void oracle_conv_weight_rows(const uint16_t *w, int64_t o, int64_t c, int kh, int kw, uint16_t *out)
{
    int64_t k = (int64_t)kh * kw * c;
    for (int64_t oo = 0; oo < o; ++oo)
        for (int ky = 0; ky < kh; ++ky)
            for (int kx = 0; kx < kw; ++kx)
                for (int64_t ch = 0; ch < c; ++ch)
                    out[oo * k + ((int64_t)ky * kw + kx) * c + ch] =
                        w[((oo * c + ch) * kh + ky) * kw + kx];
}

/* ------------------------------------------------------------------ */
/* INT8 GEMM with INT32 result                                         */
/* ------------------------------------------------------------------ */

/*
 * acc[m,n] = sum_k xq[m,k] * wq[n,k], summed exactly in int64.
 * xq [m,k] and wq [n,k] are row-major; acc [m,n] row-major.
 * Returns the number of sums that do not fit in int32 (those are stored
 * wrapped; the caller treats a nonzero return as an error).
 */
int64_t oracle_gemm_i32(const int8_t *xq, const int8_t *wq, int64_t m,
                        int64_t n, int64_t k, int32_t *acc)
{
    int64_t overflow = 0;
#ifdef _OPENMP
#pragma omp parallel for collapse(2) reduction(+:overflow) schedule(static)
#endif
    for (int64_t i = 0; i < m; ++i)
        for (int64_t j = 0; j < n; ++j) {
            int64_t sum = 0;
            for (int64_t c = 0; c < k; ++c)
                sum += (int64_t)xq[i * k + c] * (int64_t)wq[j * k + c];
            if (sum > INT32_MAX || sum < INT32_MIN) ++overflow;
            acc[i * n + j] = (int32_t)sum;
        }
    return overflow;
}

/* ------------------------------------------------------------------ */
/* Dequantisation to BF16                                              */
/* ------------------------------------------------------------------ */

/* y[m,n] = bf16_rne( ((float)acc[m,n] * sx[m]) * sw[n] ), FP32 products. */
void oracle_dequant_bf16(const int32_t *acc, const float *sx, const float *sw,
                         int64_t m, int64_t n, uint16_t *y)
{
#ifdef _OPENMP
#pragma omp parallel for collapse(2) schedule(static)
#endif
    for (int64_t i = 0; i < m; ++i)
        for (int64_t j = 0; j < n; ++j) {
            float v = (float)acc[i * n + j];
            v = v * sx[i];
            v = v * sw[j];
            y[i * n + j] = oracle_float_to_bf16(v);
        }
}

/*
 * The same with an optional per-output-channel bias (BF16 bits [n], or
 * NULL for none): y[m,n] = bf16_rne( ((float)acc * sx[m]) * sw[n] + b[n] ),
 * the bias added to the FP32 product and the sum rounded once to BF16.  The
 * source pages quantise bias-free projections; the bias is this library's
 * extension for layers that carry one.
 */
void oracle_dequant_bf16_bias(const int32_t *acc, const float *sx, const float *sw,
                              const uint16_t *bias, int64_t m, int64_t n, uint16_t *y)
{
#ifdef _OPENMP
#pragma omp parallel for collapse(2) schedule(static)
#endif
    for (int64_t i = 0; i < m; ++i)
        for (int64_t j = 0; j < n; ++j) {
            float v = (float)acc[i * n + j];
            v = v * sx[i];
            v = v * sw[j];
            if (bias) v = v + bf16_bits_to_float(bias[j]);
            y[i * n + j] = oracle_float_to_bf16(v);
        }
}

/* ------------------------------------------------------------------ */
/* Composites                                                          */
/* ------------------------------------------------------------------ */

/* Rotate and quantise the rows of a BF16 matrix (weights offline, or
   activations at call time).  Returns the count of inexact groups, or -1. */
int64_t oracle_rotate_quantize(const uint16_t *a, int64_t rows, int64_t k,
                               int group, int8_t *q, float *s)
{
    float *y = (float *)malloc(sizeof(float) * (size_t)(rows * k > 0 ? rows * k : 1));
    if (!y) return -1;
    int64_t bad = 0;
    if (oracle_rotate_rows(a, rows, k, group, y, &bad) != 0) { free(y); return -1; }
    oracle_quantize_rows(y, rows, k, q, s);
    free(y);
    return bad;
}

/*
 * Full forward of the layer on pre-quantised weights:
 *   x (BF16 [m,k]) -> rotate -> quantise (xq, sx) -> GEMM with wq -> dequant.
 * Intermediate outputs are written when their pointers are non-NULL.
 * Returns 0 on success, -1 on bad arguments, -2 on an inexact rotation group,
 * -3 on an INT32 overflow.
 */
int oracle_linear_int8(const uint16_t *x, int64_t m, int64_t k, int group,
                       const int8_t *wq, const float *sw, int64_t n,
                       uint16_t *y, int8_t *xq_out, float *sx_out,
                       int32_t *acc_out)
{
    int8_t *xq = xq_out ? xq_out : (int8_t *)malloc((size_t)(m * k > 0 ? m * k : 1));
    float *sx = sx_out ? sx_out : (float *)malloc(sizeof(float) * (size_t)(m > 0 ? m : 1));
    int32_t *acc = acc_out ? acc_out
                           : (int32_t *)malloc(sizeof(int32_t) * (size_t)(m * n > 0 ? m * n : 1));
    int rc = 0;
    if (!xq || !sx || !acc) { rc = -1; goto done; }
    int64_t bad = oracle_rotate_quantize(x, m, k, group, xq, sx);
    if (bad < 0) { rc = -1; goto done; }
    if (bad > 0) { rc = -2; goto done; }
    if (oracle_gemm_i32(xq, wq, m, n, k, acc) != 0) { rc = -3; goto done; }
    oracle_dequant_bf16(acc, sx, sw, m, n, y);
done:
    if (!xq_out) free(xq);
    if (!sx_out) free(sx);
    if (!acc_out) free(acc);
    return rc;
}

/* ------------------------------------------------------------------ */
/* FP64 references for error reporting                                 */
/* ------------------------------------------------------------------ */

/* c[m,n] = sum_k a[m,k] * b[n,k] in FP64 (both operands row-major). */
void oracle_matmul_nt_f64(const double *a, const double *b, int64_t m,
                          int64_t n, int64_t k, double *c)
{
    for (int64_t i = 0; i < m; ++i)
        for (int64_t j = 0; j < n; ++j) {
            double s = 0.0;
            for (int64_t t = 0; t < k; ++t)
                s += a[i * k + t] * b[j * k + t];
            c[i * n + j] = s;
        }
}
