/*
 * convrot.h -- C ABI of libconvrot, the INT8 ConvRot linear layer for
 * NVIDIA B200 (sm_100a).
 *
 * The layer (from the source pages):
 *   - "ConvRot" is a grouped Hadamard pre-rotation: the input dimension K is
 *     cut into fixed groups of 256 and each group is Hadamard-rotated before
 *     quantisation, which spreads outlier energy so INT8 can hold it
 *     [0539edu.com "minimax-h3-nvfp4-convrot", section 4 "INT8 ConvRot";
 *      zskr.cn "Qwen3-VL-32B ... INT8-ConvRot", "INT8 ConvRot quantisation
 *      details": row-wise, group size 256].
 *   - Weights are rotated offline and quantised to INT8 with one FP32 scale
 *     per output row, by round-to-nearest [zskr.cn conversion command:
 *     "--int8 --scaling_mode row --convrot --convrot-group-size 256";
 *     0539edu.com section 4 "INT8 row-scale", section 5 "--simple" = RTN].
 *   - Activations are rotated the same way and quantised per token row at
 *     call time, so the product runs on INT8 tensor cores [0539edu.com
 *     section 4 (INT8 tensor-core throughput), section 5 (activations and
 *     weights both rotated), section 7 (INT8 activation path on Blackwell)].
 *
 * Arithmetic contract (identical to the CPU oracle bit for bit):
 *   y_j  = fp32( (sum_i a_i * H[i][j]) / 16 )   per 256-group, H Sylvester,
 *          the sum exact (FP64; exact while the nonzero magnitudes inside a
 *          group span at most 37 binades -- finite BF16 inputs outside that
 *          range give unspecified low bits; non-finite inputs give
 *          unspecified codes).  Every rotating kernel records
 *          CONVROT_WARN_INEXACT_DOMAIN for convrot_device_status() when a row
 *          holds a nonzero input |a| < 2^(e(amax) - 33), amax the row's
 *          largest |y| and e() the frexp exponent: every group spanning more
 *          than 37 binades meets this (its largest input is at most 16 amax),
 *          so rows without the warning are inside the exact domain; a row
 *          whose groups differ greatly in scale can raise it although each
 *          group is exact.  Groups G of 16 .. 128 (the
 *          sizes --dynamic-convrot falls back to, see convrot_dynamic_group):
 *          the same with H_G and sqrt(G); for G = 32 and 128 the exact sum
 *          is divided by fp64(sqrt(G)) in FP64 and that quotient rounded to
 *          FP32.
 *   s    = fp32(max_k |y_k| / 127);  q = clamp(rne(y / s), -127, 127), q = 0
 *          and s = 0 for an all-zero row
 *   acc  = sum_k xq[m,k] * wq[n,k]   (INT32, exact for K <= 133144)
 *   Y    = bf16_rne( ((float)acc * sx[m]) * sw[n] )
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers, owned by the caller, row-major,
 *     16-byte aligned.  BF16 tensors are passed as `const void *`/`void *`
 *     (IEEE bfloat16 bit patterns, 2 bytes each).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is
 *     enqueued asynchronously; the call returns once it is launched.
 *   - Argument errors are detected on the host before anything is launched
 *     and returned as a status; nothing is written then.  A launch failure
 *     returns CONVROT_ERR_CUDA.
 *   - Kernels never trap.  Every wait inside a kernel is bounded; a wait that
 *     runs out records CONVROT_ERR_DEVICE_TIMEOUT in a device-side status
 *     word that convrot_device_status() reads.
 *   - The library allocates no device memory.  Scratch space is the
 *     caller-provided workspace.
 *   - Calls on different streams are independent provided they do not share
 *     a workspace.
 */
#ifndef CONVROT_H
#define CONVROT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CONVROT_OK = 0,
    CONVROT_ERR_INVALID_ARG = 1,       /* null pointer, non-positive size */
    CONVROT_ERR_ALIGNMENT = 2,         /* a pointer is not 16-byte aligned */
    CONVROT_ERR_UNSUPPORTED_SHAPE = 3, /* bad group, k % group != 0, k too large */
    CONVROT_ERR_UNSUPPORTED_ARCH = 4,  /* current device is not compute capability 10.0 */
    CONVROT_ERR_WORKSPACE = 5,         /* workspace missing or smaller than required */
    CONVROT_ERR_CUDA = 6,              /* a CUDA runtime/driver call failed */
    CONVROT_ERR_DEVICE_TIMEOUT = 7,    /* a bounded in-kernel wait ran out */
    CONVROT_WARN_INEXACT_DOMAIN = 8    /* an input row may lie outside the exact-rotation domain (see below) */
} convrot_status_t;

/*
 * Quantised-weight handle: a VIEW of caller-owned device memory.
 *   q     : int8  [n, k] row-major -- the rotated, row-quantised weight Wq
 *   scale : fp32  [n]              -- sw, one scale per output row
 *   n     : out_features, k : in_features (the rotation runs along k)
 *   group : rotation group size: 256 (the pages' setting), or a smaller power
 *           of two >= 16 dividing k (convrot_dynamic_group)
 * The offline converter's record is an INT8 tensor, an FP32 row scale and the
 * ConvRot group size [zskr.cn "Qwen3-VL-32B ... INT8-ConvRot": 350 INT8
 * ConvRot matrices with FP32 scales; 0539edu.com section 4: "INT8 row-scale
 * + ConvRot metadata"].
 */
typedef struct {
    int8_t *q;
    float *scale;
    int64_t n;
    int64_t k;
    int32_t group;
} convrot_weight_t;

/* Human-readable name of a status code (static string, never NULL). */
const char *convrot_status_string(convrot_status_t status);

/* Library version as 10000 * major + 100 * minor + patch. */
int convrot_version(void);

/* Identity of this build: 16 hex digits of SHA-256 over the compile flags
   and the CUDA sources the library was compiled from ("unknown" for a build
   made without the build script).  Static string, never NULL.  The Python
   binding refuses a library whose id differs from its sources' hash and
   rebuilds it; no passage of the source pages corresponds to this call. */
const char *convrot_build_id(void);

/* Text of the last CUDA error this thread's calls turned into
   CONVROT_ERR_CUDA ("no error" if none).  Static string, never NULL. */
const char *convrot_last_error_string(void);

/*
 * Fill a handle.  Checks: w, q, scale non-NULL; n, k >= 1; group a power
 * of two in 16 .. 256 with k % group == 0; k <= 133120 (INT32 accumulation
 * bound); q and scale 16-byte aligned.  Host only; touches no device.
 */
convrot_status_t convrot_weight_init(convrot_weight_t *w, int8_t *q, float *scale,
                                     int64_t n, int64_t k, int32_t group);

/*
 * The rotation group --dynamic-convrot picks for a layer with k input
 * features: the largest power of two <= max_group (the configured group
 * size, 256) that divides k [0539edu.com "minimax-h3-nvfp4-convrot",
 * section 4, item 3: the flag picks the largest compatible group size per
 * layer; in_features 5376 keeps 256].  Returns 0 when that group would be
 * below 16 (k not a multiple of 16: INT8 rows must be 16-byte multiples
 * for the tensor-memory-access loads), which the other entry points reject.
 * Host only.
 */
int32_t convrot_dynamic_group(int64_t k, int32_t max_group);

/*
 * Offline weight conversion: rotate every row of the BF16 weight w [n, k]
 * (PyTorch Linear layout, out x in) per group and quantise it row-wise
 * by round-to-nearest into out->q and out->scale.  The pages quantise from
 * the BF16 source, never from an already quantised tensor [0539edu.com
 * section 4, engineering detail 1] and use RTN in "--simple" mode
 * [0539edu.com section 5].
 */
convrot_status_t convrot_quantize_weight(const void *w_bf16, const convrot_weight_t *out,
                                         void *stream);

/*
 * Activation prologue: rotate each row of x [m, k] (BF16) per group (the
 * weight's group) and quantise it per row into xq (int8 [m, k]) and sx
 * (fp32 [m]).  Same arithmetic as the weight conversion.
 */
convrot_status_t convrot_quantize_act(const void *x_bf16, int64_t m, int64_t k, int32_t group,
                                      int8_t *xq, float *sx, void *stream);

/*
 * Scratch bytes convrot_gemm_i8 needs for an [m x k] x [n x k]^T product on
 * the current device (0 when no device is present is never returned: the
 * B200's 148 SMs are assumed then).  The workspace must be zero-filled
 * (convrot_workspace_init) before its first use; every successful call
 * leaves it zero-filled again.
 */
size_t convrot_gemm_workspace_bytes(int64_t m, int64_t n, int64_t k);

/*
 * How the GEMM kernel would tile a product (host arithmetic only: no device
 * is touched; for tests and tuning).  count == 1: the single-product entry
 * points (convrot_gemm_i8 / convrot_linear_int8) for m x k against n x k;
 * count in 2..8 (m <= 512): one batched launch of `count` products with the
 * same m (convrot_gemm_i8_batch / convrot_linear_int8_batch), w4 = 1 for
 * INT4 weights unpacked inside the GEMM (what convrot_linear_w4a8 launches
 * for m <= 512; for larger m it unpacks the weights to INT8 first and runs
 * the INT8 plan, w4 = 0).  A CTA c of the `grid` takes, in order: whole
 * tiles wave * grid + c for wave < full_waves while below full_tiles; piece
 * c of the split tail when c < split_pieces (tile full_tiles + c / split_ways,
 * K blocks [s * kbpt / ways, (s + 1) * kbpt / ways) with s = c % ways); then
 * the stream-K units [tail_units * q / Q, tail_units * (q + 1) / Q) with
 * q = c / rep, Q = grid / rep, where unit u of job j (u - unit0[j] = t * kbpt
 * + kb) is K block kb of tile tile_base[j] + t * rep + c % rep.  A tile of
 * job j is (A tile, B tile) with tiles_a[j] x tiles_b[j] tiles; 128-byte K
 * blocks, kbpt[j] per tile.  swap = 1: the weights are the 128-row A operand.
 * Errors: CONVROT_ERR_INVALID_ARG (null pointers, count out of range, sizes
 * < 1, sms < 1), CONVROT_ERR_UNSUPPORTED_SHAPE (a batch with m > 512).
 */
typedef struct {
    int32_t njobs, swap, bn, grid;
    int32_t full_waves, full_tiles, split_ways, split_pieces;
    int32_t rep, stages, tmem_cols, slots;
    int64_t tail_units, smem_bytes, ws_bytes;
    int32_t tiles_a[8], tiles_b[8], group_a[8], kbpt[8], tile_base[8];
    int64_t unit0[8];
} convrot_gemm_plan_t;
convrot_status_t convrot_gemm_plan(int64_t m, int32_t count, const int64_t *n, const int64_t *k, int32_t w4,
                                   int32_t sms, convrot_gemm_plan_t *out);

/* Scratch bytes convrot_linear_int8 needs: the GEMM scratch followed by the
   quantised activations xq [m, k] and their scales sx [m]. */
size_t convrot_linear_workspace_bytes(int64_t m, int64_t n, int64_t k);

/* Zero-fill a workspace on `stream` (an asynchronous memset). */
convrot_status_t convrot_workspace_init(void *ws, size_t ws_bytes, void *stream);

/*
 * INT8 GEMM with INT32 accumulation on the tcgen05 tensor cores, with the
 * dequantisation fused into the epilogue:
 *   acc[m, n] = sum_k xq[m, k] * w->q[n, k]
 *   y[m, n]   = bf16_rne(((float)acc * sx[m]) * w->scale[n])
 * y (BF16 [m, n]) and acc (int32 [m, n]) are optional outputs; at least one
 * must be non-NULL (acc exists for bit-exact checking).  ws/ws_bytes: see
 * convrot_gemm_workspace_bytes.
 */
convrot_status_t convrot_gemm_i8(const int8_t *xq, const float *sx, int64_t m,
                                 const convrot_weight_t *w, void *y_bf16, int32_t *acc,
                                 void *ws, size_t ws_bytes, void *stream);

/*
 * The whole layer: y = ConvRotLinearINT8(x) for BF16 x [m, k] against the
 * quantised weight w, BF16 y [m, n].  Runs the activation prologue into the
 * workspace, then the GEMM; the GEMM is launched as a programmatic
 * dependent of the prologue so its weight prefetch overlaps the prologue.
 */
convrot_status_t convrot_linear_int8(const void *x_bf16, int64_t m, const convrot_weight_t *w,
                                     void *y_bf16, void *ws, size_t ws_bytes, void *stream);

/*
 * One product of a batched GEMM call (see convrot_gemm_i8 for the maths).
 *   xq : int8 [m, w->k] quantised activations;  sx : fp32 [m] their scales
 *   y_bf16 : BF16 [m, w->n] output or NULL;  acc : int32 [m, w->n] or NULL
 *   bias_bf16 : BF16 [w->n] per-output-channel bias or NULL (none).  With a
 *     bias, y = bf16_rne( ((float)acc * sx[m]) * sw[n] + bias[n] ): the bias
 *     joins the FP32 product and the sum is rounded once.  The source pages
 *     quantise bias-free projections; the bias is this library's extension
 *     for layers that carry one.  16-byte aligned.
 */
typedef struct {
    const int8_t *xq;
    const float *sx;
    const convrot_weight_t *w;
    void *y_bf16;
    int32_t *acc;
    const void *bias_bf16;
} convrot_gemm_job_t;

/*
 * Several INT8 GEMMs with the same m (1 <= m <= 512) in ONE launch: every
 * 128-byte K block of every output tile of every product is dealt out
 * evenly to the SMs (stream-K), so the whole set streams its weights as one
 * long read.  m > 512: CONVROT_ERR_INVALID_ARG.
 * count <= 8.  Workspace: convrot_gemm_batch_workspace_bytes, zero-filled
 * before first use, left zero-filled.
 */
convrot_status_t convrot_gemm_i8_batch(int64_t m, int count, const convrot_gemm_job_t *jobs,
                                       void *ws, size_t ws_bytes, void *stream);

size_t convrot_gemm_batch_workspace_bytes(int64_t m, int count, const convrot_gemm_job_t *jobs);

/*
 * One linear of a batched call: y = ConvRotLinearINT8(x) (+ bias) against w.
 *   x_bf16 : BF16 [m, w->k] input (device).  Jobs that pass the same x_bf16
 *            pointer (same k) share one activation prologue.
 *   w      : quantised weight handle
 *   y_bf16 : BF16 [m, w->n] output (device)
 *   bias_bf16 : BF16 [w->n] bias or NULL, as in convrot_gemm_job_t
 */
typedef struct {
    const void *x_bf16;
    const convrot_weight_t *w;
    void *y_bf16;
    const void *bias_bf16;
} convrot_linear_job_t;

/*
 * Several ConvRot INT8 linears with the same token count m, in two
 * launches: one activation prologue over the rows of every distinct input
 * (jobs with the same x_bf16 share its rotated INT8 copy), then one GEMM
 * whose K blocks of all weights are dealt out evenly to every SM (m <= 512;
 * larger m runs the GEMMs one after another).  This is how the linears of
 * one decoder layer that share an input (q/k/v, gate/up) or that are
 * otherwise ready together run at decode size, where a per-linear launch
 * would spend more time starting and draining than streaming its weight.
 * The pages quantise exactly these projections of every layer [zskr.cn
 * "Qwen3-VL-32B ... INT8-ConvRot": 350 = 50 layers x 7 row-wise INT8 ConvRot
 * matrices; 0539edu.com section 4: the attention QKV projections].
 * count <= 8.  No job's output may overlap any job's input or another
 * job's output (CONVROT_ERR_INVALID_ARG).  Results equal count calls of
 * convrot_linear_int8.
 */
convrot_status_t convrot_linear_int8_batch(int64_t m, int count, const convrot_linear_job_t *jobs,
                                           void *ws, size_t ws_bytes, void *stream);

/* Workspace bytes convrot_linear_int8_batch needs for these jobs (0 if the
   jobs are invalid).  Zero-fill before first use, as for the others. */
size_t convrot_linear_batch_workspace_bytes(int64_t m, int count, const convrot_linear_job_t *jobs);

/*
 * convrot_gemm_i8 for callers that cannot allocate device memory: the same
 * product and outputs (xq, sx, w, y_bf16, acc as for convrot_gemm_i8), but
 * with no workspace argument.  Its scratch is an array of 8 MiB built into
 * the library.  The array is part of the library's single device module, so
 * every process that loads libconvrot pays its 8 MiB on each device the
 * library is used on, until the process exits, whether or not it ever calls
 * this entry point.  It is meant for code that must not call cudaMalloc
 * where it runs the layer -- for example a plugin inside an engine that owns
 * all device memory through its own pool -- and cannot be handed a
 * workspace either.  (The source pages have no counterpart of this entry
 * point; it is an integration convenience.)
 *   - The first call in a CUDA context looks up the array's device address
 *     (with cudaGetSymbolAddress, with that context's device current) and
 *     keeps it for that context; a new context (after cudaDeviceReset, for
 *     instance) looks it up again.  The lookup can load the library's
 *     module (lazily, under CUDA_MODULE_LOADING=LAZY), which must not
 *     happen during a stream capture: make the first call on each device
 *     before any stream capture starts, whatever is being captured.
 *   - Problems whose scratch needs more than 8 MiB are rejected with
 *     CONVROT_ERR_WORKSPACE before anything is launched
 *     (convrot_last_error_string says so).  convrot_gemm_workspace_bytes
 *     gives the need.
 *   - Each call clears the part of the array it uses (an asynchronous memset
 *     on `stream`) and then launches the GEMM; it allocates nothing.
 *   - Every call on a device shares the one array: calls whose GPU work can
 *     overlap (other streams, other host threads) race and corrupt each
 *     other's results.  Serialise them.
 */
convrot_status_t convrot_gemm_i8_noalloc(const int8_t *xq, const float *sx, int64_t m,
                                         const convrot_weight_t *w, void *y_bf16, int32_t *acc,
                                         void *stream);

/*
 * ---------------------------------------------------------------- INT4 ConvRot weights (W4A8)
 * The INT4 variants rotate weights and activations with the same grouped
 * Hadamard and quantise to 4 bits by round-to-nearest [0539edu.com
 * "minimax-h3-nvfp4-convrot", section 5 "INT4 W4A4 ConvRot", --simple = RTN];
 * on Blackwell those kernels take the INT8-activation path [same page,
 * section 7].  Here: weights INT4 (levels -7..7, one FP32 scale per row,
 * s = max|Wr[n,:]| / 7), activations INT8 exactly as in the INT8 layer, the
 * product on the INT8 tensor cores after unpacking the weight tile in shared
 * memory, so the weight stream (the decode bound) is half as many bytes.
 *
 * Packed INT4 weight handle (caller-owned device memory):
 *   q     : uint8 [n, k/2] -- within each 16-code chunk c of a row, byte
 *           8c + j holds code 16c + j in its low nibble and code 16c + 8 + j
 *           in its high nibble (two's complement)
 *   scale : fp32 [n];  group as in convrot_weight_t;  k % 32 == 0
 */
typedef struct {
    uint8_t *q;
    float *scale;
    int64_t n;
    int64_t k;
    int32_t group;
} convrot_weight4_t;

/* Fill an INT4 handle; the checks of convrot_weight_init plus k % 32 == 0. */
convrot_status_t convrot_weight4_init(convrot_weight4_t *w, uint8_t *q, float *scale,
                                      int64_t n, int64_t k, int32_t group);

/* Offline: rotate every row of the BF16 weight w [n, k] per group, quantise
   it to INT4 (row scale max/7, RTN, clamp to -7..7) and pack it into out->q. */
convrot_status_t convrot_quantize_weight4(const void *w_bf16, const convrot_weight4_t *out, void *stream);

/* One W4A8 linear of a call: y [m, w->n] = the ConvRot layer of x [m, w->k]. */
typedef struct {
    const void *x_bf16;
    const convrot_weight4_t *w;
    void *y_bf16;
    const void *bias_bf16;      /* BF16 [w->n] or NULL, as in convrot_linear_job_t */
} convrot_linear4_job_t;

/*
 * count (<= 8) W4A8 linears with the same token count m: the activation
 * prologue (INT8 codes, shared by jobs with the same input), then the INT8
 * tensor-core GEMM with the packed weight tiles unpacked to INT8 in shared
 * memory by eight dedicated warps per CTA.  m <= 512: one GEMM launch for all
 * jobs (for m <= 256 weight-streaming, the K blocks of all weights dealt out
 * to every SM).  Larger m (prefill, video tokens), where the layer is
 * tensor-bound: per job, the weight is first unpacked to INT8 into the
 * workspace (one pass over it) and then multiplied by the INT8 GEMM (whole
 * 128 x 256 tiles); the workspace then also holds one unpacked weight (the
 * largest n * k of the jobs, in bytes).  Results:
 * y = bf16(((float)acc * sx[m]) * sw[n] [+ bias[n]]) with acc the exact INT32
 * product of the INT8 activation codes and the INT4 weight codes.
 * Workspace: convrot_linear_w4a8_workspace_bytes, zero-filled before first
 * use, left zero-filled.
 */
convrot_status_t convrot_linear_w4a8(int64_t m, int count, const convrot_linear4_job_t *jobs,
                                     void *ws, size_t ws_bytes, void *stream);

size_t convrot_linear_w4a8_workspace_bytes(int64_t m, int count, const convrot_linear4_job_t *jobs);

/*
 * ---------------------------------------------------------------- 2-D convolutions (int8_convrot)
 * The pages apply int8_convrot to the VAE's convolutions (a reported ~1.5x
 * decode speed-up; feinterview.poetries.top "MiniMax-H3在ComfyUI的W4A8量化与
 * VAE加速实战", the int8_convrot VAE paragraph) without further detail.
 * Here a convolution is the ConvRot INT8 layer on its im2col matrix: row
 * (b, oy, ox) holds, tap by tap (ky, kx row-major) and channel by channel,
 * x[b, oy*stride - pad + ky*dil, ox*stride - pad + kx*dil, c] (zero outside
 * the image); the weight row o holds w[o, c, ky, kx] in the same order; the
 * rotation groups lie inside one tap's channels (group divides C), so
 * rotating both sides preserves the convolution.  For kernels larger than
 * 1x1 every input pixel is rotated once (FP32 copy and its maximum in the
 * workspace) and a second kernel gathers the im2col rows from those pixels
 * and quantises them (a row's maximum is the maximum of its pixels'); a 1x1
 * convolution gathers and rotates in one step.  No BF16 im2col copy exists.
 */
typedef struct {
    int32_t n, h, w, c;             /* input NHWC: batch, height, width, channels (c % 16 == 0) */
    int32_t kh, kw;                 /* kernel size */
    int32_t stride, pad, dilation;  /* the same along both axes */
} convrot_conv2d_t;

/* Output height and width: (size + 2 pad - dil (k - 1) - 1) / stride + 1. */
convrot_status_t convrot_conv2d_shape(const convrot_conv2d_t *g, int32_t *oh, int32_t *ow);

/*
 * How convrot_conv2d_int8 gathers the im2col rows of a kernel larger than
 * 1x1 on a GPU of `sms` SMs (host arithmetic only: no device is touched;
 * for tests and tuning).  tiled = 1: persistent CTAs (one per SM, at most
 * `tiles`) quantise th x tw tiles of output pixels of one image from the
 * rotated pixels of the tile's input region, rh x rw pixels, staged in one of
 * two shared-memory buffers of buf_bytes each (the region's FP32 values, one
 * zero pixel, then the region's pixel maxima).  tiled = 0: more than 32 taps
 * or no tile fits, and a warp per row gathers straight from global memory
 * (the other fields are 0).  Errors: CONVROT_ERR_INVALID_ARG for a null
 * pointer, sms < 1 or an invalid geometry, CONVROT_ERR_UNSUPPORTED_SHAPE for
 * a 1x1 kernel (its rows are gathered and rotated in one step).
 */
typedef struct {
    int32_t tiled;
    int32_t th, tw;                 /* output pixels per tile (rows x columns) */
    int32_t rh, rw;                 /* input pixels the tile reads */
    int64_t tiles;                  /* n * ceil(oh / th) * ceil(ow / tw) */
    int64_t buf_bytes;              /* one region buffer */
} convrot_conv2d_plan_t;
convrot_status_t convrot_conv2d_gather_plan(const convrot_conv2d_t *g, int32_t sms, convrot_conv2d_plan_t *out);

/*
 * Offline: rotate and quantise a BF16 OIHW weight [c_out, c, kh, kw] into
 * the handle `out` (out->n = c_out, out->k = kh * kw * c, out->group dividing
 * c; convrot_dynamic_group(c, 256) picks it), rows in the im2col order.
 */
convrot_status_t convrot_quantize_conv_weight(const void *w_oihw_bf16, const convrot_conv2d_t *g,
                                              const convrot_weight_t *out, void *stream);

/* Workspace of convrot_conv2d_int8: GEMM scratch + the INT8 im2col codes and
 * their row scales, and for kernels larger than 1x1 every input pixel's
 * rotated FP32 values (n*h*w x c) and maxima.  0 for an invalid argument. */
size_t convrot_conv2d_workspace_bytes(const convrot_conv2d_t *g, const convrot_weight_t *w);

/*
 * y [n, oh, ow, w->n] (NHWC, BF16) = the INT8 ConvRot convolution of x
 * [n, h, w, c] (NHWC, BF16) with the handle from convrot_quantize_conv_weight.
 * Launches: the activation prologue (two kernels, one for 1x1: every input
 * pixel rotated once, then the im2col rows gathered from the rotated pixels
 * and quantised), then the INT8 GEMM with M = n * oh * ow, N = c_out,
 * K = kh * kw * c.  The codes equal those of rotating and quantising each
 * im2col row directly.
 */
convrot_status_t convrot_conv2d_int8(const void *x_nhwc_bf16, const convrot_conv2d_t *g, const convrot_weight_t *w,
                                     void *y_nhwc_bf16, void *ws, size_t ws_bytes, void *stream);

/*
 * Tensor-wise "simple" INT8 of a BF16 tensor of `count` elements (the
 * word-embedding table [vocab, dim]): no rotation, ONE scale for the whole
 * tensor, round-to-nearest-even --
 *   a = max |x|;  *scale = fl(a / 127);  q = clamp(rne(fl(x / s)), -127, 127)
 * (q = 0, s = 0 for an all-zero tensor) -- the treatment the converter gives
 * the embedding table instead of ConvRot [zskr.cn "Qwen3-VL-32B ...
 * INT8-ConvRot": word embedding "simple tensor-wise INT8"; conversion
 * command --custom-layers embed_tokens --custom-type int8
 * --custom-scaling-mode tensor --custom-simple].
 *   w_bf16 : BF16 [count] (device);  q : int8 [count] (device)
 *   scale  : ONE fp32 (device), overwritten; it also holds the running
 *            maximum between the launches, so it may not alias w or q.
 * count >= 16 and a multiple of 16.  Offline: four stream-ordered steps (a
 * memset of *scale and three kernels).
 */
convrot_status_t convrot_quantize_tensor(const void *w_bf16, int64_t count, int8_t *q, float *scale,
                                         void *stream);

/*
 * Rows of the tensor-wise table: out[i, :] = bf16_rne(fl((float)q[tokens[i], :]
 * * scale)) for i < t.
 *   tokens : int32 [t] (device);  q : int8 [vocab, dim];  scale : one fp32
 *   out_bf16 : BF16 [t, dim]
 * dim a multiple of 16.  A token id outside [0, vocab) cannot be checked on
 * the host: its row is written as zeros and CONVROT_ERR_INVALID_ARG is
 * recorded for convrot_device_status().
 */
convrot_status_t convrot_embed_lookup(const int32_t *tokens, int64_t t, const int8_t *q, const float *scale,
                                      int64_t vocab, int64_t dim, void *out_bf16, void *stream);

/*
 * Synchronise `stream`, then read and clear the device-side status word of
 * the current device.  Returns CONVROT_OK, CONVROT_ERR_DEVICE_TIMEOUT if a
 * bounded wait ran out in some kernel since the last call (the workspace
 * must then be re-initialised), CONVROT_ERR_INVALID_ARG if a lookup met a
 * token outside its table, CONVROT_WARN_INEXACT_DOMAIN if a rotation met an
 * input row that may lie outside the exact-sum domain (the results were
 * written; their low bits may differ from the exact-sum definition), or
 * CONVROT_ERR_CUDA.  A timeout overrides an earlier warning; the first
 * other status recorded is kept until this call clears it.
 */
convrot_status_t convrot_device_status(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* CONVROT_H */
