/*
 * tq.h -- C ABI of libtq: the TQ4_1S weight codec and its fused dequant-GEMV
 * for NVIDIA B200 (sm_100a).
 *
 * Source of the method: the web page titled "企业官网建设流程全解析"
 * (hotelren.com/news/5458160; below "TQ page"), which describes TQ4_1S weight
 * compression: paragraph 格式原理 items 1-3 (sign flip + 32-point Walsh-Hadamard
 * rotation per block, nearest of 16 Lloyd-Max N(0,1) centroids, separate
 * scales d0/d1 for elements 0-15 and 16-31), the paragraph after them (16
 * centroids, nibble packing, no correction term; the reference dequantiser
 * inverse-rotates and rescales) and section 解码速度：分硬件汇总 (decode
 * pre-rotates the activation once, so dequantisation becomes centroid
 * lookup times scale).
 *
 * ---------------------------------------------------------------------------
 * Conventions shared by every entry point
 * ---------------------------------------------------------------------------
 *  - W is N x K (out_features x in_features), row-major; y = W x.  Blocks of
 *    32 run along K; K must be a positive multiple of 32.
 *  - Pointers named codes/scales/w/x/y/workspace/xrot are DEVICE pointers on
 *    the current CUDA device; the caller owns and allocates all of them.
 *    The library allocates no memory and keeps no state beyond constant
 *    tables.  stream is a cudaStream_t (NULL = legacy default stream).
 *  - Calls are asynchronous on `stream` and never synchronise.  Argument
 *    errors are detected on the host before any launch and nothing is
 *    launched; a launch failure returns TQ_ERR_CUDA.
 *  - n == 0 or m == 0 is an empty problem: TQ_OK, nothing launched.
 *  - All results are deterministic run to run (no floating-point atomics).
 *
 * Packed format (5.0 bits per weight when N % 16 == 0 and K % 128 == 0):
 *  - code: 4 bits; bit 3 = sign (1 = negative), bits 0-2 = magnitude rank
 *    0..7 into the eight positive Lloyd-Max centroids.
 *  - superblock = four consecutive 32-element blocks of one row (128
 *    columns); NSB = ceil(K/128).  Rows are grouped in tiles of 16
 *    (T = ceil(N/16)).  A unit = (tile, superblock) is stored contiguously and
 *    units are tile-major, so the fused kernel streams 1024 + 256 contiguous
 *    bytes per unit.  Blocks past K/32 and rows past N are zero.
 *  - codes plane: uint8 [T][NSB][16 rows][64].  Within a row's 64 bytes,
 *    logical byte L (0..15) of block j (0..3) holds the codes of elements 2L
 *    (low nibble) and 2L+1 (high nibble) and is stored at byte
 *    16*(L%4) + 4*j + L/4.
 *  - scales plane: uint16 [T][NSB][16 rows][4 blocks][2], IEEE fp16 bit
 *    patterns d0, d1: d_h = fp16(sqrt(mean of the 16 squared rotated values)).
 *  - rotation: y = H (s .* w) per block, H the unnormalised 32x32 Sylvester
 *    Hadamard matrix; s_k = -1 where bit 31 of hash(k) is set, with
 *    hash(k) = g(k * 0x9E3779B9) and g(h) = ((h ^ h>>16) * 0x85EBCA6B) ^ (...>>13)
 *    on 32-bit words, k = global column index (same for every row).
 *  - dequantisation: w~ = s .* (H c) / 32, c_e = +-M[mag_e] * d_h(e).
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TQ_API __attribute__((visibility("default")))
#else
#define TQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TQ_OK = 0,
    TQ_ERR_INVALID_ARG = 1, /* null pointer, bad leading dimension, negative size */
    TQ_ERR_SHAPE = 2,       /* k <= 0, k % 32 != 0, or a size above the supported maximum */
    TQ_ERR_ALIGNMENT = 3,   /* a pointer or leading dimension breaks the alignment rule */
    TQ_ERR_DTYPE = 4,       /* unknown tq_dtype value */
    TQ_ERR_WORKSPACE = 5,   /* workspace null or smaller than the *_workspace_bytes query */
    TQ_ERR_CUDA = 6,        /* a CUDA runtime call or launch failed */
    TQ_ERR_UNSUPPORTED = 7, /* valid request that this build does not implement */
    TQ_ERR_TIMEOUT = 8      /* a kernel's bounded wait expired (tq_workspace_status) */
} tq_status;

typedef enum { TQ_F32 = 0, TQ_BF16 = 1, TQ_F16 = 2 } tq_dtype;

/* Largest supported sizes (checked; TQ_ERR_SHAPE above them). */
#define TQ_MAX_N ((int64_t)1 << 30)
#define TQ_MAX_K ((int64_t)1 << 26)
#define TQ_MAX_BATCH 8

/* Human-readable name of a status code (static string, never NULL). */
TQ_API const char *tq_status_string(tq_status s);

/* Bytes of the codes plane / of the scales plane for an N x K matrix
 * (ceil(n/16) * ceil(k/128) * 1024 and ceil(n/16) * ceil(k/128) * 256).
 * 0 for invalid sizes. */
TQ_API size_t tq_codes_bytes(int64_t n, int64_t k);
TQ_API size_t tq_scales_bytes(int64_t n, int64_t k);

/*
 * tq_quantize -- encode W into the packed TQ4_1S planes.
 * TQ page, 格式原理 items 1-3 and the paragraph after them: per 32-block,
 * sign flip + Walsh-Hadamard rotation, two fp16 RMS half-block scales, then
 * for every rotated value y the code sign(y) / #{j : |y| > B_j * d} with the
 * seven Lloyd-Max decision thresholds B_j (ties go to the smaller magnitude,
 * +0 and -0 count as positive).  Every step is IEEE fp32 in a fixed order,
 * so codes and scales are bit-reproducible by a CPU implementation.
 *   w      device, n x k of dtype wt (F32, BF16 or F16), row stride ldw
 *          elements (ldw >= k, ldw % 8 == 0, w 16-byte aligned)
 *   codes  device, tq_codes_bytes(n, k) bytes, 16-byte aligned (written)
 *   scales device, tq_scales_bytes(n, k) bytes, 16-byte aligned (written)
 * Inputs with |w| large enough to overflow fp16 scales (RMS >= 65520) or
 * containing NaN/Inf are outside the contract.
 */
TQ_API tq_status tq_quantize(const void *w, tq_dtype wt, int64_t n, int64_t k, int64_t ldw, uint8_t *codes,
                      uint16_t *scales, void *stream);

/*
 * tq_dequantize -- reconstruct w~ = s .* (H c) / 32 (TQ page, paragraph after
 * 格式原理: inverse rotation and rescale).  fp32 arithmetic, output rounded
 * to ot (nearest-even).
 *   codes, scales  device, as written by tq_quantize for the same n, k
 *   w_out  device, n x k of dtype ot, row stride ldo (ldo >= k, ldo % 8 == 0,
 *          16-byte aligned)
 */
TQ_API tq_status tq_dequantize(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, void *w_out,
                        tq_dtype ot, int64_t ldo, void *stream);

/*
 * tq_dequantize_batch -- tq_dequantize of count (1..TQ_MAX_BATCH) matrices in
 * one launch, every output of dtype ot (e.g. all seven matrices of a layer;
 * one launch has one ramp and one tail instead of seven).  The same argument
 * rules as tq_dequantize per descriptor; descriptors with n == 0 are skipped.
 * Outputs must not overlap one another or any codes/scales.
 */
typedef struct {
    const uint8_t *codes;   /* device, packed planes of an n x k matrix (tq_quantize) */
    const uint16_t *scales;
    int64_t n;              /* >= 0 */
    int64_t k;              /* positive multiple of 32 */
    void *w_out;            /* device, n x k of dtype ot, row stride ldo (ldo >= k, ldo % 8 == 0, 16-byte aligned) */
    int64_t ldo;
} tq_dequant_desc;
TQ_API tq_status tq_dequantize_batch(const tq_dequant_desc *descs, int count, tq_dtype ot, void *stream);

/*
 * Pre-rotated activations (TQ page, 解码速度 section: the activation is
 * rotated once and shared, so the per-weight work is lookup x scale).
 * xrot holds fp16 values H(s .* x)/32 per 32-block, in the order the fused
 * kernel's tensor-core fragments read them: [m][NSB][4 blocks][4][8], where
 * entry [t][q] of a block is element (q/2)*8 + 2t + (q%2).  Padding blocks
 * are zero.  |x| must stay below 65504 (fp16 range).
 */
TQ_API size_t tq_xrot_bytes(int64_t m, int64_t k);

/*
 * tq_prerotate -- xrot = fragment-ordered fp16(H (s .* x) / 32) for each of the
 * m rows of X.
 *   X     device, m x k of dtype xt, row stride ldx (ldx >= k, ldx % 8 == 0,
 *         16-byte aligned)
 *   xrot  device, tq_xrot_bytes(m, k) bytes, 16-byte aligned (written)
 */
TQ_API tq_status tq_prerotate(const void *X, tq_dtype xt, int64_t m, int64_t k, int64_t ldx, uint16_t *xrot,
                       void *stream);

/* Workspace bytes needed by tq_gemm / tq_gemv / tq_gemm_xrot on the CURRENT
 * device for these sizes (the split-K partition depends on its SM count).
 * Layout: a 256-byte header (status word, call tag), the split-K partial
 * sums and the pre-rotated activation.
 *
 * Every call clears the status word and advances the 32-bit call tag before
 * its product; split-K partial sums are stored together with the tag of
 * their call, so words left by earlier calls never match.  A workspace that
 * has never been used holds arbitrary bytes and a stale word could match the
 * first call's tag by chance (probability 2^-32 per word read): zero-fill a
 * new workspace once (later calls need no clearing). */
TQ_API size_t tq_gemm_workspace_bytes(int64_t m, int64_t n, int64_t k);

/*
 * tq_gemm -- Y[i][r] = sum_k w~[r][k] X[i][k] for i < m, r < n, computed as
 * (1/32) sum_blocks sum_halves d * sum_e c_e xrot_e with the activation
 * pre-rotated once per call (TQ page, 解码速度 section).  Centroids and xrot
 * enter the tensor cores as fp16; products accumulate in fp32.
 * Kernels: m <= 8 runs the mma.sync kernel (half-block sums scaled in fp32);
 * m = 9..32 runs the tcgen05 kernel that stages the decoded weights in tensor
 * memory; m > 32 runs the prefill product.  From m = 9 (and for m = 25..32
 * on the mma.sync kernel when a test hook forces it) the centroid enters
 * already multiplied by its half-block scale, fp16(c * d): that product
 * overflows once d exceeds about 23,970 (weights of magnitude around 4,000
 * and up) and becomes an fp16 subnormal, with coarser relative precision,
 * once 0.128 * d falls below 6.1e-5, i.e. d below about 4.8e-4 (weights of
 * RMS below about 1e-4).
 *   X          device, m x k of dtype xt, row stride ldx (as tq_prerotate)
 *   Y          device, m x n of dtype yt (F32, BF16 or F16), row stride ldy
 *              (ldy >= n)
 *   workspace  device, >= tq_gemm_workspace_bytes(m, n, k) bytes, 256-byte
 *              aligned, exclusively owned by this call until it completes
 *              on `stream` (zero-filled once when new, see above; calls
 *              that overlap on the GPU must use different workspaces)
 * m <= 32 runs the skinny kernel in one pass; larger m runs the tensor-core
 * prefill product of tq_gemm_prefill (its workspace is then the size that
 * tq_gemm_workspace_bytes(m, n, k) returns for that m).
 */
TQ_API tq_status tq_gemm(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, const void *X, tq_dtype xt,
                  int64_t m, int64_t ldx, void *Y, tq_dtype yt, int64_t ldy, void *workspace, size_t ws_bytes,
                  void *stream);

/* tq_gemv -- tq_gemm with m = 1 (x: k elements, y: n elements). */
TQ_API tq_status tq_gemv(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, const void *x, tq_dtype xt,
                  void *y, tq_dtype yt, void *workspace, size_t ws_bytes, void *stream);

/*
 * tq_gemm_prefill -- the same product for many activation rows (prefill) on
 * the fifth-generation tensor cores (TQ page, 解码速度 section: rotate the
 * activation once, then every weight is centroid times scale).  X is first
 * pre-rotated into a plain row-major fp16 matrix in the workspace; then each
 * CTA takes 256 weight rows x 256 activation rows: it decodes its weight rows
 * 64 columns at a time into shared memory (centroid x half-block scale, fp16),
 * receives the matching activation columns by TMA, and accumulates
 * tcgen05.mma products (fp16 operands, two fp32 accumulators in tensor
 * memory, one per 128-row half of the weight tile).
 * Compared with tq_gemm's skinny path the weight enters as fp16(c * d), one
 * more rounding per weight (relative 2^-11).  Same operand rules as tq_gemm;
 * any m >= 1 (m <= 16,776,960).  Returns TQ_ERR_UNSUPPORTED if the driver
 * offers no tensor-map encoder.
 *   workspace  >= tq_gemm_prefill_workspace_bytes(m, k) bytes (256-byte
 *              header + m*k fp16), 256-byte aligned
 */
TQ_API size_t tq_gemm_prefill_workspace_bytes(int64_t m, int64_t k);
TQ_API tq_status tq_gemm_prefill(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, const void *X,
                                 tq_dtype xt, int64_t m, int64_t ldx, void *Y, tq_dtype yt, int64_t ldy,
                                 void *workspace, size_t ws_bytes, void *stream);

/*
 * The two steps of tq_gemm_prefill as separate calls, so that one rotated
 * activation serves every matrix that consumes it (e.g. q/k/v in a prefill;
 * TQ page, paragraph 适用前提与边界, the attention tensors share one rotation).
 *
 * tq_prefill_xrot_bytes -- m * k * 2: the plain pre-rotated activation, a
 * row-major m x k fp16 matrix, element [i][c] = fp16(H(s .* x_i)/32) at
 * column c (blocks of 32 along k, in order).
 *
 * tq_prerotate_plain -- writes that matrix for the m rows of X.
 *   X     device, m x k of dtype xt, row stride ldx (as tq_prerotate)
 *   xrot  device, tq_prefill_xrot_bytes(m, k) bytes, 16-byte aligned
 *         (written; read by tensor-memory-accelerator copies afterwards)
 *
 * tq_gemm_prefill_xrot -- the tensor-core product of tq_gemm_prefill over an
 * xrot written by tq_prerotate_plain (same m and k).  The workspace needs
 * only its 256-byte header (>= 256 bytes, 256-byte aligned); a one-thread
 * launch clears its status word first.  Y, yt, ldy as tq_gemm.
 */
TQ_API size_t tq_prefill_xrot_bytes(int64_t m, int64_t k);
TQ_API tq_status tq_prerotate_plain(const void *X, tq_dtype xt, int64_t m, int64_t k, int64_t ldx, uint16_t *xrot,
                                    void *stream);
TQ_API tq_status tq_gemm_prefill_xrot(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k,
                                      const uint16_t *xrot, int64_t m, void *Y, tq_dtype yt, int64_t ldy,
                                      void *workspace, size_t ws_bytes, void *stream);

/*
 * tq_gemm_xrot -- the product with an activation already pre-rotated by
 * tq_prerotate (one xrot shared by every matrix that consumes the same
 * input, e.g. q/k/v).  m <= 32.  Same workspace rules as tq_gemm (a
 * one-thread launch on `stream` clears the status word and advances the call
 * tag before the product).
 */
TQ_API tq_status tq_gemm_xrot(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, const uint16_t *xrot,
                       int64_t m, void *Y, tq_dtype yt, int64_t ldy, void *workspace, size_t ws_bytes, void *stream);

/*
 * Several matrices in one launch (TQ page, paragraph 适用前提与边界: the
 * attention tensors of a layer share one in-place rotation, i.e. matrices
 * that consume the same input can share one pre-rotated activation).
 * Every descriptor is one product Y = X w~^T with its own codes/scales;
 * descriptors with the same X pointer, k and ldx share one pre-rotation.
 * One launch pre-rotates every distinct input, one launch computes every
 * product (no per-matrix launch overhead).
 */
typedef struct {
    const uint8_t *codes;   /* device, packed planes of an n x k matrix */
    const uint16_t *scales;
    int64_t n;              /* >= 1 */
    int64_t k;              /* positive multiple of 32 */
    const void *X;          /* device, m x k activations (dtype xt), row stride ldx */
    int64_t ldx;
    void *Y;                /* device, m x n outputs (dtype yt), row stride ldy */
    int64_t ldy;
} tq_gemm_desc;

/* Workspace bytes for tq_gemm_batch on the current device (0 if invalid). */
TQ_API size_t tq_gemm_batch_workspace_bytes(const tq_gemm_desc *descs, int count, int64_t m);

/* tq_gemm_batch -- count (1..TQ_MAX_BATCH) products with m <= 32 activation
 * rows each; the same argument rules as tq_gemm per descriptor. */
TQ_API tq_status tq_gemm_batch(const tq_gemm_desc *descs, int count, int64_t m, tq_dtype xt, tq_dtype yt,
                               void *workspace, size_t ws_bytes, void *stream);

/*
 * tq_workspace_status -- synchronises `stream`, then reports whether the last
 * product that used this workspace hit a bounded wait (TQ_ERR_TIMEOUT: the
 * kernel gave up on a bulk copy after ~1 s, recorded it and returned; its
 * outputs are then incomplete).  clear != 0 resets the flag.  The flag is
 * also reset by the next tq_gemm / tq_gemv / tq_gemm_xrot / tq_gemm_batch
 * on the workspace.
 */
TQ_API tq_status tq_workspace_status(void *workspace, int clear, void *stream);

/*
 * tq_debug_set_flags -- test hook, process-wide, 0 by default.  Bit 0: in
 * later fused-product launches (m <= 32) the first copy of the first warp
 * (mma.sync kernel) or of the first CTA (tensor-memory kernel) is never
 * issued, so its bounded wait expires after ~5 ms and the timeout path runs
 * (status word set, kernel returns normally; no fault, no trap).  Bits 2 and
 * 3: every product with m <= 32 runs on the tensor-memory kernel (bit 2) or
 * on the mma.sync kernel (bit 3) instead of the kernel chosen by m.  Bit 4:
 * in the mma.sync kernel the first warp of every split tile recomputes the
 * later warps' contributions from the packed weights instead of reading
 * them (the path it takes when a contribution does not arrive within 50 us,
 * e.g. because another kernel holds the SMs its CTA needs); the result is
 * bit-identical.  Bit 1:
 * the same for the tensor-core prefill product (tq_gemm_prefill and m > 32):
 * the first CTA never issues its second activation-tile copy (nor counts its
 * bytes), its waits expire after ~5 ms, every tensor-memory column is still
 * released, and the status word is set.
 */
TQ_API void tq_debug_set_flags(uint32_t flags);

/*
 * tq_gemv_static_scratch -- the GEMV of tq_gemv for callers that cannot
 * allocate device memory (code inside an allocator or memory-pool callback,
 * plugins that only receive an operation's tensors, processes whose device
 * memory is all reserved up front).  The pages this library follows have no
 * counterpart to it: it exists only for such callers.
 *
 * Inputs and outputs are as for tq_gemv (x: k elements, y: n elements, both
 * device memory supplied by the caller); no workspace is passed.  Instead the
 * scratch lives in one fixed device array of TQ_STATIC_SCRATCH_BYTES inside
 * the library, present on every GPU that loads it until the process exits.
 * The call allocates nothing (no cudaMalloc, cudaFree or allocating library
 * routine) and returns TQ_ERR_SHAPE when the problem's scratch,
 * tq_gemm_workspace_bytes(1, n, k), exceeds TQ_STATIC_SCRATCH_BYTES.
 *
 * The first call in a CUDA context looks up the array's device address
 * (cudaGetSymbolAddress) with that context's device current; make that first
 * call before any stream capture.  The address is cached per context (keyed
 * by the driver's unique context id), so after cudaDeviceReset, or from
 * another context on the same device, the next call looks it up again; do
 * that call outside stream capture too.  All calls share the array, and each
 * starts by clearing what must start at zero: calls that overlap on the GPU
 * (other streams, other host threads, without ordering between them) race
 * and give wrong results.  Run them in order on one stream (or order the
 * streams with events), or use tq_gemv.
 *
 * A bounded wait that expires inside this call is recorded in the array's
 * status word like tq_gemv's: read it with tq_static_scratch_status.
 */
#define TQ_STATIC_SCRATCH_BYTES (4u << 20)

TQ_API tq_status tq_gemv_static_scratch(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k,
                                        const void *x, tq_dtype xt, void *y, tq_dtype yt, void *stream);

/*
 * tq_static_scratch_status -- tq_workspace_status for the fixed array of
 * tq_gemv_static_scratch in the current context: synchronises `stream`, then
 * returns TQ_ERR_TIMEOUT if the last tq_gemv_static_scratch call on this
 * device gave up a bounded wait (its y is then incomplete), else TQ_OK;
 * clear != 0 resets the flag (the next call also resets it).  Allocates
 * nothing.
 */
TQ_API tq_status tq_static_scratch_status(int clear, void *stream);

/*
 * ---------------------------------------------------------------------------
 * NVFP4 comparison codec
 * ---------------------------------------------------------------------------
 * NVFP4 is named, without a bit recipe, by the llm-compressor page
 * (ai-insight.org/news/11771: NVFP4 checkpoints) and the llama.cpp quantizer
 * page (bittide.aicompass.dev: "NVFP4 weight and input tensor scales").  This
 * library implements the plainest reading of the format, for comparison with
 * TQ4_1S on the same shapes:
 *   g   = amax|W| / (6 * 448)                       fp32, one per tensor
 *   s_b = E4M3(amax_b / (6 * g))                    one per 16 elements
 *   q   = E2M1(w / (value(s_b) * g))                4 bits per element, 0 when
 *                                                   the scale is 0
 *   w~  = value(q) * value(s_b) * g
 * Each quotient and product is one IEEE fp32 operation; both conversions
 * round to nearest-even and saturate (E4M3 at 448, E2M1 at 6); a zero code
 * carries no sign.  No rotation.  4.5 bits per weight.
 *
 * Layout: the codes plane is the TQ4_1S one (tq_codes_bytes; the two
 * 16-element blocks of a 32-column pair take the place of one 32-element
 * block, byte order unchanged: element 2L in the low nibble of logical byte
 * L).  E2M1 code: bit 3 = sign, bits 0-2 = magnitude index into
 * {0, 0.5, 1, 1.5, 2, 3, 4, 6}.  The scales plane is E4M3 bytes
 * [T][NSB][16 rows][8 blocks of 16] (tq_nvfp4_scales_bytes).  The tensor
 * block is TQ_NVFP4_TENSOR_BYTES of device memory: float g at offset 0, the
 * fp32 amax|W| at offset 4, the rest reserved.
 */
#define TQ_NVFP4_TENSOR_BYTES 16

/* ceil(n/16) * ceil(k/128) * 128 bytes; 0 for invalid sizes. */
TQ_API size_t tq_nvfp4_scales_bytes(int64_t n, int64_t k);

/*
 * tq_nvfp4_quantize -- encode W (n x k, dtype wt, row stride ldw; the operand
 * rules of tq_quantize) into codes (tq_codes_bytes), scales
 * (tq_nvfp4_scales_bytes) and the tensor block (TQ_NVFP4_TENSOR_BYTES); all
 * device, 16-byte aligned, written.  Three operations on `stream`: a memset of
 * the amax word, a reduction of amax|W|, the encode.  NaN/Inf inputs are
 * outside the contract.
 */
TQ_API tq_status tq_nvfp4_quantize(const void *w, tq_dtype wt, int64_t n, int64_t k, int64_t ldw, uint8_t *codes,
                                   uint8_t *scales, float *tensor_scale, void *stream);

/* tq_nvfp4_dequantize -- w~ in fp32, rounded to ot; the operand rules of
 * tq_dequantize plus the tensor block written by tq_nvfp4_quantize. */
TQ_API tq_status tq_nvfp4_dequantize(const uint8_t *codes, const uint8_t *scales, const float *tensor_scale,
                                     int64_t n, int64_t k, void *w_out, tq_dtype ot, int64_t ldo, void *stream);

/*
 * tq_nvfp4_gemm -- Y[i][r] = sum_k w~[r][k] X[i][k] for i < m <= 32 with the
 * fused kernel of tq_gemm: codes enter the tensor cores as fp16 E2M1 values,
 * the activation as fp16 (converted once per call, no rotation), each
 * 16-column partial sum is scaled by its E4M3 block scale in fp32 and the
 * row total by g.  Workspace: tq_gemm_workspace_bytes(m, n, k), same rules.
 * m > 32 returns TQ_ERR_SHAPE.
 */
TQ_API tq_status tq_nvfp4_gemm(const uint8_t *codes, const uint8_t *scales, const float *tensor_scale, int64_t n,
                               int64_t k, const void *X, tq_dtype xt, int64_t m, int64_t ldx, void *Y, tq_dtype yt,
                               int64_t ldy, void *workspace, size_t ws_bytes, void *stream);

/* Several NVFP4 products in one launch pair, as tq_gemm_batch. */
typedef struct {
    const uint8_t *codes;
    const uint8_t *scales;
    const float *tensor_scale; /* device tensor block of this matrix */
    int64_t n;
    int64_t k;
    const void *X;
    int64_t ldx;
    void *Y;
    int64_t ldy;
} tq_nvfp4_gemm_desc;

TQ_API size_t tq_nvfp4_gemm_batch_workspace_bytes(const tq_nvfp4_gemm_desc *descs, int count, int64_t m);
TQ_API tq_status tq_nvfp4_gemm_batch(const tq_nvfp4_gemm_desc *descs, int count, int64_t m, tq_dtype xt, tq_dtype yt,
                                     void *workspace, size_t ws_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H_ */
