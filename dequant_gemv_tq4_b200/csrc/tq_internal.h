// tq_internal.h -- launchers behind the C ABI (host side, no validation here:
// the C ABI checks every argument before calling them).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace tq {

constexpr int kMaxInputs = 8;    // distinct activations pre-rotated by one launch
constexpr int kMaxProblems = 8;  // matrices in one fused-product launch

struct DeviceInfo {
    int device;
    int sm_count;
};

// Current device and its SM count (cached per device).
cudaError_t device_info(DeviceInfo *out);

inline int64_t superblocks(int64_t k) { return (k / 32 + 3) / 4; }
inline int64_t tiles(int64_t n) { return (n + 15) / 16; }
inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

cudaError_t launch_quantize(const void *w, int dtype, int64_t n, int64_t k, int64_t ldw, uint8_t *codes,
                            uint16_t *scales, cudaStream_t stream);

cudaError_t launch_dequantize(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, void *w_out,
                              int dtype, int64_t ldo, cudaStream_t stream);

// Several matrices dequantised by one launch (all outputs of one dtype).
struct DequantJob {
    const uint8_t *codes;
    const uint16_t *scales;
    int64_t n;
    int64_t k;
    void *out;
    int64_t ldo;
};
cudaError_t launch_dequantize_batch(const DequantJob *jobs, int count, int dtype, cudaStream_t stream);

// ---- pre-rotation ----------------------------------------------------------
struct RotInput {  // device-side description of one activation matrix
    const char *x;
    uint32_t *xrot;
    int64_t ldx;
    int64_t unit_begin;  // first warp unit (row, superblock) of this input
    int nb;
    int nsb;
};

struct RotParams {
    RotInput in[kMaxInputs];
    int count;
    int64_t units;
    unsigned *header;  // product workspace header (see below), or nullptr
    int m;             // activation rows (rows past m are written as zeros)
    int npad;          // rows of the core-matrix layout
};

// Output layouts of the pre-rotation (see launch_prerotate).
enum RotLayout : int { kRotFragment = 0, kRotPlain = 1, kRotCore = 2 };

struct RotJob {  // host-side request
    const void *x;
    int64_t ldx;
    int64_t k;
    uint16_t *xrot;
};

// Header of a fused-product workspace (its first 256 bytes): word 0 is the
// status word (timeout flag), word 1 the call tag.  Every call first clears
// the status and advances the tag; the product's split-K partial sums are
// stored with the tag of their call, so entries of earlier calls never match.
constexpr int kHeaderStatus = 0;
constexpr int kHeaderTag = 1;

// xrot for m rows of every job (same dtype); also prepares `header` (status
// cleared, tag advanced) when it is not null.  With rotate = false the
// activation is only converted to fp16 (fragment or core-matrix order).
// Layouts: kRotFragment (tq_xrot_bytes per input; the mma.sync kernel),
// kRotPlain (one row, NSB*128 fp16 with zero padding; the tensor-memory
// kernel for m = 1), kRotCore (npad rows, NSB*16*npad*16 bytes; the
// tensor-memory kernel for m > 1).
cudaError_t launch_prerotate(const RotJob *jobs, int count, int dtype, int64_t m, unsigned *header,
                             cudaStream_t stream, bool rotate = true, int layout = kRotFragment, int npad = 0);

// Only the header preparation (for products whose activation is already
// pre-rotated).  Launched as a programmatic dependent like the pre-rotation.
cudaError_t launch_prepare_header(unsigned *header, cudaStream_t stream);

// ---- fused product ---------------------------------------------------------
struct GemvProblem {  // host-side request, m <= 32 rows of pre-rotated activations
    const uint8_t *codes;
    const uint16_t *scales;
    const uint16_t *xrot;
    void *y;
    int64_t ldy;
    int64_t n;
    int64_t k;
    const float *tensor_scale = nullptr;  // NVFP4 only (device pointer)
};

struct GroupPlan {
    int64_t units;        // sum over problems of tiles * nsb
    int64_t tiles;        // sum over problems of ceil(n / 16)
    int grid;             // CTAs (<= SM count)
    int total_warps;      // min(grid * warps per CTA, units); warp w owns [w*U/W, (w+1)*U/W)
    int mcap;             // 8 * ceil(m / 8)
    size_t partial_bytes; // (tiles + total_warps) * 16 * mcap * 8 (value + tag), rounded up to 256
};

GroupPlan plan_group(const int64_t *n, const int64_t *k, int count, int64_t m, int sm_count);

// Debug hooks (tq_debug_set_flags): bit 0 makes one bulk copy of the fused
// GEMV go missing, bit 1 one activation-tile copy of the prefill product, so
// that the kernel's bounded wait expires and reports a timeout.
constexpr uint32_t kDebugSkipGemvCopy = 1u;
constexpr uint32_t kDebugSkipPrefillCopy = 2u;
// bits 2 and 3: run every product of m <= 32 on the tensor-memory kernel
// (bit 2) or on the mma.sync kernel (bit 3) instead of choosing by m (lets
// tests and measurements cover both kernels at every m)
constexpr uint32_t kDebugUseTmem = 4u;
constexpr uint32_t kDebugUseMmaSync = 8u;
// bit 4: in the mma.sync kernel, the first warp of every split tile computes
// the later contributions itself instead of reading them (the path taken
// when a contributor cannot run)
constexpr uint32_t kDebugStealAll = 16u;
void set_debug_flags(uint32_t flags);
uint32_t debug_flags();

cudaError_t launch_group(const GemvProblem *probs, int count, int64_t m, int ydtype, const GroupPlan &plan,
                         unsigned *header, uint64_t *partials, bool programmatic, cudaStream_t stream);

// ---- fused product on tcgen05 with the weights in tensor memory (tq_tcgemv.cu)
// Big units of 128 weight rows x 128 columns split into equal ranges, one per
// CTA; split row blocks combine through per-row-block call-tagged counters
// (the last contributor adds the partial sums).  The activation operand is
// the pre-rotation in kRotPlain layout (m = 1) or kRotCore layout with
// npad = 16 (m <= 16) or 32 rows.
struct TcPlan {
    int64_t units;        // big units over all problems
    int64_t rblocks;      // row blocks over all problems (counter slots)
    int grid;             // CTAs (<= SM count)
    int npad;             // activation rows of the operand: 0 (one row, plain layout), 16 or 32
    int mld;              // accumulator columns read back per row: 1, 2, 4, 8, 16 or 32
    size_t counter_bytes; // rblocks * 8, rounded up to 256
    size_t partial_bytes; // 2 * grid * mld * 128 fp32, rounded up to 256
};
int tc_npad(int64_t m);
int tc_mld(int64_t m);
size_t tc_xrot_bytes(int64_t m, int64_t k);  // the activation operand of one input
TcPlan plan_tc(const int64_t *n, const int64_t *k, int count, int64_t m, int sm_count);
cudaError_t launch_tc(const GemvProblem *probs, int count, int64_t m, int ydtype, const TcPlan &plan,
                      unsigned *header, unsigned long long *counters, float *partials, bool programmatic,
                      cudaStream_t stream);
// Which kernel runs a TQ4_1S product of m <= 32 activation rows: the mma.sync
// kernel up to 8 rows, the tensor-memory kernel from 9 rows (measured on B200:
// from 9 rows the mma.sync kernel reloads four activation fragments per unit
// and falls below it); the test hooks kDebugUseTmem / kDebugUseMmaSync force
// one kernel.
bool use_tc(int64_t m);

// ---- large-M product on tcgen05 (tq_prefill.cu) ---------------------------------
// Y = X w~^T for any m: X is first pre-rotated into plain row-major fp16 xrot
// (prefill_xrot_bytes), then one CTA per 256 weight rows x 256 activation rows
// decodes the weight tile into shared memory and multiplies on the tensor cores.
size_t prefill_xrot_bytes(int64_t m, int64_t k);
cudaError_t launch_prefill(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, const void *X,
                           int xdtype, int64_t m, int64_t ldx, uint16_t *xrot, void *y, int ydtype, int64_t ldy,
                           unsigned *header, cudaStream_t stream);
// The two steps of launch_prefill on their own: the plain pre-rotation (header
// may be null; otherwise it clears the status word and advances the call tag)
// and the product over an xrot it wrote.
cudaError_t launch_prerotate_plain(const void *X, int xdtype, int64_t m, int64_t k, int64_t ldx, uint16_t *xrot,
                                   unsigned *header, cudaStream_t stream);
cudaError_t launch_prefill_product(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k,
                                   const uint16_t *xrot, int64_t m, void *y, int ydtype, int64_t ldy,
                                   unsigned *header, cudaStream_t stream);

// ---- NVFP4 comparison codec ---------------------------------------------------
// Same fused product over NVFP4 planes (E2M1 codes in the TQ4_1S unit layout,
// E4M3 block scales, a device fp32 tensor scale per problem); xrot holds the
// activation in fragment order without rotation (launch_prerotate, rotate=false).
cudaError_t launch_group_nvfp4(const GemvProblem *probs, int count, int64_t m, int ydtype, const GroupPlan &plan,
                               unsigned *header, uint64_t *partials, bool programmatic, cudaStream_t stream);

cudaError_t launch_nvfp4_amax(const void *w, int dtype, int64_t n, int64_t k, int64_t ldw, unsigned *amax_bits,
                              cudaStream_t stream);
cudaError_t launch_nvfp4_quantize(const void *w, int dtype, int64_t n, int64_t k, int64_t ldw,
                                  const unsigned *amax_bits, uint8_t *codes, uint8_t *scales, float *tensor_scale,
                                  cudaStream_t stream);
cudaError_t launch_nvfp4_dequantize(const uint8_t *codes, const uint8_t *scales, const float *tensor_scale,
                                    int64_t n, int64_t k, void *w_out, int dtype, int64_t ldo, cudaStream_t stream);

}  // namespace tq
