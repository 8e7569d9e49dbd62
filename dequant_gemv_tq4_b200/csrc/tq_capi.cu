// tq_capi.cu -- the extern "C" boundary (include/tq.h): argument checks on
// the host, workspace carving, dispatch to the launchers.  No allocation.
#include <mutex>

#include "../../include/tq.h"
#include "tq_internal.h"

namespace tq {

cudaError_t device_info(DeviceInfo *out) {
    static std::mutex mu;
    static int cached_sm[256] = {0};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 256) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (cached_sm[dev] == 0) {
        int sms = 0;
        err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (err != cudaSuccess) return err;
        cached_sm[dev] = sms;
    }
    out->device = dev;
    out->sm_count = cached_sm[dev];
    return cudaSuccess;
}

}  // namespace tq

namespace {

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool valid_dtype(tq_dtype d) { return d == TQ_F32 || d == TQ_BF16 || d == TQ_F16; }

tq_status check_nk(int64_t n, int64_t k) {
    if (n < 0 || k < 0) return TQ_ERR_INVALID_ARG;
    if (k == 0 || k % 32 != 0 || k > TQ_MAX_K || n > TQ_MAX_N) return TQ_ERR_SHAPE;
    return TQ_OK;
}

tq_status check_matrix_operand(const void *p, int64_t ld, int64_t cols) {
    if (!p) return TQ_ERR_INVALID_ARG;
    if (ld < cols) return TQ_ERR_INVALID_ARG;
    if (!aligned(p, 16) || ld % 8 != 0) return TQ_ERR_ALIGNMENT;
    return TQ_OK;
}

tq_status check_planes(const uint8_t *codes, const uint16_t *scales) {
    if (!codes || !scales) return TQ_ERR_INVALID_ARG;
    if (!aligned(codes, 16) || !aligned(scales, 16)) return TQ_ERR_ALIGNMENT;
    return TQ_OK;
}

tq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA; }

struct GemmLayout {
    size_t xrot_off, xrot_bytes, counter_off, partial_off, total;
    tq::SkinnyPlan plan;
};

// Workspace: [xrot for <= 32 rows][split-K counters][partial slots].
tq_status gemm_layout(int64_t m, int64_t n, int64_t k, bool with_xrot, GemmLayout *lay) {
    tq::DeviceInfo di;
    if (tq::device_info(&di) != cudaSuccess) return TQ_ERR_CUDA;
    const int64_t ms = m > 32 ? 32 : m;
    lay->plan = tq::plan_skinny(ms, n, k, di.sm_count);
    lay->xrot_off = 0;
    lay->xrot_bytes = with_xrot ? tq::round_up(tq_xrot_bytes(ms, k), 256) : 0;
    lay->counter_off = lay->xrot_bytes;
    lay->partial_off = lay->counter_off + lay->plan.counter_bytes;
    lay->total = lay->partial_off + lay->plan.partial_bytes;
    return TQ_OK;
}

}  // namespace

extern "C" {

const char *tq_status_string(tq_status s) {
    switch (s) {
        case TQ_OK: return "TQ_OK";
        case TQ_ERR_INVALID_ARG: return "TQ_ERR_INVALID_ARG: null pointer, bad leading dimension or negative size";
        case TQ_ERR_SHAPE: return "TQ_ERR_SHAPE: k must be a positive multiple of 32 within the supported maximum";
        case TQ_ERR_ALIGNMENT: return "TQ_ERR_ALIGNMENT: pointers must be 16-byte aligned and leading dimensions multiples of 8";
        case TQ_ERR_DTYPE: return "TQ_ERR_DTYPE: unknown element type";
        case TQ_ERR_WORKSPACE: return "TQ_ERR_WORKSPACE: workspace missing, misaligned or too small";
        case TQ_ERR_CUDA: return "TQ_ERR_CUDA: a CUDA call or kernel launch failed";
        case TQ_ERR_UNSUPPORTED: return "TQ_ERR_UNSUPPORTED: request not implemented by this build";
    }
    return "unknown tq_status";
}

size_t tq_codes_bytes(int64_t n, int64_t k) {
    if (check_nk(n, k) != TQ_OK) return 0;
    return (size_t)n * (size_t)tq::superblocks(k) * 64u;
}

size_t tq_scales_bytes(int64_t n, int64_t k) {
    if (check_nk(n, k) != TQ_OK) return 0;
    return (size_t)n * (size_t)tq::superblocks(k) * 16u;
}

size_t tq_xrot_bytes(int64_t m, int64_t k) {
    if (m < 0 || check_nk(0, k) != TQ_OK) return 0;
    return (size_t)m * (size_t)tq::superblocks(k) * 4u * 32u * 2u;
}

tq_status tq_quantize(const void *w, tq_dtype wt, int64_t n, int64_t k, int64_t ldw, uint8_t *codes,
                      uint16_t *scales, void *stream) {
    tq_status st = check_nk(n, k);
    if (st != TQ_OK) return st;
    if (!valid_dtype(wt)) return TQ_ERR_DTYPE;
    if (n == 0) return TQ_OK;
    if ((st = check_matrix_operand(w, ldw, k)) != TQ_OK) return st;
    if ((st = check_planes(codes, scales)) != TQ_OK) return st;
    return from_cuda(tq::launch_quantize(w, wt, n, k, ldw, codes, scales, (cudaStream_t)stream));
}

tq_status tq_dequantize(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, void *w_out,
                        tq_dtype ot, int64_t ldo, void *stream) {
    tq_status st = check_nk(n, k);
    if (st != TQ_OK) return st;
    if (!valid_dtype(ot)) return TQ_ERR_DTYPE;
    if (n == 0) return TQ_OK;
    if ((st = check_planes(codes, scales)) != TQ_OK) return st;
    if ((st = check_matrix_operand(w_out, ldo, k)) != TQ_OK) return st;
    return from_cuda(tq::launch_dequantize(codes, scales, n, k, w_out, ot, ldo, (cudaStream_t)stream));
}

tq_status tq_prerotate(const void *X, tq_dtype xt, int64_t m, int64_t k, int64_t ldx, uint16_t *xrot,
                       void *stream) {
    tq_status st = check_nk(m, k);
    if (st != TQ_OK) return st;
    if (!valid_dtype(xt)) return TQ_ERR_DTYPE;
    if (m == 0) return TQ_OK;
    if ((st = check_matrix_operand(X, ldx, k)) != TQ_OK) return st;
    if (!xrot) return TQ_ERR_INVALID_ARG;
    if (!aligned(xrot, 16)) return TQ_ERR_ALIGNMENT;
    return from_cuda(tq::launch_prerotate(X, xt, m, k, ldx, xrot, nullptr, 0, (cudaStream_t)stream));
}

size_t tq_gemm_workspace_bytes(int64_t m, int64_t n, int64_t k) {
    if (m < 0 || check_nk(n, k) != TQ_OK) return 0;
    GemmLayout lay;
    if (gemm_layout(m < 1 ? 1 : m, n, k, true, &lay) != TQ_OK) return 0;
    return lay.total;
}

static tq_status check_gemm_common(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, int64_t m,
                                   void *Y, tq_dtype yt, int64_t ldy) {
    tq_status st = check_nk(n, k);
    if (st != TQ_OK) return st;
    if (m < 0) return TQ_ERR_INVALID_ARG;
    if (m > TQ_MAX_N) return TQ_ERR_SHAPE;
    if (!valid_dtype(yt)) return TQ_ERR_DTYPE;
    if (n == 0 || m == 0) return TQ_OK;
    if ((st = check_planes(codes, scales)) != TQ_OK) return st;
    if (!Y) return TQ_ERR_INVALID_ARG;
    if (ldy < n) return TQ_ERR_INVALID_ARG;
    const size_t esize = yt == TQ_F32 ? 4 : 2;
    if (!aligned(Y, esize)) return TQ_ERR_ALIGNMENT;
    return TQ_OK;
}

tq_status tq_gemm_xrot(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, const uint16_t *xrot,
                       int64_t m, void *Y, tq_dtype yt, int64_t ldy, void *workspace, size_t ws_bytes, void *stream) {
    tq_status st = check_gemm_common(codes, scales, n, k, m, Y, yt, ldy);
    if (st != TQ_OK || n == 0 || m == 0) return st;
    if (m > 32) return TQ_ERR_SHAPE;
    if (!xrot) return TQ_ERR_INVALID_ARG;
    if (!aligned(xrot, 16)) return TQ_ERR_ALIGNMENT;
    GemmLayout lay;
    if ((st = gemm_layout(m, n, k, false, &lay)) != TQ_OK) return st;
    if (!workspace || !aligned(workspace, 256) || ws_bytes < lay.total) return TQ_ERR_WORKSPACE;
    char *ws = static_cast<char *>(workspace);
    auto *counters = reinterpret_cast<unsigned *>(ws + lay.counter_off);
    // the arrival counters must start at zero; the workspace may have held
    // anything (another call's partial sums or pre-rotated activations)
    cudaError_t e = cudaMemsetAsync(counters, 0, (size_t)lay.plan.tiles * sizeof(unsigned), (cudaStream_t)stream);
    if (e != cudaSuccess) return TQ_ERR_CUDA;
    return from_cuda(tq::launch_skinny(codes, scales, n, k, xrot, m, Y, yt, ldy, lay.plan, counters,
                                       reinterpret_cast<float *>(ws + lay.partial_off), true, (cudaStream_t)stream));
}

tq_status tq_gemm(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, const void *X, tq_dtype xt,
                  int64_t m, int64_t ldx, void *Y, tq_dtype yt, int64_t ldy, void *workspace, size_t ws_bytes,
                  void *stream) {
    tq_status st = check_gemm_common(codes, scales, n, k, m, Y, yt, ldy);
    if (st != TQ_OK || n == 0 || m == 0) return st;
    if (!valid_dtype(xt)) return TQ_ERR_DTYPE;
    if ((st = check_matrix_operand(X, ldx, k)) != TQ_OK) return st;
    GemmLayout lay;
    if ((st = gemm_layout(m, n, k, true, &lay)) != TQ_OK) return st;
    if (!workspace || !aligned(workspace, 256) || ws_bytes < lay.total) return TQ_ERR_WORKSPACE;
    char *ws = static_cast<char *>(workspace);
    auto *xrot = reinterpret_cast<uint16_t *>(ws + lay.xrot_off);
    auto *counters = reinterpret_cast<unsigned *>(ws + lay.counter_off);
    auto *partials = reinterpret_cast<float *>(ws + lay.partial_off);
    const size_t xsize = xt == TQ_F32 ? 4 : 2, ysize = yt == TQ_F32 ? 4 : 2;
    cudaStream_t s = (cudaStream_t)stream;
    for (int64_t i0 = 0; i0 < m; i0 += 32) {
        const int64_t ms = (m - i0) < 32 ? (m - i0) : 32;
        const char *Xs = static_cast<const char *>(X) + (size_t)i0 * (size_t)ldx * xsize;
        char *Ys = static_cast<char *>(Y) + (size_t)i0 * (size_t)ldy * ysize;
        cudaError_t e = tq::launch_prerotate(Xs, xt, ms, k, ldx, xrot, counters, lay.plan.tiles, s);
        if (e != cudaSuccess) return TQ_ERR_CUDA;
        e = tq::launch_skinny(codes, scales, n, k, xrot, ms, Ys, yt, ldy, lay.plan, counters, partials, true, s);
        if (e != cudaSuccess) return TQ_ERR_CUDA;
    }
    return TQ_OK;
}

tq_status tq_gemv(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, const void *x, tq_dtype xt,
                  void *y, tq_dtype yt, void *workspace, size_t ws_bytes, void *stream) {
    return tq_gemm(codes, scales, n, k, x, xt, 1, k, y, yt, n, workspace, ws_bytes, stream);
}

}  // extern "C"
