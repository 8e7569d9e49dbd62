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

// Workspace of a fused-product call (m <= 32):
//   [0, 256)           header: status word (timeout flag of the last call),
//                      call tag (advanced by every call)
//   tensor-memory kernel:
//     counters         one call-tagged 64-bit counter per 128-row block
//     partial slots    2 * CTAs * mld * 128 fp32 partial sums of split row blocks
//   mma.sync kernel:
//     partial slots    (tiles + warps) * 16 * mcap tagged sums (8 bytes each)
//   pre-rotated inputs one area per distinct activation, in the layout of the
//                      kernel that runs
struct Layout {
    size_t partial_off, counter_off, xrot_off[tq::kMaxInputs], total;
    int inputs;
    bool tc;             // the tensor-memory kernel runs the product
    tq::GroupPlan plan;  // mma.sync kernel
    tq::TcPlan tplan;    // tensor-memory kernel
};

constexpr size_t kStatusBytes = 256;

tq_status make_layout(const int64_t *n, const int64_t *k, int count, const int64_t *input_k, int inputs, int64_t m,
                      Layout *lay, bool allow_tc) {
    tq::DeviceInfo di;
    if (tq::device_info(&di) != cudaSuccess) return TQ_ERR_CUDA;
    const int64_t ms = m > 32 ? 32 : (m < 1 ? 1 : m);
    lay->inputs = inputs;
    lay->tc = allow_tc && tq::use_tc(ms);
    size_t off;
    if (lay->tc) {
        lay->tplan = tq::plan_tc(n, k, count, ms, di.sm_count);
        if (lay->tplan.units >= ((int64_t)1 << 31)) return TQ_ERR_SHAPE;  // > 2^41 weights per call
        lay->counter_off = kStatusBytes;
        lay->partial_off = lay->counter_off + lay->tplan.counter_bytes;
        off = lay->partial_off + lay->tplan.partial_bytes;
        for (int i = 0; i < inputs; ++i) {
            lay->xrot_off[i] = off;
            off += tq::round_up(tq::tc_xrot_bytes(ms, input_k[i]), 256);
        }
    } else {
        lay->plan = tq::plan_group(n, k, count, ms, di.sm_count);
        if (lay->plan.units >= ((int64_t)1 << 31)) return TQ_ERR_SHAPE;  // > 2^42 weights per call
        lay->counter_off = 0;
        lay->partial_off = kStatusBytes;
        off = lay->partial_off + lay->plan.partial_bytes;
        for (int i = 0; i < inputs; ++i) {
            lay->xrot_off[i] = off;
            off += tq::round_up(tq_xrot_bytes(ms, input_k[i]), 256);
        }
    }
    lay->total = off;
    return TQ_OK;
}

// Bytes a product of these shapes needs whichever kernel runs it.
tq_status workspace_need(const int64_t *n, const int64_t *k, int count, const int64_t *input_k, int inputs, int64_t m,
                         size_t *need) {
    Layout a, b;
    tq_status st = make_layout(n, k, count, input_k, inputs, m, &a, false);
    if (st != TQ_OK) return st;
    st = make_layout(n, k, count, input_k, inputs, m, &b, true);
    if (st != TQ_OK) return st;
    *need = a.total > b.total ? a.total : b.total;
    return TQ_OK;
}

// Pre-rotation (which also clears the status word and advances the call tag)
// and product of a laid-out call: jobs[q] feeds the problems whose input is q.
cudaError_t run_layout(const Layout &lay, const tq::RotJob *jobs, const tq::GemvProblem *pbs, int count, int64_t m,
                       tq_dtype xt, tq_dtype yt, char *ws, cudaStream_t s) {
    unsigned *header = reinterpret_cast<unsigned *>(ws);
    if (lay.tc) {
        const int np = lay.tplan.npad;
        cudaError_t e = tq::launch_prerotate(jobs, lay.inputs, xt, m, header, s, true,
                                             np == 0 ? tq::kRotPlain : tq::kRotCore, np);
        if (e != cudaSuccess) return e;
        return tq::launch_tc(pbs, count, m, yt, lay.tplan, header,
                             reinterpret_cast<unsigned long long *>(ws + lay.counter_off),
                             reinterpret_cast<float *>(ws + lay.partial_off), true, s);
    }
    cudaError_t e = tq::launch_prerotate(jobs, lay.inputs, xt, m, header, s);
    if (e != cudaSuccess) return e;
    return tq::launch_group(pbs, count, m, yt, lay.plan, header, reinterpret_cast<uint64_t *>(ws + lay.partial_off),
                            true, s);
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
        case TQ_ERR_TIMEOUT: return "TQ_ERR_TIMEOUT: a kernel's bounded wait expired (see tq_workspace_status)";
    }
    return "unknown tq_status";
}

size_t tq_codes_bytes(int64_t n, int64_t k) {
    if (check_nk(n, k) != TQ_OK) return 0;
    return (size_t)tq::tiles(n) * (size_t)tq::superblocks(k) * 1024u;
}

size_t tq_scales_bytes(int64_t n, int64_t k) {
    if (check_nk(n, k) != TQ_OK) return 0;
    return (size_t)tq::tiles(n) * (size_t)tq::superblocks(k) * 256u;
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

tq_status tq_dequantize_batch(const tq_dequant_desc *descs, int count, tq_dtype ot, void *stream) {
    if (!descs) return TQ_ERR_INVALID_ARG;
    if (count < 1 || count > TQ_MAX_BATCH) return TQ_ERR_SHAPE;
    if (!valid_dtype(ot)) return TQ_ERR_DTYPE;
    tq::DequantJob jobs[TQ_MAX_BATCH];
    int rows = 0;  // descriptors with rows
    for (int i = 0; i < count; ++i) {
        const tq_dequant_desc &d = descs[i];
        tq_status st = check_nk(d.n, d.k);
        if (st != TQ_OK) return st;
        if (d.n == 0) continue;
        if ((st = check_planes(d.codes, d.scales)) != TQ_OK) return st;
        if ((st = check_matrix_operand(d.w_out, d.ldo, d.k)) != TQ_OK) return st;
        jobs[rows++] = {d.codes, d.scales, d.n, d.k, d.w_out, d.ldo};
    }
    if (rows == 0) return TQ_OK;  // nothing to launch
    return from_cuda(tq::launch_dequantize_batch(jobs, rows, ot, (cudaStream_t)stream));
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
    tq::RotJob job = {X, ldx, k, xrot};
    return from_cuda(tq::launch_prerotate(&job, 1, xt, m, nullptr, (cudaStream_t)stream));
}

// Products with more activation rows than the skinny kernel takes run on
// the tcgen05 prefill kernel.
constexpr int64_t kSkinnyMaxM = 32;

static size_t prefill_workspace(int64_t m, int64_t k) {
    return kStatusBytes + tq::prefill_xrot_bytes(m < 1 ? 1 : m, k);
}

size_t tq_gemm_workspace_bytes(int64_t m, int64_t n, int64_t k) {
    if (m < 0 || check_nk(n, k) != TQ_OK) return 0;
    if (m > kSkinnyMaxM) return prefill_workspace(m, k);
    size_t need = 0;
    if (workspace_need(&n, &k, 1, &k, 1, m, &need) != TQ_OK) return 0;
    return need;
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

static tq_status check_workspace(void *workspace, size_t ws_bytes, size_t need) {
    if (!workspace || !aligned(workspace, 256) || ws_bytes < need) return TQ_ERR_WORKSPACE;
    return TQ_OK;
}

static tq_status run_prefill(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, const void *X,
                             tq_dtype xt, int64_t m, int64_t ldx, void *Y, tq_dtype yt, int64_t ldy, void *workspace,
                             size_t ws_bytes, void *stream) {
    tq_status st;
    if ((st = check_workspace(workspace, ws_bytes, prefill_workspace(m, k))) != TQ_OK) return st;
    if ((m + 255) / 256 > 65535) return TQ_ERR_SHAPE;
    char *ws = static_cast<char *>(workspace);
    const cudaError_t e =
        tq::launch_prefill(codes, scales, n, k, X, xt, m, ldx, reinterpret_cast<uint16_t *>(ws + kStatusBytes), Y, yt,
                           ldy, reinterpret_cast<unsigned *>(ws), (cudaStream_t)stream);
    if (e == cudaErrorNotSupported) return TQ_ERR_UNSUPPORTED;
    return from_cuda(e);
}

tq_status tq_gemm_xrot(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, const uint16_t *xrot,
                       int64_t m, void *Y, tq_dtype yt, int64_t ldy, void *workspace, size_t ws_bytes, void *stream) {
    tq_status st = check_gemm_common(codes, scales, n, k, m, Y, yt, ldy);
    if (st != TQ_OK || n == 0 || m == 0) return st;
    if (m > 32) return TQ_ERR_SHAPE;
    if (!xrot) return TQ_ERR_INVALID_ARG;
    if (!aligned(xrot, 16)) return TQ_ERR_ALIGNMENT;
    Layout lay;  // the activation is in the mma.sync kernel's fragment order: that kernel runs
    if ((st = make_layout(&n, &k, 1, nullptr, 0, m, &lay, false)) != TQ_OK) return st;
    if ((st = check_workspace(workspace, ws_bytes, lay.total)) != TQ_OK) return st;
    char *ws = static_cast<char *>(workspace);
    cudaStream_t s = (cudaStream_t)stream;
    // clear the status word and advance the call tag (the pre-rotation does
    // this in the calls that rotate)
    if (tq::launch_prepare_header(reinterpret_cast<unsigned *>(ws), s) != cudaSuccess) return TQ_ERR_CUDA;
    tq::GemvProblem pb = {codes, scales, xrot, Y, ldy, n, k};
    return from_cuda(tq::launch_group(&pb, 1, m, yt, lay.plan, reinterpret_cast<unsigned *>(ws),
                                      reinterpret_cast<uint64_t *>(ws + lay.partial_off), true, s));
}

tq_status tq_gemm(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, const void *X, tq_dtype xt,
                  int64_t m, int64_t ldx, void *Y, tq_dtype yt, int64_t ldy, void *workspace, size_t ws_bytes,
                  void *stream) {
    tq_status st = check_gemm_common(codes, scales, n, k, m, Y, yt, ldy);
    if (st != TQ_OK || n == 0 || m == 0) return st;
    if (!valid_dtype(xt)) return TQ_ERR_DTYPE;
    if ((st = check_matrix_operand(X, ldx, k)) != TQ_OK) return st;
    if (m > kSkinnyMaxM) return run_prefill(codes, scales, n, k, X, xt, m, ldx, Y, yt, ldy, workspace, ws_bytes, stream);
    Layout lay;
    if ((st = make_layout(&n, &k, 1, &k, 1, m, &lay, true)) != TQ_OK) return st;
    if ((st = check_workspace(workspace, ws_bytes, lay.total)) != TQ_OK) return st;
    char *ws = static_cast<char *>(workspace);
    const tq::RotJob job = {X, ldx, k, reinterpret_cast<uint16_t *>(ws + lay.xrot_off[0])};
    const tq::GemvProblem pb = {codes, scales, job.xrot, Y, ldy, n, k};
    return from_cuda(run_layout(lay, &job, &pb, 1, m, xt, yt, ws, (cudaStream_t)stream));
}

tq_status tq_gemv(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, const void *x, tq_dtype xt,
                  void *y, tq_dtype yt, void *workspace, size_t ws_bytes, void *stream) {
    return tq_gemm(codes, scales, n, k, x, xt, 1, k, y, yt, n, workspace, ws_bytes, stream);
}

size_t tq_gemm_prefill_workspace_bytes(int64_t m, int64_t k) {
    if (m < 0 || check_nk(0, k) != TQ_OK) return 0;
    return prefill_workspace(m, k);
}

tq_status tq_gemm_prefill(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, const void *X,
                          tq_dtype xt, int64_t m, int64_t ldx, void *Y, tq_dtype yt, int64_t ldy, void *workspace,
                          size_t ws_bytes, void *stream) {
    tq_status st = check_gemm_common(codes, scales, n, k, m, Y, yt, ldy);
    if (st != TQ_OK || n == 0 || m == 0) return st;
    if (!valid_dtype(xt)) return TQ_ERR_DTYPE;
    if ((st = check_matrix_operand(X, ldx, k)) != TQ_OK) return st;
    return run_prefill(codes, scales, n, k, X, xt, m, ldx, Y, yt, ldy, workspace, ws_bytes, stream);
}

size_t tq_prefill_xrot_bytes(int64_t m, int64_t k) {
    if (m < 0 || check_nk(0, k) != TQ_OK) return 0;
    return (size_t)m * (size_t)k * 2u;
}

tq_status tq_prerotate_plain(const void *X, tq_dtype xt, int64_t m, int64_t k, int64_t ldx, uint16_t *xrot,
                             void *stream) {
    tq_status st = check_nk(m, k);
    if (st != TQ_OK) return st;
    if (!valid_dtype(xt)) return TQ_ERR_DTYPE;
    if (m == 0) return TQ_OK;
    if (m > TQ_MAX_N) return TQ_ERR_SHAPE;
    if ((st = check_matrix_operand(X, ldx, k)) != TQ_OK) return st;
    if (!xrot) return TQ_ERR_INVALID_ARG;
    if (!aligned(xrot, 16)) return TQ_ERR_ALIGNMENT;
    return from_cuda(tq::launch_prerotate_plain(X, xt, m, k, ldx, xrot, nullptr, (cudaStream_t)stream));
}

tq_status tq_gemm_prefill_xrot(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k,
                               const uint16_t *xrot, int64_t m, void *Y, tq_dtype yt, int64_t ldy, void *workspace,
                               size_t ws_bytes, void *stream) {
    tq_status st = check_gemm_common(codes, scales, n, k, m, Y, yt, ldy);
    if (st != TQ_OK || n == 0 || m == 0) return st;
    if (!xrot) return TQ_ERR_INVALID_ARG;
    if (!aligned(xrot, 16)) return TQ_ERR_ALIGNMENT;
    if ((m + 255) / 256 > 65535) return TQ_ERR_SHAPE;
    if ((st = check_workspace(workspace, ws_bytes, kStatusBytes)) != TQ_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned *header = static_cast<unsigned *>(workspace);
    if (tq::launch_prepare_header(header, s) != cudaSuccess) return TQ_ERR_CUDA;
    const cudaError_t e = tq::launch_prefill_product(codes, scales, n, k, xrot, m, Y, yt, ldy, header, s);
    if (e == cudaErrorNotSupported) return TQ_ERR_UNSUPPORTED;
    return from_cuda(e);
}

// ---- batch: several matrices, one pre-rotation per distinct input ----------
static tq_status batch_layout(const tq_gemm_desc *descs, int count, int64_t m, Layout *lay, int *input_of,
                              bool allow_tc) {
    int64_t n[tq::kMaxProblems], k[tq::kMaxProblems], ik[tq::kMaxInputs];
    int inputs = 0;
    for (int i = 0; i < count; ++i) {
        n[i] = descs[i].n;
        k[i] = descs[i].k;
        int found = -1;
        for (int j = 0; j < i; ++j)
            if (descs[j].X == descs[i].X && descs[j].k == descs[i].k && descs[j].ldx == descs[i].ldx) {
                found = input_of[j];
                break;
            }
        if (found < 0) {
            found = inputs;
            ik[inputs++] = descs[i].k;
        }
        input_of[i] = found;
    }
    return make_layout(n, k, count, ik, inputs, m, lay, allow_tc);
}

size_t tq_gemm_batch_workspace_bytes(const tq_gemm_desc *descs, int count, int64_t m) {
    if (!descs || count < 1 || count > TQ_MAX_BATCH || m < 0 || m > 32) return 0;
    for (int i = 0; i < count; ++i)
        if (check_nk(descs[i].n, descs[i].k) != TQ_OK) return 0;
    Layout a, b;
    int input_of[tq::kMaxProblems];
    if (batch_layout(descs, count, m, &a, input_of, false) != TQ_OK) return 0;
    if (batch_layout(descs, count, m, &b, input_of, true) != TQ_OK) return 0;
    return a.total > b.total ? a.total : b.total;
}

tq_status tq_gemm_batch(const tq_gemm_desc *descs, int count, int64_t m, tq_dtype xt, tq_dtype yt, void *workspace,
                        size_t ws_bytes, void *stream) {
    if (!descs) return TQ_ERR_INVALID_ARG;
    if (count < 1 || count > TQ_MAX_BATCH) return TQ_ERR_SHAPE;
    if (m < 0) return TQ_ERR_INVALID_ARG;
    if (m > 32) return TQ_ERR_SHAPE;
    if (!valid_dtype(xt) || !valid_dtype(yt)) return TQ_ERR_DTYPE;
    tq_status st;
    for (int i = 0; i < count; ++i) {
        const tq_gemm_desc &d = descs[i];
        if ((st = check_gemm_common(d.codes, d.scales, d.n, d.k, m, d.Y, yt, d.ldy)) != TQ_OK) return st;
        if (d.n == 0) return TQ_ERR_SHAPE;  /* every matrix of a batch must be non-empty */
        if (m > 0 && (st = check_matrix_operand(d.X, d.ldx, d.k)) != TQ_OK) return st;
    }
    if (m == 0) return TQ_OK;
    Layout lay;
    int input_of[tq::kMaxProblems];
    if ((st = batch_layout(descs, count, m, &lay, input_of, true)) != TQ_OK) return st;
    if ((st = check_workspace(workspace, ws_bytes, lay.total)) != TQ_OK) return st;
    char *ws = static_cast<char *>(workspace);
    tq::RotJob jobs[tq::kMaxInputs];
    tq::GemvProblem pbs[tq::kMaxProblems];
    for (int i = 0; i < count; ++i) {
        const int q = input_of[i];
        auto *xrot = reinterpret_cast<uint16_t *>(ws + lay.xrot_off[q]);
        jobs[q] = {descs[i].X, descs[i].ldx, descs[i].k, xrot};
        pbs[i] = {descs[i].codes, descs[i].scales, xrot, descs[i].Y, descs[i].ldy, descs[i].n, descs[i].k};
    }
    return from_cuda(run_layout(lay, jobs, pbs, count, m, xt, yt, ws, (cudaStream_t)stream));
}

// ---- NVFP4 comparison codec -------------------------------------------------
size_t tq_nvfp4_scales_bytes(int64_t n, int64_t k) {
    if (check_nk(n, k) != TQ_OK) return 0;
    return (size_t)tq::tiles(n) * (size_t)tq::superblocks(k) * 128u;
}

static tq_status check_nv_planes(const uint8_t *codes, const uint8_t *scales, const float *tensor_scale) {
    if (!codes || !scales || !tensor_scale) return TQ_ERR_INVALID_ARG;
    if (!aligned(codes, 16) || !aligned(scales, 16) || !aligned(tensor_scale, 16)) return TQ_ERR_ALIGNMENT;
    return TQ_OK;
}

tq_status tq_nvfp4_quantize(const void *w, tq_dtype wt, int64_t n, int64_t k, int64_t ldw, uint8_t *codes,
                            uint8_t *scales, float *tensor_scale, void *stream) {
    tq_status st = check_nk(n, k);
    if (st != TQ_OK) return st;
    if (!valid_dtype(wt)) return TQ_ERR_DTYPE;
    if (n == 0) return TQ_OK;
    if ((st = check_matrix_operand(w, ldw, k)) != TQ_OK) return st;
    if ((st = check_nv_planes(codes, scales, tensor_scale)) != TQ_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    // word 1 of the tensor block accumulates amax|W| (as non-negative float bits)
    unsigned *amax = reinterpret_cast<unsigned *>(tensor_scale) + 1;
    if (cudaMemsetAsync(amax, 0, sizeof(unsigned), s) != cudaSuccess) return TQ_ERR_CUDA;
    if (tq::launch_nvfp4_amax(w, wt, n, k, ldw, amax, s) != cudaSuccess) return TQ_ERR_CUDA;
    return from_cuda(tq::launch_nvfp4_quantize(w, wt, n, k, ldw, amax, codes, scales, tensor_scale, s));
}

tq_status tq_nvfp4_dequantize(const uint8_t *codes, const uint8_t *scales, const float *tensor_scale, int64_t n,
                              int64_t k, void *w_out, tq_dtype ot, int64_t ldo, void *stream) {
    tq_status st = check_nk(n, k);
    if (st != TQ_OK) return st;
    if (!valid_dtype(ot)) return TQ_ERR_DTYPE;
    if (n == 0) return TQ_OK;
    if ((st = check_nv_planes(codes, scales, tensor_scale)) != TQ_OK) return st;
    if ((st = check_matrix_operand(w_out, ldo, k)) != TQ_OK) return st;
    return from_cuda(
        tq::launch_nvfp4_dequantize(codes, scales, tensor_scale, n, k, w_out, ot, ldo, (cudaStream_t)stream));
}

size_t tq_nvfp4_gemm_batch_workspace_bytes(const tq_nvfp4_gemm_desc *descs, int count, int64_t m) {
    if (!descs || count < 1 || count > TQ_MAX_BATCH) return 0;
    tq_gemm_desc plain[TQ_MAX_BATCH];
    for (int i = 0; i < count; ++i)
        plain[i] = {descs[i].codes, nullptr, descs[i].n, descs[i].k, descs[i].X, descs[i].ldx, descs[i].Y,
                    descs[i].ldy};
    return tq_gemm_batch_workspace_bytes(plain, count, m);
}

tq_status tq_nvfp4_gemm_batch(const tq_nvfp4_gemm_desc *descs, int count, int64_t m, tq_dtype xt, tq_dtype yt,
                              void *workspace, size_t ws_bytes, void *stream) {
    if (!descs) return TQ_ERR_INVALID_ARG;
    if (count < 1 || count > TQ_MAX_BATCH) return TQ_ERR_SHAPE;
    if (m < 0) return TQ_ERR_INVALID_ARG;
    if (m > 32) return TQ_ERR_SHAPE;
    if (!valid_dtype(xt) || !valid_dtype(yt)) return TQ_ERR_DTYPE;
    tq_status st;
    tq_gemm_desc plain[TQ_MAX_BATCH];
    for (int i = 0; i < count; ++i) {
        const tq_nvfp4_gemm_desc &d = descs[i];
        // the scale plane of an NVFP4 matrix is bytes; the shared checks only look at pointers
        if ((st = check_gemm_common(d.codes, reinterpret_cast<const uint16_t *>(d.scales), d.n, d.k, m, d.Y, yt,
                                    d.ldy)) != TQ_OK)
            return st;
        if (d.n == 0) return TQ_ERR_SHAPE;
        if (!d.tensor_scale) return TQ_ERR_INVALID_ARG;
        if (!aligned(d.tensor_scale, 16)) return TQ_ERR_ALIGNMENT;
        if (m > 0 && (st = check_matrix_operand(d.X, d.ldx, d.k)) != TQ_OK) return st;
        plain[i] = {d.codes, nullptr, d.n, d.k, d.X, d.ldx, d.Y, d.ldy};
    }
    if (m == 0) return TQ_OK;
    Layout lay;
    int input_of[tq::kMaxProblems];
    if ((st = batch_layout(plain, count, m, &lay, input_of, false)) != TQ_OK) return st;
    if ((st = check_workspace(workspace, ws_bytes, lay.total)) != TQ_OK) return st;
    char *ws = static_cast<char *>(workspace);
    tq::RotJob jobs[tq::kMaxInputs];
    tq::GemvProblem pbs[tq::kMaxProblems];
    for (int i = 0; i < count; ++i) {
        const int q = input_of[i];
        auto *xf = reinterpret_cast<uint16_t *>(ws + lay.xrot_off[q]);
        jobs[q] = {descs[i].X, descs[i].ldx, descs[i].k, xf};
        pbs[i] = {descs[i].codes, reinterpret_cast<const uint16_t *>(descs[i].scales), xf, descs[i].Y,
                  descs[i].ldy, descs[i].n, descs[i].k, descs[i].tensor_scale};
    }
    cudaStream_t s = (cudaStream_t)stream;
    // no rotation: the activation is only converted to fp16 in fragment order
    cudaError_t e = tq::launch_prerotate(jobs, lay.inputs, xt, m, reinterpret_cast<unsigned *>(ws), s, false);
    if (e != cudaSuccess) return TQ_ERR_CUDA;
    e = tq::launch_group_nvfp4(pbs, count, m, yt, lay.plan, reinterpret_cast<unsigned *>(ws),
                               reinterpret_cast<uint64_t *>(ws + lay.partial_off), true, s);
    return from_cuda(e);
}

tq_status tq_nvfp4_gemm(const uint8_t *codes, const uint8_t *scales, const float *tensor_scale, int64_t n, int64_t k,
                        const void *X, tq_dtype xt, int64_t m, int64_t ldx, void *Y, tq_dtype yt, int64_t ldy,
                        void *workspace, size_t ws_bytes, void *stream) {
    if (m > 32) return TQ_ERR_SHAPE;
    if (n == 0 && check_nk(n, k) == TQ_OK && m >= 0) return TQ_OK;
    tq_nvfp4_gemm_desc d = {codes, scales, tensor_scale, n, k, X, ldx, Y, ldy};
    return tq_nvfp4_gemm_batch(&d, 1, m, xt, yt, workspace, ws_bytes, stream);
}

tq_status tq_workspace_status(void *workspace, int clear, void *stream) {
    if (!workspace) return TQ_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned word = 0;
    if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess) return TQ_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return TQ_ERR_CUDA;
    if (clear && word != 0) {
        if (cudaMemsetAsync(workspace, 0, sizeof(word), s) != cudaSuccess) return TQ_ERR_CUDA;
    }
    return word ? TQ_ERR_TIMEOUT : TQ_OK;
}

void tq_debug_set_flags(uint32_t flags) { tq::set_debug_flags(flags); }

}  // extern "C"

// ---------------------------------------------------------------------------
// GEMV for callers that cannot allocate device memory.
//
// Some callers have no way to obtain a workspace: code running inside a
// custom allocator or a memory-pool callback (where allocating would recurse),
// plugins handed only the tensors of one operation by a host framework, or
// processes whose device memory is entirely reserved up front.  For them the
// scratch of the fused GEMV (header: status word and call tag, partial sums,
// pre-rotated activation) lives in this fixed device array instead, sized
// TQ_STATIC_SCRATCH_BYTES, resident on every GPU that loads the library until
// the process exits.
// ---------------------------------------------------------------------------
namespace {

static __device__ __align__(256) unsigned char g_static_scratch[TQ_STATIC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
struct ScratchAddr {
    unsigned long long ctx_id;  // the context the address belongs to (0: none yet)
    void *ptr;
};
ScratchAddr g_scratch_addr[256];

using CtxGetCurrent = int (*)(void **);
using CtxGetId = int (*)(void *, unsigned long long *);

// Unique id of the calling thread's current context (cuCtxGetId through the
// runtime's driver entry point, no link to the driver library).  A device
// reset or another context on the same device yields a new id.
cudaError_t current_context_id(unsigned long long *id) {
    static std::once_flag once;
    static CtxGetCurrent get_current = nullptr;
    static CtxGetId get_id = nullptr;
    std::call_once(once, [] {
        void *a = nullptr, *b = nullptr;
        cudaDriverEntryPointQueryResult qa = cudaDriverEntryPointSymbolNotFound, qb = qa;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
            qa == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
            qb == cudaDriverEntryPointSuccess) {
            get_current = reinterpret_cast<CtxGetCurrent>(a);
            get_id = reinterpret_cast<CtxGetId>(b);
        }
    });
    if (!get_current || !get_id) return cudaErrorNotSupported;
    void *ctx = nullptr;
    if (get_current(&ctx) != 0 || !ctx) return cudaErrorDeviceUninitialized;
    return get_id(ctx, id) == 0 ? cudaSuccess : cudaErrorDeviceUninitialized;
}

// Device address of g_static_scratch in the current context.  In host code the
// array's name is only a host-side stand-in, so the address is asked from the
// runtime with the device current, once per context: the cache is keyed by
// the context's unique id, so a device reset (which reloads the module, and
// may place the array elsewhere) or a different context on the same device
// looks the address up again.
cudaError_t static_scratch_address(void **out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 256) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    unsigned long long id = 0;
    void *p = nullptr;
    if (current_context_id(&id) != cudaSuccess) {
        // no current context yet: the runtime creates the device's primary
        // context on its first call, here the address lookup itself
        if ((err = cudaGetSymbolAddress(&p, g_static_scratch)) != cudaSuccess) return err;
        if ((err = current_context_id(&id)) != cudaSuccess) return err;
        g_scratch_addr[dev] = {id, p};
    } else if (g_scratch_addr[dev].ctx_id != id || !g_scratch_addr[dev].ptr) {
        if ((err = cudaGetSymbolAddress(&p, g_static_scratch)) != cudaSuccess) return err;
        g_scratch_addr[dev] = {id, p};
    }
    *out = g_scratch_addr[dev].ptr;
    return cudaSuccess;
}

}  // namespace

extern "C" tq_status tq_gemv_static_scratch(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k,
                                            const void *x, tq_dtype xt, void *y, tq_dtype yt, void *stream) {
    tq_status st = check_gemm_common(codes, scales, n, k, 1, y, yt, n);
    if (st != TQ_OK || n == 0) return st;
    if (!valid_dtype(xt)) return TQ_ERR_DTYPE;
    if ((st = check_matrix_operand(x, k, k)) != TQ_OK) return st;
    Layout lay;
    if ((st = make_layout(&n, &k, 1, &k, 1, 1, &lay, true)) != TQ_OK) return st;
    if (lay.total > (size_t)TQ_STATIC_SCRATCH_BYTES) return TQ_ERR_SHAPE;  // does not fit the fixed scratch
    void *scratch = nullptr;
    if (static_scratch_address(&scratch) != cudaSuccess) return TQ_ERR_CUDA;
    char *ws = static_cast<char *>(scratch);
    const tq::RotJob job = {x, k, k, reinterpret_cast<uint16_t *>(ws + lay.xrot_off[0])};
    const tq::GemvProblem pb = {codes, scales, job.xrot, y, n, n, k};
    // the pre-rotation launch also clears the status word and advances the
    // call tag: the array keeps whatever the previous call left in it
    return from_cuda(run_layout(lay, &job, &pb, 1, 1, xt, yt, ws, (cudaStream_t)stream));
}

extern "C" tq_status tq_static_scratch_status(int clear, void *stream) {
    void *scratch = nullptr;
    if (static_scratch_address(&scratch) != cudaSuccess) return TQ_ERR_CUDA;
    return tq_workspace_status(scratch, clear, stream);
}
