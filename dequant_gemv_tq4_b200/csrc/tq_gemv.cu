// tq_gemv.cu -- fused TQ4_1S dequant-GEMV / skinny GEMM (m <= 32) for sm_100a,
// over a group of up to eight matrices in one launch.
//
// Method: TQ4_1S page ("企业官网建设流程全解析", hotelren.com/news/5458160),
// section 解码速度：分硬件汇总: the activation is rotated once with the block
// transform, after which each weight contributes centroid(code) * scale * x_rot;
// no per-block inverse transform of the weights.
//
//   Y[i][r] = sum_b sum_h d[r][b][h] * sum_{e in half h} c(code[r][32b+e]) * xrot[i][32b+e]
//
// with xrot = H(s .* x)/32 in fp16 (the pre-rotation kernel) and c() the 16
// signed centroids in fp16.
//
// B200 design (the page's Metal kernel is prior art only):
//  * Work unit = 16 weight rows x one 128-column superblock: 1024 contiguous
//    code bytes + 256 contiguous scale bytes in the tile-major packed layout.
//    The units of all matrices in the group form one index space, split evenly
//    over every warp of a one-CTA-per-SM grid (stream-K style), so each warp
//    streams one contiguous stretch of memory.
//  * Each warp keeps a ring of kStages units in shared memory filled by
//    cp.async.bulk (TMA bulk copies, one lane issues, an mbarrier per stage
//    counts the bytes).  No registers are spent on loads in flight; waits are
//    bounded in time and report a timeout through a status word.
//  * The per-weight work is a 4-bit -> fp16 lookup.  A byte holds two codes, so
//    a 256-entry table of half2 pairs turns one byte into a ready tensor-core
//    operand.  The table lives in shared memory replicated per lane (entry v,
//    lane l at byte 256*v + 4*l): 32 lanes with arbitrary bytes hit 32 distinct
//    banks; one PRMT builds the address (lane*4 in byte 0, code byte in byte 1).
//  * The multiply-accumulate runs on the tensor pipe (mma.sync m16n8k16, f16 in,
//    f32 out): A = 16 weight rows x one 16-element half-block, B = the
//    pre-rotated activation fragment (X rows as the n dimension, 8 per mma,
//    NT n-tiles for m <= 8*NT).  One k16 step is exactly one half-block, so the
//    fp16 half-block scale multiplies the fp32 mma result before it joins the
//    accumulator.
//  * Tiles split across warps combine fixed-order partial sums: each
//    contributor writes its slot, the last to arrive (atomic counter, no
//    waiting) adds the slots in warp order.  Deterministic for a given GPU.
#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {

namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kStages = 6;
constexpr int kUnitCodeBytes = 1024;
constexpr int kUnitScaleBytes = 256;
constexpr int kUnitBytes = kUnitCodeBytes + kUnitScaleBytes;
constexpr int kLutBytes = 256 * 256;  // 256 entries x 256 B (32 lanes x 4 B used)
constexpr int kRingBytes = kWarps * kStages * kUnitBytes;
constexpr int kBarBytes = kWarps * kStages * 8;
constexpr int kSmemBytes = kLutBytes + kRingBytes + kBarBytes;
constexpr unsigned kStatusTimeout = 1u;
constexpr uint64_t kTimeoutNs = 1000000000ull;     // 1 s
constexpr uint64_t kDebugTimeoutNs = 5000000ull;   // 5 ms under fault injection

static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

__constant__ uint16_t c_mag_f16[8] = TQ_MAG_F16_INIT;

uint32_t g_debug_flags = 0;

struct DevProblem {
    const uint8_t *codes;
    const uint8_t *scales;
    const uint16_t *xrot;
    char *y;
    int64_t ldy;
    int64_t unit_begin;
    int64_t tile_begin;
    int n;
    int nsb;
};

struct GroupParams {
    DevProblem prob[kMaxProblems];
    int count;
    int m;
    int64_t units;
    int total_warps;
    float *partials;
    unsigned *counters;
    unsigned *status;
    uint64_t timeout_ns;
    int inject_skip;
};

// ---- PTX helpers ------------------------------------------------------------
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for phase `parity` of the barrier; false after `timeout_ns` (or 2^30 polls).
__device__ __noinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
    if (mbar_try(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t it = 0; it < (1u << 30); ++it) {
        if (mbar_try(bar, parity)) return true;
        if (global_ns() - t0 > timeout_ns) return false;
    }
    return false;
}

// One unit (1024 code bytes + 256 scale bytes) into a ring stage.
__device__ __forceinline__ void issue_unit(const GroupParams &P, int64_t v, uint32_t dst, uint32_t bar) {
    int q = 0;
    while (q + 1 < P.count && v >= P.prob[q + 1].unit_begin) ++q;
    const int64_t local = v - P.prob[q].unit_begin;
    const uint8_t *src_c = P.prob[q].codes + local * kUnitCodeBytes;
    const uint8_t *src_s = P.prob[q].scales + local * kUnitScaleBytes;
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(kUnitBytes) : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src_c), "r"(kUnitCodeBytes), "r"(bar)
                 : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     dst + kUnitCodeBytes),
                 "l"(src_s), "r"(kUnitScaleBytes), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ float h2f_lo(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w & 0xffffu))); }
__device__ __forceinline__ float h2f_hi(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w >> 16))); }

// Warp that owns unit x under the even split of `units` over `warps`.
__device__ __forceinline__ int owner_warp(int64_t x, int64_t units, int warps) {
    return (int)(((x + 1) * (int64_t)warps - 1) / units);
}

template <int NT, bool M1, int OT>
__global__ void __launch_bounds__(kThreads, 1) gemv_group_kernel(const __grid_constant__ GroupParams P) {
    extern __shared__ __align__(1024) uint8_t smem[];
    uint32_t *lut = reinterpret_cast<uint32_t *>(smem);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gw = blockIdx.x * kWarps + warp;
    const uint32_t smem_base = (uint32_t)__cvta_generic_to_shared(smem);
    const uint32_t ring = smem_base + kLutBytes + warp * (kStages * kUnitBytes);
    const uint32_t bars = smem_base + kLutBytes + kRingBytes + warp * (kStages * 8);
    const bool active = gw < P.total_warps;
    const int64_t U = P.units;
    const int64_t u0 = active ? (int64_t)gw * U / P.total_warps : 0;
    const int64_t u1 = active ? (int64_t)(gw + 1) * U / P.total_warps : 0;

    // ---- prologue: barriers, first bulk copies, lookup table -------------
    // (the packed weights never depend on the preceding grid, so the copies
    // start before the programmatic-dependency wait)
    if (active && lane == 0) {
        for (int i = 0; i < kStages; ++i) mbar_init(bars + 8 * i, 1);
        fence_mbar_init();
        for (int i = 0; i < kStages; ++i) {
            const int64_t v = u0 + i;
            if (v < u1 && !(P.inject_skip && gw == 0 && i == 1))
                issue_unit(P, v, ring + i * kUnitBytes, bars + 8 * i);
        }
    }
    for (int idx = threadIdx.x; idx < 256 * 32; idx += kThreads) {
        const int v = idx >> 5, l = idx & 31;
        const uint32_t lo = c_mag_f16[v & 7] | ((v & 8) ? 0x8000u : 0u);
        const uint32_t hi = c_mag_f16[(v >> 4) & 7] | ((v & 0x80) ? 0x8000u : 0u);
        lut[v * 64 + l] = lo | (hi << 16);
    }
    __syncthreads();
    grid_dependency_wait();  // pre-rotated activations and counters are ready
    if (!active) return;

    const int g = lane >> 2, t = lane & 3;
    const uint32_t lane4 = (uint32_t)lane * 4u;
    constexpr int kMcap = 8 * NT;

    int q = 0;
    while (q + 1 < P.count && u0 >= P.prob[q + 1].unit_begin) ++q;
    int nsb = P.prob[q].nsb;
    int64_t r;
    int sb;
    {
        const int64_t local = u0 - P.prob[q].unit_begin;
        r = local / nsb;
        sb = (int)(local % nsb);
    }
    int64_t prob_end = (q + 1 < P.count) ? P.prob[q + 1].unit_begin : U;

    float acc[NT][4];
#pragma unroll
    for (int a = 0; a < NT; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;

    int stage = 0;
    uint32_t parity = 0;
    const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
    for (int64_t u = u0; u < u1; ++u) {
        const uint32_t st = ring + stage * kUnitBytes, bar = bars + 8 * stage;
        const bool ok = mbar_wait_bounded(bar, parity, P.timeout_ns);
        if (!__all_sync(kFull, ok)) {
            // report, then let the copies still in flight land before leaving
            if (lane == 0) {
                atomicOr(P.status, kStatusTimeout);
                int s2 = stage;
                uint32_t p2 = parity;
                for (int64_t v = u + 1; v < u1 && v < u + kStages; ++v) {
                    if (++s2 == kStages) { s2 = 0; p2 ^= 1u; }
                    mbar_wait_bounded(bars + 8 * s2, p2, P.timeout_ns);
                }
            }
            __syncwarp();
            return;
        }
        const uint4 c0 = lds128(st + g * 64 + t * 16);
        const uint4 c1 = lds128(st + (g + 8) * 64 + t * 16);
        const uint4 s0 = lds128(st + kUnitCodeBytes + g * 16);
        const uint4 s1 = lds128(st + kUnitCodeBytes + (g + 8) * 16);
        __syncwarp();
        if (lane == 0 && u + kStages < u1) {
            fence_proxy_async();
            issue_unit(P, u + kStages, st, bar);
        }
        if (++stage == kStages) { stage = 0; parity ^= 1u; }

        const uint16_t *xr = P.prob[q].xrot;
        const uint32_t cw0[4] = {c0.x, c0.y, c0.z, c0.w};
        const uint32_t cw1[4] = {c1.x, c1.y, c1.z, c1.w};
        const uint32_t sw0[4] = {s0.x, s0.y, s0.z, s0.w};
        const uint32_t sw1[4] = {s1.x, s1.y, s1.z, s1.w};
#pragma unroll
        for (int j = 0; j < kSbBlocks; ++j) {
            uint4 xb[NT];
#pragma unroll
            for (int a = 0; a < NT; ++a) {
                const int xrow = 8 * a + g;
                xb[a] = (xrow < P.m) ? ldg_keep(xr + (((int64_t)xrow * nsb + sb) * kSbBlocks + j) * 32 + t * 8) : z4;
            }
            // code byte b of word cw: logical byte t + 4b of the block
            const uint32_t a00 = lds_u32(smem_base + prmt(cw0[j], lane4, 0x5504u));
            const uint32_t a01 = lds_u32(smem_base + prmt(cw1[j], lane4, 0x5504u));
            const uint32_t a02 = lds_u32(smem_base + prmt(cw0[j], lane4, 0x5514u));
            const uint32_t a03 = lds_u32(smem_base + prmt(cw1[j], lane4, 0x5514u));
            const uint32_t a10 = lds_u32(smem_base + prmt(cw0[j], lane4, 0x5524u));
            const uint32_t a11 = lds_u32(smem_base + prmt(cw1[j], lane4, 0x5524u));
            const uint32_t a12 = lds_u32(smem_base + prmt(cw0[j], lane4, 0x5534u));
            const uint32_t a13 = lds_u32(smem_base + prmt(cw1[j], lane4, 0x5534u));
            const float d0g = h2f_lo(sw0[j]), d1g = h2f_hi(sw0[j]);
            const float d0g8 = h2f_lo(sw1[j]), d1g8 = h2f_hi(sw1[j]);
#pragma unroll
            for (int a = 0; a < NT; ++a) {
                float d[4];
                mma_16816_zero(d, a00, a01, a02, a03, xb[a].x, xb[a].y);
                acc[a][0] = fmaf(d[0], d0g, acc[a][0]);
                acc[a][2] = fmaf(d[2], d0g8, acc[a][2]);
                if (!M1) {
                    acc[a][1] = fmaf(d[1], d0g, acc[a][1]);
                    acc[a][3] = fmaf(d[3], d0g8, acc[a][3]);
                }
                mma_16816_zero(d, a10, a11, a12, a13, xb[a].z, xb[a].w);
                acc[a][0] = fmaf(d[0], d1g, acc[a][0]);
                acc[a][2] = fmaf(d[2], d1g8, acc[a][2]);
                if (!M1) {
                    acc[a][1] = fmaf(d[1], d1g, acc[a][1]);
                    acc[a][3] = fmaf(d[3], d1g8, acc[a][3]);
                }
            }
        }

        // ---- end of a tile segment: write Y or combine partial sums --------
        if (sb == nsb - 1 || u + 1 == u1) {
            const DevProblem &pr = P.prob[q];
            const int64_t tile_lo = pr.unit_begin + r * nsb, tile_hi = tile_lo + nsb;
            const int64_t gt = pr.tile_begin + r;
            const int row_g = (int)(r * 16) + g, row_g8 = row_g + 8;
            if (u0 <= tile_lo && tile_hi <= u1) {
#pragma unroll
                for (int a = 0; a < NT; ++a)
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        if (M1 && (b & 1)) continue;
                        const int xrow = 8 * a + 2 * t + (b & 1);
                        const int wrow = (b & 2) ? row_g8 : row_g;
                        if (xrow < P.m && wrow < pr.n)
                            store1<OT>(pr.y + ((int64_t)xrow * pr.ldy + wrow) * ElemSize<OT>::value, acc[a][b]);
                    }
            } else {
                float *slot = P.partials + (gt + gw) * (int64_t)(16 * kMcap);
#pragma unroll
                for (int a = 0; a < NT; ++a)
#pragma unroll
                    for (int b = 0; b < 4; ++b) {
                        const int xrow = 8 * a + 2 * t + (b & 1);
                        const int wrow = g + ((b & 2) ? 8 : 0);
                        slot[xrow * 16 + wrow] = acc[a][b];
                    }
                __threadfence();
                __syncwarp();
                const int first = owner_warp(tile_lo, U, P.total_warps);
                const int last = owner_warp(tile_hi - 1, U, P.total_warps);
                unsigned arrived = 0;
                if (lane == 0) arrived = atomicAdd(P.counters + gt, 1u);
                arrived = __shfl_sync(kFull, arrived, 0);
                if (arrived == (unsigned)(last - first)) {
                    __threadfence();
                    for (int e = lane; e < 16 * P.m; e += 32) {
                        const int xrow = e >> 4, wl = e & 15;
                        float sum = 0.f;
                        for (int c = first; c <= last; ++c)
                            sum += __ldcg(P.partials + (gt + c) * (int64_t)(16 * kMcap) + xrow * 16 + wl);
                        const int wrow = (int)(r * 16) + wl;
                        if (wrow < pr.n)
                            store1<OT>(pr.y + ((int64_t)xrow * pr.ldy + wrow) * ElemSize<OT>::value, sum);
                    }
                    if (lane == 0) P.counters[gt] = 0u;
                }
            }
#pragma unroll
            for (int a = 0; a < NT; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
        }

        // ---- advance (superblock, tile, problem) ---------------------------
        if (++sb == nsb) {
            sb = 0;
            ++r;
        }
        if (u + 1 == prob_end && q + 1 < P.count) {
            ++q;
            nsb = P.prob[q].nsb;
            r = 0;
            sb = 0;
            prob_end = (q + 1 < P.count) ? P.prob[q + 1].unit_begin : U;
        }
    }
}

template <int NT, bool M1>
cudaError_t launch_nt(const GroupParams &prm, int dtype, int grid, bool programmatic, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = programmatic ? 1 : 0;
    cudaError_t err;
    switch (dtype) {
        case kF32:
            err = cudaFuncSetAttribute(gemv_group_kernel<NT, M1, kF32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
            if (err != cudaSuccess) return err;
            return cudaLaunchKernelEx(&cfg, gemv_group_kernel<NT, M1, kF32>, prm);
        case kBF16:
            err = cudaFuncSetAttribute(gemv_group_kernel<NT, M1, kBF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
            if (err != cudaSuccess) return err;
            return cudaLaunchKernelEx(&cfg, gemv_group_kernel<NT, M1, kBF16>, prm);
        case kF16:
            err = cudaFuncSetAttribute(gemv_group_kernel<NT, M1, kF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
            if (err != cudaSuccess) return err;
            return cudaLaunchKernelEx(&cfg, gemv_group_kernel<NT, M1, kF16>, prm);
        default:
            return cudaErrorInvalidValue;
    }
}

}  // namespace

void set_debug_flags(uint32_t flags) { g_debug_flags = flags; }

GroupPlan plan_group(const int64_t *n, const int64_t *k, int count, int64_t m, int sm_count) {
    GroupPlan pl = {};
    for (int i = 0; i < count; ++i) {
        pl.tiles += tiles(n[i]);
        pl.units += tiles(n[i]) * superblocks(k[i]);
    }
    int64_t want = (pl.units + kWarps - 1) / kWarps;  // at least one unit per warp
    if (want > sm_count) want = sm_count;
    if (want < 1) want = 1;
    pl.grid = (int)want;
    const int64_t warps = (int64_t)pl.grid * kWarps;
    pl.total_warps = (int)(pl.units < warps ? pl.units : warps);
    const int64_t mm = m < 1 ? 1 : (m > 32 ? 32 : m);
    pl.mcap = (int)(8 * ((mm + 7) / 8));
    pl.counter_bytes = round_up((size_t)pl.tiles * 4u, 256);
    pl.partial_bytes = round_up((size_t)(pl.tiles + pl.total_warps) * 16u * (size_t)pl.mcap * 4u, 256);
    return pl;
}

cudaError_t launch_group(const GemvProblem *probs, int count, int64_t m, int ydtype, const GroupPlan &plan,
                         unsigned *counters, float *partials, unsigned *status, bool programmatic,
                         cudaStream_t stream) {
    if (count < 1 || count > kMaxProblems) return cudaErrorInvalidValue;
    GroupParams prm = {};
    int64_t ub = 0, tb = 0;
    for (int i = 0; i < count; ++i) {
        DevProblem &d = prm.prob[i];
        d.codes = probs[i].codes;
        d.scales = reinterpret_cast<const uint8_t *>(probs[i].scales);
        d.xrot = probs[i].xrot;
        d.y = static_cast<char *>(probs[i].y);
        d.ldy = probs[i].ldy;
        d.unit_begin = ub;
        d.tile_begin = tb;
        d.n = (int)probs[i].n;
        d.nsb = (int)superblocks(probs[i].k);
        ub += tiles(probs[i].n) * d.nsb;
        tb += tiles(probs[i].n);
    }
    prm.count = count;
    prm.m = (int)m;
    prm.units = ub;
    prm.total_warps = plan.total_warps;
    prm.partials = partials;
    prm.counters = counters;
    prm.status = status;
    prm.inject_skip = (g_debug_flags & 1u) ? 1 : 0;
    prm.timeout_ns = prm.inject_skip ? kDebugTimeoutNs : kTimeoutNs;
    // the partial-slot stride is 16 * 8 * NT floats: NT must match plan.mcap
    const int nt = plan.mcap / 8;
    if (m == 1 && nt == 1) return launch_nt<1, true>(prm, ydtype, plan.grid, programmatic, stream);
    switch (nt) {
        case 1: return launch_nt<1, false>(prm, ydtype, plan.grid, programmatic, stream);
        case 2: return launch_nt<2, false>(prm, ydtype, plan.grid, programmatic, stream);
        case 3: return launch_nt<3, false>(prm, ydtype, plan.grid, programmatic, stream);
        case 4: return launch_nt<4, false>(prm, ydtype, plan.grid, programmatic, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace tq
