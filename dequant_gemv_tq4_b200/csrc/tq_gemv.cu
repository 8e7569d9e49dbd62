// tq_gemv.cu -- fused TQ4_1S dequant-GEMV / skinny GEMM (m <= 32) for sm_100a.
//
// Method: TQ4_1S page ("企业官网建设流程全解析", hotelren.com/news/5458160),
// section 解码速度：分硬件汇总: the activation is rotated once with the block
// transform, after which each weight contributes centroid(code) * scale * x_rot;
// no per-block inverse transform of the weights.
//
//   Y[i][r] = sum_b sum_h d[r][b][h] * sum_{e in half h} c(code[r][32b+e]) * xrot[i][32b+e]
//
// with xrot = H(s .* x)/32 in fp16 (tq_prerotate) and c() the 16 signed
// centroids in fp16.
//
// B200 design (the page's Metal kernel is prior art only):
//  * The per-weight work is a 4-bit -> fp16 lookup.  A byte holds two codes,
//    so a 256-entry table of half2 pairs turns one byte into a ready tensor-core
//    operand.  The table lives in shared memory replicated per lane (entry v,
//    lane l at byte 256*v + 4*l), so 32 lanes with arbitrary bytes hit 32
//    distinct banks; one PRMT builds the address (lane*4 in byte 0, code byte in
//    byte 1).  Per two weights: PRMT + LDS.
//  * The multiply-accumulate runs on the tensor pipe (mma.sync m16n8k16, f16
//    in, f32 out): A = 16 weight rows x one 16-element half-block, B = the
//    pre-rotated activation fragment (X rows as the n dimension, up to 8 per
//    mma, 4 n-tiles for m <= 32).  One k16 step is exactly one half-block, so
//    the fp16 half-block scale multiplies the fp32 mma result (FFMA) before it
//    joins the accumulator.
//  * Packed codes are read with 128-bit streaming loads (one per lane per
//    superblock and row), four superblocks in flight per warp.
//  * Stream-K style partition: the (16-row tile, superblock) units of the
//    matrix are split evenly over all warps of a one-CTA-per-SM grid.  A warp
//    whose range covers a whole tile writes Y; tiles shared by several warps
//    combine fixed-order partial sums: each contributor writes its slot, the
//    last to arrive (atomic counter, no waiting) adds the slots in warp order.
//    Results are deterministic for a given GPU.
#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {

namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kLutBytes = 256 * 256;  // 256 entries x 256 B (32 lanes x 4 B used)
constexpr int kPF = 2;                // superblocks in flight per warp (register budget: 128/thread)

__constant__ uint16_t c_mag_f16[8] = TQ_MAG_F16_INIT;

struct SkinnyParams {
    const uint8_t *codes;
    const uint8_t *scales;
    const uint16_t *xrot;
    char *y;
    float *partials;
    unsigned *counters;
    int64_t ldy;
    int64_t units;
    int n;
    int nsb;
    int m;
    int total_warps;
};

__device__ __forceinline__ float h2f_lo(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w & 0xffffu))); }
__device__ __forceinline__ float h2f_hi(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w >> 16))); }

// Warp that owns unit x under the even split of `units` over `warps`.
__device__ __forceinline__ int owner_warp(int64_t x, int64_t units, int warps) {
    return (int)(((x + 1) * (int64_t)warps - 1) / units);
}

template <int NT, bool M1, int OT>
__global__ void __launch_bounds__(kThreads, 1) skinny_kernel(const SkinnyParams p) {
    extern __shared__ __align__(1024) uint32_t lut[];

    // ---- prologue (overlaps the pre-rotation kernel under PDL) ------------
    for (int idx = threadIdx.x; idx < 256 * 32; idx += kThreads) {
        const int v = idx >> 5, l = idx & 31;
        const uint32_t lo = c_mag_f16[v & 7] | ((v & 8) ? 0x8000u : 0u);
        const uint32_t hi = c_mag_f16[(v >> 4) & 7] | ((v & 0x80) ? 0x8000u : 0u);
        lut[v * 64 + l] = lo | (hi << 16);
    }
    __syncthreads();
    grid_dependency_wait();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int gw = blockIdx.x * kWarps + warp;
    // total_warps <= units, so every participating warp owns >= 1 unit and the
    // contributors of a tile are exactly the warps owner(first)..owner(last)
    if (gw >= p.total_warps) return;
    const int64_t U = p.units;
    const int64_t u0 = (int64_t)gw * U / p.total_warps;
    const int64_t u1 = (int64_t)(gw + 1) * U / p.total_warps;
    const uint32_t lut_base = (uint32_t)__cvta_generic_to_shared(lut);
    const uint32_t lane4 = (uint32_t)lane * 4u;
    const int nsb = p.nsb;
    const int64_t row_code_bytes = (int64_t)nsb * kSbCodeBytes;
    const int64_t row_scale_bytes = (int64_t)nsb * kSbScaleBytes;
    constexpr int kMcap = 8 * NT;

    int64_t u = u0;
    while (u < u1) {
        const int64_t r = u / nsb;
        const int sb_begin = (int)(u % nsb);
        const int64_t sb_lim = (int64_t)sb_begin + (u1 - u);
        const int sb_end = (int)(sb_lim < nsb ? sb_lim : (int64_t)nsb);
        const int row_g = (int)(r * 16) + g, row_g8 = row_g + 8;
        const bool ok_g = row_g < p.n, ok_g8 = row_g8 < p.n;
        const uint8_t *cg = p.codes + (int64_t)row_g * row_code_bytes + 16 * t;
        const uint8_t *cg8 = p.codes + (int64_t)row_g8 * row_code_bytes + 16 * t;
        const uint8_t *sg = p.scales + (int64_t)row_g * row_scale_bytes;
        const uint8_t *sg8 = p.scales + (int64_t)row_g8 * row_scale_bytes;

        float acc[NT][4];
#pragma unroll
        for (int a = 0; a < NT; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;

        uint4 bc0[kPF], bc1[kPF], bs0[kPF], bs1[kPF];
        const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int i = 0; i < kPF; ++i) {
            const int s = sb_begin + i;
            const bool in = s < sb_end;
            bc0[i] = (in && ok_g) ? ldg_stream(cg + (int64_t)s * kSbCodeBytes) : z4;
            bc1[i] = (in && ok_g8) ? ldg_stream(cg8 + (int64_t)s * kSbCodeBytes) : z4;
            bs0[i] = (in && ok_g) ? ldg_stream(sg + (int64_t)s * kSbScaleBytes) : z4;
            bs1[i] = (in && ok_g8) ? ldg_stream(sg8 + (int64_t)s * kSbScaleBytes) : z4;
        }

        for (int base = sb_begin; base < sb_end; base += kPF) {
#pragma unroll
            for (int i = 0; i < kPF; ++i) {
                const int s = base + i;
                if (s < sb_end) {
                    const uint4 c0 = bc0[i], c1 = bc1[i], s0 = bs0[i], s1 = bs1[i];
                    // refill this stage with superblock s + kPF
                    const int sn = s + kPF;
                    const bool in = sn < sb_end;
                    bc0[i] = (in && ok_g) ? ldg_stream(cg + (int64_t)sn * kSbCodeBytes) : z4;
                    bc1[i] = (in && ok_g8) ? ldg_stream(cg8 + (int64_t)sn * kSbCodeBytes) : z4;
                    bs0[i] = (in && ok_g) ? ldg_stream(sg + (int64_t)sn * kSbScaleBytes) : z4;
                    bs1[i] = (in && ok_g8) ? ldg_stream(sg8 + (int64_t)sn * kSbScaleBytes) : z4;

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
                            xb[a] = (xrow < p.m)
                                        ? ldg_keep(p.xrot + (((int64_t)xrow * nsb + s) * kSbBlocks + j) * 32 + t * 8)
                                        : z4;
                        }
                        // code byte b of word cw: logical byte t + 4b of the block
                        const uint32_t a00 = lds_u32(lut_base + prmt(cw0[j], lane4, 0x5504u));
                        const uint32_t a01 = lds_u32(lut_base + prmt(cw1[j], lane4, 0x5504u));
                        const uint32_t a02 = lds_u32(lut_base + prmt(cw0[j], lane4, 0x5514u));
                        const uint32_t a03 = lds_u32(lut_base + prmt(cw1[j], lane4, 0x5514u));
                        const uint32_t a10 = lds_u32(lut_base + prmt(cw0[j], lane4, 0x5524u));
                        const uint32_t a11 = lds_u32(lut_base + prmt(cw1[j], lane4, 0x5524u));
                        const uint32_t a12 = lds_u32(lut_base + prmt(cw0[j], lane4, 0x5534u));
                        const uint32_t a13 = lds_u32(lut_base + prmt(cw1[j], lane4, 0x5534u));
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
                }
            }
        }

        // ---- flush the tile segment ---------------------------------------
        const int64_t tile_lo = r * nsb, tile_hi = (r + 1) * nsb;
        if (u0 <= tile_lo && tile_hi <= u1) {
#pragma unroll
            for (int a = 0; a < NT; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    if (M1 && (b & 1)) continue;
                    const int xrow = 8 * a + 2 * t + (b & 1);
                    const int wrow = (b & 2) ? row_g8 : row_g;
                    if (xrow < p.m && wrow < p.n)
                        store1<OT>(p.y + ((int64_t)xrow * p.ldy + wrow) * ElemSize<OT>::value, acc[a][b]);
                }
        } else {
            float *slot = p.partials + (r + gw) * (int64_t)(16 * kMcap);
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
            const int first = owner_warp(tile_lo, U, p.total_warps);
            const int last = owner_warp(tile_hi - 1, U, p.total_warps);
            unsigned arrived = 0;
            if (lane == 0) arrived = atomicAdd(p.counters + r, 1u);
            arrived = __shfl_sync(kFull, arrived, 0);
            if (arrived == (unsigned)(last - first)) {
                __threadfence();
                for (int e = lane; e < 16 * p.m; e += 32) {
                    const int xrow = e >> 4, wl = e & 15;
                    float sum = 0.f;
                    for (int c = first; c <= last; ++c)
                        sum += __ldcg(p.partials + (r + c) * (int64_t)(16 * kMcap) + xrow * 16 + wl);
                    const int wrow = (int)(r * 16) + wl;
                    if (wrow < p.n) store1<OT>(p.y + ((int64_t)xrow * p.ldy + wrow) * ElemSize<OT>::value, sum);
                }
                if (lane == 0) p.counters[r] = 0u;
            }
        }
        u += sb_end - sb_begin;
    }
}

template <int NT, bool M1>
cudaError_t launch_nt(const SkinnyParams &prm, int dtype, int grid, bool programmatic, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kLutBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = programmatic ? 1 : 0;
    cudaError_t err;
    switch (dtype) {
        case kF32:
            err = cudaFuncSetAttribute(skinny_kernel<NT, M1, kF32>, cudaFuncAttributeMaxDynamicSharedMemorySize, kLutBytes);
            if (err != cudaSuccess) return err;
            return cudaLaunchKernelEx(&cfg, skinny_kernel<NT, M1, kF32>, prm);
        case kBF16:
            err = cudaFuncSetAttribute(skinny_kernel<NT, M1, kBF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, kLutBytes);
            if (err != cudaSuccess) return err;
            return cudaLaunchKernelEx(&cfg, skinny_kernel<NT, M1, kBF16>, prm);
        case kF16:
            err = cudaFuncSetAttribute(skinny_kernel<NT, M1, kF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, kLutBytes);
            if (err != cudaSuccess) return err;
            return cudaLaunchKernelEx(&cfg, skinny_kernel<NT, M1, kF16>, prm);
        default:
            return cudaErrorInvalidValue;
    }
}

}  // namespace

SkinnyPlan plan_skinny(int64_t m, int64_t n, int64_t k, int sm_count) {
    SkinnyPlan pl;
    pl.tiles = (n + 15) / 16;
    pl.units = pl.tiles * superblocks(k);
    int64_t want = (pl.units + kWarps - 1) / kWarps;  // at least one unit per warp
    if (want > sm_count) want = sm_count;
    if (want < 1) want = 1;
    pl.grid = (int)want;
    pl.total_warps = (int)(pl.units < (int64_t)pl.grid * kWarps ? pl.units : (int64_t)pl.grid * kWarps);
    const int64_t mm = m < 1 ? 1 : (m > 32 ? 32 : m);
    pl.mcap = (int)(8 * ((mm + 7) / 8));
    pl.counter_bytes = round_up((size_t)pl.tiles * 4u, 256);
    pl.partial_bytes = round_up((size_t)(pl.tiles + pl.total_warps) * 16u * (size_t)pl.mcap * 4u, 256);
    return pl;
}

cudaError_t launch_skinny(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, const uint16_t *xrot,
                          int64_t m, void *Y, int dtype, int64_t ldy, const SkinnyPlan &plan, unsigned *counters,
                          float *partials, bool programmatic, cudaStream_t stream) {
    SkinnyParams prm;
    prm.codes = codes;
    prm.scales = reinterpret_cast<const uint8_t *>(scales);
    prm.xrot = xrot;
    prm.y = static_cast<char *>(Y);
    prm.partials = partials;
    prm.counters = counters;
    prm.ldy = ldy;
    prm.units = plan.units;
    prm.n = (int)n;
    prm.nsb = (int)superblocks(k);
    prm.m = (int)m;
    prm.total_warps = plan.total_warps;
    // the partial-slot stride is 16 * 8 * NT floats: NT must match plan.mcap
    const int nt = plan.mcap / 8;
    if (m == 1 && nt == 1) return launch_nt<1, true>(prm, dtype, plan.grid, programmatic, stream);
    switch (nt) {
        case 1: return launch_nt<1, false>(prm, dtype, plan.grid, programmatic, stream);
        case 2: return launch_nt<2, false>(prm, dtype, plan.grid, programmatic, stream);
        case 3: return launch_nt<3, false>(prm, dtype, plan.grid, programmatic, stream);
        case 4: return launch_nt<4, false>(prm, dtype, plan.grid, programmatic, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace tq
