// tq_codec.cu -- TQ4_1S quantise, dequantise and activation pre-rotation.
//
// Method: TQ4_1S page ("企业官网建设流程全解析", hotelren.com/news/5458160),
// paragraph 格式原理 items 1-3 and the paragraph after them; section
// 解码速度：分硬件汇总 for the pre-rotated activation.
//
// Thread layout used by all three kernels: one warp owns one 128-column
// superblock (four 32-element blocks) of one row per step; lane = 8*j + p
// holds elements 4p..4p+3 of block j.  The 32-point transform runs as two
// butterfly stages in registers (h = 1, 2) and three across lanes (h = 4, 8,
// 16 via shfl_xor 1, 2, 4), in the codec's stage order, so every fp32 result
// equals the sequential definition bit for bit.
#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {

namespace {

constexpr int kCodecWarps = 8;
constexpr int kCodecThreads = kCodecWarps * 32;

__constant__ uint32_t c_thr_bits[7] = TQ_THR_F32_INIT;
__constant__ uint32_t c_mag_bits[8] = TQ_MAG_F32_INIT;

// Full 32-point transform of the warp's four blocks (see file comment).
__device__ __forceinline__ void fwht32_warp(float (&v)[4], int p) {
    butterfly_local4(v);
#pragma unroll
    for (int s = 0; s < 3; ++s) {
        const int x = 1 << s;
        const bool upper = (p & x) != 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = butterfly_xlane(v[i], x, upper);
    }
}

// Index of a row's 64-byte code slot (and 16-byte scale slot) for superblock
// sb in the tile-major layout [tile][sb][16 rows].
__device__ __forceinline__ size_t unit_row(int row, int sb, int nsb) {
    return ((size_t)(row >> 4) * nsb + sb) * 16 + (row & 15);
}

// #{j : a > t_j} for ascending t (binary search over the seven thresholds).
__device__ __forceinline__ uint32_t magnitude_rank(float a, const float (&t)[7]) {
    const bool b2 = a > t[3];
    const float tm = b2 ? t[5] : t[1];
    const bool b1 = a > tm;
    const float tl = b2 ? (b1 ? t[6] : t[4]) : (b1 ? t[2] : t[0]);
    const bool b0 = a > tl;
    return (b2 ? 4u : 0u) | (b1 ? 2u : 0u) | (b0 ? 1u : 0u);
}

// -------------------------------------------------------------------------
// Quantise.  grid.x = superblock column, grid.y * 8 warps stride the rows.
// -------------------------------------------------------------------------
template <int DT>
__global__ void __launch_bounds__(kCodecThreads) quantize_kernel(const char *__restrict__ w, int64_t ldw, int n,
                                                                   int nb, int nsb, uint32_t *__restrict__ codes,
                                                                   uint32_t *__restrict__ scales) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int j = lane >> 3, p = lane & 7;
    const int sb = blockIdx.x;
    const bool valid = sb * kSbBlocks + j < nb;
    const uint32_t col0 = (uint32_t)sb * kSbElems + 32u * j + 4u * p;

    uint32_t smask[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) smask[i] = sign_mask(col0 + i);
    float thr[7];
#pragma unroll
    for (int i = 0; i < 7; ++i) thr[i] = __uint_as_float(c_thr_bits[i]);

    // code gather for the packed store: output word o = 4*tw + jw holds logical
    // bytes tw, tw+4, tw+8, tw+12 of block jw; logical byte L comes from lane
    // 8*jw + L/2 (low or high byte of its 16-bit code group).
    const int o = lane & 15, tw = o >> 2, jw = o & 3;
    const int byte_shift = 8 * (tw & 1);

    const int rows_padded = (n + 15) & ~15;  // rows past n are written as zeros
    for (int row = blockIdx.y * kCodecWarps + warp; row < rows_padded; row += gridDim.y * kCodecWarps) {
        float v[4] = {0.f, 0.f, 0.f, 0.f};
        if (valid && row < n) load4<DT>(w + ((int64_t)row * ldw + col0) * ElemSize<DT>::value, v);
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = flip(v[i], smask[i]);
        fwht32_warp(v, p);

        // half-block scale: adjacent pairwise tree of the 16 squares
        float q0 = __fmul_rn(v[0], v[0]), q1 = __fmul_rn(v[1], v[1]);
        float q2 = __fmul_rn(v[2], v[2]), q3 = __fmul_rn(v[3], v[3]);
        float s = __fadd_rn(__fadd_rn(q0, q1), __fadd_rn(q2, q3));
        s = __fadd_rn(s, __shfl_xor_sync(kFull, s, 1));
        s = __fadd_rn(s, __shfl_xor_sync(kFull, s, 2));
        const __half hd = __float2half_rn(__fsqrt_rn(__fmul_rn(s, 0.0625f)));
        const float D = __half2float(hd);
        float t[7];
#pragma unroll
        for (int i = 0; i < 7; ++i) t[i] = __fmul_rn(thr[i], D);

        uint32_t c16 = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t code = (v[i] < 0.0f ? 8u : 0u) | magnitude_rank(fabsf(v[i]), t);
            c16 |= code << (4 * i);
        }

        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t src = __shfl_sync(kFull, c16, 8 * jw + 2 * i + (tw >> 1));
            word |= ((src >> byte_shift) & 0xffu) << (8 * i);
        }
        const size_t sb_index = unit_row(row, sb, nsb);
        if (lane < 16) codes[sb_index * 16 + o] = word;

        const uint32_t hbits = __half_as_ushort(hd);
        const uint32_t hbits_hi = __shfl_xor_sync(kFull, hbits, 4);
        if (p == 0) scales[sb_index * 4 + j] = hbits | (hbits_hi << 16);
    }
}

// -------------------------------------------------------------------------
// Dequantise: w~ = s .* (H c) / 32, fp32, rounded to the output dtype.
// -------------------------------------------------------------------------
template <int DT>
__global__ void __launch_bounds__(kCodecThreads) dequantize_kernel(const uint32_t *__restrict__ codes,
                                                                     const uint32_t *__restrict__ scales, int n,
                                                                     int nb, int nsb, char *__restrict__ out,
                                                                     int64_t ldo) {
    __shared__ float smag[8];
    if (threadIdx.x < 8) smag[threadIdx.x] = __uint_as_float(c_mag_bits[threadIdx.x]);
    __syncthreads();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int j = lane >> 3, p = lane & 7;
    const int sb = blockIdx.x;
    const bool valid = sb * kSbBlocks + j < nb;
    const uint32_t col0 = (uint32_t)sb * kSbElems + 32u * j + 4u * p;
    uint32_t smask[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) smask[i] = sign_mask(col0 + i);

    // logical bytes 2p and 2p+1 of block j live in words 4*((2p)%4)+j and
    // 4*((2p+1)%4)+j, byte p/2
    const int src0 = 4 * ((2 * p) & 3) + j, src1 = 4 * ((2 * p + 1) & 3) + j;
    const int bsh = 8 * (p >> 1);
    const int half = p >> 2;

    for (int row = blockIdx.y * kCodecWarps + warp; row < n; row += gridDim.y * kCodecWarps) {
        const size_t sb_index = unit_row(row, sb, nsb);
        const uint32_t cw = __ldg(codes + sb_index * 16 + (lane & 15));
        const uint32_t sw = __ldg(scales + sb_index * 4 + j);
        const uint32_t b0 = (__shfl_sync(kFull, cw, src0) >> bsh) & 0xffu;
        const uint32_t b1 = (__shfl_sync(kFull, cw, src1) >> bsh) & 0xffu;
        const uint32_t code[4] = {b0 & 15u, b0 >> 4, b1 & 15u, b1 >> 4};
        const float D = __half2float(__ushort_as_half((unsigned short)(half ? (sw >> 16) : (sw & 0xffffu))));
        float v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float c = __fmul_rn(smag[code[i] & 7u], D);
            v[i] = (code[i] & 8u) ? -c : c;
        }
        fwht32_warp(v, p);
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = flip(__fmul_rn(v[i], 0.03125f), smask[i]);
        if (valid) store4<DT>(out + ((int64_t)row * ldo + col0) * ElemSize<DT>::value, v);
    }
}

// -------------------------------------------------------------------------
// Pre-rotation of activations into the fused kernel's fragment order:
// element e of a block goes to slot t*8 + q with t = (e%8)/2, q = 2*(e/8) + e%2.
// Handles a list of inputs (one warp per (input, row, superblock)) and zeroes
// the split-K arrival counters of the product that follows.
// -------------------------------------------------------------------------
template <int DT>
__global__ void __launch_bounds__(kCodecThreads) prerotate_kernel(const __grid_constant__ RotParams prm) {
    grid_dependents_launch();
    const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (int64_t i = gtid; i < prm.counters_count; i += (int64_t)gridDim.x * blockDim.x) prm.counters[i] = 0u;

    const int lane = threadIdx.x & 31;
    const int j = lane >> 3, p = lane & 7;
    const int64_t unit = (int64_t)blockIdx.x * kCodecWarps + (threadIdx.x >> 5);
    if (unit >= prm.units) return;
    int q = 0;
    while (q + 1 < prm.count && unit >= prm.in[q + 1].unit_begin) ++q;
    const RotInput &in = prm.in[q];
    const int64_t local = unit - in.unit_begin;
    const int row = (int)(local / in.nsb), sb = (int)(local % in.nsb);
    const bool valid = sb * kSbBlocks + j < in.nb;
    const uint32_t col0 = (uint32_t)sb * kSbElems + 32u * j + 4u * p;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (valid) load4<DT>(in.x + ((int64_t)row * in.ldx + col0) * ElemSize<DT>::value, v);
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = flip(v[i], sign_mask(col0 + i));
    fwht32_warp(v, p);
    const __half2 lo = __floats2half2_rn(__fmul_rn(v[0], 0.03125f), __fmul_rn(v[1], 0.03125f));
    const __half2 hi = __floats2half2_rn(__fmul_rn(v[2], 0.03125f), __fmul_rn(v[3], 0.03125f));
    // elements 4p, 4p+1 -> t = 2(p&1), q = 2(p>>1) + {0,1}; 4p+2, 4p+3 -> t + 1
    const size_t blk_words = ((size_t)local * kSbBlocks + j) * 16;  // 32 halves per block
    const int t0 = 2 * (p & 1), q0 = 2 * (p >> 1);
    in.xrot[blk_words + (t0 * 8 + q0) / 2] = *reinterpret_cast<const uint32_t *>(&lo);
    in.xrot[blk_words + ((t0 + 1) * 8 + q0) / 2] = *reinterpret_cast<const uint32_t *>(&hi);
}

int rows_grid(int64_t n, int64_t nsb, int sm_count) {
    // aim for ~8 resident CTAs per SM in total, at least one warp-row per CTA
    int64_t target = (int64_t)sm_count * 8;
    int64_t gy = (target + nsb - 1) / nsb;
    int64_t max_gy = (((n + 15) & ~(int64_t)15) + kCodecWarps - 1) / kCodecWarps;
    if (gy > max_gy) gy = max_gy;
    if (gy > 65535) gy = 65535;
    if (gy < 1) gy = 1;
    return (int)gy;
}

}  // namespace

cudaError_t launch_quantize(const void *w, int dtype, int64_t n, int64_t k, int64_t ldw, uint8_t *codes,
                            uint16_t *scales, cudaStream_t stream) {
    DeviceInfo di;
    cudaError_t err = device_info(&di);
    if (err != cudaSuccess) return err;
    const int64_t nb = k / 32, nsb = superblocks(k);
    dim3 grid((unsigned)nsb, (unsigned)rows_grid(n, nsb, di.sm_count));
    auto *c = reinterpret_cast<uint32_t *>(codes);
    auto *s = reinterpret_cast<uint32_t *>(scales);
    const char *wp = static_cast<const char *>(w);
    switch (dtype) {
        case kF32: quantize_kernel<kF32><<<grid, kCodecThreads, 0, stream>>>(wp, ldw, (int)n, (int)nb, (int)nsb, c, s); break;
        case kBF16: quantize_kernel<kBF16><<<grid, kCodecThreads, 0, stream>>>(wp, ldw, (int)n, (int)nb, (int)nsb, c, s); break;
        case kF16: quantize_kernel<kF16><<<grid, kCodecThreads, 0, stream>>>(wp, ldw, (int)n, (int)nb, (int)nsb, c, s); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, void *w_out,
                              int dtype, int64_t ldo, cudaStream_t stream) {
    DeviceInfo di;
    cudaError_t err = device_info(&di);
    if (err != cudaSuccess) return err;
    const int64_t nb = k / 32, nsb = superblocks(k);
    dim3 grid((unsigned)nsb, (unsigned)rows_grid(n, nsb, di.sm_count));
    auto *c = reinterpret_cast<const uint32_t *>(codes);
    auto *s = reinterpret_cast<const uint32_t *>(scales);
    char *o = static_cast<char *>(w_out);
    switch (dtype) {
        case kF32: dequantize_kernel<kF32><<<grid, kCodecThreads, 0, stream>>>(c, s, (int)n, (int)nb, (int)nsb, o, ldo); break;
        case kBF16: dequantize_kernel<kBF16><<<grid, kCodecThreads, 0, stream>>>(c, s, (int)n, (int)nb, (int)nsb, o, ldo); break;
        case kF16: dequantize_kernel<kF16><<<grid, kCodecThreads, 0, stream>>>(c, s, (int)n, (int)nb, (int)nsb, o, ldo); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_prerotate(const RotJob *jobs, int count, int dtype, int64_t m, unsigned *counters,
                             int64_t counters_count, cudaStream_t stream) {
    if (count < 1 || count > kMaxInputs) return cudaErrorInvalidValue;
    RotParams prm = {};
    int64_t units = 0;
    for (int i = 0; i < count; ++i) {
        RotInput &in = prm.in[i];
        in.x = static_cast<const char *>(jobs[i].x);
        in.xrot = reinterpret_cast<uint32_t *>(jobs[i].xrot);
        in.ldx = jobs[i].ldx;
        in.unit_begin = units;
        in.nb = (int)(jobs[i].k / 32);
        in.nsb = (int)superblocks(jobs[i].k);
        units += m * in.nsb;
    }
    prm.count = count;
    prm.units = units;
    prm.counters = counters;
    prm.counters_count = counters ? counters_count : 0;
    int64_t grid = (units + kCodecWarps - 1) / kCodecWarps;
    if (grid < 1) grid = 1;
    switch (dtype) {
        case kF32: prerotate_kernel<kF32><<<(unsigned)grid, kCodecThreads, 0, stream>>>(prm); break;
        case kBF16: prerotate_kernel<kBF16><<<(unsigned)grid, kCodecThreads, 0, stream>>>(prm); break;
        case kF16: prerotate_kernel<kF16><<<(unsigned)grid, kCodecThreads, 0, stream>>>(prm); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace tq
