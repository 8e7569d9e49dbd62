// tq_nvfp4.cu -- NVFP4 comparison codec: tensor amax, quantise, dequantise.
//
// NVFP4 is named by the llm-compressor page (ai-insight.org/news/11771) and the
// llama.cpp quantizer page (bittide.aicompass.dev, "NVFP4 weight and input
// tensor scales"); neither gives a bit recipe, so the codec takes the plainest
// reading of the format:
//   g   = amax|W| / (6 * 448)                       fp32, per tensor
//   s_b = E4M3(amax_b / (6 g))                       per 16-element block
//   q   = E2M1(w / (E4M3value(s_b) * g))             per element, 0 if the scale is 0
// each quotient and product one IEEE fp32 operation, conversions round to
// nearest-even and saturate (cvt.rn.satfinite), zeros carry no sign.
// Storage reuses the TQ4_1S units: codes [T][NSB][16][64 B] with the same byte
// order (two 16-element blocks take the place of one 32-element block), and
// E4M3 scales [T][NSB][16 rows][8 blocks]; no rotation.
#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {

namespace {

constexpr int kNvWarps = 8;
constexpr int kNvThreads = kNvWarps * 32;

__device__ __forceinline__ size_t nv_unit_row(int row, int sb, int nsb) {
    return ((size_t)(row >> 4) * nsb + sb) * 16 + (row & 15);
}

// Two fp32 -> two E4M3 bytes: (hi << 8) | lo.
__device__ __forceinline__ uint32_t e4m3x2(float hi, float lo) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two fp32 -> one byte of E2M1 codes: (code(hi) << 4) | code(lo).
__device__ __forceinline__ uint32_t e2m1x2(float hi, float lo) {
    uint16_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u16.u8 %0, t;\n\t}"
        : "=h"(r)
        : "f"(hi), "f"(lo));
    return r;
}

// E4M3 byte pair -> two floats (.x from the low byte).
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t two) {
    uint32_t h;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((uint16_t)two));
    return __half22float2(*reinterpret_cast<const __half2 *>(&h));
}

// E2M1 code byte -> two floats (.x from the low nibble).
__device__ __forceinline__ float2 e2m1x2_to_float2(uint32_t byte) {
    uint32_t h;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(h) : "r"(byte));
    return __half22float2(*reinterpret_cast<const __half2 *>(&h));
}

// Clear the sign bit of every zero-magnitude nibble (a zero carries no sign).
__device__ __forceinline__ uint32_t unsign_zero_nibbles(uint32_t w) {
    const uint32_t mag = w & 0x77777777u;
    const uint32_t nz = (mag | (mag >> 1) | (mag >> 2)) & 0x11111111u;
    return mag | (w & (nz << 3));
}

template <int DT>
__device__ __forceinline__ void load32(const char *p, float (&v)[32]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float q[4];
        load4<DT>(p + (size_t)4 * i * ElemSize<DT>::value, q);
#pragma unroll
        for (int c = 0; c < 4; ++c) v[4 * i + c] = q[c];
    }
}

template <int DT>
__global__ void __launch_bounds__(kNvThreads) nvfp4_amax_kernel(const char *__restrict__ w, int64_t ldw, int n, int k,
                                                                 unsigned *__restrict__ amax_bits) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float m = 0.f;
    for (int row = blockIdx.x * kNvWarps + warp; row < n; row += gridDim.x * kNvWarps)
        for (int c = lane * 4; c < k; c += 128) {
            float v[4];
            load4<DT>(w + ((int64_t)row * ldw + c) * ElemSize<DT>::value, v);
#pragma unroll
            for (int i = 0; i < 4; ++i) m = fmaxf(m, fabsf(v[i]));
        }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
    if (lane == 0) atomicMax(amax_bits, __float_as_uint(m));  // non-negative floats order as integers
}

// One lane per 32-column pair of 16-element blocks; the warp walks rows.
template <int DT>
__global__ void __launch_bounds__(kNvThreads) nvfp4_quantize_kernel(const char *__restrict__ w, int64_t ldw, int n,
                                                                     int nb, int nsb,
                                                                     const unsigned *__restrict__ amax_bits,
                                                                     uint32_t *__restrict__ codes,
                                                                     uint16_t *__restrict__ scales,
                                                                     float *__restrict__ tensor_scale) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int blk = blockIdx.x * 32 + lane;  // 32-column pair index
    const bool exists = blk < nsb * kSbBlocks;
    const bool valid = blk < nb;
    const int sb = blk >> 2, j = blk & 3;
    const float amax = __uint_as_float(__ldg(amax_bits));
    const float g = __fdiv_rn(amax, 2688.0f);  // 6 * 448
    const float denom = __fmul_rn(6.0f, g);
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *tensor_scale = g;

    const int rows_padded = (n + 15) & ~15;
    for (int row = blockIdx.y * kNvWarps + warp; row < rows_padded; row += gridDim.y * kNvWarps) {
        float v[32];
        if (valid && row < n) {
            load32<DT>(w + ((int64_t)row * ldw + (int64_t)blk * 32) * ElemSize<DT>::value, v);
        } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = 0.f;
        }
        float am[2] = {0.f, 0.f};
#pragma unroll
        for (int e = 0; e < 32; ++e) am[e >> 4] = fmaxf(am[e >> 4], fabsf(v[e]));
        const float x0 = denom > 0.f ? __fdiv_rn(am[0], denom) : 0.f;
        const float x1 = denom > 0.f ? __fdiv_rn(am[1], denom) : 0.f;
        const uint32_t sbytes = e4m3x2(x1, x0);  // byte 0: block 2j, byte 1: block 2j+1
        const float2 sv = e4m3x2_to_float2(sbytes);
        const float scale[2] = {__fmul_rn(sv.x, g), __fmul_rn(sv.y, g)};
        uint32_t lw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t word = 0;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int e = 8 * i + 2 * b;  // logical byte 4i + b: elements e, e+1
                const float sc = scale[e >> 4];
                const float lo = sc > 0.f ? __fdiv_rn(v[e], sc) : 0.f;
                const float hi = sc > 0.f ? __fdiv_rn(v[e + 1], sc) : 0.f;
                word |= e2m1x2(hi, lo) << (8 * b);
            }
            lw[i] = unsign_zero_nibbles(word);
        }
        if (exists) {
            uint32_t sw[4];
            transpose4(lw, sw);
            const size_t slot = nv_unit_row(row, sb, nsb);
#pragma unroll
            for (int tt = 0; tt < 4; ++tt) codes[slot * 16 + 4 * tt + j] = sw[tt];
            scales[slot * 4 + j] = (uint16_t)sbytes;
        }
    }
}

template <int DT>
__global__ void __launch_bounds__(kNvThreads) nvfp4_dequantize_kernel(const uint32_t *__restrict__ codes,
                                                                       const uint16_t *__restrict__ scales,
                                                                       const float *__restrict__ tensor_scale, int n,
                                                                       int nb, int nsb, char *__restrict__ out,
                                                                       int64_t ldo) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int blk = blockIdx.x * 32 + lane;
    if (blk >= nb) return;
    const int sb = blk >> 2, j = blk & 3;
    const float g = __ldg(tensor_scale);
    for (int row = blockIdx.y * kNvWarps + warp; row < n; row += gridDim.y * kNvWarps) {
        const size_t slot = nv_unit_row(row, sb, nsb);
        uint32_t sw[4], lw[4];
#pragma unroll
        for (int tt = 0; tt < 4; ++tt) sw[tt] = __ldg(codes + slot * 16 + 4 * tt + j);
        transpose4(sw, lw);
        const float2 sv = e4m3x2_to_float2(__ldg(scales + slot * 4 + j));
        const float scale[2] = {__fmul_rn(sv.x, g), __fmul_rn(sv.y, g)};
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
            const float2 q = e2m1x2_to_float2((lw[e >> 3] >> (4 * (e & 7))) & 0xffu);
            v[e] = __fmul_rn(q.x, scale[e >> 4]);
            v[e + 1] = __fmul_rn(q.y, scale[e >> 4]);
        }
        char *o = out + ((int64_t)row * ldo + (int64_t)blk * 32) * ElemSize<DT>::value;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float q[4] = {v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]};
            store4<DT>(o + (size_t)4 * i * ElemSize<DT>::value, q);
        }
    }
}

int nv_rows_grid(int64_t n, int64_t segs, int sm_count) {
    int64_t target = (int64_t)sm_count * 4;
    int64_t gy = (target + segs - 1) / segs;
    int64_t max_gy = (((n + 15) & ~(int64_t)15) + kNvWarps - 1) / kNvWarps;
    if (gy > max_gy) gy = max_gy;
    if (gy > 65535) gy = 65535;
    if (gy < 1) gy = 1;
    return (int)gy;
}

}  // namespace

cudaError_t launch_nvfp4_amax(const void *w, int dtype, int64_t n, int64_t k, int64_t ldw, unsigned *amax_bits,
                              cudaStream_t stream) {
    DeviceInfo di;
    cudaError_t err = device_info(&di);
    if (err != cudaSuccess) return err;
    int64_t grid = (n + kNvWarps - 1) / kNvWarps;
    if (grid > (int64_t)di.sm_count * 8) grid = (int64_t)di.sm_count * 8;
    if (grid < 1) grid = 1;
    const char *wp = static_cast<const char *>(w);
    switch (dtype) {
        case kF32: nvfp4_amax_kernel<kF32><<<(unsigned)grid, kNvThreads, 0, stream>>>(wp, ldw, (int)n, (int)k, amax_bits); break;
        case kBF16: nvfp4_amax_kernel<kBF16><<<(unsigned)grid, kNvThreads, 0, stream>>>(wp, ldw, (int)n, (int)k, amax_bits); break;
        case kF16: nvfp4_amax_kernel<kF16><<<(unsigned)grid, kNvThreads, 0, stream>>>(wp, ldw, (int)n, (int)k, amax_bits); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_nvfp4_quantize(const void *w, int dtype, int64_t n, int64_t k, int64_t ldw,
                                  const unsigned *amax_bits, uint8_t *codes, uint8_t *scales, float *tensor_scale,
                                  cudaStream_t stream) {
    DeviceInfo di;
    cudaError_t err = device_info(&di);
    if (err != cudaSuccess) return err;
    const int64_t nb = k / 32, nsb = superblocks(k);
    const int64_t segs = (nsb * kSbBlocks + 31) / 32;
    dim3 grid((unsigned)segs, (unsigned)nv_rows_grid(n, segs, di.sm_count));
    const char *wp = static_cast<const char *>(w);
    auto *c = reinterpret_cast<uint32_t *>(codes);
    auto *s = reinterpret_cast<uint16_t *>(scales);
    switch (dtype) {
        case kF32: nvfp4_quantize_kernel<kF32><<<grid, kNvThreads, 0, stream>>>(wp, ldw, (int)n, (int)nb, (int)nsb, amax_bits, c, s, tensor_scale); break;
        case kBF16: nvfp4_quantize_kernel<kBF16><<<grid, kNvThreads, 0, stream>>>(wp, ldw, (int)n, (int)nb, (int)nsb, amax_bits, c, s, tensor_scale); break;
        case kF16: nvfp4_quantize_kernel<kF16><<<grid, kNvThreads, 0, stream>>>(wp, ldw, (int)n, (int)nb, (int)nsb, amax_bits, c, s, tensor_scale); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_nvfp4_dequantize(const uint8_t *codes, const uint8_t *scales, const float *tensor_scale,
                                    int64_t n, int64_t k, void *w_out, int dtype, int64_t ldo, cudaStream_t stream) {
    DeviceInfo di;
    cudaError_t err = device_info(&di);
    if (err != cudaSuccess) return err;
    const int64_t nb = k / 32, nsb = superblocks(k);
    const int64_t segs = (nb + 31) / 32;
    dim3 grid((unsigned)segs, (unsigned)nv_rows_grid(n, segs, di.sm_count));
    auto *c = reinterpret_cast<const uint32_t *>(codes);
    auto *s = reinterpret_cast<const uint16_t *>(scales);
    char *o = static_cast<char *>(w_out);
    switch (dtype) {
        case kF32: nvfp4_dequantize_kernel<kF32><<<grid, kNvThreads, 0, stream>>>(c, s, tensor_scale, (int)n, (int)nb, (int)nsb, o, ldo); break;
        case kBF16: nvfp4_dequantize_kernel<kBF16><<<grid, kNvThreads, 0, stream>>>(c, s, tensor_scale, (int)n, (int)nb, (int)nsb, o, ldo); break;
        case kF16: nvfp4_dequantize_kernel<kF16><<<grid, kNvThreads, 0, stream>>>(c, s, tensor_scale, (int)n, (int)nb, (int)nsb, o, ldo); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace tq
