// tq_device.cuh -- device-side building blocks shared by the TQ4_1S kernels.
//
// Method: TQ4_1S page ("企业官网建设流程全解析", hotelren.com/news/5458160),
// paragraph 格式原理 (sign flip + 32-point Walsh-Hadamard rotation per block,
// 16 Lloyd-Max centroids, two half-block scales) and section 解码速度：分硬件汇总
// (the activation is pre-rotated once; decode is centroid lookup x scale).
//
// Floating-point rule for everything that decides a code or a scale: one
// IEEE fp32 operation per step, round-to-nearest-even, in the order the codec
// defines (explicit __fadd_rn/__fmul_rn/__fsqrt_rn so nothing is contracted
// into an FMA); this file is compiled without fast-math, so no flush-to-zero.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "tq_codebook.h"

namespace tq {

constexpr int kBlock = 32;        // elements per block
constexpr int kSbBlocks = 4;      // blocks per superblock
constexpr int kSbElems = 128;     // elements per superblock
constexpr int kSbCodeBytes = 64;  // code bytes per superblock
constexpr int kSbScaleBytes = 16; // scale bytes per superblock (4 blocks x 2 fp16)
constexpr unsigned kFull = 0xffffffffu;

// Element dtypes, same numbering as tq_dtype in tq.h.
enum Dtype : int { kF32 = 0, kBF16 = 1, kF16 = 2 };

// Sign pattern of global column k: golden-ratio multiplicative hash followed by
// one MurmurHash3-style mixing round; -1 where bit 31 is set.  Returned as the
// mask to XOR into an fp32 bit pattern (0x80000000 = negate, 0 = keep).
__device__ __forceinline__ uint32_t sign_mask(uint32_t k) {
    uint32_t h = k * 0x9E3779B9u;
    h ^= h >> 16;
    h *= 0x85EBCA6Bu;
    h ^= h >> 13;
    return h & 0x80000000u;
}

__device__ __forceinline__ float flip(float v, uint32_t mask) { return __uint_as_float(__float_as_uint(v) ^ mask); }

// One butterfly stage across lanes: this lane holds element i, the partner lane
// (lane ^ lane_xor) holds element i ^ h.  The lower index becomes a + b, the
// upper a - b, exactly as the sequential transform computes them (fp32 add is
// commutative, and partner - own == a - b for the upper element).
__device__ __forceinline__ float butterfly_xlane(float v, int lane_xor, bool upper) {
    float o = __shfl_xor_sync(kFull, v, lane_xor);
    return upper ? __fsub_rn(o, v) : __fadd_rn(v, o);
}

// In-register stages h = 1 and h = 2 on four consecutive elements v[0..3].
__device__ __forceinline__ void butterfly_local4(float (&v)[4]) {
    float a0 = __fadd_rn(v[0], v[1]), a1 = __fsub_rn(v[0], v[1]);
    float a2 = __fadd_rn(v[2], v[3]), a3 = __fsub_rn(v[2], v[3]);
    v[0] = __fadd_rn(a0, a2);
    v[2] = __fsub_rn(a0, a2);
    v[1] = __fadd_rn(a1, a3);
    v[3] = __fsub_rn(a1, a3);
}

// Loads of 4 consecutive elements converted (exactly) to fp32.
template <int DT>
__device__ __forceinline__ void load4(const void *p, float (&v)[4]);

template <>
__device__ __forceinline__ void load4<kF32>(const void *p, float (&v)[4]) {
    float4 q = __ldg(reinterpret_cast<const float4 *>(p));
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
}

template <>
__device__ __forceinline__ void load4<kBF16>(const void *p, float (&v)[4]) {
    uint2 q = __ldg(reinterpret_cast<const uint2 *>(p));
    v[0] = __uint_as_float(q.x << 16);
    v[1] = __uint_as_float(q.x & 0xffff0000u);
    v[2] = __uint_as_float(q.y << 16);
    v[3] = __uint_as_float(q.y & 0xffff0000u);
}

template <>
__device__ __forceinline__ void load4<kF16>(const void *p, float (&v)[4]) {
    uint2 q = __ldg(reinterpret_cast<const uint2 *>(p));
    __half2 h0 = *reinterpret_cast<__half2 *>(&q.x), h1 = *reinterpret_cast<__half2 *>(&q.y);
    float2 f0 = __half22float2(h0), f1 = __half22float2(h1);
    v[0] = f0.x; v[1] = f0.y; v[2] = f1.x; v[3] = f1.y;
}

// Stores of 4 consecutive fp32 values rounded (nearest-even) to the dtype.
template <int DT>
__device__ __forceinline__ void store4(void *p, const float (&v)[4]);

template <>
__device__ __forceinline__ void store4<kF32>(void *p, const float (&v)[4]) {
    *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
}

template <>
__device__ __forceinline__ void store4<kBF16>(void *p, const float (&v)[4]) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
    uint2 q;
    q.x = *reinterpret_cast<uint32_t *>(&a);
    q.y = *reinterpret_cast<uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p) = q;
}

template <>
__device__ __forceinline__ void store4<kF16>(void *p, const float (&v)[4]) {
    __half2 a = __floats2half2_rn(v[0], v[1]), b = __floats2half2_rn(v[2], v[3]);
    uint2 q;
    q.x = *reinterpret_cast<uint32_t *>(&a);
    q.y = *reinterpret_cast<uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p) = q;
}

template <int DT>
__device__ __forceinline__ void store1(void *p, float v);

template <>
__device__ __forceinline__ void store1<kF32>(void *p, float v) { *reinterpret_cast<float *>(p) = v; }

template <>
__device__ __forceinline__ void store1<kBF16>(void *p, float v) {
    *reinterpret_cast<__nv_bfloat16 *>(p) = __float2bfloat16_rn(v);
}

template <>
__device__ __forceinline__ void store1<kF16>(void *p, float v) { *reinterpret_cast<__half *>(p) = __float2half_rn(v); }

template <int DT>
struct ElemSize {
    static constexpr int value = DT == kF32 ? 4 : 2;
};

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------

// 128-bit global load that may stay in L1 (small, reused operands).
__device__ __forceinline__ uint4 ldg_keep(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

// Byte permute: result byte i = byte sel_i of the 8-byte value {b, a}.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ float lds_f32(uint32_t saddr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(saddr));
    return v;
}

// ---------------------------------------------------------------------------
// Register-table decode of TQ4_1S codes (no shared-memory table): the eight
// fp16 Lloyd-Max magnitudes as byte tables for PRMT.
// ---------------------------------------------------------------------------
// 4x4 byte transpose: out[i] byte b = in[b] byte i (its own inverse).  Logical
// code words W0..W3 (bytes 0-3, 4-7, 8-11, 12-15 of a block) <-> stored words
// T0..T3 (T_t = logical bytes t, t+4, t+8, t+12).
__device__ __forceinline__ void transpose4(const uint32_t (&w)[4], uint32_t (&o)[4]) {
    const uint32_t a = prmt(w[0], w[1], 0x5140u), b = prmt(w[2], w[3], 0x5140u);
    const uint32_t c = prmt(w[0], w[1], 0x7362u), d = prmt(w[2], w[3], 0x7362u);
    o[0] = prmt(a, b, 0x5410u);
    o[1] = prmt(a, b, 0x7632u);
    o[2] = prmt(c, d, 0x5410u);
    o[3] = prmt(c, d, 0x7632u);
}

// fp16 Lloyd-Max magnitudes as byte tables for PRMT: low bytes of magnitudes
// 0..3 / 4..7 and high bytes of magnitudes 0..3 / 4..7.
constexpr uint16_t kMagF16[8] = TQ_MAG_F16_INIT;
constexpr uint32_t mag_bytes(int i0, bool hi) {
    uint32_t v = 0;
    for (int i = 0; i < 4; ++i) v |= (uint32_t)((hi ? kMagF16[i0 + i] >> 8 : kMagF16[i0 + i]) & 0xFF) << (8 * i);
    return v;
}
constexpr uint32_t kMagLo0 = mag_bytes(0, false), kMagLo1 = mag_bytes(4, false);
constexpr uint32_t kMagHi0 = mag_bytes(0, true), kMagHi1 = mag_bytes(4, true);

// Eight codes (one logical word: element 2L in the low nibble of byte L,
// element 2L+1 in the high nibble) to four fp16 pairs of signed centroids.
//  * magnitudes: PRMT with the three magnitude bits of four codes as its
//    selector nibbles picks their low (high) bytes from the byte tables;
//  * signs: a code's sign is bit 3 of its nibble, i.e. the top bit of a byte
//    of w (odd elements) or of w << 4 (even elements); PRMT in sign-replicate
//    mode turns those top bits into 0xFF / 0x00 bytes, one per code, whose
//    top bit is merged into the high bytes;
//  * two more PRMTs interleave low and high bytes into fp16 pairs.
__device__ __forceinline__ void decode_word(uint32_t w, uint32_t (&o)[4]) {
    const uint32_t m = w & 0x77777777u;  // magnitude ranks (PRMT reads the low 16 bits)
    const uint32_t m2 = m >> 16;
    const uint32_t w4 = w << 4;
    // byte j of the mask: sign of element j (selector nibbles: 8 | byte, a = w4, b = w)
    const uint32_t s03 = prmt(w4, w, 0xD9C8u), s47 = prmt(w4, w, 0xFBEAu);
    const uint32_t lo03 = prmt(kMagLo0, kMagLo1, m), lo47 = prmt(kMagLo0, kMagLo1, m2);
    const uint32_t hi03 = prmt(kMagHi0, kMagHi1, m) | (s03 & 0x80808080u);
    const uint32_t hi47 = prmt(kMagHi0, kMagHi1, m2) | (s47 & 0x80808080u);
    o[0] = prmt(lo03, hi03, 0x5140u);  // elements 0, 1
    o[1] = prmt(lo03, hi03, 0x7362u);  // elements 2, 3
    o[2] = prmt(lo47, hi47, 0x5140u);  // elements 4, 5
    o[3] = prmt(lo47, hi47, 0x7362u);  // elements 6, 7
}

// L2 prefetch hint for the line holding p (no data returned, no fault on a
// valid address).
__device__ __forceinline__ void prefetch_l2(const void *p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

// Programmatic dependent launch: wait for the preceding grid's results / let
// the next grid start its prologue.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dependents_launch() { asm volatile("griddepcontrol.launch_dependents;" :::); }

// ---------------------------------------------------------------------------
// Activation pre-rotation (TQ page, section 解码速度: the activation is
// rotated once per call with the weights' sign pattern and transform, scaled
// by 1/32, and stored as fp16).  One warp rotates the 128 columns of one
// (row, superblock) "rotation unit": lane = 8*j + p holds elements 4p..4p+3 of
// block j; stages h = 1, 2 run in registers, h = 4, 8, 16 across lanes.
// ---------------------------------------------------------------------------
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

// This lane's four rotated (or, without ROTATE, only converted) values of
// rotation unit (row, sb) of an activation with nb blocks per row, as two
// fp16 pairs; blocks past nb and rows >= m give zeros.
template <int DT, bool ROTATE>
__device__ __forceinline__ void rotate_unit_lane(const char *x, int64_t ldx, int nb, int m, int row, int sb, int lane,
                                                 __half2 &lo, __half2 &hi) {
    const int j = lane >> 3, p = lane & 7;
    const bool valid = sb * kSbBlocks + j < nb && row < m;
    const uint32_t col0 = (uint32_t)sb * kSbElems + 32u * j + 4u * p;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (valid) load4<DT>(x + ((int64_t)row * ldx + col0) * ElemSize<DT>::value, v);
    if (ROTATE) {
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = flip(v[i], sign_mask(col0 + i));
        fwht32_warp(v, p);
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = __fmul_rn(v[i], 0.03125f);
    }
    lo = __floats2half2_rn(v[0], v[1]);
    hi = __floats2half2_rn(v[2], v[3]);
}

// Store of one lane's values in the mma.sync kernel's fragment order: element
// e of a block goes to slot t*8 + q with t = (e%8)/2, q = 2*(e/8) + e%2
// (`local` = row * nsb + sb within the input).
__device__ __forceinline__ void store_fragment(uint32_t *xrot, int64_t local, int lane, __half2 lo, __half2 hi) {
    const int j = lane >> 3, p = lane & 7;
    const size_t blk_words = ((size_t)local * kSbBlocks + j) * 16;  // 32 halves per block
    // elements 4p, 4p+1 -> t = 2(p&1), q = 2(p>>1) + {0,1}; 4p+2, 4p+3 -> t + 1
    const int t0 = 2 * (p & 1), q0 = 2 * (p >> 1);
    xrot[blk_words + (t0 * 8 + q0) / 2] = *reinterpret_cast<const uint32_t *>(&lo);
    xrot[blk_words + ((t0 + 1) * 8 + q0) / 2] = *reinterpret_cast<const uint32_t *>(&hi);
}

}  // namespace tq
