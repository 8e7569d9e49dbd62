// tq_codec.cu -- TQ4_1S quantise, dequantise and activation pre-rotation.
//
// Method: TQ4_1S page ("企业官网建设流程全解析", hotelren.com/news/5458160),
// paragraph 格式原理 items 1-3 and the paragraph after them; section
// 解码速度：分硬件汇总 for the pre-rotated activation.
//
// Quantise and dequantise: lane l of a warp owns one 32-element block (32
// consecutive columns) and the warp walks rows, so the sign pattern of the
// lane's columns is computed once; the whole 32-point transform runs in
// registers in the codec's stage order, so every fp32 result equals the
// sequential definition bit for bit.
// Pre-rotation: one warp owns one 128-column superblock of one row per step;
// lane = 8*j + p holds elements 4p..4p+3 of block j; two butterfly stages in
// registers (h = 1, 2), three across lanes (h = 4, 8, 16 via shfl_xor).
#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {

namespace {

constexpr int kCodecWarps = 8;
constexpr int kCodecThreads = kCodecWarps * 32;

__constant__ uint32_t c_thr_bits[7] = TQ_THR_F32_INIT;
__constant__ uint32_t c_mag_bits[8] = TQ_MAG_F32_INIT;

// Index of a row's 64-byte code slot (and 16-byte scale slot) for superblock
// sb in the tile-major layout [tile][sb][16 rows].
__device__ __forceinline__ size_t unit_row(int row, int sb, int nsb) {
    return ((size_t)(row >> 4) * nsb + sb) * 16 + (row & 15);
}

// Code of one rotated value y against the ascending thresholds t of its half,
// added into `word` at nibble position `sh`: bit 3 = [y < 0], bits 0..2 =
// #{j : |y| > t_j} by a three-compare binary search.  Each bit is a
// conditional add consumed right after its compare, so the compiler can
// predicate the adds instead of materialising (or spilling) the predicates.
__device__ __forceinline__ uint32_t add_code(uint32_t word, float y, const float (&t)[7], int sh) {
    const float a = fabsf(y);
    const bool b2 = a > t[3];
    const bool b1 = a > (b2 ? t[5] : t[1]);
    const bool b0 = a > (b1 ? (b2 ? t[6] : t[2]) : (b2 ? t[4] : t[0]));
    if (b2) word += 4u << sh;
    if (b1) word += 2u << sh;
    if (b0) word += 1u << sh;
    if (y < 0.0f) word += 8u << sh;
    return word;
}

// -------------------------------------------------------------------------
// Block-per-lane helpers (quantise / dequantise): lane l of a warp owns block
// 32*seg + l of its rows, i.e. 32 consecutive columns; the whole 32-point
// transform runs in registers in the codec's stage order.
// -------------------------------------------------------------------------

// Sign bits of the lane's 32 columns (bit e = 1 where column k0+e flips).
__device__ __forceinline__ uint32_t block_sign_bits(uint32_t k0) {
    uint32_t m = 0;
#pragma unroll
    for (int e = 0; e < 32; ++e) m |= (sign_mask(k0 + e) >> 31) << e;
    return m;
}

// Packed 16-bit sign masks: word i flips elements 2i (bit 15) and 2i+1 (bit 31).
__device__ __forceinline__ void packed_sign_words(uint32_t bits, uint32_t (&ps)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) ps[i] = (((bits >> (2 * i)) & 1u) << 15) | (((bits >> (2 * i + 1)) & 1u) << 31);
}

// Packed fp32 pairs (sm_100 add/sub.rn.f32x2): each half is one IEEE fp32
// operation rounded to nearest even, exactly the scalar __fadd_rn/__fsub_rn.
// Their operands here are loads or scalar products, never a packed product
// (a packed multiply feeding a packed add may be contracted into an FMA).
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void unpack2(uint64_t r, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// The 32-point transform in the codec's stage order h = 1, 2, 4, 8, 16.
// Element t and element t + 16 share one packed register: stages h < 16 pair
// register t with register t + h (both halves at once), stage 16 combines
// the two halves of each register in scalar.  Every element sees the same
// operations on the same operands as the sequential definition.
__device__ __forceinline__ void fwht32_regs(float (&v)[32]) {
    uint64_t P[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) P[t] = pack2(v[t], v[t + 16]);
#pragma unroll
    for (int h = 1; h < 16; h <<= 1)
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if ((i & h) == 0) {
                const uint64_t a = P[i], b = P[i + h];
                P[i] = add2(a, b);
                P[i + h] = sub2(a, b);
            }
#pragma unroll
    for (int t = 0; t < 16; ++t) {
        float lo, hi;
        unpack2(P[t], lo, hi);
        v[t] = __fadd_rn(lo, hi);
        v[t + 16] = __fsub_rn(lo, hi);
    }
}

// 32 input elements -> fp32 with the sign flip applied (exact).
template <int DT>
__device__ __forceinline__ void load_block(const char *p, uint32_t bits, const uint32_t (&ps)[16], float (&v)[32]);

template <>
__device__ __forceinline__ void load_block<kF32>(const char *p, uint32_t bits, const uint32_t (&)[16],
                                                 float (&v)[32]) {
    const uint4 *q = reinterpret_cast<const uint4 *>(p);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint4 w = __ldg(q + i);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int e = 4 * i + c;
            v[e] = __uint_as_float(ws[c] ^ ((bits << (31 - e)) & 0x80000000u));
        }
    }
}

template <>
__device__ __forceinline__ void load_block<kBF16>(const char *p, uint32_t, const uint32_t (&ps)[16],
                                                  float (&v)[32]) {
    const uint4 *q = reinterpret_cast<const uint4 *>(p);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 w = __ldg(q + i);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint32_t x = ws[c] ^ ps[4 * i + c];
            v[8 * i + 2 * c] = __uint_as_float(x << 16);
            v[8 * i + 2 * c + 1] = __uint_as_float(x & 0xffff0000u);
        }
    }
}

template <>
__device__ __forceinline__ void load_block<kF16>(const char *p, uint32_t, const uint32_t (&ps)[16],
                                                 float (&v)[32]) {
    const uint4 *q = reinterpret_cast<const uint4 *>(p);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 w = __ldg(q + i);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint32_t x = ws[c] ^ ps[4 * i + c];
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&x));
            v[8 * i + 2 * c] = f.x;
            v[8 * i + 2 * c + 1] = f.y;
        }
    }
}

// -------------------------------------------------------------------------
// Quantise.  grid.x = 1024-column segment (32 blocks, one per lane),
// grid.y * 8 warps stride the rows (padded to a multiple of 16).
// -------------------------------------------------------------------------
template <int DT>
__global__ void __launch_bounds__(kCodecThreads) quantize_kernel(const char *__restrict__ w, int64_t ldw, int n,
                                                                   int nb, int nsb, uint32_t *__restrict__ codes,
                                                                   uint32_t *__restrict__ scales) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int blk = blockIdx.x * 32 + lane;  // block column of this lane
    const bool exists = blk < nsb * kSbBlocks;  // padding blocks still get zero codes
    const bool valid = blk < nb;
    const int sb = blk >> 2, j = blk & 3;
    const uint32_t k0 = (uint32_t)blk * kBlock;
    const uint32_t bits = block_sign_bits(k0);
    uint32_t ps[16];
    packed_sign_words(bits, ps);
    float thr[7];
#pragma unroll
    for (int i = 0; i < 7; ++i) thr[i] = __uint_as_float(c_thr_bits[i]);

    const int rows_padded = (n + 15) & ~15;
    for (int row = blockIdx.y * kCodecWarps + warp; row < rows_padded; row += gridDim.y * kCodecWarps) {
        float v[32];
        if (valid && row < n) {
            load_block<DT>(w + ((int64_t)row * ldw + k0) * ElemSize<DT>::value, bits, ps, v);
        } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = 0.f;
        }
        fwht32_regs(v);

        // half-block scales: adjacent pairwise tree of the squares
        uint32_t dbits[2];
        float D[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float q[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) q[e] = __fmul_rn(v[16 * h + e], v[16 * h + e]);
#pragma unroll
            for (int step = 1; step < 16; step <<= 1)
#pragma unroll
                for (int i = 0; i < 16; i += 2 * step) q[i] = __fadd_rn(q[i], q[i + step]);
            const __half hd = __float2half_rn(__fsqrt_rn(__fmul_rn(q[0], 0.0625f)));
            dbits[h] = __half_as_ushort(hd);
            D[h] = __half2float(hd);
        }

        uint32_t lw[4] = {0u, 0u, 0u, 0u};  // logical code words
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float t[7];
#pragma unroll
            for (int i = 0; i < 7; ++i) t[i] = __fmul_rn(thr[i], D[h]);
#pragma unroll
            for (int e = 16 * h; e < 16 * h + 16; ++e) lw[e >> 3] = add_code(lw[e >> 3], v[e], t, 4 * (e & 7));
        }
        if (exists) {
            uint32_t sw[4];
            transpose4(lw, sw);
            const size_t slot = unit_row(row, sb, nsb);
#pragma unroll
            for (int tt = 0; tt < 4; ++tt) codes[slot * 16 + 4 * tt + j] = sw[tt];
            scales[slot * 4 + j] = dbits[0] | (dbits[1] << 16);
        }
    }
}

// -------------------------------------------------------------------------
// Dequantise: w~ = s .* (H c) / 32, fp32, rounded to the output dtype.
// The 1/32 is folded into the fp16 scale (exact power-of-two scaling).
// A warp writes one row segment of 32 blocks per step: each lane's block goes
// through a per-warp shared-memory stage (16-byte chunks, XOR-placed so that
// neither side has bank conflicts) and leaves as fully coalesced 512-byte
// stores; the next row's codes and scales are loaded one step ahead.
// -------------------------------------------------------------------------
template <int DT>
struct DeqOut {
    static constexpr int kWords = DT == kF32 ? 32 : 16;  // 32-bit output words per block
    static constexpr int kChunks = kWords / 4;            // 16-byte chunks per block
};

// A block's output words: elements rounded to DT, sign flip applied.
template <int DT>
__device__ __forceinline__ void block_words(uint32_t bits, const uint32_t (&ps)[16], const float (&v)[32],
                                            uint32_t (&o)[DeqOut<DT>::kWords]);

template <>
__device__ __forceinline__ void block_words<kF32>(uint32_t bits, const uint32_t (&)[16], const float (&v)[32],
                                                  uint32_t (&o)[32]) {
#pragma unroll
    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(v[e]) ^ ((bits << (31 - e)) & 0x80000000u);
}

template <>
__device__ __forceinline__ void block_words<kBF16>(uint32_t, const uint32_t (&ps)[16], const float (&v)[32],
                                                   uint32_t (&o)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        o[i] = *reinterpret_cast<uint32_t *>(&h) ^ ps[i];
    }
}

template <>
__device__ __forceinline__ void block_words<kF16>(uint32_t, const uint32_t (&ps)[16], const float (&v)[32],
                                                  uint32_t (&o)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        __half2 h = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
        o[i] = *reinterpret_cast<uint32_t *>(&h) ^ ps[i];
    }
}

// Stage slot of chunk i of lane l's block: l * C + (i ^ key(l)); within any
// 8 consecutive lanes writing chunk i, and within any 8 consecutive chunks
// read back, the slots fall in 8 different 16-byte bank groups.
template <int C>
__device__ __forceinline__ int stage_key(int l) {
    return C == 8 ? (l & 7) : ((l >> 1) & 3);
}

// Work items of a (batched) dequantise launch: (matrix, 1024-column segment,
// 8-row group), numbered matrix by matrix and, within a matrix, segment by
// segment; each CTA takes one contiguous range of items, so its lanes'
// sign patterns change only where the segment does.  Warp w of a CTA
// writes row 8 * group + w of each item.
struct DeqProblem {
    const uint32_t *codes;
    const uint32_t *scales;
    char *out;
    int64_t ldo;
    int64_t item_begin;
    int n, nb, nsb, segs, groups;
};
struct DeqParams {
    DeqProblem p[kMaxProblems];
    int count;
    int64_t items;
};

struct DeqItem {
    int q, seg, group;
};

__device__ __forceinline__ void next_item(const DeqParams &P, DeqItem &it) {
    if (++it.group == P.p[it.q].groups) {
        it.group = 0;
        if (++it.seg == P.p[it.q].segs) {
            it.seg = 0;
            ++it.q;
        }
    }
}

template <int DT>
__global__ void __launch_bounds__(kCodecThreads, DT == kF32 ? 2 : 3) dequantize_kernel(const __grid_constant__ DeqParams P) {
    constexpr int C = DeqOut<DT>::kChunks;
    __shared__ float cent[16];  // signed centroids c(code)
    __shared__ __align__(16) uint4 stage[kCodecWarps * 32 * C];
    if (threadIdx.x < 16) {
        const float m = __uint_as_float(c_mag_bits[threadIdx.x & 7]);
        cent[threadIdx.x] = (threadIdx.x & 8) ? -m : m;
    }
    __syncthreads();
    const uint32_t cent_base = (uint32_t)__cvta_generic_to_shared(cent);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint4 *st = stage + warp * 32 * C;
    const int key = stage_key<C>(lane);

    const int64_t i0 = P.items * blockIdx.x / gridDim.x, i1 = P.items * (blockIdx.x + 1) / gridDim.x;
    if (i0 >= i1) return;
    DeqItem cur;
    cur.q = 0;
    while (cur.q + 1 < P.count && i0 >= P.p[cur.q + 1].item_begin) ++cur.q;
    {
        const int64_t local = i0 - P.p[cur.q].item_begin;
        cur.seg = (int)(local / P.p[cur.q].groups);
        cur.group = (int)(local % P.p[cur.q].groups);
    }
    // codes and scales of this warp's row of an item (nothing past the matrix)
    auto load_row = [&](const DeqItem &it, uint32_t (&w)[4], uint32_t &sc) {
        const DeqProblem &pr = P.p[it.q];
        const int row = it.group * kCodecWarps + warp, blk = it.seg * 32 + lane;
        if (row < pr.n && blk < pr.nb) {
            const size_t slot = unit_row(row, blk >> 2, pr.nsb);
#pragma unroll
            for (int tt = 0; tt < 4; ++tt) w[tt] = __ldg(pr.codes + slot * 16 + 4 * tt + (blk & 3));
            sc = __ldg(pr.scales + slot * 4 + (blk & 3));
        }
    };
    int seg_bits = -1;  // segment whose sign pattern `bits` / `ps` hold
    uint32_t bits = 0, ps[16];
    uint32_t nsw[4] = {0u, 0u, 0u, 0u}, nsc = 0u;  // the next item's row, loaded one step ahead
    load_row(cur, nsw, nsc);
    for (int64_t i = i0; i < i1; ++i) {
        const DeqProblem &pr = P.p[cur.q];
        const int row = cur.group * kCodecWarps + warp, blk = cur.seg * 32 + lane;
        if (cur.seg != seg_bits) {
            seg_bits = cur.seg;
            bits = block_sign_bits((uint32_t)blk * kBlock);
            packed_sign_words(bits, ps);
        }
        uint32_t sw[4], sc = nsc;
#pragma unroll
        for (int tt = 0; tt < 4; ++tt) sw[tt] = nsw[tt];
        DeqItem nx = cur;
        next_item(P, nx);
        if (i + 1 < i1) load_row(nx, nsw, nsc);
        float v[32];
        if (row < pr.n && blk < pr.nb) {
            uint32_t lw[4];
            transpose4(sw, lw);  // the transpose is its own inverse
            const float2 D = __half22float2(*reinterpret_cast<const __half2 *>(&sc));
            const float Ds[2] = {__fmul_rn(D.x, 0.03125f), __fmul_rn(D.y, 0.03125f)};
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const uint32_t code = (lw[e >> 3] >> (4 * (e & 7))) & 15u;
                v[e] = __fmul_rn(lds_f32(cent_base + 4 * code), Ds[e >> 4]);
            }
            fwht32_regs(v);
        } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = 0.f;
        }
        uint32_t o[DeqOut<DT>::kWords];
        block_words<DT>(bits, ps, v, o);
#pragma unroll
        for (int c = 0; c < C; ++c) st[lane * C + (c ^ key)] = make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
        __syncwarp();
        if (row < pr.n) {
            const int nvalid = min(32, pr.nb - cur.seg * 32);  // blocks of this segment
            uint4 *rowp = reinterpret_cast<uint4 *>(pr.out + ((int64_t)row * pr.ldo + (int64_t)cur.seg * 32 * kBlock) *
                                                                 ElemSize<DT>::value);
#pragma unroll
            for (int c0 = 0; c0 < C; ++c0) {
                const int c = c0 * 32 + lane;  // 16-byte chunk of the warp's row segment
                const int L = c / C;           // the lane (block) it belongs to
                const uint4 val = st[L * C + ((c % C) ^ stage_key<C>(L))];
                if (L < nvalid) rowp[c] = val;
            }
        }
        __syncwarp();
        cur = nx;
    }
}

// -------------------------------------------------------------------------
// Pre-rotation of activations.  Output layouts (RotLayout):
//  * kRotFragment: the mma.sync kernel's fragment order: element e of a block
//    goes to slot t*8 + q with t = (e%8)/2, q = 2*(e/8) + e%2;
//  * kRotPlain: row-major fp16 [rows][NSB*128], padding columns zero (the
//    tensor-memory kernel's one-row operand);
//  * kRotCore: the tensor-memory kernel's B operand for npad rows, in 16-byte
//    core-matrix rows: [NSB][16 column groups of 8][npad rows][8], rows m ..
//    npad-1 and padding columns zero.
// Handles a list of inputs (one warp per (input, row, superblock)) and
// prepares the header of the product that follows (status cleared, tag
// advanced).
// -------------------------------------------------------------------------
template <int DT, bool ROTATE, int LAYOUT>
__global__ void __launch_bounds__(kCodecThreads) prerotate_kernel(const __grid_constant__ RotParams prm) {
    // Launched as a programmatic dependent of the previous kernel in the
    // stream.  The fused product that follows may launch at once: before its
    // own dependency wait it only fills shared memory and copies packed
    // weights, which no kernel still running writes (a product's weights are
    // written by a quantise launch that completed before this kernel could
    // start), so its CTAs can take the SMs that the previous product frees
    // in its tail.  Then wait until every earlier kernel has completed.
    //
    // The activation lines this lane will read are prefetched into L2 before
    // the wait (L2 is where writes meet, so a line a still-running kernel
    // rewrites is current there when the load after the wait reads it): the
    // loads then do not queue behind the product's weight prefetch in DRAM.
    const int lane = threadIdx.x & 31;
    const int j = lane >> 3, p = lane & 7;
    const int64_t unit = (int64_t)blockIdx.x * kCodecWarps + (threadIdx.x >> 5);
    int q = 0;
    while (q + 1 < prm.count && unit >= prm.in[q + 1].unit_begin) ++q;
    const RotInput &in = prm.in[q];
    const int64_t local = unit - in.unit_begin;
    const int row = (int)(local / in.nsb), sb = (int)(local % in.nsb);
    const uint32_t col0 = (uint32_t)sb * kSbElems + 32u * j + 4u * p;
    if (unit < prm.units && sb * kSbBlocks + j < in.nb && row < prm.m)
        prefetch_l2(in.x + ((int64_t)row * in.ldx + col0) * ElemSize<DT>::value);
    grid_dependents_launch();
    grid_dependency_wait();
    if (prm.header && blockIdx.x == 0 && threadIdx.x == 0) {
        prm.header[kHeaderStatus] = 0u;
        prm.header[kHeaderTag] += 1u;  // the previous call (and its product) has completed
    }
    if (unit >= prm.units) return;
    __half2 lo, hi;
    rotate_unit_lane<DT, ROTATE>(in.x, in.ldx, in.nb, prm.m, row, sb, lane, lo, hi);
    if constexpr (LAYOUT == kRotFragment) {
        store_fragment(in.xrot, local, lane, lo, hi);
    } else {
        size_t half_off;
        if constexpr (LAYOUT == kRotPlain) {
            half_off = (size_t)row * in.nsb * kSbElems + col0;
        } else {  // kRotCore: column group 4j + p/2, element 4(p&1) .. +3 of its 16-byte row
            half_off = ((size_t)sb * 16 + 4 * j + (p >> 1)) * (size_t)prm.npad * 8 + (size_t)row * 8 + 4 * (p & 1);
        }
        uint2 o;
        o.x = *reinterpret_cast<const uint32_t *>(&lo);
        o.y = *reinterpret_cast<const uint32_t *>(&hi);
        *reinterpret_cast<uint2 *>(reinterpret_cast<uint16_t *>(in.xrot) + half_off) = o;
    }
}

// Row groups per column segment: one wave of the CTAs that fit on the GPU at
// once (`per_sm` resident per SM), each striding the rows.
int rows_grid(int64_t n, int64_t segs, int sm_count, int per_sm) {
    int64_t target = (int64_t)sm_count * (per_sm > 0 ? per_sm : 1);
    int64_t gy = target / segs;
    int64_t max_gy = (((n + 15) & ~(int64_t)15) + kCodecWarps - 1) / kCodecWarps;
    if (gy > max_gy) gy = max_gy;
    if (gy > 65535) gy = 65535;
    if (gy < 1) gy = 1;
    return (int)gy;
}

}  // namespace

// Resident CTAs per SM of a kernel (queried once per kernel).
template <typename K>
int resident_per_sm(K kernel, int *cache) {
    if (*cache <= 0) {
        int nb = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kernel, kCodecThreads, 0) != cudaSuccess || nb < 1)
            nb = 1;
        *cache = nb;
    }
    return *cache;
}

template <int DT>
int quantize_per_sm() {
    static int cache = 0;
    return resident_per_sm(quantize_kernel<DT>, &cache);
}

template <int DT>
int dequantize_per_sm() {
    static int cache = 0;
    return resident_per_sm(dequantize_kernel<DT>, &cache);
}

cudaError_t launch_quantize(const void *w, int dtype, int64_t n, int64_t k, int64_t ldw, uint8_t *codes,
                            uint16_t *scales, cudaStream_t stream) {
    DeviceInfo di;
    cudaError_t err = device_info(&di);
    if (err != cudaSuccess) return err;
    const int64_t nb = k / 32, nsb = superblocks(k);
    const int64_t segs = (nsb * kSbBlocks + 31) / 32;
    const int per_sm = dtype == kF32 ? quantize_per_sm<kF32>() : dtype == kBF16 ? quantize_per_sm<kBF16>()
                                                                                 : quantize_per_sm<kF16>();
    dim3 grid((unsigned)segs, (unsigned)rows_grid(n, segs, di.sm_count, per_sm));
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

cudaError_t launch_dequantize_batch(const DequantJob *jobs, int count, int dtype, cudaStream_t stream) {
    if (count < 1 || count > kMaxProblems) return cudaErrorInvalidValue;
    DeviceInfo di;
    cudaError_t err = device_info(&di);
    if (err != cudaSuccess) return err;
    DeqParams prm = {};
    int64_t items = 0;
    int used = 0;  // matrices with rows (an empty one has no items to walk)
    for (int i = 0; i < count; ++i) {
        if (jobs[i].n <= 0) continue;
        DeqProblem &d = prm.p[used++];
        d.codes = reinterpret_cast<const uint32_t *>(jobs[i].codes);
        d.scales = reinterpret_cast<const uint32_t *>(jobs[i].scales);
        d.out = static_cast<char *>(jobs[i].out);
        d.ldo = jobs[i].ldo;
        d.item_begin = items;
        d.n = (int)jobs[i].n;
        d.nb = (int)(jobs[i].k / 32);
        d.nsb = (int)superblocks(jobs[i].k);
        d.segs = (d.nb + 31) / 32;
        d.groups = (int)((jobs[i].n + kCodecWarps - 1) / kCodecWarps);
        items += (int64_t)d.segs * d.groups;
    }
    prm.count = used;
    prm.items = items;
    if (items == 0) return cudaSuccess;
    const int per_sm = dtype == kF32 ? dequantize_per_sm<kF32>() : dtype == kBF16 ? dequantize_per_sm<kBF16>()
                                                                                   : dequantize_per_sm<kF16>();
    int64_t grid = (int64_t)di.sm_count * per_sm;  // one wave, persistent
    if (grid > items) grid = items;
    switch (dtype) {
        case kF32: dequantize_kernel<kF32><<<(unsigned)grid, kCodecThreads, 0, stream>>>(prm); break;
        case kBF16: dequantize_kernel<kBF16><<<(unsigned)grid, kCodecThreads, 0, stream>>>(prm); break;
        case kF16: dequantize_kernel<kF16><<<(unsigned)grid, kCodecThreads, 0, stream>>>(prm); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, void *w_out,
                              int dtype, int64_t ldo, cudaStream_t stream) {
    const DequantJob job = {codes, scales, n, k, w_out, ldo};
    return launch_dequantize_batch(&job, 1, dtype, stream);
}

namespace {

__global__ void __launch_bounds__(32) prepare_header_kernel(unsigned *header) {
    grid_dependents_launch();  // as in the pre-rotation: the product's prologue may overlap
    grid_dependency_wait();
    if (threadIdx.x == 0) {
        header[kHeaderStatus] = 0u;
        header[kHeaderTag] += 1u;
    }
}

}  // namespace

cudaError_t launch_prepare_header(unsigned *header, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(32);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prepare_header_kernel, header);
}

cudaError_t launch_prerotate(const RotJob *jobs, int count, int dtype, int64_t m, unsigned *header,
                             cudaStream_t stream, bool rotate, int layout, int npad) {
    if (count < 1 || count > kMaxInputs) return cudaErrorInvalidValue;
    if (layout == kRotCore && (npad < m || npad % 8 != 0)) return cudaErrorInvalidValue;
    if (layout == kRotPlain && !rotate) return cudaErrorInvalidValue;
    // rows written per input: m, or npad in the core-matrix layout (rows past
    // m are written as zeros)
    const int64_t rows = layout == kRotCore ? npad : m;
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
        units += rows * in.nsb;
    }
    prm.count = count;
    prm.units = units;
    prm.header = header;
    prm.m = (int)m;
    prm.npad = npad;
    int64_t grid = (units + kCodecWarps - 1) / kCodecWarps;
    if (grid < 1) grid = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kCodecThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (layout == kRotPlain) {
        switch (dtype) {
            case kF32: return cudaLaunchKernelEx(&cfg, prerotate_kernel<kF32, true, kRotPlain>, prm);
            case kBF16: return cudaLaunchKernelEx(&cfg, prerotate_kernel<kBF16, true, kRotPlain>, prm);
            case kF16: return cudaLaunchKernelEx(&cfg, prerotate_kernel<kF16, true, kRotPlain>, prm);
            default: return cudaErrorInvalidValue;
        }
    }
    if (layout == kRotCore) {
        switch (dtype * 2 + (rotate ? 1 : 0)) {
            case kF32 * 2 + 1: return cudaLaunchKernelEx(&cfg, prerotate_kernel<kF32, true, kRotCore>, prm);
            case kBF16 * 2 + 1: return cudaLaunchKernelEx(&cfg, prerotate_kernel<kBF16, true, kRotCore>, prm);
            case kF16 * 2 + 1: return cudaLaunchKernelEx(&cfg, prerotate_kernel<kF16, true, kRotCore>, prm);
            default: return cudaErrorInvalidValue;
        }
    }
    switch (dtype * 2 + (rotate ? 1 : 0)) {
        case kF32 * 2 + 1: return cudaLaunchKernelEx(&cfg, prerotate_kernel<kF32, true, kRotFragment>, prm);
        case kBF16 * 2 + 1: return cudaLaunchKernelEx(&cfg, prerotate_kernel<kBF16, true, kRotFragment>, prm);
        case kF16 * 2 + 1: return cudaLaunchKernelEx(&cfg, prerotate_kernel<kF16, true, kRotFragment>, prm);
        case kF32 * 2: return cudaLaunchKernelEx(&cfg, prerotate_kernel<kF32, false, kRotFragment>, prm);
        case kBF16 * 2: return cudaLaunchKernelEx(&cfg, prerotate_kernel<kBF16, false, kRotFragment>, prm);
        case kF16 * 2: return cudaLaunchKernelEx(&cfg, prerotate_kernel<kF16, false, kRotFragment>, prm);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace tq
