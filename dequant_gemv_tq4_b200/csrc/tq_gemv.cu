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
//  * Each warp keeps a ring of two stages of four units (one activation row)
//    or two units (more rows) in shared memory,
//    filled by cp.async.bulk (TMA bulk copies, one lane issues, an mbarrier
//    per stage counts the bytes).  No registers are spent on loads in flight;
//    waits are bounded in time and report a timeout through a status word.
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
//    accumulator; with four n-tiles (m > 24) it multiplies the decoded
//    centroids instead (fp16(c * d), shared by the n-tiles) and the mmas
//    accumulate directly.
//  * One activation row (the decode case) would leave seven of the eight mma
//    columns idle.  Instead column c carries half-block c of the superblock
//    (four blocks x two halves): the B fragment is the activation in the four
//    lanes of column c and zero elsewhere, so the eight mmas of a unit chain
//    into accumulators whose columns stay separate half-block sums.  Each
//    lane then applies two scales per row pair per unit (not sixteen), and the
//    four lanes of a row add their blocks once per tile.  Two and four
//    activation rows share the eight columns the same way (four and two
//    half-block slots per row).
//  * Tiles split across warps combine fixed-order partial sums: the later
//    contributors store (value, call tag) words without fences or atomics,
//    and the tile's first warp, which reaches its part of the tile last, adds
//    them in warp order once each carries this call's tag (a bounded poll).
//    Deterministic for a given GPU.
#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {

namespace {

// Warps per CTA and units per ring stage.  One activation row: 12 warps of up
// to 168 registers, four units per stage (fewer, longer-lived warps with deeper
// stages beat 16 or 20 warps of two or three units: the per-stage loop and
// copy bookkeeping is paid once per four units, and each warp's stretch of the
// unit space is longer).  Up to 16 rows: 16 warps (128 registers), two units
// per stage; 17..32 rows: 12 warps, whose three or four accumulator tiles need
// up to 168 registers without spilling.
__host__ __device__ constexpr int warps_for(bool one_row, int nt = 1) { return one_row ? 12 : (nt >= 3 ? 12 : 16); }
// Activation rows per half-block-combination kernel for m rows (1, 2 or 4; 0:
// the multi-row kernel).  3 rows run the 4-row kernel with the last row
// repeated (never stored).
constexpr int combo_rows(int64_t m) { return m == 1 ? 1 : m == 2 ? 2 : (m == 3 || m == 4) ? 4 : 0; }
constexpr int kStages = 2;  // ring stages per warp
constexpr int kUnitCodeBytes = 1024;
constexpr int kUnitScaleBytes = 256;  // TQ4_1S: 16 rows x 4 blocks x 2 fp16; NVFP4 uses 128 (16 x 8 E4M3)
constexpr int kUnitBytes = kUnitCodeBytes + kUnitScaleBytes;
// stage = [codes of units 0 .. P-1 | scales of units 0 .. P-1]
template <bool M1>
struct Ring {
    static constexpr int kPerStage = M1 ? 4 : 2;  // consecutive units per stage
    static constexpr int kStageScaleOff = kPerStage * kUnitCodeBytes;
    static constexpr int kStageBytes = kPerStage * kUnitBytes;  // room for either codec
    static constexpr int kRingWarpBytes = kStages * kStageBytes;
};
// Shared-memory map (addresses in the CTA's shared window; the dynamic
// allocation starts at a small base B <= kMaxSmemBase):
//   [kBarAddr, kLowRings)       the mbarriers
//   [kLowRings, 0x10000)        rings of the first kLowWarps warps
//   [0x10000, 0x20000)          lookup table, 64 KB aligned so that one PRMT
//                               yields the full address of an entry
//   [0x20000, kTop)             rings of the other warps
constexpr uint32_t kLutAddr = 0x10000;
constexpr uint32_t kHighRings = 0x20000;
template <int W, bool M1>
struct Geometry {
    static constexpr int kWarps = W;
    static constexpr int kThreads = W * 32;
    static constexpr int kRingWarpBytes = Ring<M1>::kRingWarpBytes;
    static constexpr uint32_t kBarBytes = W * kStages * 8;
    static constexpr int kLowFit = (int)((0x10000u - 1024u - kBarBytes) / kRingWarpBytes);
    static constexpr int kLowWarps = W < kLowFit ? W : kLowFit;
    static constexpr uint32_t kLowRings = 0x10000u - kLowWarps * kRingWarpBytes;
    static constexpr uint32_t kBarAddr = kLowRings - kBarBytes;
    static constexpr uint32_t kMaxSmemBase = kBarAddr;
    static constexpr uint32_t kTop = kHighRings + (W - kLowWarps) * kRingWarpBytes;
    static_assert(kMaxSmemBase >= 1024, "barriers and rings below the table");
    static_assert(kTop - 1024 <= 227 * 1024, "dynamic shared memory per CTA");
    // dynamic shared memory to request for a dynamic base of `base` bytes
    static uint32_t smem_bytes_for_base(uint32_t base) { return kTop - base; }
};
constexpr unsigned kStatusTimeout = 1u;
constexpr unsigned kStatusLayout = 2u;
constexpr uint64_t kTimeoutNs = 1000000000ull;     // 1 s
constexpr uint64_t kDebugTimeoutNs = 5000000ull;   // 5 ms under fault injection
constexpr uint64_t kStealAfterNs = 50000ull;       // 50 us (later contributors store at the start of their ranges)


// Dynamic shared memory to request for a dynamic base of `base` bytes.

__constant__ uint16_t c_mag_f16[8] = TQ_MAG_F16_INIT;

uint32_t g_debug_flags = 0;

struct DevProblem {
    const uint8_t *codes;
    const uint8_t *scales;
    const uint16_t *xrot;  // TQ4_1S: pre-rotated activation; NVFP4: activation in fragment order
    const float *tscale;   // NVFP4 tensor scale (device), nullptr for TQ4_1S
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
    int64_t units;    // < 2^31 (checked on the host)
    int total_warps;  // <= units: warp w owns [w*units/W, (w+1)*units/W)
    uint64_t *partials;  // tagged partial sums (value bits | call tag << 32)
    unsigned *header;    // workspace header: status word, call tag
    uint64_t timeout_ns;
    uint64_t steal_after_ns;  // a split tile's first warp computes a contribution missing for this long
    int inject_skip;
    int steal_all;            // test hook: compute every later contribution instead of reading it
    double inv_units;  // 1.0 / units and 1.0 / total_warps (host-computed):
    double inv_warps;  // the split arithmetic divides without 64-bit integer division
};

// floor(n / d) for 0 <= n < 2^52, 0 < d < 2^31, given inv_d = 1.0 / d.  The
// double estimate is within one of the quotient (n is exact in a double and
// the product's relative error is ~2^-52), and one integer step corrects it.
// A 64-bit integer division is a long instruction sequence; this is a few.
__device__ __forceinline__ int64_t div_floor(int64_t n, int64_t d, double inv_d) {
    int64_t q = __double2ll_rz((double)n * inv_d);
    if ((q + 1) * d <= n)
        ++q;
    else if (q * d > n)
        --q;
    return q;
}

// ---- PTX helpers ------------------------------------------------------------
// LUT read: the table is written once before the CTA barrier and never again,
// so its loads may be scheduled freely (no volatile)
__device__ __forceinline__ uint32_t lds_lut(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ void mma_nv(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}
__device__ __forceinline__ void mma_acc(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// fp16x2 product, round to nearest even
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 ldg64(const void *p) {
    uint2 r;
    asm volatile("ld.global.nc.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

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
__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
    const uint64_t t0 = global_ns();
    for (uint32_t it = 0; it < (1u << 30); ++it) {
        if (mbar_try(bar, parity)) return true;
        if (global_ns() - t0 > timeout_ns) return false;
    }
    return false;
}

__device__ __forceinline__ void arrive_expect_tx_pred(uint32_t pred, uint32_t bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %0, 0;\n\t"
        "@p mbarrier.arrive.expect_tx.shared::cta.b64 _, [%1], %2;\n\t}" ::"r"(pred),
        "r"(bar), "r"(bytes)
        : "memory");
}

// Bulk copy global -> shared completing on `bar`, issued by the lanes with
// `pred` set (one lane), without a branch.
__device__ __forceinline__ void bulk_copy_pred(uint32_t pred, uint32_t dst, const void *src, uint32_t bytes,
                                               uint32_t bar) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %0, 0;\n\t"
        "@p cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%1], [%2], %3, [%4];\n\t}" ::"r"(pred),
        "r"(dst), "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Producer cursor: the next unit this warp will copy, walked incrementally.
struct Cursor {
    const uint8_t *c;
    const uint8_t *s;
    int left;           // units left in the current problem
    int sb_left;        // units left in the current tile
    int q;
};

__device__ __forceinline__ int problem_of(const GroupParams &P, int v) {
    // the largest q with unit_begin <= v (independent loads, not a dependent walk)
    int q = 0;
#pragma unroll
    for (int i = 1; i < kMaxProblems; ++i)
        if (i < P.count && v >= P.prob[i].unit_begin) q = i;
    return q;
}

__device__ __forceinline__ int problem_end(const GroupParams &P, int q) {
    return (int)((q + 1 < P.count) ? P.prob[q + 1].unit_begin : P.units);
}

template <int SB>
__device__ __forceinline__ Cursor cursor_at(const GroupParams &P, int v) {
    const int q = problem_of(P, v);
    const int local = v - (int)P.prob[q].unit_begin;
    const int nsb = P.prob[q].nsb;
    Cursor cu;
    cu.c = P.prob[q].codes + (int64_t)local * kUnitCodeBytes;
    cu.s = P.prob[q].scales + (int64_t)local * SB;
    cu.left = problem_end(P, q) - v;
    cu.sb_left = nsb - local % nsb;
    cu.q = q;
    return cu;
}

// Advance by `units` (at most cu.sb_left: never past the end of a tile).
template <int SB>
__device__ __forceinline__ void cursor_step(const GroupParams &P, Cursor &cu, int units) {
    cu.c += units * kUnitCodeBytes;
    cu.s += units * SB;
    cu.left -= units;
    cu.sb_left -= units;
    if (cu.sb_left == 0) {  // next tile
        if (cu.left == 0 && cu.q + 1 < P.count) {  // of the next problem
            ++cu.q;
            cu.c = P.prob[cu.q].codes;
            cu.s = P.prob[cu.q].scales;
            cu.left = problem_end(P, cu.q) - (int)P.prob[cu.q].unit_begin;
        }
        cu.sb_left = P.prob[cu.q].nsb;
    }
}

// Copy the next `cnt` (1 or 2) units of the cursor into a stage.  Units of one
// tile are contiguous in both planes, so a pair is one copy per plane; a pair
// that straddles two tiles takes one copy per unit and plane.
template <int SB, int SOFF>  // scale bytes per unit, offset of the scales in a stage
__device__ __forceinline__ void issue_stage(const GroupParams &P, Cursor &cu, int cnt, uint32_t dst, uint32_t bar,
                                            uint32_t leader) {
    arrive_expect_tx_pred(leader, bar, (uint32_t)(cnt * (kUnitCodeBytes + SB)));
    if (cu.sb_left >= cnt) {
        bulk_copy_pred(leader, dst, cu.c, (uint32_t)(cnt * kUnitCodeBytes), bar);
        bulk_copy_pred(leader, dst + SOFF, cu.s, (uint32_t)(cnt * SB), bar);
        cursor_step<SB>(P, cu, cnt);
    } else {
        for (int h = 0; h < cnt; ++h) {
            bulk_copy_pred(leader, dst + h * kUnitCodeBytes, cu.c, kUnitCodeBytes, bar);
            bulk_copy_pred(leader, dst + SOFF + h * SB, cu.s, SB, bar);
            cursor_step<SB>(P, cu, 1);
        }
    }
}

// ---- codec traits -----------------------------------------------------------
// TQ4_1S: codes are sign-magnitude ranks into the Lloyd-Max magnitudes, scales
// are fp16 (d0, d1) per 32-block.  NVFP4: codes are E2M1 values, scales are
// E4M3 bytes per 16-block, plus a per-tensor fp32 scale applied to y.
enum Codec : int { kCodecTQ4 = 0, kCodecNVFP4 = 1 };

__constant__ uint16_t c_e2m1_f16[8] = {0x0000u, 0x3800u, 0x3c00u, 0x3e00u, 0x4000u, 0x4200u, 0x4400u, 0x4600u};

template <int CODEC>
struct CodecTraits;

template <>
struct CodecTraits<kCodecTQ4> {
    static constexpr int kScaleBytes = 256;
    // fp16 value of a 4-bit code
    __device__ static uint32_t code_f16(int c) { return c_mag_f16[c & 7] | ((c & 8) ? 0x8000u : 0u); }
    // this lane's scale words for row `row` of the unit (4 blocks x (d0, d1))
    __device__ static uint4 load(uint32_t ss, int row) { return lds128(ss + row * 16); }
    // (scale of half 0, scale of half 1) of 32-column block j
    __device__ static float2 pair(const uint4 &w, int j) {
        const uint32_t v = pair_h2(w, j);
        return __half22float2(*reinterpret_cast<const __half2 *>(&v));
    }
    // the same pair as one fp16x2 word
    __device__ static uint32_t pair_h2(const uint4 &w, int j) { return j == 0 ? w.x : j == 1 ? w.y : j == 2 ? w.z : w.w; }
    // (d0, d1) of block j of row `row`
    __device__ static float2 block(uint32_t ss, int row, int j) {
        const uint32_t v = lds32(ss + row * 16 + j * 4);
        return __half22float2(*reinterpret_cast<const __half2 *>(&v));
    }
};

template <>
struct CodecTraits<kCodecNVFP4> {
    static constexpr int kScaleBytes = 128;
    __device__ static uint32_t code_f16(int c) { return c_e2m1_f16[c & 7] | ((c & 8) ? 0x8000u : 0u); }
    // 8 E4M3 bytes of row `row` (16-element blocks 0..7 of the superblock)
    __device__ static uint4 load(uint32_t ss, int row) {
        uint32_t a, b;
        asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(a), "=r"(b) : "r"(ss + row * 8));
        return make_uint4(a, b, 0u, 0u);
    }
    // 32-column block j covers 16-element blocks 2j (half 0) and 2j+1 (half 1)
    __device__ static float2 pair(const uint4 &w, int j) {
        const uint32_t h = pair_h2(w, j);
        return __half22float2(*reinterpret_cast<const __half2 *>(&h));
    }
    // the same pair as one fp16x2 word (E4M3 values are exact in fp16)
    __device__ static uint32_t pair_h2(const uint4 &w, int j) {
        const uint32_t word = (j < 2) ? w.x : w.y;
        const uint16_t two = (uint16_t)(word >> (16 * (j & 1)));
        uint32_t h;
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(two));
        return h;
    }
    // block scales of the two halves of 32-column block j of row `row`
    __device__ static float2 block(uint32_t ss, int row, int j) {
        uint16_t two;
        asm volatile("ld.shared.u16 %0, [%1];" : "=h"(two) : "r"(ss + row * 8 + j * 2));
        uint32_t h;
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(two));
        return __half22float2(*reinterpret_cast<const __half2 *>(&h));
    }
};

// Relaxed 64-bit global store / load (single-copy atomic: a value and its
// call tag are seen together or not at all).
__device__ __forceinline__ void st_relaxed_u64(uint64_t *p, uint64_t v) {
    asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t *p) {
    uint64_t v;
    asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

template <int NT>
struct AccTile {
    float v[NT][4];
};

// Activation row of accumulator v[a][b] of lane (g, t) once a tile segment is
// complete, or 32 (never below m) for an entry that carries nothing.  CM = 0:
// the multi-row kernel (column 2t + (b & 1) of n-tile a).  CM = 1, 2, 4: the
// half-block-combination kernels for 1, 2 and 4 activation rows, whose sums
// end in entries b = 0 (weight row g) and b = 2 (row g + 8) of the lanes that
// own an activation row: t = 0 (CM = 1), t = 0 and 2 (CM = 2), every t (CM = 4).
template <int CM>
__device__ __forceinline__ int acc_xrow(int a, int b, int t) {
    if constexpr (CM == 0) return 8 * a + 2 * t + (b & 1);
    else if constexpr (CM == 1) return (b & 1) ? 32 : 2 * t;
    else if constexpr (CM == 2) return ((b & 1) || (t & 1)) ? 32 : (t >> 1);
    else return (b & 1) ? 32 : t;
}

// Activation row whose fragments lane group g loads (rows past m repeat row
// m - 1; their results are never stored).  CM = 0: row 8a + g of n-tile a;
// CM = 1, 2, 4: the activation row of the B column g, g / (8 / CM).
template <int CM>
__device__ __forceinline__ int lane_xrow(int a, int g, int m) {
    if constexpr (CM == 0) return min(8 * a + g, m - 1);
    else return min(g / (8 / CM), m - 1);
}

// Products of one unit (16 rows x 128 columns) accumulated into acc: the
// unit's codes at shared address sc, its scales at ss, the activation
// fragments at xcur[a] + xoff.
template <int NT, typename CT>
__device__ __forceinline__ void unit_product(uint32_t sc, uint32_t ss, const uint16_t *const (&xcur)[NT], int xoff,
                                             uint32_t lut_lane, uint32_t off_c, int g, float (&acc)[NT][4]) {
    const uint4 c0 = lds128(sc + off_c);
    const uint4 c1 = lds128(sc + off_c + 512);
    const uint4 s0 = CT::load(ss, g);
    const uint4 s1 = CT::load(ss, g + 8);
    const uint32_t cw0[4] = {c0.x, c0.y, c0.z, c0.w};
    const uint32_t cw1[4] = {c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int j = 0; j < kSbBlocks; ++j) {
        uint4 xb[NT];
#pragma unroll
        for (int a = 0; a < NT; ++a) xb[a] = ldg_keep(xcur[a] + xoff + j * 32);
        // code byte b of word cw: logical byte t + 4b of the block
        const uint32_t a00 = lds_lut(prmt(cw0[j], lut_lane, 0x7604u));
        const uint32_t a01 = lds_lut(prmt(cw1[j], lut_lane, 0x7604u));
        const uint32_t a02 = lds_lut(prmt(cw0[j], lut_lane, 0x7614u));
        const uint32_t a03 = lds_lut(prmt(cw1[j], lut_lane, 0x7614u));
        const uint32_t a10 = lds_lut(prmt(cw0[j], lut_lane, 0x7624u));
        const uint32_t a11 = lds_lut(prmt(cw1[j], lut_lane, 0x7624u));
        const uint32_t a12 = lds_lut(prmt(cw0[j], lut_lane, 0x7634u));
        const uint32_t a13 = lds_lut(prmt(cw1[j], lut_lane, 0x7634u));
        if constexpr (NT >= 4) {
            // four n-tiles share A: scale the decoded centroids once, fp16(c *
            // d) (the prefill kernel's operand), and let the tensor cores
            // accumulate every half-block in fp32 (no FFMA per n-tile; with
            // fewer n-tiles the dependent-mma chains this makes cost more than
            // the FFMAs they save)
            const uint32_t pg = CT::pair_h2(s0, j), pg8 = CT::pair_h2(s1, j);
            const uint32_t g0 = prmt(pg, pg, 0x1010u), g1 = prmt(pg, pg, 0x3232u);    // (d0, d0), (d1, d1) of row g
            const uint32_t e0 = prmt(pg8, pg8, 0x1010u), e1 = prmt(pg8, pg8, 0x3232u);  // the same for row g + 8
            const uint32_t b00 = hmul2(a00, g0), b01 = hmul2(a01, e0), b02 = hmul2(a02, g0), b03 = hmul2(a03, e0);
            const uint32_t b10 = hmul2(a10, g1), b11 = hmul2(a11, e1), b12 = hmul2(a12, g1), b13 = hmul2(a13, e1);
#pragma unroll
            for (int a = 0; a < NT; ++a) {
                mma_acc(acc[a], b00, b01, b02, b03, xb[a].x, xb[a].y);
                mma_acc(acc[a], b10, b11, b12, b13, xb[a].z, xb[a].w);
            }
        } else {
            const float2 dg = CT::pair(s0, j);
            const float2 dg8 = CT::pair(s1, j);
#pragma unroll
            for (int a = 0; a < NT; ++a) {
                float d[4];
                mma_nv(d, a00, a01, a02, a03, xb[a].x, xb[a].y);
                acc[a][0] = fmaf(d[0], dg.x, acc[a][0]);
                acc[a][2] = fmaf(d[2], dg8.x, acc[a][2]);
                acc[a][1] = fmaf(d[1], dg.x, acc[a][1]);
                acc[a][3] = fmaf(d[3], dg8.x, acc[a][3]);
                mma_nv(d, a10, a11, a12, a13, xb[a].z, xb[a].w);
                acc[a][0] = fmaf(d[0], dg.y, acc[a][0]);
                acc[a][2] = fmaf(d[2], dg8.y, acc[a][2]);
                acc[a][1] = fmaf(d[1], dg.y, acc[a][1]);
                acc[a][3] = fmaf(d[3], dg8.y, acc[a][3]);
            }
        }
    }
}

// One activation row: the eight columns of B carry the eight half-blocks
// (c = 2j + h) of the unit, column c non-zero only in the products of
// half-block c (its four lanes g == c hold the activation, the others zero),
// so one accumulator chain keeps the eight partial sums apart.  Lane (g, t)
// ends with the half-block sums of block t for rows g and g + 8 and scales
// them with that block's two scales; the lanes' block sums are added when the
// tile segment is flushed.  xv: this lane's four activation values of
// half-block g (from the stage).
template <typename CT>
__device__ __forceinline__ void unit_product_m1(uint32_t sc, uint32_t ss, uint2 xv, uint32_t lut_lane,
                                                uint32_t off_c, int g, int t, float (&acc)[1][4]) {
    const uint4 c0 = lds128(sc + off_c);
    const uint4 c1 = lds128(sc + off_c + 512);
    const uint32_t cw0[4] = {c0.x, c0.y, c0.z, c0.w};
    const uint32_t cw1[4] = {c1.x, c1.y, c1.z, c1.w};
    // two accumulator chains, first halves (even columns) in d, second halves
    // (odd columns) in e: half the dependent-mma depth, and lane (g, t) reads
    // column 2t from d and column 2t + 1 from e
    float d[4], e[4];
#pragma unroll
    for (int j = 0; j < kSbBlocks; ++j) {
        // code byte b of word cw: logical byte t + 4b of the block
        const uint32_t a00 = lds_lut(prmt(cw0[j], lut_lane, 0x7604u));
        const uint32_t a01 = lds_lut(prmt(cw1[j], lut_lane, 0x7604u));
        const uint32_t a02 = lds_lut(prmt(cw0[j], lut_lane, 0x7614u));
        const uint32_t a03 = lds_lut(prmt(cw1[j], lut_lane, 0x7614u));
        const uint32_t a10 = lds_lut(prmt(cw0[j], lut_lane, 0x7624u));
        const uint32_t a11 = lds_lut(prmt(cw1[j], lut_lane, 0x7624u));
        const uint32_t a12 = lds_lut(prmt(cw0[j], lut_lane, 0x7634u));
        const uint32_t a13 = lds_lut(prmt(cw1[j], lut_lane, 0x7634u));
        const bool p0 = g == 2 * j, p1 = g == 2 * j + 1;
        if (j == 0) {
            mma_nv(d, a00, a01, a02, a03, p0 ? xv.x : 0u, p0 ? xv.y : 0u);
            mma_nv(e, a10, a11, a12, a13, p1 ? xv.x : 0u, p1 ? xv.y : 0u);
        } else {
            mma_acc(d, a00, a01, a02, a03, p0 ? xv.x : 0u, p0 ? xv.y : 0u);
            mma_acc(e, a10, a11, a12, a13, p1 ? xv.x : 0u, p1 ? xv.y : 0u);
        }
    }
    const float2 sg = CT::block(ss, g, t), sg8 = CT::block(ss, g + 8, t);
    acc[0][0] = fmaf(d[0], sg.x, acc[0][0]);
    acc[0][1] = fmaf(e[1], sg.y, acc[0][1]);
    acc[0][2] = fmaf(d[2], sg8.x, acc[0][2]);
    acc[0][3] = fmaf(e[3], sg8.y, acc[0][3]);
}

// Two or four activation rows (CM): the eight B columns hold CM rows x S = 8 /
// CM half-block slots.  Block j of the unit goes to accumulator chain k = j %
// CM and slot pair u = j / CM (its halves in slots 2u and 2u + 1), so column
// n = S * row + 2u + h carries half h of block u * CM + k of activation row
// `row`; the CM chains are independent, 8 / CM dependent MMAs deep each, and
// keep their half-block sums apart.  Lane (g, t) feeds column g:
// in chain k it supplies its words of block (g % S) / 2 * CM + k, half g % 2,
// of activation row g / S (xv[k], loaded by the caller), and zero in the
// other slots.  It ends with, per chain k, columns 2t and 2t + 1: the two
// halves of block (t % (S / 2)) * CM + k of activation row 2t / S, which it
// scales by that block's (d0, d1).
template <int CM, typename CT>
__device__ __forceinline__ void unit_product_cm(uint32_t sc, uint32_t ss, const uint2 (&xv)[CM], uint32_t lut_lane,
                                                uint32_t off_c, int g, int t, float (&acc)[1][4]) {
    static_assert(CM == 2 || CM == 4, "two or four activation rows");
    constexpr int S = 8 / CM;
    const uint4 c0 = lds128(sc + off_c);
    const uint4 c1 = lds128(sc + off_c + 512);
    const uint32_t cw0[4] = {c0.x, c0.y, c0.z, c0.w};
    const uint32_t cw1[4] = {c1.x, c1.y, c1.z, c1.w};
    const int slot = g % S;  // this lane's B column slot
    float d[CM][4];
#pragma unroll
    for (int j = 0; j < kSbBlocks; ++j) {
        const uint32_t a00 = lds_lut(prmt(cw0[j], lut_lane, 0x7604u));
        const uint32_t a01 = lds_lut(prmt(cw1[j], lut_lane, 0x7604u));
        const uint32_t a02 = lds_lut(prmt(cw0[j], lut_lane, 0x7614u));
        const uint32_t a03 = lds_lut(prmt(cw1[j], lut_lane, 0x7614u));
        const uint32_t a10 = lds_lut(prmt(cw0[j], lut_lane, 0x7624u));
        const uint32_t a11 = lds_lut(prmt(cw1[j], lut_lane, 0x7624u));
        const uint32_t a12 = lds_lut(prmt(cw0[j], lut_lane, 0x7634u));
        const uint32_t a13 = lds_lut(prmt(cw1[j], lut_lane, 0x7634u));
        const int k = j % CM, u = j / CM;
        const bool p0 = slot == 2 * u, p1 = slot == 2 * u + 1;
        if (u == 0)
            mma_nv(d[k], a00, a01, a02, a03, p0 ? xv[k].x : 0u, p0 ? xv[k].y : 0u);
        else
            mma_acc(d[k], a00, a01, a02, a03, p0 ? xv[k].x : 0u, p0 ? xv[k].y : 0u);
        mma_acc(d[k], a10, a11, a12, a13, p1 ? xv[k].x : 0u, p1 ? xv[k].y : 0u);
    }
#pragma unroll
    for (int k = 0; k < CM; ++k) {
        const int blk = (t % (S / 2)) * CM + k;
        const float2 sg = CT::block(ss, g, blk), sg8 = CT::block(ss, g + 8, blk);
        acc[0][0] = fmaf(d[k][0], sg.x, acc[0][0]);
        acc[0][1] = fmaf(d[k][1], sg.y, acc[0][1]);
        acc[0][2] = fmaf(d[k][2], sg8.x, acc[0][2]);
        acc[0][3] = fmaf(d[k][3], sg8.y, acc[0][3]);
    }
}

// Activation words a half-block-combination lane needs per unit (CM = 1, 2,
// 4): one 8-byte word per chain.
template <int CM>
struct XWords {
    uint2 w[CM == 0 ? 1 : CM];
};

// Half-block-combination unit with its activation words already loaded (a
// no-op for the multi-row kernels, which never take that path).
template <int NT, int CM, typename CT>
__device__ __forceinline__ void unit_xv(uint32_t sc, uint32_t ss, const XWords<CM> &xv, uint32_t lut_lane,
                                        uint32_t off_c, int g, int t, float (&acc)[NT][4]) {
    if constexpr (CM == 1) unit_product_m1<CT>(sc, ss, xv.w[0], lut_lane, off_c, g, t, acc);
    else if constexpr (CM == 2 || CM == 4) unit_product_cm<CM, CT>(sc, ss, xv.w, lut_lane, off_c, g, t, acc);
}

// The activation words of one unit for a half-block-combination lane: chain k
// at byte offset 64 k from the lane's first word (xb).
template <int CM>
__device__ __forceinline__ XWords<CM> load_xwords(const char *xb) {
    XWords<CM> xv;
#pragma unroll
    for (int k = 0; k < (CM == 0 ? 1 : CM); ++k) xv.w[k] = ldg64(xb + 64 * k);
    return xv;
}

// One unit's products; the activation fragments of its superblock start at
// xcur[a] + xoff.
template <int NT, int CM, typename CT>
__device__ __forceinline__ void unit_any(uint32_t sc, uint32_t ss, const uint16_t *const (&xcur)[NT], int xoff,
                                         uint32_t lut_lane, uint32_t off_c, uint32_t off_x, int g, int t,
                                         float (&acc)[NT][4]) {
    if constexpr (CM > 0) {
        static_assert(NT == 1, "the half-block-combination kernels use one n-tile");
        const XWords<CM> xv = load_xwords<CM>(reinterpret_cast<const char *>(xcur[0] + xoff) + off_x);
        unit_xv<NT, CM, CT>(sc, ss, xv, lut_lane, off_c, g, t, acc);
    } else {
        unit_product<NT, CT>(sc, ss, xcur, xoff, lut_lane, off_c, g, acc);
    }
}

// What the first contributor of a split tile needs to compute a missing
// contribution itself: a free shared-memory stage of its ring and its lane
// constants for the unit products.
struct StealCtx {
    uint32_t smem;
    uint32_t lut_lane;
    uint32_t off_c;
    uint32_t off_x;
};

// Half-block-combination kernels: add the two halves of every weight row,
// then the blocks the lanes of one activation row share (as when a tile
// segment ends).
template <int NT, int CM>
__device__ __forceinline__ void combine_rows(float (&acc)[NT][4]) {
    if constexpr (CM > 0) {
        float vg = acc[0][0] + acc[0][1], vg8 = acc[0][2] + acc[0][3];
        if constexpr (CM <= 2) {
            vg += __shfl_xor_sync(kFull, vg, 1);
            vg8 += __shfl_xor_sync(kFull, vg8, 1);
        }
        if constexpr (CM == 1) {
            vg += __shfl_xor_sync(kFull, vg, 2);
            vg8 += __shfl_xor_sync(kFull, vg8, 2);
        }
        acc[0][0] = vg;
        acc[0][2] = vg8;
    }
}

// The sums warp w would store for its part [va, vb) of tile (q, r),
// recomputed by this warp (same units, same order, same arithmetic: the
// result is bit-identical).  Each unit is copied into the free stage with
// plain loads and multiplied as in the main loop.
template <int NT, int CM, int CODEC>
__device__ __noinline__ AccTile<NT> steal_partial(const GroupParams &P, int q, int va, int vb, const StealCtx &cx) {
    using CT = CodecTraits<CODEC>;
    constexpr int SB = CT::kScaleBytes;
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const DevProblem &pr = P.prob[q];
    float acc[NT][4];
#pragma unroll
    for (int a = 0; a < NT; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
    for (int v = va; v < vb; ++v) {
        const int local = v - (int)pr.unit_begin;
        const int sb = local % pr.nsb;
        const uint8_t *c = pr.codes + (int64_t)local * kUnitCodeBytes;
        const uint8_t *sc = pr.scales + (int64_t)local * SB;
        const uint4 c0 = ldg_keep(c + 32 * lane), c1 = ldg_keep(c + 32 * lane + 16);
        __syncwarp();  // the previous unit's products have read the stage
        asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(cx.smem + 32 * lane), "r"(c0.x), "r"(c0.y),
                     "r"(c0.z), "r"(c0.w)
                     : "memory");
        asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(cx.smem + 32 * lane + 16), "r"(c1.x), "r"(c1.y),
                     "r"(c1.z), "r"(c1.w)
                     : "memory");
        if (lane < SB / 16) {
            const uint4 s4 = ldg_keep(sc + 16 * lane);
            asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(cx.smem + kUnitCodeBytes + 16 * lane),
                         "r"(s4.x), "r"(s4.y), "r"(s4.z), "r"(s4.w)
                         : "memory");
        }
        __syncwarp();
        const uint16_t *xcur[NT];
#pragma unroll
        for (int a = 0; a < NT; ++a)
            xcur[a] = pr.xrot + ((int64_t)lane_xrow<CM>(a, g, P.m) * pr.nsb + sb) * 128 + t * 8;
        unit_any<NT, CM, CT>(cx.smem, cx.smem + kUnitCodeBytes, xcur, 0, cx.lut_lane, cx.off_c, cx.off_x, g, t, acc);
    }
    __syncwarp();
    combine_rows<NT, CM>(acc);
    const float ts = pr.tscale ? __ldg(pr.tscale) : 1.0f;  // NVFP4 tensor scale
    AccTile<NT> out;
#pragma unroll
    for (int a = 0; a < NT; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) out.v[a][b] = acc[a][b] * ts;
    return out;
}

// The first contributor of a split tile: its own sums plus those of warps
// gw+1 .. last (the owner of the tile's last unit), added in warp order.
// The later contributors store their sums at the start of their ranges, so
// normally every word already carries this call's tag; a contribution still
// missing after a short bounded poll (its warp may not have been able to
// start: nothing guarantees that the grid is resident at once) is computed
// here from the packed weights instead.  Nothing waits unboundedly for
// another CTA, and the result is the same bits either way.
template <int NT, int CM, int OT, int CODEC>
__device__ __noinline__ void reduce_first(const GroupParams &P, int q, int r, int tile_lo, int tile_hi, int gw,
                                          uint32_t tag, AccTile<NT> acc, uint32_t smem, uint32_t lut_lane,
                                          uint32_t off_c, uint32_t off_x) {
    constexpr int kMcap = 8 * NT;
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const DevProblem &pr = P.prob[q];
    const int64_t gt = pr.tile_begin + r;
    const int U = (int)P.units, W = P.total_warps;
    const int last = (int)div_floor((int64_t)tile_hi * W - 1, U, P.inv_units);
    const StealCtx cx = {smem, lut_lane, off_c, off_x};
    const float ts = pr.tscale ? __ldg(pr.tscale) : 1.0f;  // NVFP4 tensor scale
    AccTile<NT> sum;
#pragma unroll
    for (int a = 0; a < NT; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) sum.v[a][b] = acc.v[a][b] * ts;
    uint64_t t0 = 0;
    for (int w = gw + 1; w <= last; ++w) {
        const uint64_t *slot = P.partials + (gt + w) * (int64_t)(16 * kMcap);
        bool present = false;
        AccTile<NT> part;
        for (uint32_t it = 0;; ++it) {  // bounded poll for the tagged words
            bool ok = !P.steal_all;
#pragma unroll
            for (int a = 0; a < NT; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int xrow = acc_xrow<CM>(a, b, t);
                    part.v[a][b] = 0.f;
                    if (xrow >= P.m) continue;
                    const uint64_t v = ld_relaxed_u64(slot + xrow * 16 + g + ((b & 2) ? 8 : 0));
                    ok = ok && (uint32_t)(v >> 32) == tag;
                    part.v[a][b] = __uint_as_float((uint32_t)v);
                }
            present = __all_sync(kFull, ok);
            if (present || P.steal_all) break;
            if (t0 == 0) t0 = __shfl_sync(kFull, global_ns(), 0);
            // a vote, so that all 32 lanes stop polling together (a lane that
            // left alone would leave the others in the next full-warp vote)
            if (__any_sync(kFull, global_ns() - t0 > P.steal_after_ns || it >= (1u << 24))) break;
        }
        if (!present) {
            const int64_t wa = div_floor((int64_t)w * U, W, P.inv_warps), wb = div_floor((int64_t)(w + 1) * U, W, P.inv_warps);
            part = steal_partial<NT, CM, CODEC>(P, q, (int)max(wa, (int64_t)tile_lo), (int)min(wb, (int64_t)tile_hi),
                                                cx);
        }
#pragma unroll
        for (int a = 0; a < NT; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) sum.v[a][b] += part.v[a][b];
    }
#pragma unroll
    for (int a = 0; a < NT; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int xrow = acc_xrow<CM>(a, b, t);
            const int wrow = r * 16 + g + ((b & 2) ? 8 : 0);
            if (xrow < P.m && wrow < pr.n)
                store1<OT>(pr.y + ((int64_t)xrow * pr.ldy + wrow) * ElemSize<OT>::value, sum.v[a][b]);
        }
}

// Write the accumulators of a finished tile segment: straight to Y when this
// warp covered the whole tile, else (a later contributor of a split tile)
// through the tagged partial sums.
//
// A tile split over warps gw0 < ... < gwk: the tile starts in gw0's range and
// is that warp's last segment, reached at the end of its work; for every
// later contributor it is the first segment, reached at the start.  So the
// later contributors store their sums, each as one 64-bit word (fp32 value,
// call tag), with no fence and no atomic, and gw0 adds them (own part first,
// then warp order: deterministic) in reduce_first, after its main loop.
template <int NT, int CM, int OT>
__device__ __forceinline__ void flush_segment(const GroupParams &P, int q, int r, int tile_lo, int tile_hi, int u0,
                                           int u1, int gw, uint32_t tag, const float (&acc_in)[NT][4]) {
    constexpr int kMcap = 8 * NT;
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const DevProblem &pr = P.prob[q];
    float acc[NT][4];
    const float ts = pr.tscale ? __ldg(pr.tscale) : 1.0f;  // NVFP4 tensor scale
#pragma unroll
    for (int a = 0; a < NT; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = acc_in[a][b] * ts;
    const int64_t gt = pr.tile_begin + r;
    const int row_g = r * 16 + g, row_g8 = row_g + 8;
    if (u0 <= tile_lo && tile_hi <= u1) {
#pragma unroll
        for (int a = 0; a < NT; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int xrow = acc_xrow<CM>(a, b, t);
                const int wrow = (b & 2) ? row_g8 : row_g;
                if (xrow < P.m && wrow < pr.n)
                    store1<OT>(pr.y + ((int64_t)xrow * pr.ldy + wrow) * ElemSize<OT>::value, acc[a][b]);
            }
        return;
    }
    // a later contributor: store the tagged sums and go on
    const uint64_t tag_hi = (uint64_t)tag << 32;
    uint64_t *slot = P.partials + (gt + gw) * (int64_t)(16 * kMcap);
#pragma unroll
    for (int a = 0; a < NT; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int xrow = acc_xrow<CM>(a, b, t);
            const int wrow = g + ((b & 2) ? 8 : 0);
            if (xrow < P.m) st_relaxed_u64(slot + xrow * 16 + wrow, tag_hi | __float_as_uint(acc[a][b]));
        }
}

// The tile segment ending at unit u is complete: write it out, reset the
// accumulators and move the segment state to the tile of unit u.
template <int NT, int CM, int OT, int CODEC>
__device__ __forceinline__ void end_segment(const GroupParams &P, int u, int u0, int u1, int gw, int g, int t,
                                         uint32_t tag, int &q,
                                         int &prob_end, int &nsb, int &r, int &tile_lo, int &seg_end,
                                         const uint16_t *(&xcur)[NT], float (&acc)[NT][4]) {
    // weight rows g, g + 8: add the two halves, then the blocks the lanes of
    // one activation row share (four lanes for CM = 1, two for CM = 2)
    combine_rows<NT, CM>(acc);
    // the first contributor of a split tile meets it at the end of its range
    // (u == u1): its sums stay in acc for reduce_first after the main loop
    if (tile_lo >= u0 && tile_lo + nsb > u1) return;
    flush_segment<NT, CM, OT>(P, q, r, tile_lo, tile_lo + nsb, u0, u1, gw, tag, acc);
#pragma unroll
    for (int a = 0; a < NT; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
    if (u < u1) {
        if (u == prob_end) {  // next problem: new tiles, new activation
            ++q;
            prob_end = problem_end(P, q);
            nsb = P.prob[q].nsb;
            r = 0;
            tile_lo = u;
        } else {
            ++r;
            tile_lo += nsb;
        }
        seg_end = min(tile_lo + nsb, u1);
#pragma unroll
        for (int a = 0; a < NT; ++a) {  // back to superblock 0 of the activation
            const int xrow = lane_xrow<CM>(a, g, P.m);
            xcur[a] = P.prob[q].xrot + (int64_t)xrow * nsb * 128 + t * 8;
        }
    }
}

template <int NT, int CM, int OT, int CODEC>
__global__ void __launch_bounds__(warps_for(CM > 0, NT) * 32, 1) gemv_group_kernel(const __grid_constant__ GroupParams P) {
    using G = Geometry<warps_for(CM > 0, NT), (CM > 0)>;
    using RG = Ring<(CM > 0)>;
    using CT = CodecTraits<CODEC>;
    constexpr int SB = CT::kScaleBytes;
    constexpr int kPerStage = RG::kPerStage, kStageBytes = RG::kStageBytes, kStageScaleOff = RG::kStageScaleOff;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gw = blockIdx.x * G::kWarps + warp;
    const uint32_t base = (uint32_t)__cvta_generic_to_shared(smem);
    if (base > G::kMaxSmemBase) {  // layout precondition (checked, never expected)
        if (threadIdx.x == 0) atomicOr(P.header + kHeaderStatus, kStatusLayout);
        return;
    }
    const uint32_t ring =
        warp < G::kLowWarps ? G::kLowRings + warp * G::kRingWarpBytes : kHighRings + (warp - G::kLowWarps) * G::kRingWarpBytes;
    const uint32_t bars = G::kBarAddr + warp * (kStages * 8);
    const bool active = gw < P.total_warps;
    const int U = (int)P.units;
    const int W = P.total_warps;
    const int u0 = active ? (int)div_floor((int64_t)gw * U, W, P.inv_warps) : 0;
    const int u1 = active ? (int)div_floor((int64_t)(gw + 1) * U, W, P.inv_warps) : 0;

    // ---- prologue: barriers, first bulk copies, lookup table -------------
    // (the packed weights never depend on the preceding grid, so the first
    // stage's copies start before the programmatic-dependency wait; the
    // other stages follow it: a smaller burst ahead of the wait lets the
    // pre-rotation's activation loads, which run meanwhile, come back sooner)
    Cursor cu = {nullptr, nullptr, 0, 0, 0};
    int pv = u0;  // next unit to copy
    if (active) {
        if (lane == 0) {
            for (int i = 0; i < kStages; ++i) mbar_init(bars + 8 * i, 1);
            fence_mbar_init();
        }
        __syncwarp();
        cu = cursor_at<SB>(P, u0);
        if (pv < u1) {
            const int cnt = min(kPerStage, u1 - pv);
            const bool skip = P.inject_skip && gw == 0;
            issue_stage<SB, kStageScaleOff>(P, cu, cnt, ring, bars, lane == 0 && !skip);
            pv += cnt;
        }
    }
    {
        // entry v holds the same half2 in all 32 lane slots (the first 128 of
        // its 256 bytes)
        uint4 *lut = reinterpret_cast<uint4 *>(smem + (kLutAddr - base));
        for (int idx = threadIdx.x; idx < 256 * 8; idx += G::kThreads) {  // entry v: 8 x 16 bytes
            const int v = idx >> 3;
            const uint32_t e = CT::code_f16(v & 15) | (CT::code_f16(v >> 4) << 16);
            lut[v * 16 + (idx & 7)] = make_uint4(e, e, e, e);
        }
    }
    __syncthreads();
    grid_dependency_wait();  // pre-rotated activations and the header are ready
    // every CTA of this grid is resident: the next pre-rotation may launch and
    // wait (it waits for this grid's completion before writing anything)
    grid_dependents_launch();
    if (!active) return;
    for (int i = 1; i < kStages && pv < u1; ++i) {  // the ring's other stages
        const int cnt = min(kPerStage, u1 - pv);
        issue_stage<SB, kStageScaleOff>(P, cu, cnt, ring + i * kStageBytes, bars + 8 * i, lane == 0);
        pv += cnt;
    }
    // this call's tag (advanced by the launch that prepared the header)
    const uint32_t tag = *reinterpret_cast<volatile const unsigned *>(P.header + kHeaderTag);

    const int g = lane >> 2, t = lane & 3;
    // PRMT operand: byte 0 = lane*4, bytes 2..3 = table base >> 16
    const uint32_t lut_lane = kLutAddr | ((uint32_t)lane * 4u);
    // this lane's 16 code bytes of rows g and g+8 in a unit
    const uint32_t off_c = g * 64 + t * 16;
    // half-block-combination kernels: byte offset of this lane's first 8-byte
    // activation word (block (g % S) / 2 * CM, half g % 2, S = 8 / CM) in a
    // superblock's fragments [4 blocks][4 t][8 halves], relative to xcur
    // (which already holds t); chain k adds 64 k
    constexpr int kSlots = 8 / (CM == 0 ? 1 : CM);
    const uint32_t off_x = ((g % kSlots) >> 1) * (CM == 0 ? 1 : CM) * 64 + (g & 1) * 8;

    // ---- segment state: the tile the current unit belongs to ---------------
    int q = problem_of(P, u0);
    int prob_end = problem_end(P, q);
    int nsb = P.prob[q].nsb;
    int r, sb, tile_lo;
    {
        const int local = u0 - (int)P.prob[q].unit_begin;
        r = local / nsb;
        sb = local - r * nsb;
        tile_lo = (int)P.prob[q].unit_begin + r * nsb;
    }
    int seg_end = min(tile_lo + nsb, u1);
    // activation fragments: rows past m repeat row m-1 (their outputs are never
    // stored), so every lane loads without a predicate; xcur[a] walks the
    // superblocks of the current unit (128 halves per superblock)
    const uint16_t *xcur[NT];
#pragma unroll
    for (int a = 0; a < NT; ++a) {
        const int xrow = lane_xrow<CM>(a, g, P.m);
        xcur[a] = P.prob[q].xrot + ((int64_t)xrow * nsb + sb) * 128 + t * 8;
    }

    float acc[NT][4];
#pragma unroll
    for (int a = 0; a < NT; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;

    int stage = 0;
    uint32_t parity = 0;
    int u = u0;
    while (u < u1) {
        const uint32_t st = ring + stage * kStageBytes, bar = bars + 8 * stage;
        {
            bool ok = mbar_try(bar, parity);
            if (!__all_sync(kFull, ok)) {
                ok = ok || mbar_wait_slow(bar, parity, P.timeout_ns);
                if (!__all_sync(kFull, ok)) {
                    // report, then let the copies still in flight land before leaving
                    if (lane == 0) {
                        atomicOr(P.header + kHeaderStatus, kStatusTimeout);
                        int s2 = stage;
                        uint32_t p2 = parity;
                        for (int i = 1; i < kStages && u + kPerStage * i < pv; ++i) {
                            if (++s2 == kStages) { s2 = 0; p2 ^= 1u; }
                            mbar_wait_slow(bars + 8 * s2, p2, P.timeout_ns);
                        }
                    }
                    __syncwarp();
                    return;
                }
            }
        }
        const int cnt = min(kPerStage, u1 - u);  // units held by this stage
        if (CM > 0 && cnt == kPerStage && u + kPerStage <= seg_end) {
            // common half-block-combination case: every unit of the stage
            // belongs to the current tile segment; their activation words are
            // loaded first (the multi-row kernels take the loop below, which
            // keeps one unit's operands live at a time)
            const char *xb = reinterpret_cast<const char *>(xcur[0]) + off_x;
            XWords<CM> xv[kPerStage];
#pragma unroll
            for (int h = 0; h < kPerStage; ++h) xv[h] = load_xwords<CM>(xb + 256 * h);  // 128 halves per superblock
#pragma unroll
            for (int h = 0; h < kPerStage; ++h)
                unit_xv<NT, CM, CT>(st + h * kUnitCodeBytes, st + kStageScaleOff + h * SB, xv[h], lut_lane, off_c, g,
                                    t, acc);
#pragma unroll
            for (int a = 0; a < NT; ++a) xcur[a] += 128 * kPerStage;
            u += kPerStage;
            if (u == seg_end)
                end_segment<NT, CM, OT, CODEC>(P, u, u0, u1, gw, g, t, tag, q, prob_end, nsb, r, tile_lo, seg_end, xcur, acc);
        } else {
            for (int h = 0; h < cnt; ++h) {
                unit_any<NT, CM, CT>(st + h * kUnitCodeBytes, st + kStageScaleOff + h * SB, xcur, 0, lut_lane, off_c,
                                     off_x, g, t, acc);
#pragma unroll
                for (int a = 0; a < NT; ++a) xcur[a] += 128;
                ++u;
                if (u == seg_end)
                    end_segment<NT, CM, OT, CODEC>(P, u, u0, u1, gw, g, t, tag, q, prob_end, nsb, r, tile_lo, seg_end, xcur, acc);
            }
        }
        __syncwarp();  // every lane has read the stage: it may be refilled
        if (pv < u1) {
            const int c2 = min(kPerStage, u1 - pv);
            issue_stage<SB, kStageScaleOff>(P, cu, c2, st, bar, lane == 0);
            pv += c2;
        }
        stage = (stage == kStages - 1) ? 0 : stage + 1;
        parity ^= (stage == 0) ? 1u : 0u;
    }
    // the first contributor of a split tile (its last segment, still in acc);
    // no copy is in flight any more, so the ring may serve as scratch
    if (tile_lo >= u0 && tile_lo + nsb > u1) {
        AccTile<NT> own;
#pragma unroll
        for (int a = 0; a < NT; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) own.v[a][b] = acc[a][b];
        reduce_first<NT, CM, OT, CODEC>(P, q, r, tile_lo, tile_lo + nsb, gw, tag, own, ring, lut_lane, off_c, off_x);
    }
}

// Base offset of dynamic shared memory in a CTA's shared window (the
// per-block reserved system area), queried once per device.
uint32_t dynamic_smem_base() {
    static uint32_t cached[256];
    static bool have[256];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return 1024;
    if (!have[dev]) {
        int reserved = 0;
        if (cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess)
            reserved = 1024;
        cached[dev] = (uint32_t)reserved;
        have[dev] = true;
    }
    return cached[dev];
}

template <int NT, int CM, int CODEC>
cudaError_t launch_nt(const GroupParams &prm, int dtype, int grid, bool programmatic, cudaStream_t stream) {
    using G = Geometry<warps_for(CM > 0, NT), (CM > 0)>;
    const uint32_t smem = G::smem_bytes_for_base(dynamic_smem_base());
    const int kSmemBytes = (int)smem;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(G::kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    // (no warp depends on another CTA being resident: a split tile's first warp
    // computes a contribution that does not arrive, so a plain launch, which
    // may start on the SMs that the previous kernel frees, is enough)
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = programmatic ? 1 : 0;
    cudaError_t err;
    switch (dtype) {
        case kF32:
            err = cudaFuncSetAttribute(gemv_group_kernel<NT, CM, kF32, CODEC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
            if (err != cudaSuccess) return err;
            return cudaLaunchKernelEx(&cfg, gemv_group_kernel<NT, CM, kF32, CODEC>, prm);
        case kBF16:
            err = cudaFuncSetAttribute(gemv_group_kernel<NT, CM, kBF16, CODEC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
            if (err != cudaSuccess) return err;
            return cudaLaunchKernelEx(&cfg, gemv_group_kernel<NT, CM, kBF16, CODEC>, prm);
        case kF16:
            err = cudaFuncSetAttribute(gemv_group_kernel<NT, CM, kF16, CODEC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
            if (err != cudaSuccess) return err;
            return cudaLaunchKernelEx(&cfg, gemv_group_kernel<NT, CM, kF16, CODEC>, prm);
        default:
            return cudaErrorInvalidValue;
    }
}

}  // namespace

void set_debug_flags(uint32_t flags) { g_debug_flags = flags; }
uint32_t debug_flags() { return g_debug_flags; }

GroupPlan plan_group(const int64_t *n, const int64_t *k, int count, int64_t m, int sm_count) {
    GroupPlan pl = {};
    for (int i = 0; i < count; ++i) {
        pl.tiles += tiles(n[i]);
        pl.units += tiles(n[i]) * superblocks(k[i]);
    }
    // up to four activation rows run a half-block-combination kernel (see
    // launch_group_codec)
    const int kWarps = warps_for(combo_rows(m) > 0, (int)((m > 32 ? 32 : (m < 1 ? 1 : m)) + 7) / 8);
    int64_t want = (pl.units + kWarps - 1) / kWarps;  // at least one unit per warp
    if (want > sm_count) want = sm_count;
    if (want < 1) want = 1;
    pl.grid = (int)want;
    const int64_t warps = want * kWarps;
    pl.total_warps = (int)(pl.units < warps ? pl.units : warps);
    const int64_t mm = m < 1 ? 1 : (m > 32 ? 32 : m);
    pl.mcap = (int)(8 * ((mm + 7) / 8));
    pl.partial_bytes = round_up((size_t)(pl.tiles + pl.total_warps) * 16u * (size_t)pl.mcap * 8u, 256);
    return pl;
}

template <int CODEC>
cudaError_t launch_group_codec(const GemvProblem *probs, int count, int64_t m, int ydtype, const GroupPlan &plan,
                               unsigned *header, uint64_t *partials, bool programmatic, cudaStream_t stream) {
    if (count < 1 || count > kMaxProblems) return cudaErrorInvalidValue;
    GroupParams prm = {};
    int64_t ub = 0, tb = 0;
    for (int i = 0; i < count; ++i) {
        DevProblem &d = prm.prob[i];
        d.codes = probs[i].codes;
        d.scales = reinterpret_cast<const uint8_t *>(probs[i].scales);
        d.xrot = probs[i].xrot;
        d.tscale = probs[i].tensor_scale;
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
    if (ub != plan.units || ub >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    prm.units = ub;
    prm.total_warps = plan.total_warps;
    prm.partials = partials;
    prm.header = header;
    prm.inject_skip = (g_debug_flags & 1u) ? 1 : 0;
    prm.inv_units = 1.0 / (double)prm.units;
    prm.inv_warps = 1.0 / (double)prm.total_warps;
    prm.timeout_ns = prm.inject_skip ? kDebugTimeoutNs : kTimeoutNs;
    prm.steal_after_ns = kStealAfterNs;
    prm.steal_all = (g_debug_flags & kDebugStealAll) ? 1 : 0;
    // the partial-slot stride is 16 * 8 * NT floats: NT must match plan.mcap
    const int nt = plan.mcap / 8;
    const int cm = nt == 1 ? combo_rows(m) : 0;
    // the plan's warps must all exist in the launched grid
    if (plan.total_warps > (int64_t)plan.grid * warps_for(cm > 0, nt)) return cudaErrorInvalidValue;
    if (cm == 1) return launch_nt<1, 1, CODEC>(prm, ydtype, plan.grid, programmatic, stream);
    if (cm == 2) return launch_nt<1, 2, CODEC>(prm, ydtype, plan.grid, programmatic, stream);
    if (cm == 4) return launch_nt<1, 4, CODEC>(prm, ydtype, plan.grid, programmatic, stream);
    switch (nt) {
        case 1: return launch_nt<1, 0, CODEC>(prm, ydtype, plan.grid, programmatic, stream);
        case 2: return launch_nt<2, 0, CODEC>(prm, ydtype, plan.grid, programmatic, stream);
        case 3: return launch_nt<3, 0, CODEC>(prm, ydtype, plan.grid, programmatic, stream);
        case 4: return launch_nt<4, 0, CODEC>(prm, ydtype, plan.grid, programmatic, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_group(const GemvProblem *probs, int count, int64_t m, int ydtype, const GroupPlan &plan,
                         unsigned *header, uint64_t *partials, bool programmatic, cudaStream_t stream) {
    return launch_group_codec<kCodecTQ4>(probs, count, m, ydtype, plan, header, partials, programmatic, stream);
}

cudaError_t launch_group_nvfp4(const GemvProblem *probs, int count, int64_t m, int ydtype, const GroupPlan &plan,
                               unsigned *header, uint64_t *partials, bool programmatic, cudaStream_t stream) {
    return launch_group_codec<kCodecNVFP4>(probs, count, m, ydtype, plan, header, partials, programmatic, stream);
}

}  // namespace tq
