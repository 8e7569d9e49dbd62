// tq_tcgemv.cu -- fused TQ4_1S dequant skinny GEMM (9 <= m <= 32 by default)
// on the fifth-generation tensor cores, with the decoded weights in tensor
// memory.
//
// Method: TQ4_1S page ("企业官网建设流程全解析", hotelren.com/news/5458160),
// section 解码速度：分硬件汇总: the activation is rotated once with the block
// transform, after which each weight contributes centroid(code) * scale * x_rot:
//
//   Y[i][r] = sum_blocks sum_e (c(code[r][e]) * d[r][half(e)]) * xrot[i][e]
//
// with xrot = fp16(H(s .* x)/32) and the weight operand fp16(c * d).
//
// B200 design:
//  * Big unit (BU) = 128 weight rows (eight 16-row tiles) x one 128-column
//    superblock; a pipeline step is a BU pair (two consecutive superblocks of
//    one row block).  The pairs of all matrices of a group form one index
//    space, split into equal contiguous ranges, one per CTA (one per SM).
//  * Warp 0 streams each pair's codes and scales into a weight stage with two
//    3-D TMA box copies (eight 2 KB code runs, eight 512-byte scale runs) and
//    the pair's two activation superblocks into an activation slot.
//  * Sixteen decode warps in four groups (group g takes the pairs i = g mod 4):
//    thread = one weight row.  It reads its row's code and scale bytes from the
//    stage, turns them into fp16 centroids with byte permutes against register
//    tables (no shared-memory table), multiplies by the half-block scale in
//    fp16 and writes the row's operands into tensor memory with tcgen05.st,
//    half a superblock (64 columns) at a time, double buffered.
//  * One MMA-issuing thread per group issues tcgen05.mma (M = 128, N = 16 or
//    32, K = 16) with A read from tensor memory and B, the pre-rotated
//    activation, from the activation slot, into the group's own fp32
//    accumulators in tensor memory (two per group, so the epilogue of one row
//    block overlaps the next); tcgen05.commit releases the A halves, the
//    activation slot and, at a row block's end, the accumulator.
//  * Four epilogue warps add the four groups' accumulators in group order
//    (tcgen05.ld, thread = row).  A row block that one CTA covered entirely
//    goes straight to Y; one that is split between CTAs is combined by the
//    last contributor to arrive: every contributor stores its partial sums,
//    then counts itself on the row block's call-tagged counter; the one that
//    completes the count adds all partial sums in CTA order (deterministic)
//    and stores Y.  No CTA ever waits for another, so nothing depends on the
//    grid being co-resident.
//  * One activation row uses a compact B: the activation's 128 columns as one
//    contiguous 256-byte run, described with a 16-byte leading-dimension
//    stride, so B row 0 is the activation and rows 1..15 (which only feed
//    output columns nobody reads) are shifted copies.
//  * Every mbarrier wait is bounded in time and reports through the
//    workspace status word; the kernel then drains its copies and MMAs and
//    releases tensor memory.
// Measured limits on B200 (why it is used from 9 rows only): a tcgen05.mma
// issue takes ~55 cycles per issuing thread whatever N, and a 128-row unit
// reads eight separate tile streams (runs of 2 KB), which HBM serves well below
// its streaming rate; at one row the mma.sync kernel, whose warps stream 5 KB
// runs, is faster.
#include <cuda.h>

#include <mutex>

#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {

namespace {

constexpr int kTcGroups = 4;                       // decode warp groups, each with its own MMA issuer
constexpr int kTcDecWarp0 = 1;                     // warp 0: producer and tensor-memory allocator
constexpr int kTcIssWarp0 = kTcDecWarp0 + 4 * kTcGroups;  // one MMA-issuing warp per group
constexpr int kTcEpiWarp0 = kTcIssWarp0 + kTcGroups;
constexpr int kTcWarps = kTcEpiWarp0 + 4;          // + four epilogue warps
constexpr int kTcThreads = kTcWarps * 32;
constexpr int kBuCodeBytes = 8 * 1024;
constexpr int kBuScaleBytes = 8 * 256;
constexpr int kTmemCols = 512;
// tensor-memory columns: accumulator (g, b) at (2g + b) * N (N <= 32: columns
// [0, 256)); the A operands of group g at 256 + 64 g, two halves of 32
// columns (64 weights of each of the 128 rows)
constexpr uint32_t kTcACol = 256;
// shared-window addresses (the dynamic allocation starts at a base <= 1024)
constexpr uint32_t kTcMaxBase = 1024;
constexpr uint32_t kTcBars = 1024;                 // mbarriers, tensor-memory slot, reduction flag
constexpr uint32_t kTcRing = 2048;                 // activation slots, then weight stages
constexpr uint32_t kTcTopMax = kTcMaxBase + 227 * 1024;
constexpr unsigned kTcStatusTimeout = 1u;
constexpr unsigned kTcStatusLayout = 2u;
constexpr unsigned kTcStatusTmem = 4u;
constexpr uint64_t kTcTimeoutNs = 1000000000ull;   // 1 s
constexpr uint64_t kTcDebugTimeoutNs = 5000000ull; // 5 ms under the test hook

// Geometry per activation layout: NP = 0 one row (compact B), else NP rows.
// A pipeline step is a BU pair: one row block's two consecutive superblocks,
// so every tile contributes one 2 KB code run and one 512-byte scale run (runs
// of 1 KB and 256 bytes leave HBM well below its streaming rate).  Shared
// memory holds two rings: weight stages (one pair's codes and scales,
// released by its decoders as soon as they have read them) and activation
// slots (the pair's two activation superblocks, released by the MMAs that read
// them), so a weight stage is never held for the MMAs' latency.
template <int NP>
struct TcShape {
    static constexpr int kN = NP == 0 ? 16 : NP;             // MMA N
    static constexpr int kBCopy = NP == 0 ? 256 : NP * 256;  // activation bytes per superblock
    // compact form: the MMAs of a superblock read 496 bytes from its start
    static constexpr int kBSlotBytes = NP == 0 ? 1024 : 2 * NP * 256;
    static constexpr uint32_t kLBO = NP == 0 ? 16u : (uint32_t)NP * 16u;  // between 8-column groups
    static constexpr uint32_t kSBO = 128u;                              // between 8-row groups
    static constexpr int kWStage = 2 * (kBuCodeBytes + kBuScaleBytes);  // 20 KB
    static constexpr int kBSlots = NP == 32 ? 4 : 8;                   // a multiple of the group count
    static constexpr uint32_t kWRing = kTcRing + (uint32_t)(kBSlots * kBSlotBytes);
    static constexpr int kStages = (int)((kTcTopMax - kWRing) / kWStage);
    // each decode group owns every kTcGroups-th stage and slot: a waiter then
    // sees every phase of its stages in order (parity waits stay unambiguous)
    static constexpr int kGroupStages = kStages / kTcGroups;
    static constexpr int kUsedStages = kGroupStages * kTcGroups;
    static constexpr uint32_t kTop = kWRing + (uint32_t)kUsedStages * kWStage;
    // fp32 accumulator, fp16 A and B, both K-major, N, M = 128
    static constexpr uint32_t kIdesc = (1u << 4) | ((uint32_t)(kN >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
    static_assert(kUsedStages <= 16 && kBSlots <= 8, "barrier area");
    static_assert(kGroupStages >= 2, "at least two stages per decode group");
    static_assert(kBSlots % kTcGroups == 0, "activation slots owned by groups");
    static_assert(kWRing % 128 == 0 && kWStage % 128 == 0, "tensor copies land on 128-byte boundaries");
    static_assert(kTop <= kTcTopMax, "dynamic shared memory per CTA");
};

// ---- PTX wrappers ------------------------------------------------------------
__device__ __forceinline__ uint64_t tc_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void tc_mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ bool tc_mbar_try(uint32_t bar, uint32_t parity) {
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
// Wait for phase `parity`; false after timeout_ns (or 2^30 polls).
__device__ __noinline__ bool tc_mbar_wait_slow(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
    const uint64_t t0 = tc_ns();
    for (uint32_t it = 0; it < (1u << 30); ++it) {
        if (tc_mbar_try(bar, parity)) return true;
        if (tc_ns() - t0 > timeout_ns) return false;
    }
    return false;
}
__device__ __forceinline__ bool tc_mbar_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
    return tc_mbar_try(bar, parity) || tc_mbar_wait_slow(bar, parity, timeout_ns);
}
// Warp-uniform bounded wait (every lane polls; all agree on the result).
__device__ __forceinline__ bool tc_mbar_wait_warp(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
    return __all_sync(kFull, tc_mbar_wait(bar, parity, timeout_ns));
}
__device__ __forceinline__ void tc_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_arrive_expect(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// 3-D TMA load of a box at (0, y, z), no multicast; parts past the tensor
// are zero-filled and counted.
__device__ __forceinline__ void tc_tma3d(uint32_t dst, const CUtensorMap *map, int y, int z, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(y), "r"(z), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void tc_bulk(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}
__device__ __forceinline__ uint4 tc_lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t tc_hmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 16 consecutive 32-bit tensor-memory columns of this thread's lane.
__device__ __forceinline__ void tc_st16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

// MLD consecutive fp32 columns of this thread's lane (MLD = 1, 2, 4, 8, 16, 32).
template <int MLD>
__device__ __forceinline__ void tc_ld(uint32_t taddr, uint32_t (&v)[MLD]);
template <>
__device__ __forceinline__ void tc_ld<1>(uint32_t taddr, uint32_t (&v)[1]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(v[0]) : "r"(taddr));
}
template <>
__device__ __forceinline__ void tc_ld<2>(uint32_t taddr, uint32_t (&v)[2]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];" : "=r"(v[0]), "=r"(v[1]) : "r"(taddr));
}
template <>
__device__ __forceinline__ void tc_ld<4>(uint32_t taddr, uint32_t (&v)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
                 : "r"(taddr));
}
template <>
__device__ __forceinline__ void tc_ld<8>(uint32_t taddr, uint32_t (&v)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
                 : "r"(taddr));
}
template <>
__device__ __forceinline__ void tc_ld<16>(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
          "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
}
// D (tensor memory) [+]= A (tensor memory) x B (shared-memory descriptor).
__device__ __forceinline__ void tc_mma(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
// Shared-memory operand descriptor: K-major, no swizzle, 16-byte core-matrix
// rows; lbo between 8-column groups, sbo between 8-row groups; version 1.
__device__ __forceinline__ uint64_t tc_bdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}
__device__ __forceinline__ void tc_named_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
// AND of a predicate over the 128 epilogue threads (named barrier 1).
__device__ __forceinline__ bool tc_all_epilogue(bool p) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred a, b;\n\tsetp.ne.u32 a, %1, 0;\n\t"
        "bar.red.and.pred b, 1, 128, a;\n\tselp.u32 %0, 1, 0, b;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)p)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ float tc_ldcg(const float *p) {
    float v;
    asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

struct TcProblem {
    CUtensorMap cmap;   // codes plane as uint32 [T][NSB][256]: box 256 x 2 x 8 = a pair's eight 2 KB code runs
    CUtensorMap smap;   // scales plane as uint32 [T][NSB][64]: box 64 x 2 x 8 = its eight 512-byte scale runs
    const uint8_t *codes;
    const uint8_t *scales;
    const uint8_t *xb;  // activation operand (kRotPlain or kRotCore layout)
    char *y;
    int64_t ldy;
    int bu_begin;       // first BU pair of this problem in the group
    int rb_begin;       // first row block (counter slot) of this problem
    int n;
    int tiles;
    int nsb;
    int npair;          // BU pairs per row block: ceil(nsb / 2)
};

struct TcParams {
    TcProblem prob[kMaxProblems];
    int count;
    int m;
    int units;   // BU pairs over all problems (< 2^31)
    int ctas;    // grid size; CTA c owns [c*U/C, (c+1)*U/C)
    unsigned *header;
    unsigned long long *counters;  // per row block: call tag << 32 | contributors counted
    float *partials;               // [2 * ctas][mld][128] partial sums of split row blocks
    uint64_t timeout_ns;
    int inject_skip;               // test hook: CTA 0 never issues the copies of its first BU
};

static_assert(sizeof(TcParams) <= 4096, "kernel parameters");

__device__ __forceinline__ int tc_problem_of(const TcParams &P, int v) {
    int q = 0;
#pragma unroll
    for (int i = 1; i < kMaxProblems; ++i)
        if (i < P.count && v >= P.prob[i].bu_begin) q = i;
    return q;
}
__device__ __forceinline__ int tc_problem_end(const TcParams &P, int q) {
    return q + 1 < P.count ? P.prob[q + 1].bu_begin : P.units;
}
// first BU of CTA c
__device__ __forceinline__ int tc_range_begin(const TcParams &P, int c) {
    return (int)(((int64_t)c * P.units) / P.ctas);
}
// the CTA that owns BU v: the largest c with floor(c * U / C) <= v
__device__ __forceinline__ int tc_owner(const TcParams &P, int v) {
    return (int)((((int64_t)v + 1) * P.ctas - 1) / P.units);
}

// Row-block walk over a CTA's range: the segment [lo, hi) is the part of row
// block rb of problem q inside [u0, u1).
struct TcSeg {
    int q, rb, rb_lo, lo, hi;
};
__device__ __forceinline__ TcSeg tc_seg_at(const TcParams &P, int u, int u1) {
    TcSeg s;
    s.q = tc_problem_of(P, u);
    const TcProblem &pr = P.prob[s.q];
    s.rb = (u - pr.bu_begin) / pr.npair;
    s.rb_lo = pr.bu_begin + s.rb * pr.npair;
    s.lo = u;
    s.hi = min(s.rb_lo + pr.npair, u1);
    return s;
}

// Decoded operands of one row's 32-column block j (the row's 64-byte
// superblock slot in four 16-byte chunks c[0..3]; chunk b, word j holds
// logical bytes b, b + 4, b + 8, b + 12 of the block, logical byte L holding
// elements 2L and 2L + 1).  Each chunk word is decoded as it stands: register
// byte tables give the fp16 centroid pairs of its four bytes, k = 0..3 being
// elements 8k + 2b, 8k + 2b + 1, and the half-block scale multiplies them
// (elements 0..15: d0, 16..31: d1).  o[4k + b] = elements 8k + 2b, 8k + 2b +
// 1: tensor-memory column 16 j + 4 k + b.
__device__ __forceinline__ void tc_decode_block(const uint4 (&c)[4], uint32_t sw, uint32_t (&o)[16], int j) {
    const uint32_t d0 = prmt(sw, sw, 0x1010u), d1 = prmt(sw, sw, 0x3232u);
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const uint32_t w = j == 0 ? c[b].x : j == 1 ? c[b].y : j == 2 ? c[b].z : c[b].w;
        uint32_t v[4];
        decode_word(w, v);
        o[b] = tc_hmul2(v[0], d0);
        o[4 + b] = tc_hmul2(v[1], d0);
        o[8 + b] = tc_hmul2(v[2], d1);
        o[12 + b] = tc_hmul2(v[3], d1);
    }
}

template <int NP, int MLD, int OT>
__global__ void __launch_bounds__(kTcThreads, 1) tc_gemv_kernel(const __grid_constant__ TcParams P) {
    using S = TcShape<NP>;
    constexpr int kSu = S::kUsedStages;
    constexpr int kG = kTcGroups;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t base = (uint32_t)__cvta_generic_to_shared(smem);
    if (base > kTcMaxBase) {  // layout precondition (checked, never expected)
        if (threadIdx.x == 0) atomicOr(P.header + kHeaderStatus, kTcStatusLayout);
        return;
    }
    // mbarriers: full[16] empty[16] (weight stages) bfull[8] bempty[8]
    // (activation slots) afull[G][2] aempty[G][2] accfull[G][2] accempty[G][2]
    // done[G], then the tensor-memory slot and a flag
    const uint32_t full0 = kTcBars, empty0 = full0 + 8 * 16, bfull0 = empty0 + 8 * 16, bempty0 = bfull0 + 8 * 8;
    const uint32_t afull0 = bempty0 + 8 * 8;
    const uint32_t aempty0 = afull0 + 8 * 2 * kG, accfull0 = aempty0 + 8 * 2 * kG, accempty0 = accfull0 + 8 * 2 * kG;
    const uint32_t done0 = accempty0 + 8 * 2 * kG;
    const uint32_t tmem_slot = done0 + 8 * kG, flag_addr = tmem_slot + 8;
    // pair i of this CTA belongs to decode group i % G and is that group's
    // (i / G)-th pair: weight stage g + G * ((i / G) % kGroupStages), use number
    // (i / G) / kGroupStages (the stage's mbarrier phase); likewise for the
    // activation slots
    auto ring_stage = [](int i) { return i % kG + kG * ((i / kG) % S::kGroupStages); };
    auto ring_phase = [](int i) { return (uint32_t)(((i / kG) / S::kGroupStages) & 1); };
    auto stage_addr = [](int s) -> uint32_t { return S::kWRing + (uint32_t)s * S::kWStage; };
    auto bslot = [](int i) { return i % S::kBSlots; };
    auto bphase = [](int i) { return (uint32_t)((i / S::kBSlots) & 1); };
    auto bslot_addr = [](int j) -> uint32_t { return kTcRing + (uint32_t)j * S::kBSlotBytes; };
    const int c = blockIdx.x;
    const int u0 = tc_range_begin(P, c), u1 = tc_range_begin(P, c + 1);
    const int nU = u1 - u0;

    // ---- set-up ----------------------------------------------------------------
    if (threadIdx.x == 0) {
        for (int s = 0; s < kSu; ++s) {
            tc_mbar_init(full0 + 8 * s, 1);
            tc_mbar_init(empty0 + 8 * s, 4);  // the group's four warps, once they have read the stage
        }
        for (int j = 0; j < S::kBSlots; ++j) {
            tc_mbar_init(bfull0 + 8 * j, 1);
            tc_mbar_init(bempty0 + 8 * j, 1);  // the group's MMA commit
        }
        for (int j = 0; j < 2 * kG; ++j) {
            tc_mbar_init(afull0 + 8 * j, 4);
            tc_mbar_init(aempty0 + 8 * j, 1);
            tc_mbar_init(accfull0 + 8 * j, 1);
            tc_mbar_init(accempty0 + 8 * j, 4);
        }
        for (int g = 0; g < kG; ++g) tc_mbar_init(done0 + 8 * g, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tmem_slot),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + (tmem_slot - base));
    const bool tmem_ok = tmem == 0u;  // all 512 columns: base at lane 0, column 0 (checked, never expected)
    if (!tmem_ok && threadIdx.x == 0) atomicOr(P.header + kHeaderStatus, kTcStatusTmem);
    grid_dependents_launch();

    if (warp == 0) {
        // ---- producer (lane 0): TMA copies of each pair into its stage and slot.
        // Two cursors polled without blocking, so that a weight box never
        // waits for an activation slot (which the MMAs release much later) or
        // the other way round.
        if (lane == 0 && tmem_ok && nU > 0) {
            auto pair_of = [&](int i, int &q, int &pend, int &rb, int &sb) {
                const int u = u0 + i;
                while (u >= pend) pend = tc_problem_end(P, ++q);
                const TcProblem &pr = P.prob[q];
                const int local = u - pr.bu_begin;
                rb = local / pr.npair;
                sb = 2 * (local - rb * pr.npair);
            };
            const bool skip0 = P.inject_skip && c == 0;  // test hook: pair 0's copies are never issued
            auto issue_w = [&](int i, int q, int rb, int sb) {
                const TcProblem &pr = P.prob[q];
                const uint32_t st = stage_addr(ring_stage(i)), bar = full0 + 8 * ring_stage(i);
                // whole boxes (a superblock or tiles past the matrix arrive zero-filled and count)
                tc_arrive_expect(bar, (uint32_t)S::kWStage);
                if (!(skip0 && i == 0)) {
                    tc_tma3d(st, &pr.cmap, sb, rb * 8, bar);
                    tc_tma3d(st + 2 * kBuCodeBytes, &pr.smap, sb, rb * 8, bar);
                }
            };
            auto issue_b = [&](int i, int q, int sb) {
                const TcProblem &pr = P.prob[q];
                const int nb = sb + 1 < pr.nsb ? 2 : 1;  // activation superblocks of the pair
                const uint32_t bar = bfull0 + 8 * bslot(i), dst = bslot_addr(bslot(i));
                tc_arrive_expect(bar, (uint32_t)(nb * S::kBCopy));
                if (!(skip0 && i == 0))
                    for (int h = 0; h < nb; ++h)
                        tc_bulk(dst + (uint32_t)(h * S::kBCopy), pr.xb + (size_t)(sb + h) * S::kBCopy,
                                (uint32_t)S::kBCopy, bar);
            };
            // the first stages' weight boxes go out before the dependency wait
            // (the packed weights do not depend on the preceding kernel);
            // activation runs only after it
            const int pre = min(kSu, nU);  // pairs i < kSu are the first uses of their stages
            int qw = tc_problem_of(P, u0), pw = tc_problem_end(P, qw), rb, sb;
            for (int i = 0; i < pre; ++i) {
                pair_of(i, qw, pw, rb, sb);
                issue_w(i, qw, rb, sb);
            }
            grid_dependency_wait();
            int qb = tc_problem_of(P, u0), pb = tc_problem_end(P, qb);
            int iw = pre, ib = 0;
            uint64_t t_last = tc_ns();
            while (iw < nU || ib < nU) {
                bool progressed = false;
                if (iw < nU && tc_mbar_try(empty0 + 8 * ring_stage(iw), ring_phase(iw) ^ 1u)) {
                    pair_of(iw, qw, pw, rb, sb);
                    issue_w(iw, qw, rb, sb);
                    ++iw;
                    progressed = true;
                }
                if (ib < nU && (ib < S::kBSlots || tc_mbar_try(bempty0 + 8 * bslot(ib), bphase(ib) ^ 1u))) {
                    pair_of(ib, qb, pb, rb, sb);
                    issue_b(ib, qb, sb);
                    ++ib;
                    progressed = true;
                }
                if (progressed) {
                    t_last = tc_ns();
                } else if (tc_ns() - t_last <= P.timeout_ns) {
                    __nanosleep(32);  // leave the issue slots to the decoders sharing this scheduler
                } else {
                    atomicOr(P.header + kHeaderStatus, kTcStatusTimeout);
                    break;
                }
            }
            // no copy may still be in flight when the CTA exits
            for (int i = iw > kSu ? iw - kSu : 0; i < iw; ++i)
                tc_mbar_wait(full0 + 8 * ring_stage(i), ring_phase(i), P.timeout_ns);
            for (int i = ib > S::kBSlots ? ib - S::kBSlots : 0; i < ib; ++i)
                tc_mbar_wait(bfull0 + 8 * bslot(i), bphase(i), P.timeout_ns);
        }
        __syncwarp();
    } else if (warp < kTcIssWarp0) {
        // ---- decode group g: thread = weight row; per pair, superblocks 0 and 1,
        // each as two halves of 64 columns through the group's two A halves
        const int g = (warp - kTcDecWarp0) >> 2;
        const int row = 32 * (warp & 3) + lane;  // the tensor-memory lane this warp may access
        // stage layout: codes [tile][superblock][1 KB], scales [tile][superblock][256 B]
        const uint32_t code_off = (uint32_t)(row >> 4) * 2048u + (uint32_t)(row & 15) * 64u;
        const uint32_t scale_off = 2 * kBuCodeBytes + (uint32_t)(row >> 4) * 512u + (uint32_t)(row & 15) * 16u;
        const uint32_t tlane = (uint32_t)(32 * (warp & 3)) << 16;
        const uint32_t a_col = tmem + kTcACol + 64u * (uint32_t)g;
        const uint32_t afull_g = afull0 + 16 * g, aempty_g = aempty0 + 16 * g;
        bool ok = tmem_ok;
        for (int i = g, r = 0; i < nU && ok; i += kG, ++r) {
            const int s = ring_stage(i);
            if (!tc_mbar_wait_warp(full0 + 8 * s, ring_phase(i), P.timeout_ns)) {
                if (lane == 0) atomicOr(P.header + kHeaderStatus, kTcStatusTimeout);
                break;
            }
            const uint32_t st = stage_addr(s);
            uint4 cw[2][4], sw[2];
#pragma unroll
            for (int sbi = 0; sbi < 2; ++sbi) {
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) cw[sbi][k4] = tc_lds128(st + code_off + 1024u * sbi + 16u * k4);
                sw[sbi] = tc_lds128(st + scale_off + 256u * sbi);
            }
            __syncwarp();
            if (lane == 0) tc_arrive(empty0 + 8 * s);
#pragma unroll
            for (int sbi = 0; sbi < 2 && ok; ++sbi) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    // A half h is used once per superblock: its previous use has been read
                    if (!tc_mbar_wait_warp(aempty_g + 8 * h, (uint32_t)(sbi & 1) ^ 1u, P.timeout_ns)) {
                        if (lane == 0) atomicOr(P.header + kHeaderStatus, kTcStatusTimeout);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t ta = a_col + tlane + 32u * h;
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        const int j = 2 * h + jj;
                        const uint4 &w4 = sw[sbi];
                        uint32_t o[16];
                        tc_decode_block(cw[sbi], j == 0 ? w4.x : j == 1 ? w4.y : j == 2 ? w4.z : w4.w, o, j);
                        tc_st16(ta + 16u * jj, o);
                    }
                    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc_arrive(afull_g + 8 * h);
                }
            }
        }
    } else if (warp < kTcEpiWarp0) {
        // ---- MMA issuer of group g (one thread): its pairs' products into the group's
        // own accumulators, per half superblock as soon as the decoders have stored it
        const int g = warp - kTcIssWarp0;
        if (lane == 0 && tmem_ok && g < nU) {
            const uint32_t a_col = tmem + kTcACol + 64u * (uint32_t)g;
            const uint32_t afull_g = afull0 + 16 * g, aempty_g = aempty0 + 16 * g;
            const uint32_t accfull_g = accfull0 + 16 * g, accempty_g = accempty0 + 16 * g;
            int acc_use0 = 0, acc_use1 = 0;  // segments of this group so far per accumulator buffer
            int q = 0;                       // CTA segment index of the current pair
            TcSeg sg = tc_seg_at(P, u0 + g, u1);
            {
                TcSeg w = tc_seg_at(P, u0, u1);
                while (w.hi <= u0 + g) {
                    w = tc_seg_at(P, w.hi, u1);
                    ++q;
                }
            }
            bool ok = true;
            for (int i = g; i < nU && ok; i += kG) {
                const int u = u0 + i;
                while (u >= sg.hi) {  // segments without a pair of this group are skipped
                    sg = tc_seg_at(P, sg.hi, u1);
                    ++q;
                }
                const TcProblem &pr = P.prob[sg.q];
                const bool first_in_seg = i - kG < sg.lo - u0;
                const bool last_in_seg = i + kG >= sg.hi - u0;
                const bool second = 2 * (u - sg.rb_lo) + 1 < pr.nsb;  // the pair's second superblock exists
                const int b = q & 1;
                const uint32_t bsm = bslot_addr(bslot(i));
                const uint32_t d = tmem + (uint32_t)(2 * g + b) * (uint32_t)S::kN;
#pragma unroll
                for (int sbi = 0; sbi < 2 && ok; ++sbi) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        ok = tc_mbar_wait(afull_g + 8 * h, (uint32_t)(sbi & 1), P.timeout_ns);
                        if (ok && sbi == 0 && h == 0)  // the pair's activation superblocks have landed
                            ok = tc_mbar_wait(bfull0 + 8 * bslot(i), bphase(i), P.timeout_ns);
                        if (ok && sbi == 0 && h == 0 && first_in_seg)  // the epilogue has read this buffer
                            ok = tc_mbar_wait(accempty_g + 8 * b, (uint32_t)((b ? acc_use1 : acc_use0) & 1) ^ 1u,
                                              P.timeout_ns);
                        if (!ok) break;
                        tc_fence_after();
                        if (sbi == 0 || second) {
                            const uint32_t bsb = bsm + (uint32_t)(sbi * S::kBCopy);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const int ks = 4 * h + kk;  // k-step of the superblock
                                tc_mma(d, a_col + 32u * h + 8u * kk,
                                       tc_bdesc(bsb + 2u * S::kLBO * ks, S::kLBO, S::kSBO), S::kIdesc,
                                       (first_in_seg && sbi == 0 && ks == 0) ? 0u : 1u);
                            }
                        }
                        tc_commit(aempty_g + 8 * h);  // this half's A columns are free once read
                    }
                }
                if (!ok) break;
                tc_commit(bempty0 + 8 * bslot(i));  // the activation slot has been read
                if (last_in_seg) {
                    tc_commit(accfull_g + 8 * b);
                    if (b) ++acc_use1;
                    else ++acc_use0;
                }
            }
            if (!ok) atomicOr(P.header + kHeaderStatus, kTcStatusTimeout);
            // every MMA this group issued has completed before tensor memory is released
            tc_commit(done0 + 8 * g);
            tc_mbar_wait(done0 + 8 * g, 0u, P.timeout_ns);
        }
        __syncwarp();
    } else {
        // ---- epilogue: thread = weight row; the groups' accumulators -> Y -----------
        grid_dependency_wait();  // the header (call tag) is prepared by the preceding launch
        const uint32_t tag = *reinterpret_cast<volatile const unsigned *>(P.header + kHeaderTag);
        const int row = 32 * (warp & 3) + lane;
        const int et = threadIdx.x - kTcEpiWarp0 * 32;  // 0..127
        const uint32_t tlane = (uint32_t)(32 * (warp & 3)) << 16;
        volatile int *flag = reinterpret_cast<volatile int *>(smem + (flag_addr - base));
        // segments read so far per (group, buffer): 8-bit counters packed by
        // group, buffer 0 in use0 and buffer 1 in use1 (only their parity matters)
        uint32_t use0 = 0, use1 = 0;
        if (tmem_ok && nU > 0) {
            TcSeg sg = tc_seg_at(P, u0, u1);
            for (int seg = 0;; ++seg) {
                const int b = seg & 1;
                float v[MLD];
#pragma unroll
                for (int i = 0; i < MLD; ++i) v[i] = 0.f;
                bool ok = true;
#pragma unroll
                for (int g = 0; g < kG; ++g) {
                    // group g took part iff one of its BUs (i = g mod G) lies in the segment
                    const int lo = sg.lo - u0, hi = sg.hi - u0;
                    const int f = lo + ((g - lo) % kG + kG) % kG;
                    if (f >= hi) continue;
                    // one decision for all four epilogue warps (they meet at named barriers)
                    const uint32_t par = ((b ? use1 : use0) >> (8 * g)) & 1u;
                    ok = tc_all_epilogue(ok && tc_mbar_wait(accfull0 + 16 * g + 8 * b, par, P.timeout_ns));
                    if (!ok) break;
                    tc_fence_after();
                    // the group's sums, at most 16 columns at a time (registers)
                    constexpr int kChunk = MLD < 16 ? MLD : 16;
#pragma unroll
                    for (int c0 = 0; c0 < MLD; c0 += kChunk) {
                        uint32_t w[kChunk];
                        tc_ld<kChunk>(tmem + tlane + (uint32_t)(2 * g + b) * (uint32_t)S::kN + (uint32_t)c0, w);
                        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                        for (int i = 0; i < kChunk; ++i) v[c0 + i] += __uint_as_float(w[i]);
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc_arrive(accempty0 + 16 * g + 8 * b);
                    if (b) use1 += 1u << (8 * g);
                    else use0 += 1u << (8 * g);
                }
                if (!ok) {
                    if (et == 0) atomicOr(P.header + kHeaderStatus, kTcStatusTimeout);
                    break;
                }

                const TcProblem &pr = P.prob[sg.q];
                const int grow = sg.rb * 128 + row;  // weight row within the problem
                const int rb_hi = sg.rb_lo + pr.npair;
                constexpr int kM = MLD;
                if (sg.lo == sg.rb_lo && sg.hi == rb_hi) {
                    if (grow < pr.n) {
#pragma unroll
                        for (int i = 0; i < kM; ++i)
                            if (i < P.m) store1<OT>(pr.y + ((int64_t)i * pr.ldy + grow) * ElemSize<OT>::value, v[i]);
                    }
                } else {
                    // split row block: partial sums, then the last contributor adds them
                    const int e = sg.lo == u0 ? 0 : 1;
                    float *slot = P.partials + (size_t)(2 * c + e) * kM * 128;
#pragma unroll
                    for (int i = 0; i < kM; ++i)
                        if (i < P.m) slot[i * 128 + row] = v[i];
                    __threadfence();
                    tc_named_sync(1, 128);
                    const int cf = tc_owner(P, sg.rb_lo), cl = tc_owner(P, rb_hi - 1);
                    if (et == 0) {
                        unsigned long long *cnt = P.counters + (pr.rb_begin + sg.rb);
                        unsigned long long old = *reinterpret_cast<volatile unsigned long long *>(cnt), nw = 0;
                        for (int it = 0; it < (1 << 20); ++it) {
                            nw = ((uint32_t)(old >> 32) == tag) ? old + 1ull : (((unsigned long long)tag << 32) | 1ull);
                            const unsigned long long prev = atomicCAS(cnt, old, nw);
                            if (prev == old) break;
                            old = prev;
                        }
                        __threadfence();
                        *flag = ((int)(nw & 0xffffffffull) == cl - cf + 1) ? 1 : 0;
                    }
                    tc_named_sync(1, 128);
                    const bool last = *flag != 0;
                    if (last && grow < pr.n) {
                        float acc[kM];
#pragma unroll
                        for (int i = 0; i < kM; ++i) acc[i] = 0.f;
                        for (int cc = cf; cc <= cl; ++cc) {
                            const int ee = tc_range_begin(P, cc) >= sg.rb_lo ? 0 : 1;
                            const float *src = P.partials + (size_t)(2 * cc + ee) * kM * 128 + row;
#pragma unroll
                            for (int i = 0; i < kM; ++i)
                                if (i < P.m) acc[i] += tc_ldcg(src + i * 128);
                        }
#pragma unroll
                        for (int i = 0; i < kM; ++i)
                            if (i < P.m)
                                store1<OT>(pr.y + ((int64_t)i * pr.ldy + grow) * ElemSize<OT>::value, acc[i]);
                    }
                    tc_named_sync(1, 128);  // the flag may be rewritten by the next segment
                }
                if (sg.hi >= u1) break;
                sg = tc_seg_at(P, sg.hi, u1);
            }
        }
    }
    // ---- teardown ------------------------------------------------------------------
    tc_fence_before();
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
}

using TcEncode = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                              const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point.
TcEncode tc_encode() {
    static std::once_flag once;
    static TcEncode fn = nullptr;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<TcEncode>(ptr);
    });
    return fn;
}

uint32_t tc_smem_base() {
    static int cached[256];
    static bool have[256];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return 1024;
    if (!have[dev]) {
        int reserved = 0;
        if (cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess)
            reserved = 1024;
        cached[dev] = reserved;
        have[dev] = true;
    }
    return (uint32_t)cached[dev];
}

template <int NP, int MLD, int OT>
cudaError_t tc_launch_kernel(const TcParams &prm, int grid, bool programmatic, cudaStream_t stream) {
    using S = TcShape<NP>;
    const uint32_t base = tc_smem_base();
    if (base > kTcMaxBase) return cudaErrorInvalidValue;
    const int smem = (int)(S::kTop - base);
    cudaError_t err =
        cudaFuncSetAttribute(tc_gemv_kernel<NP, MLD, OT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = programmatic ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, tc_gemv_kernel<NP, MLD, OT>, prm);
}

template <int NP, int MLD>
cudaError_t tc_launch_ot(const TcParams &prm, int ydtype, int grid, bool programmatic, cudaStream_t stream) {
    switch (ydtype) {
        case kF32: return tc_launch_kernel<NP, MLD, kF32>(prm, grid, programmatic, stream);
        case kBF16: return tc_launch_kernel<NP, MLD, kBF16>(prm, grid, programmatic, stream);
        case kF16: return tc_launch_kernel<NP, MLD, kF16>(prm, grid, programmatic, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool use_tc(int64_t m) {
    if (m < 1 || m > 32) return false;
    const uint32_t f = debug_flags();
    if (f & kDebugUseTmem) return true;
    if (f & kDebugUseMmaSync) return false;
    return m >= 9;
}

int tc_npad(int64_t m) { return m <= 1 ? 0 : (m <= 16 ? 16 : 32); }
int tc_mld(int64_t m) { return m <= 1 ? 1 : m <= 2 ? 2 : m <= 4 ? 4 : m <= 8 ? 8 : m <= 16 ? 16 : 32; }

size_t tc_xrot_bytes(int64_t m, int64_t k) {
    const int np = tc_npad(m);
    return (size_t)superblocks(k) * (np == 0 ? 256u : (size_t)np * 256u);
}

TcPlan plan_tc(const int64_t *n, const int64_t *k, int count, int64_t m, int sm_count) {
    TcPlan pl = {};
    for (int i = 0; i < count; ++i) {
        const int64_t rbs = (tiles(n[i]) + 7) / 8;
        pl.rblocks += rbs;
        pl.units += rbs * ((superblocks(k[i]) + 1) / 2);  // BU pairs
    }
    int64_t grid = pl.units < sm_count ? pl.units : sm_count;
    if (grid < 1) grid = 1;
    pl.grid = (int)grid;
    pl.npad = tc_npad(m);
    pl.mld = tc_mld(m);
    pl.counter_bytes = round_up((size_t)pl.rblocks * 8u, 256);
    pl.partial_bytes = round_up((size_t)2 * (size_t)pl.grid * (size_t)pl.mld * 128u * 4u, 256);
    return pl;
}

cudaError_t launch_tc(const GemvProblem *probs, int count, int64_t m, int ydtype, const TcPlan &plan,
                      unsigned *header, unsigned long long *counters, float *partials, bool programmatic,
                      cudaStream_t stream) {
    if (count < 1 || count > kMaxProblems || m < 1 || m > 32) return cudaErrorInvalidValue;
    TcParams prm = {};
    int64_t ub = 0, rb = 0;
    for (int i = 0; i < count; ++i) {
        TcProblem &d = prm.prob[i];
        d.codes = probs[i].codes;
        d.scales = reinterpret_cast<const uint8_t *>(probs[i].scales);
        d.xb = reinterpret_cast<const uint8_t *>(probs[i].xrot);
        d.y = static_cast<char *>(probs[i].y);
        d.ldy = probs[i].ldy;
        d.bu_begin = (int)ub;
        d.rb_begin = (int)rb;
        d.n = (int)probs[i].n;
        d.tiles = (int)tiles(probs[i].n);
        d.nsb = (int)superblocks(probs[i].k);
        d.npair = (d.nsb + 1) / 2;
        const int64_t rbs = (d.tiles + 7) / 8;
        ub += rbs * d.npair;
        rb += rbs;
    }
    if (ub != plan.units || rb != plan.rblocks || ub >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    TcEncode encode = tc_encode();
    if (!encode) return cudaErrorNotSupported;
    for (int i = 0; i < count; ++i) {
        TcProblem &d = prm.prob[i];
        // [T][NSB][256 words] and [T][NSB][64 words]; a box is one row block's
        // two consecutive superblocks
        const cuuint64_t cdims[3] = {256u, (cuuint64_t)d.nsb, (cuuint64_t)d.tiles};
        const cuuint64_t cstr[2] = {1024u, (cuuint64_t)d.nsb * 1024u};
        const cuuint32_t cbox[3] = {256u, 2u, 8u};
        const cuuint64_t sdims[3] = {64u, (cuuint64_t)d.nsb, (cuuint64_t)d.tiles};
        const cuuint64_t sstr[2] = {256u, (cuuint64_t)d.nsb * 256u};
        const cuuint32_t sbox[3] = {64u, 2u, 8u};
        const cuuint32_t estr[3] = {1u, 1u, 1u};
        if (encode(&d.cmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint8_t *>(d.codes), cdims, cstr, cbox, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
            encode(&d.smap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint8_t *>(d.scales), sdims, sstr, sbox,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    if (plan.npad != tc_npad(m) || plan.mld != tc_mld(m)) return cudaErrorInvalidValue;
    prm.count = count;
    prm.m = (int)m;
    prm.units = (int)ub;
    prm.ctas = plan.grid;
    prm.header = header;
    prm.counters = counters;
    prm.partials = partials;
    prm.inject_skip = (debug_flags() & kDebugSkipGemvCopy) ? 1 : 0;
    prm.timeout_ns = prm.inject_skip ? kTcDebugTimeoutNs : kTcTimeoutNs;
    switch (plan.mld) {
        case 1: return tc_launch_ot<0, 1>(prm, ydtype, plan.grid, programmatic, stream);
        case 2: return tc_launch_ot<16, 2>(prm, ydtype, plan.grid, programmatic, stream);
        case 4: return tc_launch_ot<16, 4>(prm, ydtype, plan.grid, programmatic, stream);
        case 8: return tc_launch_ot<16, 8>(prm, ydtype, plan.grid, programmatic, stream);
        case 16: return tc_launch_ot<16, 16>(prm, ydtype, plan.grid, programmatic, stream);
        case 32: return tc_launch_ot<32, 32>(prm, ydtype, plan.grid, programmatic, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace tq
