// tq_prefill.cu -- the large-M product (prefill) on the fifth-generation
// tensor cores: Y = X w~^T for TQ4_1S weights, many activation rows.
//
// Method: TQ4_1S page ("企业官网建设流程全解析", hotelren.com/news/5458160),
// section 解码速度：分硬件汇总: the activation is rotated once with the block
// transform; afterwards every weight contributes centroid(code) * scale.  The
// same holds for a whole matrix of activations:
//
//   Y[m][r] = sum_blocks sum_e c[r][e] * xrot[m][e],   c = +-M[mag] * d_half
//
// so the weights enter the tensor cores as decoded centroids times their fp16
// half-block scale, with no per-weight inverse transform, and X enters as its
// fp16 pre-rotation H(s .* x)/32.
//
// B200 design:
//  * One CTA per output tile of 256 weight rows x 256 activation rows: two
//    tcgen05.mma of M = 128, N = 256, K = 16 per 16 columns (one per 128-row
//    half of the weight tile) share the activation operand, each into its own
//    fp32 accumulator of 128 lanes x 256 columns; together they fill the 512
//    columns of tensor memory.  Both operands are K-major in shared memory
//    with the 128-byte swizzle.  Two weight halves per activation tile halve
//    the activation bytes each flop needs from L2, which sets the pace.
//  * The activation tile (256 rows x 64 columns of fp16 per stage) arrives by
//    TMA (cp.async.bulk.tensor, no multicast); four stages.
//  * The weight tile (256 rows x 64 columns per stage) is decoded by sixteen
//    warps, one row and one 32-column block per thread: each thread reads its
//    row's 64-byte superblock slot with 16-byte loads (neighbouring threads,
//    neighbouring slots), three superblocks ahead in registers; byte
//    permutes against register tables of the fp16 magnitudes, with the sign
//    bits merged in by two more permutes, turn each stored word into four
//    fp16 centroid pairs (each byte holds two neighbouring elements, so the
//    stored byte order needs no transpose, only a choice of output chunk);
//    one fp16 multiply applies the half-block scale and 16-byte stores write
//    the swizzled rows.  A proxy
//    fence then publishes them to the tensor cores.  Three stages.
//  * One thread issues the MMAs; tcgen05.commit releases each stage to its
//    producers and finally signals the epilogue.  The sixteen decode warps
//    then read the accumulators (tcgen05.ld, one weight row per thread, four
//    warps per 32-lane quarter: accumulator half and 128 columns each) and
//    store Y with consecutive threads on consecutive columns.
//  * Every mbarrier wait is bounded in time and reports through the
//    workspace status word.
#include <cuda.h>

#include <mutex>

#include "tq_device.cuh"
#include "tq_internal.h"

namespace tq {

namespace {

constexpr int kPM = 256;                 // weight rows per tile (two MMA halves of 128)
constexpr int kMmaM = 128;               // rows of one MMA (cta_group::1 takes M = 64 or 128)
constexpr int kPN = 256;                 // activation rows per tile (MMA N)
constexpr int kPK = 64;                  // columns per stage: one 128-byte swizzle row of fp16
constexpr int kSA = 3;                   // weight-tile stages
constexpr int kSB = 4;                   // activation-tile stages
constexpr int kATile = kPM * kPK * 2;    // 32 KB (half h at + 16 KB * h)
constexpr int kAHalf = kATile / 2;
constexpr int kBTile = kPN * kPK * 2;    // 32 KB
constexpr int kDecodeWarps = 16;         // warps 2..17: (row, block) per thread
constexpr int kPThreads = (2 + kDecodeWarps) * 32;
constexpr int kTmemCols = 512;           // two accumulators of 256 fp32 columns
constexpr int kAhead = 3;       // superblocks of row slots held in registers ahead of the decode

// Shared-memory map (offsets from the 1024-aligned start of the dynamic
// allocation): weight stages, activation stages, then the mbarriers
// full_a[kSA] full_b[kSB] empty_a[kSA] empty_b[kSB] accum and the
// tensor-memory address slot.
constexpr uint32_t kPAOff = 0;
constexpr uint32_t kPBOff = kPAOff + kSA * kATile;
constexpr uint32_t kPBarOff = kPBOff + kSB * kBTile;
constexpr uint32_t kPTmemOff = kPBarOff + 8 * (2 * kSA + 2 * kSB + 1);
constexpr uint32_t kPEndOff = kPTmemOff + 16;
constexpr uint32_t kPMaxBase = 1024;     // dynamic shared memory starts at most here
static_assert(kPEndOff + kPMaxBase - 1024 <= 227 * 1024, "dynamic shared memory per CTA");

constexpr unsigned kPStatusTimeout = 1u;
constexpr unsigned kPStatusLayout = 2u;
constexpr unsigned kPStatusTmem = 4u;  // tensor-memory base not at lane 0, column 0

// ---- PTX wrappers -----------------------------------------------------------
__device__ __forceinline__ uint64_t p_global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void p_mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ bool p_mbar_try(uint32_t bar, uint32_t parity) {
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

// Wait for phase `parity` of a barrier; false after timeout_ns (or 2^30 polls).
__device__ __noinline__ bool p_mbar_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
    if (p_mbar_try(bar, parity)) return true;
    const uint64_t t0 = p_global_ns();
    for (uint32_t it = 0; it < (1u << 30); ++it) {
        if (p_mbar_try(bar, parity)) return true;
        if (p_global_ns() - t0 > timeout_ns) return false;
    }
    return false;
}

__device__ __forceinline__ void p_mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void p_mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// 2-D TMA load of box {64 columns, 256 rows} at (x = column, y = row).
__device__ __forceinline__ void p_tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
            "r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// Generic-proxy shared-memory writes become visible to the async proxy
// (tensor-core operand reads).
__device__ __forceinline__ void p_fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void p_tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void p_tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory operand descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (stride byte offset), descriptor version 1.
__device__ __forceinline__ uint64_t p_smem_desc(uint32_t addr) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor: fp32 accumulator, fp16 A and B, both K-major,
// N = 256, M = 128.
constexpr uint32_t kPIdesc = (1u << 4) | ((uint32_t)(kPN >> 3) << 17) | ((uint32_t)(kMmaM >> 4) << 24);

__device__ __forceinline__ void p_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(kPIdesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once every MMA issued so far by this thread has completed.
__device__ __forceinline__ void p_mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// 32 consecutive fp32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void p_tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t p_lds_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}

__device__ __forceinline__ void p_sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}

__device__ __forceinline__ uint32_t p_hmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

struct PrefillParams {
    const uint8_t *codes;   // TQ4_1S codes plane
    const uint8_t *scales;  // TQ4_1S scales plane (fp16 pairs)
    int n;                  // weight rows
    int tiles;              // ceil(n / 16)
    int nsb;                // superblocks per row
    int m;                  // activation rows
    int nk;                 // 64-column stages: ceil(k / 64)
    char *y;
    int64_t ldy;
    unsigned *header;       // workspace header (status word)
    uint64_t timeout_ns;
    int inject_skip;        // test hook: CTA (0, 0) never issues its second activation-tile copy
};

// One weight row's superblock slot: its four 16-byte code chunks (chunk b,
// word j holds byte b of logical words of block j, see decode_block) and its
// 16 bytes of scales ((d0, d1) of blocks 0..3).
struct RowSlot {
    uint4 c[4];
    uint4 s;
};

__device__ __forceinline__ uint4 p_ldg128(const void *ptr) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(ptr));
    return r;
}

// Whole 64-byte slots with 16-byte loads: neighbouring threads read
// neighbouring slots.
__device__ __forceinline__ RowSlot load_slot(const PrefillParams &P, int row, int sb) {
    RowSlot w;
    if (row >= P.tiles * 16 || sb >= P.nsb) {  // past the padded rows, or past the last superblock
#pragma unroll
        for (int b = 0; b < 4; ++b) w.c[b] = make_uint4(0u, 0u, 0u, 0u);
        w.s = make_uint4(0u, 0u, 0u, 0u);
        return w;
    }
    const size_t slot = ((size_t)(row >> 4) * P.nsb + sb) * 16 + (row & 15);
    const uint8_t *c = P.codes + slot * 64;
#pragma unroll
    for (int b = 0; b < 4; ++b) w.c[b] = p_ldg128(c + 16 * b);
    w.s = p_ldg128(P.scales + slot * 16);
    return w;
}

__device__ __forceinline__ uint32_t word_of(const uint4 &v, int j) {
    return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
}

// One weight row's words of one 32-column block j.
struct BlockWords {
    uint32_t c[4];
    uint32_t s;
};

__device__ __forceinline__ BlockWords block_of(const RowSlot &r, int j) {
    BlockWords w;
#pragma unroll
    for (int b = 0; b < 4; ++b) w.c[b] = word_of(r.c[b], j);
    w.s = word_of(r.s, j);
    return w;
}

// Decode one row's 32-column block jj of the stage into the swizzled weight
// tile.  In a row's 64-byte superblock slot, logical byte L of block j
// (elements 2L, 2L + 1) sits at chunk L % 4, word j, byte L / 4; so byte k of
// chunk word b holds elements 8k + 2b, 8k + 2b + 1, and each chunk word is
// decoded as it stands into fp16 pairs, k = 0..3.  The half-block scale
// multiplies in fp16.  Elements 8k .. 8k + 7 (pairs b = 0..3) form 16-byte
// chunk 4 jj + k of the tile row, stored at chunk (4 jj + k) xor (row % 8)
// (the 128-byte swizzle).
__device__ __forceinline__ void decode_block(const BlockWords &w, int row, int jj, uint32_t atile) {
    const uint32_t rbase = atile + (uint32_t)row * 128u;
    const uint32_t d0 = prmt(w.s, w.s, 0x1010u), d1 = prmt(w.s, w.s, 0x3232u);  // (d, d) of each half
    uint32_t o[4][4];  // o[k][b]: elements 8k + 2b, 8k + 2b + 1
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        uint32_t v[4];
        decode_word(w.c[b], v);
#pragma unroll
        for (int k = 0; k < 4; ++k) o[k][b] = p_hmul2(v[k], k < 2 ? d0 : d1);  // elements 0..15: d0, 16..31: d1
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t chunk = (uint32_t)(4 * jj + k) ^ (uint32_t)(row & 7);
        p_sts128(rbase + chunk * 16u, o[k][0], o[k][1], o[k][2], o[k][3]);
    }
}

template <int OT>
__global__ void __launch_bounds__(kPThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ PrefillParams P) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t base = (uint32_t)__cvta_generic_to_shared(smem);
    if (base > kPMaxBase) {  // layout precondition (checked, never expected)
        if (threadIdx.x == 0) atomicOr(P.header, kPStatusLayout);
        return;
    }
    const uint32_t sbase = (base + 1023u) & ~1023u;
    const int n0 = blockIdx.x * kPM, m0 = blockIdx.y * kPN;
    auto a_tile = [&](int s) { return sbase + kPAOff + (uint32_t)s * kATile; };
    auto b_tile = [&](int s) { return sbase + kPBOff + (uint32_t)s * kBTile; };
    const uint32_t bars = sbase + kPBarOff;
    auto full_a = [&](int s) { return bars + 8u * s; };
    auto full_b = [&](int s) { return bars + 8u * (kSA + s); };
    auto empty_a = [&](int s) { return bars + 8u * (kSA + kSB + s); };
    auto empty_b = [&](int s) { return bars + 8u * (2 * kSA + kSB + s); };
    const uint32_t accum = bars + 8u * (2 * kSA + 2 * kSB);
    const uint32_t tmem_slot = sbase + kPTmemOff;

    // ---- set-up: barriers, tensor memory -------------------------------------
    if (threadIdx.x == 0) {
        for (int s = 0; s < kSA; ++s) {
            p_mbar_init(full_a(s), 32 * kDecodeWarps);
            p_mbar_init(empty_a(s), 1);
        }
        for (int s = 0; s < kSB; ++s) {
            p_mbar_init(full_b(s), 1);
            p_mbar_init(empty_b(s), 1);
        }
        p_mbar_init(accum, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tmem_slot),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    p_tc_fence_before();
    __syncthreads();
    p_tc_fence_after();
    const uint32_t tmem = p_lds_u32(tmem_slot);
    // both accumulators need the whole of tensor memory: checked, never expected
    const bool tmem_ok = tmem == 0u;
    if (!tmem_ok && threadIdx.x == 0) atomicOr(P.header, kPStatusTmem);
    // the activation tiles are the pre-rotation's output
    grid_dependency_wait();
    grid_dependents_launch();

    if (warp == 0) {
        // ---- activation tiles by TMA ----------------------------------------
        if (lane == 0) {
            int issued = 0;
            for (int kt = 0; kt < P.nk; ++kt) {
                const int s = kt % kSB;
                const uint32_t ph = (uint32_t)(kt / kSB) & 1u;
                if (!p_mbar_wait(empty_b(s), ph ^ 1u, P.timeout_ns)) {
                    atomicOr(P.header, kPStatusTimeout);
                    break;
                }
                if (P.inject_skip && kt == 1 && blockIdx.x == 0 && blockIdx.y == 0) {
                    // neither the copy nor its byte count: the stage never
                    // completes, no copy is left in flight, and the MMA
                    // thread's bounded wait on it runs out
                    ++issued;
                    continue;
                }
                p_mbar_expect_tx(full_b(s), kBTile);
                p_tma_load_2d(b_tile(s), &xmap, kt * kPK, m0, full_b(s));
                ++issued;
            }
            // no copy may still be in flight when the CTA exits
            for (int kt = issued > kSB ? issued - kSB : 0; kt < issued; ++kt)
                p_mbar_wait(full_b(kt % kSB), (uint32_t)(kt / kSB) & 1u, P.timeout_ns);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---- MMA issue ----------------------------------------------------------
        if (lane == 0) {
            for (int kt = 0; kt < P.nk; ++kt) {
                const int sa = kt % kSA, sb = kt % kSB;
                const uint32_t pa = (uint32_t)(kt / kSA) & 1u, pb = (uint32_t)(kt / kSB) & 1u;
                if (!p_mbar_wait(full_a(sa), pa, P.timeout_ns) || !p_mbar_wait(full_b(sb), pb, P.timeout_ns)) {
                    atomicOr(P.header, kPStatusTimeout);
                    break;
                }
                p_tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kPK / 16 && tmem_ok; ++kk) {  // 16 columns = 32 bytes along the swizzled row
                    const uint64_t bdesc = p_smem_desc(b_tile(sb) + 32u * kk);
                    const uint32_t acc = (kt | kk) != 0 ? 1u : 0u;
                    p_mma(tmem, p_smem_desc(a_tile(sa) + 32u * kk), bdesc, acc);                  // rows 0..127
                    p_mma(tmem + (uint32_t)kPN, p_smem_desc(a_tile(sa) + kAHalf + 32u * kk), bdesc, acc);  // 128..255
                }
                // the stages are free once these MMAs have read them
                p_mma_commit(empty_a(sa));
                p_mma_commit(empty_b(sb));
            }
            p_mma_commit(accum);  // the accumulators are final once every MMA has completed
        }
        __syncwarp();
    } else {
        // ---- weight tiles: decode (thread = one row, one 32-column block) ---------
        const int td = (warp - 2) * 32 + lane;
        const int row = td & (kPM - 1), jj = td / kPM;
        // row slots kAhead superblocks ahead, in a register ring (the loop is
        // unrolled by kAhead so that every ring index is a constant)
        RowSlot w[kAhead];
#pragma unroll
        for (int i = 0; i < kAhead; ++i) w[i] = load_slot(P, n0 + row, i);
        const int nsb_stages = (P.nk + 1) / 2;  // superblocks touched by the stages
        bool ok = true;
        for (int sb0 = 0; sb0 < nsb_stages && ok; sb0 += kAhead) {
#pragma unroll
            for (int i = 0; i < kAhead; ++i) {
                const int sb = sb0 + i;
                if (sb >= nsb_stages || !ok) break;
#pragma unroll
                for (int hb = 0; hb < 2; ++hb) {  // the superblock's two stages
                    const int kt = 2 * sb + hb;
                    if (kt >= P.nk) break;
                    const int s = kt % kSA;
                    const uint32_t ph = (uint32_t)(kt / kSA) & 1u;
                    // (warp-uniform decision: the epilogue below runs warp-synchronous loads)
                    if (!__all_sync(kFull, p_mbar_wait(empty_a(s), ph ^ 1u, P.timeout_ns))) {
                        if (lane == 0) atomicOr(P.header, kPStatusTimeout);
                        ok = false;
                        break;
                    }
                    decode_block(block_of(w[i], 2 * hb + jj), row, jj, a_tile(s));
                    p_fence_proxy_async();
                    p_mbar_arrive(full_a(s));
                }
                w[i] = load_slot(P, n0 + row, sb + kAhead);
            }
        }
        // ---- epilogue: tensor memory -> Y (all sixteen decode warps) ---------
        // warp w may read lanes 32 (w % 4) .. +31; four warps per quarter, each
        // reads four 32-column chunks of one accumulator (h = weight-row half)
        if (tmem_ok) {
            const int q = warp & 3;
            const int iq = (warp - 2) >> 2;          // 0..3 within the quarter
            const int h = iq >> 1;
            const int c0 = (iq & 1) * (kPN / 64);
            const int wrow = n0 + h * 128 + q * 32 + lane;
            if (!__all_sync(kFull, p_mbar_wait(accum, 0u, P.timeout_ns))) {
                if (lane == 0) atomicOr(P.header, kPStatusTimeout);
            } else {
                p_tc_fence_after();
#pragma unroll 1
                for (int c = c0; c < c0 + kPN / 64; ++c) {
                    uint32_t v[32];
                    p_tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * kPN + c * 32), v);
                    if (wrow < P.n) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int mrow = m0 + c * 32 + e;
                            if (mrow < P.m)
                                store1<OT>(P.y + ((int64_t)mrow * P.ldy + wrow) * ElemSize<OT>::value,
                                           __uint_as_float(v[e]));
                        }
                    }
                }
            }
        }
    }
    // ---- teardown ---------------------------------------------------------------
    p_tc_fence_before();
    __syncthreads();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
}

// ---- pre-rotation of X into plain row-major fp16 ---------------------------------
// xrot[row][col] = fp16(H(s .* x)/32) per 32-block (one warp per row and
// superblock: lane = block j (lane / 8) and four consecutive elements
// (lane % 8)); also clears the workspace status word.
struct PlainRotParams {
    const char *x;
    int64_t ldx;
    uint16_t *xrot;
    int64_t m;
    int k;
    int nsb;
    unsigned *header;
};

template <int DT>
__global__ void __launch_bounds__(256) prerotate_plain_kernel(const __grid_constant__ PlainRotParams R) {
    grid_dependency_wait();
    grid_dependents_launch();
    if (R.header && blockIdx.x == 0 && threadIdx.x == 0) {
        R.header[kHeaderStatus] = 0u;
        R.header[kHeaderTag] += 1u;
    }
    // Warp w owns superblock w % nsb of every (w / nsb + i * groups)-th row,
    // groups = (warps in the grid) / nsb >= 1: the lane's sign masks are
    // computed once, and each step loads kRows rows before rotating any, so
    // several loads per lane are in flight.
    constexpr int kRows = 4;
    const int lane = threadIdx.x & 31;
    const int j = lane >> 3, p = lane & 7;
    const int64_t gw = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int64_t groups = (int64_t)gridDim.x * 8 / R.nsb;
    const int64_t r0 = gw / R.nsb;
    if (r0 >= groups) return;  // past the last whole set of superblocks (warp-uniform)
    const int sb = (int)(gw - r0 * R.nsb);
    const uint32_t col0 = (uint32_t)sb * 128u + 32u * j + 4u * p;
    const bool valid = (int)col0 < R.k;  // k is a multiple of 32: whole blocks
    uint32_t msk[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) msk[i] = sign_mask(col0 + i);
    for (int64_t row = r0; row < R.m; row += kRows * groups) {
        float v[kRows][4];
#pragma unroll
        for (int u = 0; u < kRows; ++u) {
            const int64_t r = row + u * groups;
#pragma unroll
            for (int i = 0; i < 4; ++i) v[u][i] = 0.f;
            if (valid && r < R.m) load4<DT>(R.x + (r * R.ldx + col0) * ElemSize<DT>::value, v[u]);
        }
#pragma unroll
        for (int u = 0; u < kRows; ++u) {
            const int64_t r = row + u * groups;
#pragma unroll
            for (int i = 0; i < 4; ++i) v[u][i] = flip(v[u][i], msk[i]);
            butterfly_local4(v[u]);
#pragma unroll
            for (int st = 0; st < 3; ++st) {
                const int xo = 1 << st;
                const bool upper = (p & xo) != 0;
#pragma unroll
                for (int i = 0; i < 4; ++i) v[u][i] = butterfly_xlane(v[u][i], xo, upper);
            }
            if (valid && r < R.m) {
                const __half2 lo = __floats2half2_rn(__fmul_rn(v[u][0], 0.03125f), __fmul_rn(v[u][1], 0.03125f));
                const __half2 hi = __floats2half2_rn(__fmul_rn(v[u][2], 0.03125f), __fmul_rn(v[u][3], 0.03125f));
                uint2 o;
                o.x = *reinterpret_cast<const uint32_t *>(&lo);
                o.y = *reinterpret_cast<const uint32_t *>(&hi);
                *reinterpret_cast<uint2 *>(R.xrot + r * R.k + col0) = o;
            }
        }
    }
}

// ---- host side ------------------------------------------------------------------
using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                 const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link to
// the driver library).
EncodeTiled encode_tiled() {
    static std::once_flag once;
    static EncodeTiled fn = nullptr;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(ptr);
    });
    return fn;
}

// Base offset of dynamic shared memory in a CTA's shared window.
uint32_t prefill_smem_base() {
    int dev = 0, reserved = 1024;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess)
        reserved = 1024;
    return (uint32_t)reserved;
}

cudaLaunchAttribute pdl_attr() {
    cudaLaunchAttribute a;
    a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a.val.programmaticStreamSerializationAllowed = 1;
    return a;
}

template <int OT>
cudaError_t launch_prefill_kernel(const CUtensorMap &map, const PrefillParams &prm, dim3 grid, uint32_t smem,
                                  cudaStream_t stream) {
    cudaError_t err =
        cudaFuncSetAttribute(prefill_kernel<OT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kPThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1] = {pdl_attr()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prefill_kernel<OT>, map, prm);
}

template <int DT>
cudaError_t launch_plain_rotation(const PlainRotParams &r, cudaStream_t stream) {
    // one (row, superblock) step per warp and four rows per step at most,
    // about one resident wave (8 CTAs of 8 warps per SM), and at least one
    // warp per superblock
    DeviceInfo di;
    const cudaError_t err = device_info(&di);
    if (err != cudaSuccess) return err;
    int64_t grid = (r.m * r.nsb + 31) / 32;
    if (grid > (int64_t)di.sm_count * 8) grid = (int64_t)di.sm_count * 8;
    const int64_t min_grid = (r.nsb + 7) / 8;
    if (grid < min_grid) grid = min_grid;
    if (grid > 0x7fffffff) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1] = {pdl_attr()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prerotate_plain_kernel<DT>, r);
}

}  // namespace

size_t prefill_xrot_bytes(int64_t m, int64_t k) { return round_up((size_t)m * (size_t)k * 2u, 256); }

cudaError_t launch_prerotate_plain(const void *X, int xdtype, int64_t m, int64_t k, int64_t ldx, uint16_t *xrot,
                                   unsigned *header, cudaStream_t stream) {
    if (m < 1 || k < 32 || k % 32 != 0) return cudaErrorInvalidValue;
    PlainRotParams r = {static_cast<const char *>(X), ldx, xrot, m, (int)k, (int)superblocks(k), header};
    switch (xdtype) {
        case kF32: return launch_plain_rotation<kF32>(r, stream);
        case kBF16: return launch_plain_rotation<kBF16>(r, stream);
        case kF16: return launch_plain_rotation<kF16>(r, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_prefill_product(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k,
                                   const uint16_t *xrot, int64_t m, void *y, int ydtype, int64_t ldy,
                                   unsigned *header, cudaStream_t stream) {
    if (n < 1 || m < 1 || k < 32 || k % 32 != 0) return cudaErrorInvalidValue;
    const int64_t grid_y = (m + kPN - 1) / kPN, grid_x = (n + kPM - 1) / kPM;
    if (grid_y > 65535 || grid_x > 0x7fffffff) return cudaErrorInvalidValue;
    EncodeTiled encode = encode_tiled();
    if (!encode) return cudaErrorNotSupported;
    // the tensor map of xrot: k x m fp16, rows of k*2 bytes, boxes of
    // 64 columns x 256 rows, 128-byte swizzle, zero fill outside
    CUtensorMap map;
    const cuuint64_t dims[2] = {(cuuint64_t)k, (cuuint64_t)m};
    const cuuint64_t strides[1] = {(cuuint64_t)k * 2u};
    const cuuint32_t box[2] = {(cuuint32_t)kPK, (cuuint32_t)kPN};
    const cuuint32_t estr[2] = {1u, 1u};
    if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t *>(xrot), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    PrefillParams prm;
    prm.codes = codes;
    prm.scales = reinterpret_cast<const uint8_t *>(scales);
    prm.n = (int)n;
    prm.tiles = (int)tiles(n);
    prm.nsb = (int)superblocks(k);
    prm.m = (int)m;
    prm.nk = (int)((k + kPK - 1) / kPK);
    prm.y = static_cast<char *>(y);
    prm.ldy = ldy;
    prm.header = header;
    prm.inject_skip = (debug_flags() & kDebugSkipPrefillCopy) ? 1 : 0;
    prm.timeout_ns = prm.inject_skip ? 5000000ull : 1000000000ull;  // 5 ms under the test hook
    const uint32_t base = prefill_smem_base();
    if (base > kPMaxBase) return cudaErrorInvalidValue;
    const uint32_t smem = ((base + 1023u) & ~1023u) + kPEndOff - base;
    const dim3 grid((unsigned)grid_x, (unsigned)grid_y);
    switch (ydtype) {
        case kF32: return launch_prefill_kernel<kF32>(map, prm, grid, smem, stream);
        case kBF16: return launch_prefill_kernel<kBF16>(map, prm, grid, smem, stream);
        case kF16: return launch_prefill_kernel<kF16>(map, prm, grid, smem, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_prefill(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, const void *X,
                           int xdtype, int64_t m, int64_t ldx, uint16_t *xrot, void *y, int ydtype, int64_t ldy,
                           unsigned *header, cudaStream_t stream) {
    if (n < 1 || m < 1 || k < 32 || k % 32 != 0) return cudaErrorInvalidValue;
    if ((m + kPN - 1) / kPN > 65535) return cudaErrorInvalidValue;
    if (!encode_tiled()) return cudaErrorNotSupported;
    // 1. X -> plain fp16 pre-rotation (clears the status word)
    cudaError_t err = launch_prerotate_plain(X, xdtype, m, k, ldx, xrot, header, stream);
    if (err != cudaSuccess) return err;
    // 2. the product
    return launch_prefill_product(codes, scales, n, k, xrot, m, y, ydtype, ldy, header, stream);
}

}  // namespace tq
