// tq_internal.h -- launchers behind the C ABI (host side, no validation here:
// the C ABI checks every argument before calling them).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace tq {

struct DeviceInfo {
    int device;
    int sm_count;
};

// Current device and its SM count (cached per device).
cudaError_t device_info(DeviceInfo *out);

cudaError_t launch_quantize(const void *w, int dtype, int64_t n, int64_t k, int64_t ldw, uint8_t *codes,
                            uint16_t *scales, cudaStream_t stream);

cudaError_t launch_dequantize(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, void *w_out,
                              int dtype, int64_t ldo, cudaStream_t stream);

// xrot for m rows; also zeroes `counters` (count entries) when non-null.
cudaError_t launch_prerotate(const void *X, int dtype, int64_t m, int64_t k, int64_t ldx, uint16_t *xrot,
                             unsigned *counters, int64_t counters_count, cudaStream_t stream);

// Skinny product for m <= 32 rows of pre-rotated activations.
struct SkinnyPlan {
    int64_t tiles;        // ceil(n / 16)
    int64_t units;        // tiles * nsb
    int grid;             // CTAs
    int total_warps;      // min(grid * warps per CTA, units): warps that own work
    int mcap;             // 8 * ceil(m / 8)
    size_t counter_bytes; // tiles * 4, rounded up to 256
    size_t partial_bytes; // (tiles + total_warps) * 16 * mcap * 4
};

SkinnyPlan plan_skinny(int64_t m, int64_t n, int64_t k, int sm_count);

cudaError_t launch_skinny(const uint8_t *codes, const uint16_t *scales, int64_t n, int64_t k, const uint16_t *xrot,
                          int64_t m, void *Y, int dtype, int64_t ldy, const SkinnyPlan &plan, unsigned *counters,
                          float *partials, bool programmatic, cudaStream_t stream);

inline int64_t superblocks(int64_t k) { return (k / 32 + 3) / 4; }
inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace tq
