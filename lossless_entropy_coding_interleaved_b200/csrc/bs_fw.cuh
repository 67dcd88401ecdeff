// bs_fw.cuh -- definitions shared by the kernels of the fixed-width lane layout
// (4-bit sign+exponent codes, 7-bit fractions, exceptions): the decode in bs_fw.cu and the fused
// GEMV in bs_fw_gemv.cu.
// Nothing here is shared with the oracle.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "bs_host.h"
#include "bs_internal.h"

namespace bs {
namespace fw {

constexpr uint32_t kFwTile = 256;
constexpr uint32_t kFwHeader = 64;
constexpr uint32_t kFwPlanesAt = kFwHeader + 32;  // after the header and the code table
constexpr uint64_t kFwMaxElems = 1ull << 40;

__host__ __device__ inline uint64_t up16(uint64_t v) { return (v + 15) & ~uint64_t(15); }

// Byte layout: section offsets from the start of the layout.
struct FwOffsets {
    uint64_t a, b, c, tile_exc, exc_pos, exc_word, total;
};
__host__ __device__ inline FwOffsets fw_offsets(uint64_t n_tiles, uint64_t n_exc) {
    FwOffsets o;
    o.a = kFwPlanesAt;
    o.b = o.a + 128 * n_tiles;
    o.c = o.b + 128 * n_tiles;
    o.tile_exc = o.c + 96 * n_tiles;
    o.exc_pos = o.tile_exc + up16(4 * (n_tiles + 1));
    o.exc_word = o.exc_pos + up16(n_exc);
    o.total = o.exc_word + up16(2 * n_exc);
    return o;
}
__host__ __device__ inline uint64_t fw_tiles(uint64_t n) { return (n + kFwTile - 1) / kFwTile; }

// The ring of a warp: groups of kFwGroup consecutive tiles, kFwStages slots.
constexpr int kFwGroup = 4;
constexpr int kFwStages = 3;
// One slot: plane A (512 B), plane B (512 B), plane C (384 B), tile_exc (5 of 8 entries).
constexpr uint32_t kSlotA = 0, kSlotB = 512, kSlotC = 1024, kSlotTE = 1408, kSlotBytes = 1440;

__device__ __forceinline__ void fw_cp16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void fw_cp4(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void fw_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N> // all but the N most recent commit groups have landed
__device__ __forceinline__ void fw_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}
__device__ __forceinline__ void fw_wait_older() { fw_wait<kFwStages - 1>(); }

// The 8 weights of one lane in one tile. Output word q is the pair of steps (2q, 2q+1).
__device__ __forceinline__ uint4 fw_octet(const uint32_t* pair_tab, uint32_t a, uint32_t b, uint32_t c0, uint32_t c1,
                                          uint32_t csh) {
    const uint32_t c = __funnelshift_r(c0, c1, csh);                        // the lane's 24-bit plane C field
    const uint32_t r4 = ((c << 4) & 0xFFFFu) | ((c << 8) & 0xFFFF0000u);   // step 2q's top bits at 4+3q, 2q+1's at 20+3q
    uint4 w;
    w.x = pair_tab[a & 0xFFu] | (b & 0x000F000Fu) | (r4 & 0x00700070u);
    w.y = pair_tab[(a >> 8) & 0xFFu] | ((b >> 4) & 0x000F000Fu) | ((r4 >> 3) & 0x00700070u);
    w.z = pair_tab[(a >> 16) & 0xFFu] | ((b >> 8) & 0x000F000Fu) | ((r4 >> 6) & 0x00700070u);
    w.w = pair_tab[a >> 24] | ((b >> 12) & 0x000F000Fu) | ((r4 >> 9) & 0x00700070u);
    return w;
}

inline bool fw_aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

inline bs_status fw_device_ok() {
    int dev = 0, major = 0, minor = 0;
    const cudaError_t ce = cudaGetDevice(&dev);
    if (ce != cudaSuccess) return cuda_status(ce);
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    return major == 10 && minor == 0 ? BS_OK : BS_E_UNSUPPORTED;
}

// The header fields of section 10 that a decode depends on, checked against each other.
inline bool fw_info_ok(const bs_fw_info& i) {
    if (i.n_elems > kFwMaxElems || i.n_tiles != fw_tiles(i.n_elems)) return false;
    if (i.n_exc >= (1ull << 32) || i.n_exc > i.n_elems) return false;
    if (i.total_bytes != fw_offsets(i.n_tiles, i.n_exc).total) return false;
    for (int k = 0; k < 16; ++k)
        if (i.table[k] >= 512) return false;
    return true;
}

} // namespace fw
} // namespace bs
