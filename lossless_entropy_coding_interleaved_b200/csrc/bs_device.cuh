// bs_device.cuh -- small device helpers shared by libbs's decode kernels.
#pragma once

#include <cstdint>

namespace bs {

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// cp.async of up to 16 bytes (the rest of the 16-byte destination is zero-filled).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
// The same, issued only when `on` is nonzero (a predicated instruction, no branch). A lane
// that is off reads nothing, so its source address need not be valid.
__device__ __forceinline__ void cp_async16_if(uint32_t on, uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("{\n .reg .pred p;\n setp.ne.u32 p, %3, 0;\n @p cp.async.cg.shared.global [%0], [%1], 16, %2;\n}\n"
                 ::"r"(dst), "l"(src), "r"(src_bytes), "r"(on) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// The item of a launch whose CTA range holds this block: a binary search over cta_begin,
// done by thread 0 into *slot.
template <typename Params>
__device__ __forceinline__ void find_item(const Params& p, int* slot) {
    int lo = 0, hi = static_cast<int>(p.n_items) - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.item[mid].cta_begin <= blockIdx.x) lo = mid;
        else hi = mid - 1;
    }
    *slot = lo;
}

} // namespace bs
