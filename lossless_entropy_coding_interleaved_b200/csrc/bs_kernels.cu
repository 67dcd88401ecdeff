// bs_kernels.cu -- sm_100a kernels of libbs.
//
// decode_kernel: the hot path. It decodes interleaved-rANS chunks of BF16 words. The method
// is the one the "Qwen3.8-27B-BF16-NVLC-Lossless" model card describes in the paragraph
// after its accounting table:
//   - the sign+exponent symbol s is decoded with the tensor's rANS model;
//   - s selects the fraction's distribution and the 7-bit fraction f is decoded with it;
//   - w = (s << 7) | f is rebuilt bitwise.
// Layout and parameters: FORMAT.md sections 2-3.
//
// Mapping onto the B200:
//  * One warp decodes two 32-lane chunks at once (two independent dependency chains per
//    lane hide the latency of the table lookups). Lane j holds rANS state j of each chunk
//    (64-bit, kept as two 32-bit halves). Under the octet map of FORMAT.md section 3, a
//    lane owns 8 contiguous output weights per 8 steps. Those leave as one 16-byte store,
//    so a warp writes 512 contiguous bytes per chunk.
//  * The tensor's decode tables (s-table 8 B/slot, f-table rows 4 B/slot) are staged once
//    per CTA in shared memory, at offset 0 so that table addresses fold into constants. A
//    CTA of 20 warps (tables up to 64 KiB), 16 (up to 96 KiB) or 8 (up to 160 KiB) decodes
//    40, 32 or 16 chunks of the same tensor; 20 warps x 2 chains is the most that the
//    register file holds (96 registers per thread).
//  * Full 256-weight blocks take a path without store bounds; the ragged tail and chunks
//    of unequal length take a checked path.
//  * The word stream of a chunk is prefetched into its own shared-memory ring with
//    cp.async (16 B per lane, in quarters of 256 words), kept 2-3 quarters ahead; the
//    upkeep runs every 16 steps.
//  * The default precisions (ns=12, nf=10) get an instantiation with constant shifts.
//  * Renormalisation reads (at most one 32-bit word per lane per weight) are assigned in
//    lane order by ballot + prefix popcount. The words a step consumes are contiguous, so
//    the ring read is conflict-free.
//  * No tensor cores: nothing here is a contraction.
//  * Error handling: a chunk whose start state is out of range, whose lanes do not end
//    at L, or which does not consume exactly its n_words sets a flag in the error block.
//    All loops are bounded by the chunk's weight count; nothing traps.
#include <cuda_runtime.h>

#include <cstdint>

#include "bs_internal.h"

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
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// One chunk in flight on a warp: lane j holds state j as two 32-bit halves.
struct Chain {
    uint32_t lo, hi;          // rANS state x = hi:lo, in [2^32, 2^64) between weights
    uint32_t posb;            // bytes of the word stream consumed (warp-uniform)
    uint32_t fq;              // ring quarters requested (warp-uniform)
    uint32_t total_q, n_words, stream_bytes, nc, n_blocks;
    uint32_t ring;            // shared-memory address of the ring
    const uint8_t* ring_ptr;  // the same ring as a pointer into the dynamic smem array
    const uint8_t* stream;
    uint16_t* out;
    uint64_t chunk;
    bool live;                // a real chunk (false: a filler chain that is never stored)
    bool bad;
};

// x = freq * (x >> n) + bias on the split state, for 1 <= n <= 31.
__device__ __forceinline__ void rans_update(uint32_t& lo, uint32_t& hi, uint32_t freq, uint32_t bias, uint32_t n) {
    const uint32_t t_lo = __funnelshift_r(lo, hi, n);
    const uint32_t t_hi = hi >> n;
    const uint64_t p = static_cast<uint64_t>(freq) * t_lo + bias;
    lo = static_cast<uint32_t>(p);
    hi = static_cast<uint32_t>(p >> 32) + freq * t_hi;
}


// NS/NF > 0: compile-time precisions (the default container); 0: read from the item.
template <int WARPS, int NS, int NF>
__global__ void __launch_bounds__(WARPS * 32, 1) decode_kernel(const __grid_constant__ DecodeParams p) {
    // dynamic smem: [s-table][f-rows][rings]; the tables start at offset 0 so that table
    // addresses are an index times the entry size plus a constant
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ int s_item;
    const uint32_t tid = threadIdx.x, lane = tid & 31u, warp = tid >> 5;

    if (tid == 0) { // the item whose CTA range holds this block
        int lo = 0, hi = static_cast<int>(p.n_items) - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.item[mid].cta_begin <= blockIdx.x) lo = mid;
            else hi = mid - 1;
        }
        s_item = lo;
    }
    __syncthreads();
    const DecodeItem& it = p.item[s_item];

    // stage the tables
    const uint32_t tb = it.table_bytes;
    {
        uint4* dst = reinterpret_cast<uint4*>(smem);
        for (uint32_t k = tid; k < tb / 16u; k += blockDim.x) dst[k] = __ldg(it.tables + k);
    }
    __syncthreads();

    const uint32_t log2c = it.log2_chunk;
    const uint64_t C = 1ull << log2c;
    const uint64_t n_elems = it.n_elems;
    const uint64_t n_chunks = (n_elems + C - 1) >> log2c;
    const uint64_t chunk0 = static_cast<uint64_t>(blockIdx.x - it.cta_begin) * (WARPS * kChains) + warp * kChains;
    if (chunk0 >= n_chunks) return;

    const uint32_t ring_off = tb + (warp * kChains) * (kRingWords * 4); // this warp's first ring
    const uint32_t ring_base = smem_u32(smem) + ring_off;
    Chain c[kChains];
    uint32_t nb = 0;
#pragma unroll
    for (int k = 0; k < kChains; ++k) {
        Chain& h = c[k];
        h.chunk = chunk0 + k;
        h.live = h.chunk < n_chunks;
        h.ring = ring_base + k * (kRingWords * 4);
        h.ring_ptr = smem + ring_off + k * (kRingWords * 4);
        h.posb = 0;
        h.fq = 0;
        h.bad = false;
        if (h.live) {
            const uint8_t* ent = it.chunk_table + 16 * h.chunk;
            const uint64_t off = __ldg(reinterpret_cast<const unsigned long long*>(ent));
            h.n_words = __ldg(reinterpret_cast<const unsigned int*>(ent + 8));
            const uint8_t* payload = it.container + off;
            h.stream = payload + 256;
            h.stream_bytes = 4u * h.n_words;
            h.total_q = (h.n_words + kQuarterWords - 1) / kQuarterWords;
            const uint64_t base = h.chunk << log2c;
            h.nc = static_cast<uint32_t>(min(C, n_elems - base));
            h.n_blocks = (h.nc + 255u) >> 8; // blocks of 8 steps
            h.out = it.out + base;
            const uint64_t x = __ldg(reinterpret_cast<const unsigned long long*>(payload) + lane);
            h.lo = static_cast<uint32_t>(x);
            h.hi = static_cast<uint32_t>(x >> 32);
            h.bad = h.hi == 0;
        } else { // filler: decodes from L and its own (unfilled) ring; nothing is stored
            h.n_words = h.stream_bytes = h.total_q = h.nc = h.n_blocks = 0;
            h.stream = nullptr;
            h.out = nullptr;
            h.lo = 0;
            h.hi = 1;
        }
        nb = max(nb, h.n_blocks);
    }

    const uint32_t ns = NS > 0 ? NS : it.ns, nf = NF > 0 ? NF : it.nf;
    const uint32_t smask = (1u << ns) - 1u, fmask = (1u << nf) - 1u;
    const uint8_t* ftab = smem + (8u << ns);
    const uint32_t lt = lanemask_lt();

    // Ring upkeep before a block of 16 steps: request up to quarter q+3 for each chain,
    // where q holds the next word. The next 16 steps need at most quarters q..q+2. Wait for
    // every copy, or for all but the newest group when those were requested earlier.
    // Quarters wholly inside the stream skip the per-piece bounds.
    auto upkeep = [&](uint32_t blk) {
        __syncwarp();
        bool newest_needed = blk == 0;
#pragma unroll
        for (int k = 0; k < kChains; ++k) {
            Chain& h = c[k];
            if (blk < h.n_blocks) {
                const uint32_t q = h.posb / (kQuarterWords * 4u);
                if (h.fq <= min(q + 2, h.total_q - 1)) newest_needed = true;
                while (h.fq < q + 4 && h.fq < h.total_q) {
                    const uint32_t qb = h.fq * (kQuarterWords * 4u);
                    if (qb + kQuarterWords * 4u <= h.stream_bytes) {
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const uint32_t byte = qb + 16u * (lane + 32u * e);
                            cp_async16(h.ring + (byte & (kRingWords * 4u - 1u)), h.stream + byte, 16u);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const uint32_t byte = qb + 16u * (lane + 32u * e);
                            if (byte < h.stream_bytes)
                                cp_async16(h.ring + (byte & (kRingWords * 4u - 1u)), h.stream + byte,
                                           min(16u, h.stream_bytes - byte));
                        }
                    }
                    ++h.fq;
                }
            }
        }
        cp_async_commit();
        if (newest_needed) cp_async_wait<0>();
        else cp_async_wait<1>();
        __syncwarp();
    };

    // 8 steps of every chain, interleaved; o[k] receives chain k's 8 words as 4 pairs
    auto octet = [&](uint32_t (&o)[kChains][4]) {
#pragma unroll
        for (int s = 0; s < 8; ++s) {
#pragma unroll
            for (int k = 0; k < kChains; ++k) {
                Chain& h = c[k];
                // sign+exponent symbol
                const uint2 se = *reinterpret_cast<const uint2*>(smem + ((h.lo & smask) << 3));
                rans_update(h.lo, h.hi, se.x & 0xFFFFu, se.x >> 16, ns);
                // fraction, from the row the symbol's exponent selects (frow_field)
                const uint32_t fslot = h.lo & fmask;
                const uint32_t fe = *reinterpret_cast<const uint32_t*>(
                    ftab + (nf <= 10 ? (se.y >> 16) + (fslot << 2) : ((se.y >> 16) + fslot) << 2));
                rans_update(h.lo, h.hi, (fe >> 7) & 0xFFFu, fe >> 19, nf);
                // renormalise: lanes below 2^32 take the next words, in lane order
                // (branch-free: every lane reads; the ones that need no word discard it)
                const bool need = h.hi == 0;
                const uint32_t m = __ballot_sync(0xFFFFFFFFu, need);
                const uint32_t w = *reinterpret_cast<const uint32_t*>(
                    h.ring_ptr + ((h.posb + (__popc(m & lt) << 2)) & (kRingWords * 4u - 1u)));
                h.hi = need ? h.lo : h.hi;
                h.lo = need ? w : h.lo;
                h.posb += __popc(m) << 2;
                // w = (s << 7) | f: s sits pre-shifted in se.y
                const uint32_t word = (se.y & 0xFF80u) | (fe & 0x7Fu);
                if (s & 1) o[k][s >> 1] = __byte_perm(o[k][s >> 1], word, 0x5410);
                else o[k][s >> 1] = word;
            }
        }
    };

    // Full blocks first: every live chain has all 256 weights of the block, so the stores
    // need no bounds; blocks are taken two at a time.
    uint32_t nb_full = 0xFFFFFFFFu;
#pragma unroll
    for (int k = 0; k < kChains; ++k)
        if (c[k].live) nb_full = min(nb_full, c[k].nc >> 8);
    uint32_t blk = 0;
    for (; blk + 2 <= nb_full; blk += 2) {
        upkeep(blk);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            uint32_t o[kChains][4];
            octet(o);
            const uint32_t b = blk + half, i0 = (b << 8) + (lane << 3);
#pragma unroll
            for (int k = 0; k < kChains; ++k) {
                Chain& h = c[k];
                if (h.live) *reinterpret_cast<uint4*>(h.out + i0) = make_uint4(o[k][0], o[k][1], o[k][2], o[k][3]);
                if (b + 1 == h.n_blocks) // end check: state back at L, every word consumed
                    h.bad |= (h.lo != 0) | (h.hi != 1) | (h.posb != h.stream_bytes);
            }
        }
    }
    // The rest (ragged tails, chains of different lengths), with bounds, two blocks at a time.
    for (; blk < nb; blk += 2) {
        upkeep(blk);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const uint32_t b = blk + half;
            if (b >= nb) break;
            uint32_t o[kChains][4];
            octet(o);
#pragma unroll
            for (int k = 0; k < kChains; ++k) {
                Chain& h = c[k];
                if (b < h.n_blocks) {
                    const uint32_t i0 = (b << 8) + (lane << 3);
                    if (i0 + 8 <= h.nc) {
                        *reinterpret_cast<uint4*>(h.out + i0) = make_uint4(o[k][0], o[k][1], o[k][2], o[k][3]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            if (i0 + e < h.nc) h.out[i0 + e] = static_cast<uint16_t>(o[k][e >> 1] >> (16 * (e & 1)));
                    }
                    if (b + 1 == h.n_blocks) // end check: state back at L, every word consumed
                        h.bad |= (h.lo != 0) | (h.hi != 1) | (h.posb != h.stream_bytes);
                }
            }
        }
    }
    cp_async_wait<0>();

#pragma unroll
    for (int k = 0; k < kChains; ++k) {
        if (c[k].live && __any_sync(0xFFFFFFFFu, c[k].bad) && lane == 0) {
            atomicOr(p.err, 1ull);
            atomicMin(p.err + 1, (static_cast<unsigned long long>(it.tensor_index) << 40) | c[k].chunk);
        }
    }
}

// Verbatim copy of STORED and RAW tensors: one CTA per 64 KiB block.
__global__ void __launch_bounds__(256) copy_kernel(const __grid_constant__ CopyParams p) {
    int lo = 0, hi = static_cast<int>(p.n_items) - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.item[mid].blk_begin <= blockIdx.x) lo = mid;
        else hi = mid - 1;
    }
    const CopyItem& it = p.item[lo];
    const uint64_t start = (blockIdx.x - it.blk_begin) * kCopyBlockBytes;
    if (start >= it.bytes) return;
    const uint64_t len = min(kCopyBlockBytes, it.bytes - start);
    const uint8_t* src = it.src + start;
    uint8_t* dst = it.dst + start;
    const bool vec = ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15u) == 0;
    const uint64_t nv = vec ? len / 16 : 0;
    for (uint64_t k = threadIdx.x; k < nv; k += blockDim.x)
        reinterpret_cast<uint4*>(dst)[k] = __ldg(reinterpret_cast<const uint4*>(src) + k);
    for (uint64_t k = nv * 16 + threadIdx.x; k < len; k += blockDim.x) dst[k] = src[k];
}

// FORMAT.md section 7: splitmix64 output for state v.
__device__ __forceinline__ unsigned long long mix64(unsigned long long v) {
    unsigned long long z = v + 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__global__ void __launch_bounds__(256) checksum_kernel(const void* data, uint64_t n, int raw_bytes,
                                                       unsigned long long* sum) {
    unsigned long long acc = 0;
    const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
    if (raw_bytes) {
        const uint8_t* b = static_cast<const uint8_t*>(data);
        for (uint64_t i = blockIdx.x * static_cast<uint64_t>(blockDim.x) + threadIdx.x; i < n; i += stride)
            acc += mix64((i << 8) | b[i]);
    } else {
        const uint16_t* w = static_cast<const uint16_t*>(data);
        for (uint64_t i = blockIdx.x * static_cast<uint64_t>(blockDim.x) + threadIdx.x; i < n; i += stride)
            acc += mix64((i << 16) | w[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
    if ((threadIdx.x & 31u) == 0) atomicAdd(sum, acc);
}

int max_dynamic_smem() {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return 0;
    return v;
}

template <int WARPS, int NS, int NF>
static int launch_decode_t(const DecodeParams& p, uint32_t smem_bytes, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<WARPS, NS, NF>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem_bytes));
    if (e != cudaSuccess) return e;
    decode_kernel<WARPS, NS, NF><<<p.total_ctas, WARPS * 32, smem_bytes, s>>>(p);
    count_launch();
    return cudaGetLastError();
}

int launch_decode(const DecodeParams& p, int warps, bool default_precision, uint32_t smem_bytes, void* stream) {
    if (p.total_ctas == 0) return cudaSuccess;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (warps == 20)
        return default_precision ? launch_decode_t<20, 12, 10>(p, smem_bytes, s) : launch_decode_t<20, 0, 0>(p, smem_bytes, s);
    if (warps == 16)
        return default_precision ? launch_decode_t<16, 12, 10>(p, smem_bytes, s) : launch_decode_t<16, 0, 0>(p, smem_bytes, s);
    return default_precision ? launch_decode_t<8, 12, 10>(p, smem_bytes, s) : launch_decode_t<8, 0, 0>(p, smem_bytes, s);
}

int launch_copy(const CopyParams& p, void* stream) {
    if (p.total_blocks == 0) return cudaSuccess;
    copy_kernel<<<static_cast<unsigned>(p.total_blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
    count_launch();
    return cudaGetLastError();
}

int launch_checksum(const void* data, uint64_t n, int raw_bytes, unsigned long long* d_sum, void* stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(d_sum, 0, sizeof(unsigned long long), s);
    if (e != cudaSuccess) return e;
    if (n == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const uint64_t want = (n + 255) / 256;
    const unsigned grid = static_cast<unsigned>(want < static_cast<uint64_t>(sms) * 8 ? want : sms * 8ull);
    checksum_kernel<<<grid, 256, 0, s>>>(data, n, raw_bytes, d_sum);
    count_launch();
    return cudaGetLastError();
}

} // namespace bs
