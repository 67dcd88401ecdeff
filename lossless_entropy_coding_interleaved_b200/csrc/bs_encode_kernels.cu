// bs_encode_kernels.cu -- sm_100a kernels of the container encoder: histograms and the lane encode.
//
// histogram_kernel: per-tensor counts of the pairs j = w >> 4 = (s << 3) | h (sign+exponent
// symbol s, the fraction's top three bits h) and of the low nibbles. The s counts and the
// (exponent, h) counts that the factored model needs are sums of pair counts, and the JOINT
// model uses the pair counts as they are. The counts go into per-CTA
// shared memory, then into global 64-bit bins.
//
// encode_kernel: one warp per chunk, lane j holds rANS state j (32-bit). It walks its
// steps backwards from L = 2^16: each weight renormalises
// at most once (one 16-bit word) and is one step of the product alphabet (s, h). The count
// pass records how many words each chunk emits. The write pass places the words of step t
// (lane order) just before those of step t+1, starting from the end of the chunk's word
// area. That is the interleaved (step, lane) order of the word stream, with no staging buffer. The
// write pass also stores the nibble words when the tensor keeps them.
#include <cuda_runtime.h>

#include <cstdint>

#include "bs_internal.h"

namespace bs {

__global__ void __launch_bounds__(512) histogram_kernel(const uint16_t* __restrict__ in, uint64_t n,
                                                        unsigned long long* __restrict__ hist) {
    extern __shared__ unsigned int h[]; // kHistBins counters
    for (uint32_t k = threadIdx.x; k < kHistBins; k += blockDim.x) h[k] = 0;
    __syncthreads();
    const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
    for (uint64_t i = blockIdx.x * static_cast<uint64_t>(blockDim.x) + threadIdx.x; i < n; i += stride) {
        const uint32_t w = in[i];
        atomicAdd(&h[w >> 4], 1u);
        atomicAdd(&h[4096 + (w & 15u)], 1u);
    }
    __syncthreads();
    for (uint32_t k = threadIdx.x; k < kHistBins; k += blockDim.x)
        if (h[k]) atomicAdd(hist + k, static_cast<unsigned long long>(h[k]));
}

int launch_histogram(const uint16_t* in, uint64_t n, unsigned long long* d_hist, void* stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(d_hist, 0, sizeof(unsigned long long) * kHistBins, s);
    if (e != cudaSuccess || n == 0) return e;
    const int smem = static_cast<int>(sizeof(unsigned int) * kHistBins);
    e = cudaFuncSetAttribute(histogram_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // each CTA counts at most 2^30 weights, so its 32-bit shared counters cannot wrap
    uint64_t grid = static_cast<uint64_t>(sms);
    while (grid * (1ull << 30) < n) grid += sms;
    const uint64_t want = (n + 4095) / 4096;
    if (want < grid) grid = want;
    histogram_kernel<<<static_cast<unsigned>(grid), 512, smem, s>>>(in, n, d_hist);
    count_launch();
    return cudaGetLastError();
}

__global__ void __launch_bounds__(kEncWarps * 32) encode_kernel(const __grid_constant__ EncParams p) {
    __shared__ int s_item;
    __shared__ uint32_t tab[kEncTableWordsMax]; // factored tables, or the JOINT table
    const uint32_t tid = threadIdx.x, lane = tid & 31u, warp = tid >> 5;
    if (tid == 0) {
        int lo = 0, hi = static_cast<int>(p.n_items) - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.item[mid].cta_begin <= blockIdx.x) lo = mid;
            else hi = mid - 1;
        }
        s_item = lo;
    }
    __syncthreads();
    const EncItem& it = p.item[s_item];
    for (uint32_t k = tid; k < it.table_words; k += blockDim.x) tab[k] = it.tables[k];
    __syncthreads();

    const uint32_t log2c = it.log2_chunk;
    const uint64_t C = 1ull << log2c;
    const uint64_t n = it.n_elems;
    const uint64_t n_chunks = (n + C - 1) >> log2c;
    const uint64_t chunk = static_cast<uint64_t>(blockIdx.x - it.cta_begin) * kEncWarps + warp;
    if (chunk >= n_chunks) return;
    const uint64_t base = chunk << log2c;
    const uint32_t nc = static_cast<uint32_t>(min(C, n - base));
    const uint32_t n_blocks = (nc + 255u) >> 8;
    const uint32_t ns = it.ns, nh = it.nh, P = ns + nh;
    const uint32_t* stab = tab;
    const uint32_t* hrows = tab + 512;
    const uint8_t* route = reinterpret_cast<const uint8_t*>(tab + 512 + 8 * (it.n_routes + 1));
    const uint16_t* in = it.in + base;
    const uint32_t lt = (1u << lane) - 1u;

    uint32_t x = kStateL;
    uint32_t cnt = 0;                                     // count pass
    uint32_t end = p.write ? it.n_words[chunk] : 0;       // write pass: next free word, from the end
    uint8_t* payload = nullptr;
    uint16_t* words = nullptr;
    if (p.write) {
        payload = p.container + it.chunk_off[chunk];
        words = reinterpret_cast<uint16_t*>(payload + 128 + (it.nib_stored ? 128u * n_blocks : 0u));
    }

    for (uint32_t b = n_blocks; b-- > 0;) {
        const uint32_t i0 = (b << 8) + (lane << 3);
        uint16_t v[8];
        if (i0 + 8 <= nc) {
            const uint4 q = *reinterpret_cast<const uint4*>(in + i0);
            const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int k = 0; k < 8; ++k) v[k] = static_cast<uint16_t>(u[k >> 1] >> (16 * (k & 1)));
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) v[k] = (i0 + k < nc) ? in[i0 + k] : it.pad_word;
        }
        if (p.write && it.nib_stored) { // step k's nibble sits at bit 4*(k >> 1) + 16*(k & 1)
            uint32_t nib = 0;
#pragma unroll
            for (int k = 0; k < 8; ++k) nib |= static_cast<uint32_t>(v[k] & 15u) << (4 * (k >> 1) + 16 * (k & 1));
            reinterpret_cast<uint32_t*>(payload + 128)[32u * b + lane] = nib;
        }
#pragma unroll
        for (int k = 7; k >= 0; --k) {
            const uint32_t w = v[k], s = w >> 7, e = s & 0xFFu, h = (w >> 4) & 7u;
            uint32_t Q, qh = 1, cs = 0, ch = 0; // JOINT: Q = Fj[j], cs = cum(j)
            if (it.joint) {
                const uint32_t je = tab[w >> 4];
                Q = je & 0xFFFFu;
                cs = je >> 16;
            } else {
                const uint32_t se = stab[s], he = hrows[route[e] * 8u + h];
                const uint32_t qs = se & 0xFFFFu;
                cs = se >> 16;
                qh = he & 0xFFFFu;
                ch = he >> 16;
                Q = qs * qh;
            }
            const bool emit = static_cast<uint64_t>(x) >= (static_cast<uint64_t>(Q) << (32 - P));
            if (p.write) {
                const uint32_t m = __ballot_sync(0xFFFFFFFFu, emit);
                const uint32_t k_t = __popc(m);
                if (k_t <= end) {
                    if (emit) words[end - k_t + __popc(m & lt)] = static_cast<uint16_t>(x);
                    end -= k_t;
                } else { // more words than the count pass saw: report, never write out of range
                    if (lane == 0) atomicOr(p.err, 1u);
                    end = 0;
                }
            } else {
                cnt += emit;
            }
            if (emit) x >>= 16;
            const uint32_t r = x % Q;
            if (it.joint) x = ((x / Q) << P) + cs + r; // the JOINT kind: x = (x / Fj) * 2^nj + cum(j) + x % Fj
            else x = ((x / Q) << P) + ((cs + r / qh) << nh) + ch + r % qh;
        }
    }
    if (p.write) {
        reinterpret_cast<uint32_t*>(payload)[lane] = x;
        if (lane == 0 && end != 0) atomicOr(p.err, 1u);
    } else {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xFFFFFFFFu, cnt, o);
        if (lane == 0) it.n_words[chunk] = cnt;
    }
}

int launch_encode(const EncParams& p, void* stream) {
    if (p.total_ctas == 0) return cudaSuccess;
    encode_kernel<<<p.total_ctas, kEncWarps * 32, 0, static_cast<cudaStream_t>(stream)>>>(p);
    count_launch();
    return cudaGetLastError();
}

} // namespace bs
