// bs_kernels.cu -- sm_100a kernels of libbs.
//
// decode_kernel: the hot path. It decodes interleaved-rANS chunks of BF16 words. The method
// is the one the "Qwen3.8-27B-BF16-NVLC-Lossless" model card describes in the paragraph
// after its accounting table:
//   - the sign+exponent symbol s is decoded with the tensor's rANS model;
//   - s selects the fraction's distribution (here over the fraction's top three bits h;
//     the low four bits u are stored verbatim) and h is decoded with it;
//   - w = (s << 7) | (h << 4) | u is rebuilt bitwise.
// Layout and parameters: the BF16RANS container, version 2.
//
// Mapping onto the B200:
//  * One warp decodes two 32-lane chunks at once (two independent dependency chains per
//    lane hide the latency of the table lookups). Lane j holds rANS state j of each chunk,
//    a 32-bit state. Under the octet map (weight i of a chunk goes to lane (i >> 3) & 31 at
//    step 8 * (i >> 8) + (i & 7)), a lane owns 8 contiguous
//    output weights per 8 steps. Those leave as one 16-byte store, so a warp writes 512
//    contiguous bytes per chunk.
//  * One weight is one state update: the P-bit slot gives the s-entry (its high ns bits)
//    and the fraction entry (its low nh bits) at once, and x = Q*(x >> P) + B with
//    Q = Fs*Fh and B = bs*Fh + bh. No 64-bit arithmetic, no second update.
//  * The s-table (8 B/entry) is staged in shared memory once per CTA. The fraction rows
//    are staged with one copy per lane, so lane c always reads bank c: that lookup never
//    conflicts. The fraction region sits at offset 0 and the s-table at a constant offset,
//    so table addresses fold into constants.
//  * Full 256-weight blocks take a path without store bounds; the ragged tail and chunks
//    of unequal length take a checked path.
//  * The 16-bit word stream of a chunk is prefetched into its own 2 KiB shared-memory ring
//    with cp.async (16 B per lane, in quarters of 512 B), kept 2-3 quarters ahead; the
//    upkeep runs every 16 steps. The same upkeep copies the nibble words (128 B per block)
//    four blocks ahead into a 1 KiB ring, so no global load sits on the decode loop.
//  * The default precisions (ns=11, nh=5) get an instantiation with constant shifts.
//  * Renormalisation reads (at most one 16-bit word per lane per weight) are assigned in
//    lane order by ballot + prefix popcount. The words a step consumes are contiguous, so
//    the ring read is conflict-free.
//  * No tensor cores: nothing here is a contraction.
//  * Error handling: a chunk whose start state is out of range, whose lanes do not end
//    at L, or which does not consume exactly its n_words sets a flag in the error block.
//    All loops are bounded by the chunk's weight count; nothing traps.
#include <cuda_runtime.h>

#include <cstdint>

#include "bs_device.cuh"
#include "bs_internal.h"

namespace bs {

// One chunk in flight on a warp: lane j holds state j.
// Only what the step loop needs stays in registers; the rest (the rings' offsets, the block
// and quarter counts, the stream and nibble pointers, the chunk index) is derived where it is
// used. Chain k's word ring sits at ring_off + k * kRingBytes and its nibble ring at
// nring_off + k * kNibRingBytes, from the warp's two offsets.
struct Chain {
    uint32_t x;               // rANS state, in [2^16, 2^32) between weights
    uint32_t posb;            // bytes of the word stream consumed (warp-uniform)
    uint32_t fq;              // ring quarters requested (warp-uniform)
    uint32_t stream_bytes, nc; // blocks of 8 steps: (nc + 255) >> 8
    uint32_t raw;             // nibble word of the current block (constant mode: c in every nibble)
    const uint8_t* payload;   // the chunk's payload: start states, nibble words (if stored), words
    bool live;                // a real chunk (false: a filler chain that is never stored)
    bool bad;
};

// NS/NH > 0: compile-time precisions (the default container); 0: read from the item.
// SHAPE_FROM_PARAMS: the launch's warps per CTA come from the parameters (small launches);
// otherwise the CTA has WARPS warps, a compile-time constant (measured 3% faster).
// JOINT: the JOINT kind: one table of 2^nj slots over the pairs (s, h) (nj = item.ns),
// one lookup and one multiply-add per weight.
// (JOINT tensors with 4-byte slot entries have a kernel of their own, bs_joint4.cu.)
template <int WARPS, int CHAINS, int NS, int NH, bool SHAPE_FROM_PARAMS, bool JOINT>
__global__ void __launch_bounds__(WARPS * 32, 1) decode_kernel(const __grid_constant__ DecodeParams p) {
    constexpr int kChains = CHAINS;
    // dynamic smem: [fraction rows, one copy per lane][s-table][rings], or for JOINT
    // [joint table][rings]
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ int s_item;
    const uint32_t tid = threadIdx.x, lane = tid & 31u, warp = tid >> 5;

    if (tid == 0) find_item(p, &s_item); // the item whose CTA range holds this block
    __syncthreads();
    const DecodeItem& it = p.item[s_item];
    const uint32_t ns = NS > 0 ? NS : it.ns, nh = NH > 0 ? NH : it.nh, P = ns + nh;

    if (JOINT) { // stage the joint table as it is
        const uint32_t jb = 8u << ns;
        uint4* jdst = reinterpret_cast<uint4*>(smem);
        for (uint32_t k = tid; k < jb / 16u; k += blockDim.x) jdst[k] = __ldg(it.tables + k);
    } else { // stage the tables: the s-table as it is, each fraction entry once per lane
        const uint32_t sb = 8u << ns;
        uint4* sdst = reinterpret_cast<uint4*>(smem + kHRegion);
        for (uint32_t k = tid; k < sb / 16u; k += blockDim.x) sdst[k] = __ldg(it.tables + k);
        const uint32_t* hsrc = reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint8_t*>(it.tables) + sb);
        uint32_t* hdst = reinterpret_cast<uint32_t*>(smem);
        const uint32_t hwords = (uint32_t(it.n_routes) + 1u) << (nh + 5);
        for (uint32_t k = tid; k < hwords; k += blockDim.x) hdst[k] = __ldg(hsrc + (k >> 5));
    }
    __syncthreads();

    const uint32_t log2c = it.log2_chunk;
    const uint64_t C = 1ull << log2c;
    const uint64_t n_elems = it.n_elems;
    const uint64_t n_chunks = (n_elems + C - 1) >> log2c;
    const uint32_t warps = SHAPE_FROM_PARAMS ? p.warps : WARPS; // WARPS also bounds the registers
    const uint64_t chunk0 = static_cast<uint64_t>(blockIdx.x - it.cta_begin) * (warps * kChains) + warp * kChains;
    if (chunk0 >= n_chunks) return;

    const bool nib_stored = it.nib_mode == 0;
    const uint32_t raw_const = (it.nib_mode & 15u) * 0x11111111u;
    const uint32_t rings = JOINT ? kJointRegion : kHRegion + s_region_bytes(ns); // a multiple of kRingBytes
    const uint32_t ring_off = rings + (warp * kChains) * kRingBytes;       // this warp's first word ring
    const uint32_t nring_off = rings + warps * kChains * kRingBytes + (warp * kChains) * kNibRingBytes;
    const uint32_t smem_base = smem_u32(smem);
    uint16_t* const out0 = it.out + (chunk0 << log2c); // chain k writes from out0 + k * C
    Chain c[kChains];
    uint32_t nb = 0;
#pragma unroll
    for (int k = 0; k < kChains; ++k) {
        Chain& h = c[k];
        const uint64_t chunk = chunk0 + k;
        h.live = chunk < n_chunks;
        h.posb = 0;
        h.fq = 0;
        h.bad = false;
        h.raw = raw_const;
        if (h.live) {
            const uint8_t* ent = it.chunk_table + 16 * chunk;
            const uint64_t off = __ldg(reinterpret_cast<const unsigned long long*>(ent));
            const uint32_t n_words = __ldg(reinterpret_cast<const unsigned int*>(ent + 8));
            h.payload = it.container + off;
            const uint64_t base = chunk << log2c;
            h.nc = static_cast<uint32_t>(min(C, n_elems - base));
            h.stream_bytes = 2u * n_words;
            h.x = __ldg(reinterpret_cast<const unsigned int*>(h.payload) + lane);
            h.bad = h.x < kStateL;
        } else { // filler: decodes from L and its own (unfilled) ring; nothing is stored
            h.stream_bytes = h.nc = 0;
            h.payload = nullptr;
            h.x = kStateL;
        }
        nb = max(nb, (h.nc + 255u) >> 8);
    }

    const uint32_t smask8 = ((1u << ns) - 1u) << 3, hmask7 = ((1u << nh) - 1u) << 7; // JOINT: smask8 masks the slot
    const uint32_t lt = lanemask_lt(), lane4 = lane << 2;
    const uint32_t mul2 = p.mul2, mul65536 = p.mul65536;

    // Ring upkeep before a block of 16 steps: request up to quarter q+3 for each chain,
    // where q holds the next word. The next 16 steps need at most quarters q..q+2 (at most
    // 32 lanes x 16 steps x 2 bytes = 1 KiB). Wait for every copy, or for all but the
    // newest group when those were requested earlier. Quarters wholly inside the stream
    // skip the per-piece bounds.
    // Nibble words: at block blk (even) the ring must hold blocks blk and blk+1, which were
    // requested one upkeep earlier (the group before the newest); this upkeep requests blocks
    // blk+2 and blk+3 (16 lanes x 16 bytes) into the other half of the 4-block ring. Sixteen
    // steps separate two upkeeps, several microseconds, far longer than a DRAM read. The
    // first upkeep requests blocks 0-3 and waits for all of them.
    auto upkeep = [&](uint32_t blk) {
        __syncwarp();
        bool newest_needed = blk == 0;
#pragma unroll
        for (int k = 0; k < kChains; ++k) {
            Chain& h = c[k];
            const uint32_t n_blocks = (h.nc + 255u) >> 8;
            if (nib_stored && blk < n_blocks) { // nibble words start after the 128-byte states
                for (uint32_t b = (blk == 0 ? 0u : blk + 2u); b < blk + 4u; b += 2u) {
                    const uint32_t byte = 128u * b + 16u * lane; // lanes 0-15: blocks b and b+1
                    if (lane < 16 && byte < 128u * n_blocks)
                        cp_async16(smem_base + nring_off + k * kNibRingBytes + (byte & (kNibRingBytes - 1u)),
                                   h.payload + 128 + byte, 16u);
                }
            }
            if (blk < n_blocks) {
                const uint32_t q = h.posb / kQuarterBytes;
                const uint32_t total_q = (h.stream_bytes + kQuarterBytes - 1) / kQuarterBytes;
                const uint8_t* stream = h.payload + 128 + (nib_stored ? 128u * n_blocks : 0u);
                if (h.fq <= min(q + 2, total_q - 1)) newest_needed = true;
                while (h.fq < q + 4 && h.fq < total_q) {
                    const uint32_t byte = h.fq * kQuarterBytes + 16u * lane;
                    const uint32_t dst = smem_base + ring_off + k * kRingBytes + (byte & (kRingBytes - 1u));
                    if ((h.fq + 1) * kQuarterBytes <= h.stream_bytes) cp_async16(dst, stream + byte, 16u);
                    else if (byte < h.stream_bytes) cp_async16(dst, stream + byte, min(16u, h.stream_bytes - byte));
                    ++h.fq;
                }
            }
        }
        cp_async_commit();
        if (newest_needed) cp_async_wait<0>();
        else cp_async_wait<1>();
        __syncwarp();
    };

    // The current block's nibble word of each chain, from its ring (or the constant). In the
    // full-block loop every live chain has block b; in the tail a chain past its end keeps
    // its last word (its output is not stored).
    auto next_raw = [&](uint32_t b, bool full) {
#pragma unroll
        for (int k = 0; k < kChains; ++k) {
            Chain& h = c[k];
            if (nib_stored && h.live && (full || b < ((h.nc + 255u) >> 8)))
                h.raw = *reinterpret_cast<const uint32_t*>(smem + nring_off + k * kNibRingBytes +
                                                           ((128u * b) & (kNibRingBytes - 1u)) + lane4);
        }
    };

    // 8 steps of every chain; o[k] receives chain k's 8 words as 4 pairs. Within a step the
    // chains advance phase by phase (lookups, update, ballot, word read, select), so the
    // independent work of the two chains sits side by side between the warp-wide votes.
    auto octet = [&](uint32_t (&o)[kChains][4]) {
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            uint2 se[kChains];
            uint32_t fe[kChains], xn[kChains], m[kChains], w[kChains];
            bool need[kChains];
            if (JOINT) { // the slot's entry: F and the word's (s, h) part in .x, the rank in .y
#pragma unroll
                for (int k = 0; k < kChains; ++k)
                    se[k] = *reinterpret_cast<const uint2*>(smem + ((c[k].x << 3) & smask8));
#pragma unroll
                for (int k = 0; k < kChains; ++k) {
                    xn[k] = (se[k].x & 0xFFFFu) * (c[k].x >> ns) + se[k].y;
                    need[k] = xn[k] < kStateL;
                    fe[k] = 0;
                }
            } else {
#pragma unroll
            for (int k = 0; k < kChains; ++k) // the s-entry from the slot's high ns bits
                se[k] = *reinterpret_cast<const uint2*>(smem + kHRegion + ((c[k].x >> (nh - 3)) & smask8));
#pragma unroll
            for (int k = 0; k < kChains; ++k) { // the fraction entry from its low nh bits
                const uint32_t u = ((c[k].x << 7) & hmask7) | lane4;
                fe[k] = *reinterpret_cast<const uint32_t*>(smem + (se[k].y >> 16) + u);
            }
#pragma unroll
            for (int k = 0; k < kChains; ++k) {
                const uint32_t t = c[k].x >> P;
                const uint32_t Fs = se[k].x & 0xFFFFu, bs = se[k].x >> 16;
                const uint32_t Fh = __byte_perm(fe[k], 0u, 0x4442), bh = fe[k] >> 24;
                xn[k] = (Fs * Fh) * t + (bs * Fh + bh);
                need[k] = xn[k] < kStateL;
            }
            }
            // renormalise: lanes below 2^16 take the next words, in lane order
            // (branch-free: every lane reads; the ones that need no word discard it)
#pragma unroll
            for (int k = 0; k < kChains; ++k) m[k] = __ballot_sync(0xFFFFFFFFu, need[k]);
#pragma unroll
            for (int k = 0; k < kChains; ++k)
                w[k] = *reinterpret_cast<const uint16_t*>(
                    smem + (((c[k].posb + __popc(m[k] & lt) * mul2) & (kRingBytes - 1u)) | (ring_off + k * kRingBytes)));
#pragma unroll
            for (int k = 0; k < kChains; ++k) {
                Chain& h = c[k];
                const uint32_t xr = xn[k] * mul65536 + w[k]; // (xn << 16) | w as one IMAD, computed by every lane
                h.x = need[k] ? xr : xn[k];
                h.posb += __popc(m[k]) * mul2;
                // (s << 7) | (h << 4): s sits pre-shifted in se.y, h in bits 4-6 of fe, and the
                // rest of fe's low half is zero, so one masked select builds the low half (the
                // high half is dropped when the pair is packed)
                if (JOINT) { // the words sit in the high halves of the entries
                    if (s & 1) o[k][s >> 1] = __byte_perm(o[k][s >> 1], se[k].x, 0x7632);
                    else o[k][s >> 1] = se[k].x;
                } else {
                    const uint32_t word = (se[k].y & 0xFF80u) | fe[k];
                    if (s & 1) o[k][s >> 1] = __byte_perm(o[k][s >> 1], word, 0x5410);
                    else o[k][s >> 1] = word;
                }
            }
        }
        // the low nibbles of the pairs (pair p of a block has its nibbles at bits 4p and 16+4p)
#pragma unroll
        for (int k = 0; k < kChains; ++k)
#pragma unroll
            for (int q = 0; q < 4; ++q) o[k][q] |= (c[k].raw >> (4 * q)) & 0x000F000Fu;
    };

    // Full blocks first: every live chain has all 256 weights of the block, so the stores
    // need no bounds; blocks are taken two at a time. A chain whose last block is the last
    // one of this loop gets its end check after the loop.
    uint32_t nb_full = 0xFFFFFFFFu;
#pragma unroll
    for (int k = 0; k < kChains; ++k)
        if (c[k].live) nb_full = min(nb_full, c[k].nc >> 8);
    uint32_t blk = 0;
    for (; blk + 2 <= nb_full; blk += 2) {
        upkeep(blk);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const uint32_t b = blk + half, i0 = (b << 8) + (lane << 3);
            next_raw(b, true);
            uint32_t o[kChains][4];
            octet(o);
#pragma unroll
            for (int k = 0; k < kChains; ++k) {
                Chain& h = c[k];
                if (h.live) *reinterpret_cast<uint4*>(out0 + k * C + i0) = make_uint4(o[k][0], o[k][1], o[k][2], o[k][3]);
            }
        }
    }
#pragma unroll
    for (int k = 0; k < kChains; ++k) // end check: state back at L, every word consumed
        if (c[k].live && ((c[k].nc + 255u) >> 8) == blk) c[k].bad |= (c[k].x != kStateL) | (c[k].posb != c[k].stream_bytes);
    // The rest (ragged tails, chains of different lengths), with bounds, two blocks at a time.
    for (; blk < nb; blk += 2) {
        upkeep(blk);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const uint32_t b = blk + half;
            if (b >= nb) break;
            next_raw(b, false);
            uint32_t o[kChains][4];
            octet(o);
#pragma unroll
            for (int k = 0; k < kChains; ++k) {
                Chain& h = c[k];
                const uint32_t n_blocks = (h.nc + 255u) >> 8;
                if (b < n_blocks) {
                    const uint32_t i0 = (b << 8) + (lane << 3);
                    if (i0 + 8 <= h.nc) {
                        *reinterpret_cast<uint4*>(out0 + k * C + i0) = make_uint4(o[k][0], o[k][1], o[k][2], o[k][3]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            if (i0 + e < h.nc) out0[k * C + i0 + e] = static_cast<uint16_t>(o[k][e >> 1] >> (16 * (e & 1)));
                    }
                    if (b + 1 == n_blocks) // end check: state back at L, every word consumed
                        h.bad |= (h.x != kStateL) | (h.posb != h.stream_bytes);
                }
            }
        }
    }
    cp_async_wait<0>();

#pragma unroll
    for (int k = 0; k < kChains; ++k) {
        if (c[k].live && __any_sync(0xFFFFFFFFu, c[k].bad) && lane == 0) {
            atomicOr(p.err, 1ull);
            atomicMin(p.err + 1, (static_cast<unsigned long long>(it.tensor_index) << 40) |
                                     (it.chunk_base + static_cast<uint64_t>(blockIdx.x - it.cta_begin) * (warps * kChains) +
                                      warp * kChains + k)); // chunk0 + k, recomputed
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

// The per-tensor checksum: the sum of splitmix64 outputs mix64((i << 16) | w[i]); mix64 is
// splitmix64's output for state v.
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

template <int WARPS, int CHAINS, int NS, int NH, bool SHAPE_FROM_PARAMS, bool JOINT>
static int launch_decode_shape(const DecodeParams& p, uint32_t smem_bytes, cudaStream_t s) {
    auto kernel = decode_kernel<WARPS, CHAINS, NS, NH, SHAPE_FROM_PARAMS, JOINT>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_bytes));
    if (e != cudaSuccess) return e;
    kernel<<<p.total_ctas, p.warps * 32, smem_bytes, s>>>(p);
    count_launch();
    return cudaGetLastError();
}

template <int WARPS, int CHAINS, int NS, int NH, bool JOINT>
static int launch_decode_t(const DecodeParams& p, uint32_t smem_bytes, cudaStream_t s) {
    if (p.warps < 1 || p.warps > WARPS) return cudaErrorInvalidValue;
    return p.warps == WARPS ? launch_decode_shape<WARPS, CHAINS, NS, NH, false, JOINT>(p, smem_bytes, s)
                            : launch_decode_shape<WARPS, CHAINS, NS, NH, true, JOINT>(p, smem_bytes, s);
}

int launch_decode(const DecodeParams& p, DecodeMode mode, uint32_t smem_bytes, void* stream) {
    if (p.total_ctas == 0) return cudaSuccess;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    switch (mode) {
    case DecodeMode::Default: return launch_decode_t<kWarpsDefault, kChainsDefault, 11, 5, false>(p, smem_bytes, s);
    case DecodeMode::Joint: return launch_decode_t<kWarpsJoint, kChainsJoint, 13, 5, true>(p, smem_bytes, s);
    case DecodeMode::JointGeneric: return launch_decode_t<kWarpsGeneric, kChainsGeneric, 0, 5, true>(p, smem_bytes, s);
    case DecodeMode::JointCompact: return launch_decode_joint4(p, smem_bytes, stream);
    default: return launch_decode_t<kWarpsGeneric, kChainsGeneric, 0, 0, false>(p, smem_bytes, s);
    }
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
