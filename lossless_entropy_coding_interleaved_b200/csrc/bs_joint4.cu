// bs_joint4.cu -- the decode kernel for JOINT tensors with 4-byte slot entries (every pair
// frequency at most 255; all large tensors of normally distributed weights qualify).
//
// It computes what decode_kernel computes for the JOINT kind: the pair j = (s << 3) | h is the
// rANS symbol of a table of 2^nj slots, the word is (j << 4) | u with the low nibble u kept
// verbatim, and the sign+exponent symbol s selects the distribution of the fraction's top
// bits h through the pair table (the field split of the "Qwen3.8-27B-BF16-NVLC-Lossless" card,
// the paragraph after its accounting table). Per weight and lane:
//
//   e  = table[x & (2^nj - 1)]            the word j << 4 in the low half, rank in byte 2, F in byte 3
//   x  = F * (x >> nj) + rank
//   if x < 2^16: x = (x << 16) | next word (the warp's lanes take words in lane order)
//   w  = (e & 0xFFFF) | u
//
// Mapping onto the B200:
//  * 32 warps of 1024 threads hold one CTA per SM at most 64 registers a thread; each warp
//    decodes two chunks at once (two independent chains per lane hide the table latency).
//  * The 32 KiB table is staged in shared memory; a 4-byte gather by 32 lanes costs about 3.5
//    wavefronts, against about 6 for the 8-byte entries of the general JOINT table.
//  * The loop is bound by issue and by the integer pipes (the ALU and the multiply-add pipe
//    each take a warp instruction every other cycle). The lane-prefix mask of the ballot is
//    a multiply-add (m * 2^(32 - lane) keeps the bits below the lane) rather than an AND on
//    the busier ALU pipe; its multiplier, like the renormalisation's 2^16 and 2, comes from
//    the launch parameters so that it stays a multiply. The table is read by slot index, so
//    the address scaling folds into the load. Multiplies-high are not used: they run at a
//    lower rate than the shifts they would replace (measured).
//  * Each chunk's word stream flows through its own 2 KiB ring of four 512-byte quarters, and
//    its nibble words through a 512-byte ring of four blocks, both filled by cp.async. The
//    upkeep between two pairs of blocks (16 steps) has no branch: at most two quarters per
//    chunk and one nibble copy for both chunks, each a predicated cp.async of whole 16-byte
//    units (a payload is padded to 16 bytes, so a unit never leaves it).
//  * The renormalisation is branch-free: ballot, prefix popcount, one ring read by every lane,
//    and a predicated multiply-add for the lanes that need the word.
//  * Eight weights per lane leave as one 16-byte store; a warp writes 512 contiguous bytes per
//    chunk and block.
//  * A chunk whose start state is below 2^16, whose lanes do not end at L = 2^16, or which does
//    not consume exactly its words sets the error block. Every loop is bounded by the chunk's
//    weight count; nothing traps.
#include <cuda_runtime.h>

#include <cstdint>

#include "bs_device.cuh"
#include "bs_internal.h"

namespace bs {

namespace {

constexpr int kChains4 = kChainsJoint4;

struct Chain4 {
    uint32_t x;           // rANS state, in [2^16, 2^32) between weights
    uint32_t posb;        // bytes of the word stream consumed (warp-uniform)
    uint32_t fb;          // bytes of the word stream requested, a multiple of 512 (warp-uniform)
    uint32_t sbytes;      // bytes of the word stream: 2 * n_words
    uint32_t nc;          // weights in the chunk; 0 for a filler chain (nothing stored)
    uint32_t raw;         // nibble word of the current block (constant mode: c in every nibble)
    const uint8_t* stream; // the word stream; in stored mode the nibble words end where it starts
    bool bad;
};

template <int WARPS, bool SHAPE_FROM_PARAMS>
__global__ void __launch_bounds__(WARPS * 32, 1) joint4_decode_kernel(const __grid_constant__ DecodeParams p) {
    // dynamic shared memory: [table, kJoint4Region][word rings][nibble rings]
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ int s_item;
    const uint32_t tid = threadIdx.x, lane = tid & 31u, warp = tid >> 5;
    if (tid == 0) find_item(p, &s_item);
    __syncthreads();
    const DecodeItem& it = p.item[s_item];
    const uint32_t nj = it.ns;
    {
        const uint32_t n16 = (4u << nj) / 16u;
        uint4* dst = reinterpret_cast<uint4*>(smem);
        for (uint32_t k = tid; k < n16; k += blockDim.x) dst[k] = __ldg(it.tables + k);
    }
    __syncthreads();

    const uint32_t log2c = it.log2_chunk;
    const uint64_t n_elems = it.n_elems;
    const uint64_t n_chunks = (n_elems + (1ull << log2c) - 1) >> log2c;
    const uint32_t warps = SHAPE_FROM_PARAMS ? p.warps : WARPS;
    const uint64_t chunk0 = static_cast<uint64_t>(blockIdx.x - it.cta_begin) * (warps * kChains4) + warp * kChains4;
    if (chunk0 >= n_chunks) return;

    const bool nib_stored = it.nib_mode == 0;
    const uint32_t raw_const = (it.nib_mode & 15u) * 0x11111111u;
    // chain k's word ring at ring0 + k * kRingBytes, its nibble ring at nring0 + k * kNibRingBytes
    // (offsets into smem; each ring starts at a multiple of its size)
    const uint32_t ring0 = kJoint4Region + warp * kChains4 * kRingBytes;
    const uint32_t nring0 = kJoint4Region + warps * kChains4 * kRingBytes + warp * kChains4 * kNibRingBytes;
    const uint32_t sbase = smem_u32(smem);
    uint16_t* const out0 = it.out + (chunk0 << log2c); // chain k writes from out0 + (k << log2c)

    Chain4 c[kChains4];
    uint32_t nb = 0, nb_full = 0xFFFFFFFFu;
#pragma unroll
    for (int k = 0; k < kChains4; ++k) {
        Chain4& h = c[k];
        const uint64_t chunk = chunk0 + k;
        h.posb = 0;
        h.fb = 0;
        h.raw = raw_const;
        h.bad = false;
        if (chunk < n_chunks) {
            const uint8_t* ent = it.chunk_table + 16 * chunk;
            const uint64_t off = __ldg(reinterpret_cast<const unsigned long long*>(ent));
            const uint32_t n_words = __ldg(reinterpret_cast<const unsigned int*>(ent + 8));
            const uint8_t* payload = it.container + off;
            h.nc = static_cast<uint32_t>(min(static_cast<uint64_t>(1ull << log2c), n_elems - (chunk << log2c)));
            const uint32_t nblk = (h.nc + 255u) >> 8;
            h.stream = payload + 128 + (nib_stored ? 128u * nblk : 0u);
            h.sbytes = 2u * n_words;
            h.x = __ldg(reinterpret_cast<const unsigned int*>(payload) + lane);
            h.bad = h.x < kStateL;
            nb = max(nb, nblk);
            nb_full = min(nb_full, h.nc >> 8);
        } else { // filler: decodes from L out of its own unfilled ring; nothing is stored
            h.nc = 0;
            h.sbytes = 0;
            h.stream = it.container;
            h.x = kStateL;
        }
    }

    const uint32_t lt_mul = lane ? 1u << (32 - lane) : 0u; // m * lt_mul keeps the bits of m below this lane
    const uint32_t lane4 = lane << 2, lane16 = lane << 4;
    const uint32_t mul2 = p.mul2, mul65536 = p.mul65536;
    const uint32_t jmask = (1u << nj) - 1u;

    // Request the 16-byte units [b, b + 16) of chain k's word stream with b < end, b = fb + i*512
    // + lane*16, into its ring.
    auto request_words = [&](int k, uint32_t i, uint32_t end) {
        const Chain4& h = c[k];
        const uint32_t b = h.fb + i * kQuarterBytes + lane16;
        cp_async16_if(b < end, sbase + (ring0 + k * kRingBytes) + (b & (kRingBytes - 1u)), h.stream + b, 16u);
    };

    // First fill: quarters 0..3 and nibble blocks 0..3 of both chains, then wait for all.
#pragma unroll
    for (int k = 0; k < kChains4; ++k) {
        const uint32_t end = min(4u * kQuarterBytes, c[k].sbytes);
#pragma unroll
        for (uint32_t i = 0; i < 4; ++i) request_words(k, i, end);
        c[k].fb = (end + kQuarterBytes - 1) & ~(kQuarterBytes - 1);
        const uint32_t nbytes = ((c[k].nc + 255u) >> 8) * 128u; // nibble words of the chunk
        cp_async16_if(nib_stored && lane16 < nbytes, sbase + nring0 + k * kNibRingBytes + lane16,
                      c[k].stream - nbytes + lane16, 16u);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncwarp();

    // Upkeep before blocks blk and blk+1 (blk even, at least 2). The next 16 steps read at most
    // 1 KiB of a chain's stream, from its position posb: at most quarters q..q+2, q = posb >> 9.
    // Each chain requests up to the end of quarter q+3 (the ring holds four), clipped at the
    // stream's end; since the last upkeep requested up to quarter q_last + 3 and q <= q_last + 2,
    // that is at most two quarters. Nibble blocks blk+2 and blk+3 of chain 0 (lanes 0-15) and
    // chain 1 (lanes 16-31) go in one copy. Then wait for every group but the newest, or for all
    // when the newest holds a quarter the next 16 steps read.
    auto upkeep = [&](uint32_t blk) {
        __syncwarp();
        bool newest = false;
#pragma unroll
        for (int k = 0; k < kChains4; ++k) {
            Chain4& h = c[k];
            const uint32_t qb = h.posb & ~(kQuarterBytes - 1u);
            const uint32_t end = min(qb + 4u * kQuarterBytes, h.sbytes);
            newest |= h.fb < h.sbytes && h.fb <= qb + 2u * kQuarterBytes;
            request_words(k, 0, end);
            request_words(k, 1, end);
            h.fb = max(h.fb, (end + kQuarterBytes - 1) & ~(kQuarterBytes - 1));
        }
        const bool hi = lane >= 16; // lanes 0-15: chain 0, 16-31: chain 1
        const uint32_t nbytes = ((hi ? c[1].nc : c[0].nc) + 255u) / 256u * 128u;
        const uint8_t* nib_end = hi ? c[1].stream : c[0].stream; // the nibble words end where the stream starts
        const uint32_t byte = 128u * (blk + 2u) + (lane16 & 255u);
        cp_async16_if(nib_stored && byte < nbytes,
                      sbase + nring0 + (hi ? kNibRingBytes : 0u) + (byte & (kNibRingBytes - 1u)), nib_end - nbytes + byte, 16u);
        cp_async_commit();
        if (newest) cp_async_wait<0>();
        else cp_async_wait<1>();
        __syncwarp();
    };

    // The current block's nibble word of each chain (a chain past its end reads a stale word;
    // its output is never stored).
    auto next_raw = [&](uint32_t b) {
        if (nib_stored) {
#pragma unroll
            for (int k = 0; k < kChains4; ++k)
                c[k].raw = *reinterpret_cast<const uint32_t*>(smem + nring0 + k * kNibRingBytes + ((b & 3u) << 7) + lane4);
        }
    };

    // 8 steps of both chains; o[k] receives chain k's 8 words as 4 pairs (low half first).
    auto octet = [&](uint32_t (&o)[kChains4][4]) {
        uint32_t ev[kChains4];
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            uint32_t e[kChains4], q[kChains4], xn[kChains4], m[kChains4], w[kChains4];
#pragma unroll
            for (int k = 0; k < kChains4; ++k) { // the slot's entry
                q[k] = c[k].x >> nj;
                e[k] = reinterpret_cast<const uint32_t*>(smem)[c[k].x & jmask]; // a scaled-index load
            }
#pragma unroll
            for (int k = 0; k < kChains4; ++k)
                xn[k] = (e[k] >> 24) * q[k] + __byte_perm(e[k], 0u, 0x4442);
#pragma unroll
            for (int k = 0; k < kChains4; ++k) m[k] = __ballot_sync(0xFFFFFFFFu, xn[k] < kStateL);
#pragma unroll
            for (int k = 0; k < kChains4; ++k)
                w[k] = *reinterpret_cast<const uint16_t*>(
                    smem + (((c[k].posb + __popc(m[k] * lt_mul) * mul2) & (kRingBytes - 1u)) | (ring0 + k * kRingBytes)));
#pragma unroll
            for (int k = 0; k < kChains4; ++k) {
                uint32_t xv = xn[k]; // (xv << 16) | w for the lanes below 2^16, as one predicated IMAD
                asm("{\n .reg .pred p;\n setp.lt.u32 p, %0, 65536;\n @p mad.lo.u32 %0, %0, %1, %2;\n}"
                    : "+r"(xv) : "r"(mul65536), "r"(w[k]));
                c[k].x = xv;
                c[k].posb += __popc(m[k]) * mul2;
                if (s & 1) o[k][s >> 1] = __byte_perm(ev[k], e[k], 0x5410);
                else ev[k] = e[k];
            }
        }
        // the low nibbles: pair p of the block has its two nibbles at bits 4p and 16 + 4p
#pragma unroll
        for (int k = 0; k < kChains4; ++k)
#pragma unroll
            for (int p4 = 0; p4 < 4; ++p4) o[k][p4] |= (c[k].raw >> (4 * p4)) & 0x000F000Fu;
    };

    // Full blocks, two at a time: every live chain has all 256 weights of both.
    uint32_t blk = 0;
    for (; blk + 2 <= nb_full; blk += 2) {
        if (blk) upkeep(blk);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const uint32_t b = blk + half, i0 = (b << 8) + (lane << 3);
            next_raw(b);
            uint32_t o[kChains4][4];
            octet(o);
#pragma unroll
            for (int k = 0; k < kChains4; ++k)
                if (c[k].nc) *reinterpret_cast<uint4*>(out0 + (uint64_t(k) << log2c) + i0) = make_uint4(o[k][0], o[k][1], o[k][2], o[k][3]);
        }
    }
#pragma unroll
    for (int k = 0; k < kChains4; ++k) // end check of chains whose last block was in the loop
        if (c[k].nc && ((c[k].nc + 255u) >> 8) == blk) c[k].bad |= (c[k].x != kStateL) | (c[k].posb != c[k].sbytes);
    // The rest (ragged tails, chains of different lengths), with bounds.
    for (; blk < nb; blk += 2) {
        if (blk) upkeep(blk);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const uint32_t b = blk + half;
            if (b >= nb) break;
            next_raw(b);
            uint32_t o[kChains4][4];
            octet(o);
#pragma unroll
            for (int k = 0; k < kChains4; ++k) {
                Chain4& h = c[k];
                const uint32_t nblk = (h.nc + 255u) >> 8;
                if (b < nblk) {
                    const uint32_t i0 = (b << 8) + (lane << 3);
                    uint16_t* dst = out0 + (uint64_t(k) << log2c) + i0;
                    if (i0 + 8 <= h.nc) {
                        *reinterpret_cast<uint4*>(dst) = make_uint4(o[k][0], o[k][1], o[k][2], o[k][3]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            if (i0 + e < h.nc) dst[e] = static_cast<uint16_t>(o[k][e >> 1] >> (16 * (e & 1)));
                    }
                    if (b + 1 == nblk) h.bad |= (h.x != kStateL) | (h.posb != h.sbytes);
                }
            }
        }
    }
    cp_async_wait<0>();

#pragma unroll
    for (int k = 0; k < kChains4; ++k) {
        if (c[k].nc && __any_sync(0xFFFFFFFFu, c[k].bad) && lane == 0) {
            atomicOr(p.err, 1ull);
            atomicMin(p.err + 1, (static_cast<unsigned long long>(it.tensor_index) << 40) |
                                     (it.chunk_base + chunk0 + k));
        }
    }
}

template <bool SHAPE_FROM_PARAMS>
int launch_shape(const DecodeParams& p, uint32_t smem_bytes, cudaStream_t s) {
    auto kernel = joint4_decode_kernel<kWarpsJoint4, SHAPE_FROM_PARAMS>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_bytes));
    if (e != cudaSuccess) return e;
    kernel<<<p.total_ctas, p.warps * 32, smem_bytes, s>>>(p);
    count_launch();
    return cudaGetLastError();
}

} // namespace

int launch_decode_joint4(const DecodeParams& p, uint32_t smem_bytes, void* stream) {
    if (p.total_ctas == 0) return cudaSuccess;
    if (p.warps < 1 || p.warps > static_cast<uint32_t>(kWarpsJoint4)) return cudaErrorInvalidValue;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return p.warps == static_cast<uint32_t>(kWarpsJoint4) ? launch_shape<false>(p, smem_bytes, s)
                                                          : launch_shape<true>(p, smem_bytes, s);
}

} // namespace bs
