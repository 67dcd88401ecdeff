// bs_fw.cu -- the fixed-width lane layout on sm_100a: the device
// transcoder from BF16 words, the decode kernel, and their C ABI (include/bs.h).
//
// The "Qwen3.8-27B-BF16-NVLC-Lossless" card says its GPU runtime derives fixed-width,
// lane-oriented streams from the rANS files once at initialisation (its Fixed7/Compact11
// runtime, about 11.36 bits per weight resident). The card gives no layout. This file
// implements this project's: a 4-bit sign+exponent code per weight (the tensor's 16 most
// frequent symbols), the 7-bit fraction in two planes, and an exception list of
// (position, word) for the rest.
//
// Decode. A warp decodes one 256-weight tile at a time: lane j reads its plane words and
// writes its 8 weights as one 16-byte store.
//   - The two codes of a pair of weights are one byte of plane A. A 256-entry shared table
//     maps it to both weights' (s << 7) in their 16-bit halves.
//   - Plane B gives both low nibbles with one shift and mask.
//   - The lane's 24-bit plane C field is spread once so that each pair's top bits come out
//     with one more shift and mask.
//   - Escapes: lane k of the warp loads the tile's k-th exception, and after the main stores
//     (ordered by __syncwarp) writes its word at its position.
// Loads run two tiles ahead, and each tile's exceptions are applied one tile later, so the
// warp never waits on a load it has just issued. The kernel is bound by HBM bandwidth:
// 11.125 bits read and 16 bits written per weight, plus 24 bits read per escape.
//
// Transcode (three passes over the input):
//   1. histogram of s, then one CTA ranks the symbols and builds the code table;
//   2. a count of escapes per tile, and a scan of the per-block sums;
//   3. the write pass: tile_exc from the scan, then the planes and the exceptions.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <vector>

#include "bs_fw.cuh"
#include "bs_host.h"
#include "bs_internal.h"

namespace bs {
namespace {
using namespace fw;


constexpr uint32_t kFwBlockTiles = 256;           // tiles per CTA of the count and write passes
constexpr uint32_t kFwPassThreads = 512;
constexpr uint8_t kEscape = 0xFF;                 // code_of[s] for a symbol outside the table

// Scratch of the transcoder (256-byte aligned sections).
struct FwScratch {
    uint64_t hist, sel, tile_cnt, blk_total, blk_base, total;
};
// The selection block: code_of[512] (u8), table[16] (u16) at 512, n_exc (u64) at 576.
constexpr uint32_t kSelBytes = 1024, kSelTable = 512, kSelNExc = 576;
inline FwScratch fw_scratch(uint64_t n) {
    const uint64_t nt = fw_tiles(n), nblk = std::max<uint64_t>(1, (nt + kFwBlockTiles - 1) / kFwBlockTiles);
    FwScratch s;
    s.hist = 0;
    s.sel = up256(sizeof(unsigned long long) * kHistBins);
    s.tile_cnt = s.sel + kSelBytes;
    s.blk_total = s.tile_cnt + up256(4 * std::max<uint64_t>(nt, 1));
    s.blk_base = s.blk_total + up256(4 * nblk);
    s.total = s.blk_base + up256(8 * nblk);
    return s;
}

// ------------------------------------------------------------------ transcode kernels
// Section 10, code table: rank every present symbol by (count down, s up); the first 16
// get codes. One CTA of 512 threads, thread s for symbol s, whose count is the sum of its
// eight (s, h) pair bins in the histogram.
__global__ void __launch_bounds__(512) fw_select_kernel(const unsigned long long* __restrict__ hist,
                                                        uint8_t* __restrict__ sel) {
    __shared__ unsigned long long cnt[512];
    const uint32_t s = threadIdx.x;
    unsigned long long c8 = 0;
    for (uint32_t h = 0; h < 8; ++h) c8 += hist[(s << 3) | h];
    cnt[s] = c8;
    uint16_t* table = reinterpret_cast<uint16_t*>(sel + kSelTable);
    if (s < 16) table[s] = 0;
    __syncthreads();
    const unsigned long long c = cnt[s];
    uint32_t rank = 0;
    for (uint32_t k = 0; k < 512; ++k) {
        const unsigned long long ck = cnt[k];
        rank += (ck > c || (ck == c && k < s)) ? 1u : 0u;
    }
    // present symbols outrank absent ones, so a present symbol's rank counts present ones only
    const bool coded = c > 0 && rank < 16;
    sel[s] = coded ? static_cast<uint8_t>(rank) : kEscape;
    if (coded) table[rank] = static_cast<uint16_t>(s);
}

// Loads the 8 words of lane `lane` in tile t. Weights at or past n read as 0, and bit k of
// `valid` says whether weight k is inside the tensor.
__device__ __forceinline__ void load_octet(const uint16_t* __restrict__ in, uint64_t n, uint64_t t, uint32_t lane,
                                           uint32_t (&w)[8], uint32_t& valid) {
    const uint64_t i0 = t * kFwTile + 8ull * lane;
    if (i0 + 8 <= n) {
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(in + i0));
        const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int k = 0; k < 8; ++k) w[k] = (u[k >> 1] >> (16 * (k & 1))) & 0xFFFFu;
        valid = 0xFFu;
    } else {
        valid = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const bool v = i0 + k < n;
            w[k] = v ? in[i0 + k] : 0u;
            valid |= (v ? 1u : 0u) << k;
        }
    }
}

__device__ __forceinline__ uint32_t escape_mask(const uint8_t* code_of, const uint32_t (&w)[8], uint32_t valid) {
    uint32_t m = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) m |= ((valid >> k) & 1u && code_of[w[k] >> 7] == kEscape ? 1u : 0u) << k;
    return m;
}

// Pass 2a: escapes per tile, and per block of kFwBlockTiles tiles.
__global__ void __launch_bounds__(kFwPassThreads) fw_count_kernel(const uint16_t* __restrict__ in, uint64_t n,
                                                                  const uint8_t* __restrict__ sel,
                                                                  uint32_t* __restrict__ tile_cnt,
                                                                  uint32_t* __restrict__ blk_total) {
    __shared__ uint8_t code_of[512];
    __shared__ uint32_t wsum[kFwPassThreads / 32];
    const uint32_t tid = threadIdx.x, lane = tid & 31u, warp = tid >> 5;
    code_of[tid] = sel[tid];
    __syncthreads();
    const uint64_t nt = fw_tiles(n), t0 = uint64_t(blockIdx.x) * kFwBlockTiles;
    uint32_t sum = 0;
    for (uint32_t k = warp; k < kFwBlockTiles; k += kFwPassThreads / 32) {
        const uint64_t t = t0 + k;
        if (t >= nt) break;
        uint32_t w[8], valid;
        load_octet(in, n, t, lane, w, valid);
        uint32_t e = __popc(escape_mask(code_of, w, valid));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) e += __shfl_xor_sync(0xFFFFFFFFu, e, o);
        if (lane == 0) tile_cnt[t] = e;
        sum += e;
    }
    if (lane == 0) wsum[warp] = sum;
    __syncthreads();
    if (tid == 0) {
        uint32_t total = 0;
        for (uint32_t k = 0; k < kFwPassThreads / 32; ++k) total += wsum[k];
        blk_total[blockIdx.x] = total;
    }
}

// Pass 2b: exclusive scan of the block sums (one CTA), and the total n_exc.
__global__ void __launch_bounds__(1024) fw_scan_kernel(const uint32_t* __restrict__ blk_total, uint32_t nblk,
                                                       unsigned long long* __restrict__ blk_base,
                                                       uint8_t* __restrict__ sel) {
    __shared__ unsigned long long wsum[32];
    __shared__ unsigned long long carry;
    const uint32_t tid = threadIdx.x, lane = tid & 31u, warp = tid >> 5;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (uint32_t b0 = 0; b0 < nblk; b0 += 1024) {
        const unsigned long long v = b0 + tid < nblk ? blk_total[b0 + tid] : 0ull;
        unsigned long long x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long y = __shfl_up_sync(0xFFFFFFFFu, x, o);
            if (lane >= static_cast<uint32_t>(o)) x += y;
        }
        if (lane == 31) wsum[warp] = x;
        __syncthreads();
        if (warp == 0) {
            unsigned long long z = wsum[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned long long y = __shfl_up_sync(0xFFFFFFFFu, z, o);
                if (lane >= static_cast<uint32_t>(o)) z += y;
            }
            wsum[lane] = z;
        }
        __syncthreads();
        const unsigned long long before = carry + (warp ? wsum[warp - 1] : 0ull);
        if (b0 + tid < nblk) blk_base[b0 + tid] = before + x - v;
        __syncthreads();
        if (tid == 0) carry += wsum[31];
        __syncthreads();
    }
    if (tid == 0) *reinterpret_cast<unsigned long long*>(sel + kSelNExc) = carry;
}

struct FwWriteParams {
    const uint16_t* in;
    uint64_t n;
    uint64_t n_exc;
    const uint8_t* sel;                  // code_of and table
    const uint32_t* tile_cnt;
    const unsigned long long* blk_base;
    uint8_t* fw;
    unsigned int* err;                   // set if the write pass disagrees with the count pass
};

// Pass 3: the layout. CTA b writes tile_exc for its tiles (its block base plus the scan of
// its tile counts), then each warp encodes tiles: planes A, B, C and the tile's exceptions.
// CTA 0 writes the header and the code table; the last CTA writes tile_exc[n_tiles] and
// zeroes the section padding.
__global__ void __launch_bounds__(kFwPassThreads) fw_write_kernel(const __grid_constant__ FwWriteParams p) {
    __shared__ uint8_t code_of[512];
    __shared__ uint32_t te[kFwBlockTiles];
    __shared__ uint32_t wsum[kFwBlockTiles / 32];
    const uint32_t tid = threadIdx.x, lane = tid & 31u, warp = tid >> 5;
    const uint64_t n = p.n, nt = fw_tiles(n), t0 = uint64_t(blockIdx.x) * kFwBlockTiles;
    const FwOffsets o = fw_offsets(nt, p.n_exc);
    uint8_t* fw = p.fw;
    code_of[tid] = p.sel[tid];
    // exclusive scan of this block's tile counts
    uint32_t v = 0, x = 0;
    if (tid < kFwBlockTiles) {
        v = t0 + tid < nt ? p.tile_cnt[t0 + tid] : 0u;
        x = v;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, d);
            if (lane >= static_cast<uint32_t>(d)) x += y;
        }
        if (lane == 31) wsum[warp] = x;
    }
    __syncthreads();
    if (tid < kFwBlockTiles) {
        uint32_t before = 0;
        for (uint32_t k = 0; k < warp; ++k) before += wsum[k];
        te[tid] = before + x - v;
    }
    __syncthreads();
    const unsigned long long base = nt ? p.blk_base[blockIdx.x] : 0ull;
    uint32_t* tile_exc = reinterpret_cast<uint32_t*>(fw + o.tile_exc);
    if (tid < kFwBlockTiles && t0 + tid < nt) tile_exc[t0 + tid] = static_cast<uint32_t>(base + te[tid]);

    if (blockIdx.x == 0 && tid < 24) { // header (16 words) and code table (8 words)
        uint32_t word = 0;
        const uint64_t total = o.total;
        switch (tid) {
        case 0: word = 0x36314642u; break; // "BF16"
        case 1: word = 0x454E414Cu; break; // "LANE"
        case 2: word = 1; break;
        case 3: word = kFwHeader; break;
        case 4: word = static_cast<uint32_t>(n); break;
        case 5: word = static_cast<uint32_t>(n >> 32); break;
        case 6: word = static_cast<uint32_t>(nt); break;
        case 7: word = static_cast<uint32_t>(nt >> 32); break;
        case 8: word = static_cast<uint32_t>(p.n_exc); break;
        case 9: word = static_cast<uint32_t>(p.n_exc >> 32); break;
        case 10: word = static_cast<uint32_t>(total); break;
        case 11: word = static_cast<uint32_t>(total >> 32); break;
        default:
            if (tid >= 16) {
                const uint16_t* table = reinterpret_cast<const uint16_t*>(p.sel + kSelTable);
                word = table[2 * (tid - 16)] | (uint32_t(table[2 * (tid - 16) + 1]) << 16);
            }
        }
        reinterpret_cast<uint32_t*>(fw)[tid] = word;
    }
    const uint64_t nblk = (nt + kFwBlockTiles - 1) / kFwBlockTiles;
    if (blockIdx.x + 1 >= nblk && tid == 0) { // the last CTA (or the only one when nt = 0)
        tile_exc[nt] = static_cast<uint32_t>(p.n_exc);
        for (uint64_t b = o.tile_exc + 4 * (nt + 1); b < o.exc_pos; ++b) fw[b] = 0;
        for (uint64_t b = o.exc_pos + p.n_exc; b < o.exc_word; ++b) fw[b] = 0;
        for (uint64_t b = o.exc_word + 2 * p.n_exc; b < o.total; ++b) fw[b] = 0;
    }
    __syncthreads();

    uint32_t* A = reinterpret_cast<uint32_t*>(fw + o.a);
    uint32_t* B = reinterpret_cast<uint32_t*>(fw + o.b);
    uint32_t* C = reinterpret_cast<uint32_t*>(fw + o.c);
    uint8_t* exc_pos = fw + o.exc_pos;
    uint16_t* exc_word = reinterpret_cast<uint16_t*>(fw + o.exc_word);
    for (uint32_t k = warp; k < kFwBlockTiles; k += kFwPassThreads / 32) {
        const uint64_t t = t0 + k;
        if (t >= nt) break;
        uint32_t w[8], valid;
        load_octet(p.in, n, t, lane, w, valid);
        const uint32_t emask = escape_mask(code_of, w, valid);
        uint32_t a = 0, b = 0, c = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const uint32_t code = code_of[w[q] >> 7];
            const uint32_t f = w[q] & 0x7Fu; // padding reads as 0: code 0, fraction 0
            const bool plain = ((valid >> q) & 1u) && code != kEscape;
            a |= (plain ? code : 0u) << (4 * q);
            b |= (f & 15u) << (4 * (q >> 1) + 16 * (q & 1));
            c |= (f >> 4) << (3 * (q >> 1) + 12 * (q & 1));
        }
        A[32 * t + lane] = a;
        B[32 * t + lane] = b;
        // plane C: lanes 4g..4g+3 fill words 3g..3g+2 of the tile's 24-word block
        const uint32_t nc = __shfl_down_sync(0xFFFFFFFFu, c, 1);
        const uint32_t r = lane & 3u;
        if (r < 3) C[24 * t + 3 * (lane >> 2) + r] = (c >> (8 * r)) | (nc << (24 - 8 * r));
        // exceptions in (lane, step) order
        const uint32_t cnt = __popc(emask);
        uint32_t off = cnt;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, off, d);
            if (lane >= static_cast<uint32_t>(d)) off += y;
        }
        const uint32_t tile_total = __shfl_sync(0xFFFFFFFFu, off, 31);
        off -= cnt;
        if (lane == 0 && tile_total != p.tile_cnt[t]) atomicOr(p.err, 1u);
        uint64_t e = base + te[k] + off;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            if ((emask >> q) & 1u) {
                if (e < p.n_exc) {
                    exc_pos[e] = static_cast<uint8_t>(8 * lane + q);
                    exc_word[e] = static_cast<uint16_t>(w[q]);
                } else {
                    atomicOr(p.err, 1u);
                }
                ++e;
            }
        }
    }
}

// ------------------------------------------------------------------ decode kernel
constexpr int kFwDecodeWarps = 16;
constexpr int kFwMaxItems = 480; // 64 B each: the parameters stay under 32 KiB
struct FwItem {
    const uint8_t* fw; // device: the layout (16-byte aligned)
    uint16_t* out;     // device: n_elems words (16-byte aligned)
    uint64_t n_elems;
    uint32_t n_exc;
    uint32_t cta_begin; // first CTA of this item in the launch
    uint16_t table[16];
};
static_assert(sizeof(FwItem) == 64, "FwItem layout");
struct FwDecodeParams {
    uint32_t n_items;
    uint32_t tiles_per_cta; // a multiple of kFwDecodeWarps * kFwGroup
    unsigned int* err;      // device: bit 0 = a tile's exception list failed its checks
    FwItem item[kFwMaxItems];
};

// A warp decodes groups of kFwGroup consecutive tiles. A group's plane A, B and C words
// and its tile_exc entries are contiguous in the layout, so each lane moves its share with
// one 16-byte cp.async per plane into the warp's ring of kFwStages shared-memory slots, and
// the copies run two groups ahead of the decode. Lane k then loads the group's k-th
// exception from global memory. The exceptions of a group are applied one group later,
// after the next group's main stores, so that their loads have a whole group's work to
// arrive.
constexpr uint32_t fw_decode_smem() { return 1024 + kFwDecodeWarps * kFwStages * kSlotBytes; }

__global__ void __launch_bounds__(kFwDecodeWarps * 32, 2) fw_decode_kernel(const __grid_constant__ FwDecodeParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t* pair_tab = reinterpret_cast<uint32_t*>(smem);
    __shared__ int s_item;
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
    const FwItem& it = p.item[s_item];
    // pair_tab[c0 | c1 << 4]: the (s << 7) of codes c0 and c1 in the low and high halves
    if (tid < 256) pair_tab[tid] = (uint32_t(it.table[tid & 15u]) << 7) | (uint32_t(it.table[tid >> 4]) << 23);
    __syncthreads();

    const uint64_t n = it.n_elems, nt = fw_tiles(n);
    const uint32_t n_exc = it.n_exc;
    const FwOffsets o = fw_offsets(nt, n_exc);
    const uint8_t* fw = it.fw;
    const uint8_t* EP = fw + o.exc_pos;
    const uint16_t* EW = reinterpret_cast<const uint16_t*>(fw + o.exc_word);
    uint16_t* out = it.out;
    // lane j's plane C field starts at bit 24j: word (3j) / 4, bit (24j) % 32; it needs the
    // next word only when it starts past bit 8
    const uint32_t cw0 = (3u * lane) >> 2, csh = (24u * lane) & 31u, cw1 = csh > 8 ? cw0 + 1 : cw0;
    const uint64_t t_first = uint64_t(blockIdx.x - it.cta_begin) * p.tiles_per_cta;
    const uint64_t t_end = min(t_first + p.tiles_per_cta, nt);
    const uint64_t T_warp = t_first + uint64_t(warp) * kFwGroup;     // this warp's first group
    constexpr uint32_t kStride = kFwDecodeWarps * kFwGroup;          // tiles between its groups
    const uint32_t groups = T_warp < t_end ? static_cast<uint32_t>((t_end - T_warp + kStride - 1) / kStride) : 0u;
    const uint32_t ring = static_cast<uint32_t>(__cvta_generic_to_shared(smem)) + 1024 + warp * kFwStages * kSlotBytes;
    const uint8_t* ring_p = smem + 1024 + warp * kFwStages * kSlotBytes;

    // Queue the copies of the warp's group k into slot k % kFwStages (an empty commit past the end).
    auto issue = [&](uint32_t k) {
        if (k < groups) {
            const uint64_t T0 = T_warp + uint64_t(k) * kStride;
            const uint32_t ng = t_end - T0 < kFwGroup ? static_cast<uint32_t>(t_end - T0) : kFwGroup;
            const uint32_t slot = ring + (k % kFwStages) * kSlotBytes;
            if (lane < 8 * ng) {
                fw_cp16(slot + kSlotA + 16 * lane, fw + o.a + 128 * T0 + 16 * lane);
                fw_cp16(slot + kSlotB + 16 * lane, fw + o.b + 128 * T0 + 16 * lane);
            }
            if (lane < 6 * ng) fw_cp16(slot + kSlotC + 16 * lane, fw + o.c + 96 * T0 + 16 * lane);
            if (lane <= ng) fw_cp4(slot + kSlotTE + 4 * lane, fw + o.tile_exc + 4 * (T0 + lane));
        }
        fw_commit();
    };

    // the previous group's exceptions: lane k holds entry k (position, word, tile in group)
    uint64_t pv_base = 0; // first weight of that group
    uint32_t pv_cnt = 0, pv_e0 = 0, pv_pos = 0, pv_word = 0, pv_tile = 0;
    uint32_t pv_d1 = 0, pv_d2 = 0, pv_d3 = 0; // tile_exc of its tiles 1..3, relative to tile 0
    auto apply = [&]() {
        if (lane < pv_cnt) {
            const uint64_t i = pv_base + (pv_tile << 8) + pv_pos;
            if (i < n) out[i] = static_cast<uint16_t>(pv_word);
            else atomicOr(p.err, 1u);
        }
        for (uint32_t k = lane + 32; k < pv_cnt; k += 32) { // a group with more than 32 escapes
            const uint32_t tile = (k >= pv_d1) + (k >= pv_d2) + (k >= pv_d3);
            const uint64_t i = pv_base + (tile << 8) + EP[pv_e0 + k];
            if (i < n) out[i] = EW[pv_e0 + k];
            else atomicOr(p.err, 1u);
        }
    };

#pragma unroll
    for (uint32_t k = 0; k < kFwStages - 1; ++k) issue(k);
    for (uint32_t k = 0; k < groups; ++k) {
        issue(k + kFwStages - 1);
        fw_wait_older();
        __syncwarp(); // every lane's copies of group k are in the slot
        const uint64_t T0 = T_warp + uint64_t(k) * kStride;
        const uint32_t ng = t_end - T0 < kFwGroup ? static_cast<uint32_t>(t_end - T0) : kFwGroup;
        const bool full = ng == kFwGroup && (T0 + kFwGroup) * kFwTile <= n;
        const uint8_t* sl = ring_p + (k % kFwStages) * kSlotBytes;
        const uint32_t* sa = reinterpret_cast<const uint32_t*>(sl + kSlotA) + lane;
        const uint32_t* sb = reinterpret_cast<const uint32_t*>(sl + kSlotB) + lane;
        const uint32_t* sc = reinterpret_cast<const uint32_t*>(sl + kSlotC);
        const uint32_t* ste = reinterpret_cast<const uint32_t*>(sl + kSlotTE);
        uint32_t te[kFwGroup + 1];
        te[0] = ste[0];
#pragma unroll
        for (int g = 1; g <= kFwGroup; ++g) te[g] = static_cast<uint32_t>(g) <= ng ? ste[g] : te[g - 1];
        // this group's exception list: lane k loads entry te[0] + k
        bool ok = te[kFwGroup] <= n_exc;
#pragma unroll
        for (int g = 0; g < kFwGroup; ++g) ok = ok && te[g] <= te[g + 1];
        const uint32_t cnt = ok ? te[kFwGroup] - te[0] : 0u;
        if (!ok && lane == 0) atomicOr(p.err, 1u);
        uint32_t pos = 0, word = 0;
        if (lane < cnt) {
            pos = EP[te[0] + lane];
            word = EW[te[0] + lane];
        }
        const uint32_t d1 = te[1] - te[0], d2 = te[2] - te[0], d3 = te[3] - te[0];
        // main words
        if (full) {
            uint16_t* po = out + (T0 << 8) + 8 * lane;
#pragma unroll
            for (int g = 0; g < kFwGroup; ++g)
                *reinterpret_cast<uint4*>(po + 256 * g) =
                    fw_octet(pair_tab, sa[32 * g], sb[32 * g], sc[24 * g + cw0], sc[24 * g + cw1], csh);
        } else {
#pragma unroll
            for (int g = 0; g < kFwGroup; ++g) {
                if (static_cast<uint32_t>(g) >= ng) break;
                const uint4 w = fw_octet(pair_tab, sa[32 * g], sb[32 * g], sc[24 * g + cw0], sc[24 * g + cw1], csh);
                const uint64_t i0 = ((T0 + g) << 8) + 8 * lane;
                if (i0 + 8 <= n) {
                    *reinterpret_cast<uint4*>(out + i0) = w;
                } else if (i0 < n) {
                    const uint32_t ow[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        if (i0 + q < n) out[i0 + q] = static_cast<uint16_t>(ow[q >> 1] >> (16 * (q & 1)));
                }
            }
        }
        // orders this group's stores before the previous group's exception stores, and every
        // lane's reads of the slot before its refill (group k + kFwStages, queued next)
        __syncwarp();
        apply();
        pv_base = T0 << 8;
        pv_cnt = cnt;
        pv_e0 = te[0];
        pv_pos = pos;
        pv_word = word;
        pv_tile = (lane >= d1) + (lane >= d2) + (lane >= d3);
        pv_d1 = d1;
        pv_d2 = d2;
        pv_d3 = d3;
    }
    asm volatile("cp.async.wait_all;\n" ::: "memory");
    __syncwarp();
    apply();
}

} // namespace
} // namespace bs

// ------------------------------------------------------------------ C ABI
using namespace bs;
using namespace bs::fw;

extern "C" size_t bs_fw_scratch_bytes(uint64_t n_elems) {
    return n_elems > kFwMaxElems ? 0 : static_cast<size_t>(fw_scratch(n_elems).total);
}

extern "C" bs_status bs_fw_measure(const void* d_in, uint64_t n_elems, void* d_scratch, size_t scratch_bytes,
                                   void* stream, bs_fw_info* info) {
    if (!info || !d_scratch || (n_elems && !d_in)) return BS_E_ARG;
    if (n_elems > kFwMaxElems) return BS_E_SIZE;
    if (!fw_aligned(d_in, 16) || !fw_aligned(d_scratch, 256)) return BS_E_ARG;
    const FwScratch sc = fw_scratch(n_elems);
    if (scratch_bytes < sc.total) return BS_E_SIZE;
    bs_status st = fw_device_ok();
    if (st != BS_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* scr = static_cast<uint8_t*>(d_scratch);
    auto* hist = reinterpret_cast<unsigned long long*>(scr + sc.hist);
    int e = launch_histogram(static_cast<const uint16_t*>(d_in), n_elems, hist, stream);
    if (e != cudaSuccess) return cuda_status(e);
    fw_select_kernel<<<1, 512, 0, s>>>(hist, scr + sc.sel);
    count_launch();
    const uint64_t nt = fw_tiles(n_elems), nblk = (nt + kFwBlockTiles - 1) / kFwBlockTiles;
    auto* tile_cnt = reinterpret_cast<uint32_t*>(scr + sc.tile_cnt);
    auto* blk_total = reinterpret_cast<uint32_t*>(scr + sc.blk_total);
    auto* blk_base = reinterpret_cast<unsigned long long*>(scr + sc.blk_base);
    if (nblk) {
        fw_count_kernel<<<static_cast<unsigned>(nblk), kFwPassThreads, 0, s>>>(static_cast<const uint16_t*>(d_in),
                                                                               n_elems, scr + sc.sel, tile_cnt,
                                                                               blk_total);
        count_launch();
    }
    fw_scan_kernel<<<1, 1024, 0, s>>>(blk_total, static_cast<uint32_t>(nblk), blk_base, scr + sc.sel);
    count_launch();
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_status(e);
    uint8_t host_sel[kSelBytes];
    e = cudaMemcpyAsync(host_sel, scr + sc.sel, kSelBytes, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_status(e);
    uint64_t n_exc = 0;
    std::memcpy(&n_exc, host_sel + kSelNExc, 8);
    if (n_exc >= (1ull << 32)) return BS_E_SIZE;
    info->n_elems = n_elems;
    info->n_tiles = nt;
    info->n_exc = n_exc;
    info->total_bytes = fw_offsets(nt, n_exc).total;
    std::memcpy(info->table, host_sel + kSelTable, sizeof(info->table));
    return BS_OK;
}

extern "C" bs_status bs_fw_write(const void* d_in, uint64_t n_elems, void* d_scratch, size_t scratch_bytes,
                                 const bs_fw_info* info, void* d_fw, size_t fw_bytes, void* stream) {
    if (!info || !d_scratch || !d_fw || (n_elems && !d_in)) return BS_E_ARG;
    if (!fw_info_ok(*info) || info->n_elems != n_elems) return BS_E_ARG;
    if (fw_bytes != info->total_bytes) return BS_E_SIZE;
    if (!fw_aligned(d_in, 16) || !fw_aligned(d_scratch, 256) || !fw_aligned(d_fw, 16)) return BS_E_ARG;
    const FwScratch sc = fw_scratch(n_elems);
    if (scratch_bytes < sc.total) return BS_E_SIZE;
    bs_status st = fw_device_ok();
    if (st != BS_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* scr = static_cast<uint8_t*>(d_scratch);
    // the error word lives in the selection block, after n_exc
    auto* err = reinterpret_cast<unsigned int*>(scr + sc.sel + kSelNExc + 8);
    int e = cudaMemsetAsync(err, 0, sizeof(unsigned int), s);
    if (e != cudaSuccess) return cuda_status(e);
    FwWriteParams p;
    p.in = static_cast<const uint16_t*>(d_in);
    p.n = n_elems;
    p.n_exc = info->n_exc;
    p.sel = scr + sc.sel;
    p.tile_cnt = reinterpret_cast<const uint32_t*>(scr + sc.tile_cnt);
    p.blk_base = reinterpret_cast<const unsigned long long*>(scr + sc.blk_base);
    p.fw = static_cast<uint8_t*>(d_fw);
    p.err = err;
    const uint64_t nblk = (info->n_tiles + kFwBlockTiles - 1) / kFwBlockTiles;
    fw_write_kernel<<<static_cast<unsigned>(std::max<uint64_t>(nblk, 1)), kFwPassThreads, 0, s>>>(p);
    count_launch();
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_status(e);
    unsigned int h_err = 0;
    e = cudaMemcpyAsync(&h_err, err, sizeof(h_err), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_status(e);
    return h_err ? BS_E_CORRUPT : BS_OK;
}

extern "C" bs_status bs_fw_parse(const void* h_head, size_t head_bytes, size_t fw_bytes, bs_fw_info* info) {
    if (!h_head || !info) return BS_E_ARG;
    if (head_bytes < kFwPlanesAt || fw_bytes < kFwPlanesAt) return BS_E_FORMAT;
    const uint8_t* b = static_cast<const uint8_t*>(h_head);
    auto le = [&](uint32_t off, uint32_t bytes) {
        uint64_t v = 0;
        for (uint32_t k = 0; k < bytes; ++k) v |= uint64_t(b[off + k]) << (8 * k);
        return v;
    };
    if (std::memcmp(b, "BF16LANE", 8) != 0) return BS_E_FORMAT;
    if (le(8, 4) != 1) return BS_E_VERSION;
    if (le(12, 4) != kFwHeader) return BS_E_FORMAT;
    for (uint32_t k = 48; k < 64; ++k)
        if (b[k]) return BS_E_FORMAT;
    bs_fw_info i;
    i.n_elems = le(16, 8);
    i.n_tiles = le(24, 8);
    i.n_exc = le(32, 8);
    i.total_bytes = le(40, 8);
    for (uint32_t k = 0; k < 16; ++k) i.table[k] = static_cast<uint16_t>(le(kFwHeader + 2 * k, 2));
    if (!fw_info_ok(i) || i.total_bytes != fw_bytes) return BS_E_FORMAT;
    *info = i;
    return BS_OK;
}

extern "C" bs_status bs_fw_decode(int32_t n, const void* const* d_fw, const bs_fw_info* infos, void* const* d_out,
                                  const size_t* out_bytes, uint32_t* d_err, void* stream) {
    if (n < 0 || !d_err || (n > 0 && (!d_fw || !infos || !d_out || !out_bytes))) return BS_E_ARG;
    uint64_t total_tiles = 0;
    for (int32_t k = 0; k < n; ++k) {
        const bs_fw_info& i = infos[k];
        if (!fw_info_ok(i)) return BS_E_ARG;
        if (out_bytes[k] != 2 * i.n_elems) return BS_E_SIZE;
        if (!d_fw[k] || !fw_aligned(d_fw[k], 16) || (i.n_elems && (!d_out[k] || !fw_aligned(d_out[k], 16))))
            return BS_E_ARG;
        total_tiles += i.n_tiles;
    }
    if (total_tiles == 0) return BS_OK;
    bs_status st = fw_device_ok();
    if (st != BS_OK) return st;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // Tiles per CTA: enough CTAs for three per SM even on a small launch, and up to 1024
    // tiles (256 Ki weights) per CTA on a large one; a multiple of the tiles one pass of the
    // CTA's warps covers.
    const uint64_t unit = uint64_t(kFwDecodeWarps) * kFwGroup;
    uint64_t tpc = (total_tiles + 3ull * sms - 1) / (3ull * sms);
    tpc = std::min<uint64_t>(1024, std::max<uint64_t>(unit, (tpc + unit - 1) / unit * unit));
    {
        const cudaError_t e = cudaFuncSetAttribute(fw_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   static_cast<int>(fw_decode_smem()));
        if (e != cudaSuccess) return cuda_status(e);
    }
    std::vector<FwDecodeParams> params(1);
    FwDecodeParams& p = params[0];
    p.tiles_per_cta = static_cast<uint32_t>(tpc);
    p.err = d_err;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t k = 0;
    while (k < n) {
        p.n_items = 0;
        uint64_t ctas = 0;
        for (; k < n && p.n_items < static_cast<uint32_t>(kFwMaxItems); ++k) {
            const bs_fw_info& i = infos[k];
            if (i.n_tiles == 0) continue;
            const uint64_t c = (i.n_tiles + tpc - 1) / tpc;
            if (ctas + c >= (1ull << 31)) break;
            FwItem& it = p.item[p.n_items++];
            it.fw = static_cast<const uint8_t*>(d_fw[k]);
            it.out = static_cast<uint16_t*>(d_out[k]);
            it.n_elems = i.n_elems;
            it.n_exc = static_cast<uint32_t>(i.n_exc);
            it.cta_begin = static_cast<uint32_t>(ctas);
            std::memcpy(it.table, i.table, sizeof(it.table));
            ctas += c;
        }
        if (p.n_items == 0) {
            if (k < n && infos[k].n_tiles) return BS_E_SIZE; // one tensor needs more than 2^31 CTAs
            continue;
        }
        fw_decode_kernel<<<static_cast<unsigned>(ctas), kFwDecodeWarps * 32, fw_decode_smem(), s>>>(p);
        count_launch();
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_status(e);
    }
    return BS_OK;
}
