// bs_fw_gemv.cu -- y = W x for a weight matrix W held in the fixed-width lane layout
// (4-bit codes, 7-bit fractions, exceptions). W is decoded in registers on its way to the multiply, so no dense
// copy of it is ever written.
//
// This is the operand path that the "Qwen3.8-27B-BF16-NVLC-Lossless" card describes for its
// runtime: the compressed weights stay resident (its runtime accounting table), the runtime
// keeps no persistent decoded-weight cache, and it reports higher decode throughput than
// stock BF16 (its DGX Spark table). The card shows no kernel. This one targets batch-1 to
// batch-8 decoding, where y = W x is a matrix-vector product bound by the bytes of W. Reading
// 11.4 instead of 16 bits per weight is the whole gain, so it runs on the CUDA cores (fp32
// accumulation) and not on the tensor cores.
//
// Work split: a warp owns whole rows of W (row r covers tiles r*cols/256 .. +cols/256) and
// walks them in the groups of 4 tiles of bs_fw.cu, through the same 3-slot cp.async ring.
// Per tile and lane, the 8 decoded weights meet 8 entries of x (one 16-byte load per batch
// row, served by L1/L2 since every warp reads the same x).
//
// Escapes: an escaped weight decodes to (table[0] << 7) | fraction, which is wrong only in its
// sign and exponent. Lane e of the warp holds the group's e-th exception and adds
// (w_true - w_decoded) * x[col] to its row's sum, so there is nothing to route to the lane
// that owns the weight. Each slot carries the next group's tile_exc entries, so a group's
// exception loads are issued one group early.
//
// Each row's sum is reduced over the warp (fixed order, no atomics) and written in fp32.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <vector>

#include "bs_fw.cuh"

namespace bs {
namespace {
using namespace fw;

constexpr int kGemvWarps = 8;
constexpr int kGemvMaxBatch = 8;
constexpr int kGemvMaxItems = 384; // 80 B each: the parameters stay under 32 KiB
struct FwGemvItem {
    const uint8_t* fw;  // device: the layout of W
    const uint16_t* x;  // device: BF16 [batch][cols]
    float* y;           // device: [batch][rows]
    uint32_t rows, cols;
    uint32_t n_exc;
    uint32_t cta_begin; // first CTA of this item in the launch
    uint32_t ctas;      // CTAs of this item
    uint16_t table[16];
    uint32_t pad;
};
static_assert(sizeof(FwGemvItem) == 80, "FwGemvItem layout");
struct FwGemvParams {
    uint32_t n_items;
    uint32_t pad;
    unsigned int* err; // device: bit 0 = an exception list failed its checks
    FwGemvItem item[kGemvMaxItems];
};

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }

// acc + w.lo * x.lo + w.hi * x.hi for two packed BF16 pairs, with the mixed-precision FMA of
// sm_100 (BF16 operands, FP32 addend). A product of two BF16 values is exact in FP32, so each
// step rounds once, exactly like fmaf on the widened operands.
__device__ __forceinline__ float fma_bf16x2(uint32_t w, uint32_t x, float acc) {
    asm("{\n\t.reg .b16 wl, wh, xl, xh;\n\tmov.b32 {wl, wh}, %1;\n\tmov.b32 {xl, xh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, wl, xl, %0;\n\tfma.rn.f32.bf16 %0, wh, xh, %0;\n}"
        : "+f"(acc)
        : "r"(w), "r"(x));
    return acc;
}

// A warp walks its rows in groups of GROUP tiles. One slot of its ring: plane A and B words
// (128 B per tile each), plane C (96 B per tile), and the tile_exc entries of the warp's
// NEXT group (GROUP + 1 of them).
template <int GROUP>
struct GemvSlot {
    static constexpr uint32_t A = 0, B = 128 * GROUP, C = 256 * GROUP, TE = 352 * GROUP;
    static constexpr uint32_t bytes = TE + ((4 * (GROUP + 1) + 15) / 16) * 16;
};
template <int GROUP>
constexpr uint32_t gemv_smem() { return 1024 + kGemvWarps * kFwStages * GemvSlot<GROUP>::bytes; }

// One group's exception list as lane e holds it: entry e's column offset in the group and its
// word, the count, and (for the path with more than 32) where each tile's entries start,
// two 16-bit offsets per word.
template <int GROUP>
struct GemvExc {
    uint32_t cnt = 0, e0 = 0, gpos = 0, word = 0;
    uint32_t d[(GROUP + 1) / 2] = {};
    __device__ uint32_t tile_of(uint32_t e) const {
        uint32_t t = 0;
#pragma unroll
        for (int g = 1; g < GROUP; ++g) t += e >= ((d[g >> 1] >> (16 * (g & 1))) & 0xFFFFu);
        return t;
    }
};

// Batches above 2 are held to 2 CTAs per SM (at most 128 registers); 1-2 need fewer anyway.
template <int BATCH, int GROUP>
__global__ void __launch_bounds__(kGemvWarps * 32, BATCH <= 2 ? 1 : 2) fw_gemv_kernel(const __grid_constant__ FwGemvParams p) {
    using Slot = GemvSlot<GROUP>;
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
    const FwGemvItem& it = p.item[s_item];
    for (uint32_t k = tid; k < 256; k += kGemvWarps * 32)
        pair_tab[k] = (uint32_t(it.table[k & 15u]) << 7) | (uint32_t(it.table[k >> 4]) << 23);
    __syncthreads();

    const uint32_t rows = it.rows, cols = it.cols, tpr = cols >> 8; // tiles per row
    const uint32_t gpr = (tpr + GROUP - 1) / GROUP;                 // groups per row
    const uint64_t nt = uint64_t(rows) * tpr;
    const uint32_t n_exc = it.n_exc;
    const FwOffsets o = fw_offsets(nt, n_exc);
    const uint8_t* fw = it.fw;
    const uint8_t* EP = fw + o.exc_pos;
    const uint16_t* EW = reinterpret_cast<const uint16_t*>(fw + o.exc_word);
    const uint16_t* x = it.x;
    const uint32_t esc_base = uint32_t(it.table[0]) << 7; // an escape decodes to this | its fraction
    const uint32_t cw0 = (3u * lane) >> 2, csh = (24u * lane) & 31u, cw1 = csh > 8 ? cw0 + 1 : cw0;
    const uint32_t wg = (blockIdx.x - it.cta_begin) * kGemvWarps + warp; // warp within the item
    const uint32_t nw = it.ctas * kGemvWarps;
    const uint32_t my_rows = wg < rows ? (rows - wg + nw - 1) / nw : 0u;
    const uint32_t groups = my_rows * gpr;
    uint8_t* wsm = smem + 1024 + warp * kFwStages * Slot::bytes;
    const uint32_t wsm_s = static_cast<uint32_t>(__cvta_generic_to_shared(wsm));

    // The warp's groups in order: row wg, then wg + nw, ...; within a row, gi = 0 .. gpr-1
    // covers tiles GROUP gi onwards. A Grp is one group's place; next() steps to the following
    // one. The loop keeps the places of groups k .. k+3 in a rolling window. Tile indices fit
    // in 32 bits (a layout has at most 2^32 tiles).
    struct Grp {
        uint32_t row, gi;
    };
    auto next = [&](Grp g) { return g.gi + 1 < gpr ? Grp{g.row, g.gi + 1} : Grp{g.row + nw, 0u}; };
    auto tile0 = [&](Grp g) { return g.row * tpr + GROUP * g.gi; };
    auto ntiles = [&](Grp g) {
        const uint32_t left = tpr - GROUP * g.gi;
        return left < GROUP ? left : static_cast<uint32_t>(GROUP);
    };
    // this lane's 16-byte share of a group's plane bytes, and of its exception arrays
    const uint8_t* gA = fw + o.a + 16 * lane;
    const uint8_t* gB = fw + o.b + 16 * lane;
    const uint8_t* gC = fw + o.c + 16 * lane;
    const uint8_t* gT = fw + o.tile_exc + 4 * lane;
    const uint8_t* EPl = EP + lane;
    const uint16_t* EWl = EW + lane;
    const uint16_t* xl = x + 8 * lane;
    // Queue the copies of a group (place g; h is the next group's place) into the slot at
    // shared address `slot`. Every call commits one cp.async group, empty or not.
    auto issue = [&](bool live, Grp g, bool hlive, Grp h, uint32_t slot) {
        if (live) {
            const uint32_t T0 = tile0(g), ng = ntiles(g);
            const uint64_t ba = uint64_t(T0) * 128, bc = uint64_t(T0) * 96;
#pragma unroll
            for (uint32_t j = 0; j < 8 * GROUP; j += 32)
                if (lane + j < 8 * ng) {
                    fw_cp16(slot + Slot::A + 16 * (lane + j), gA + ba + 16 * j);
                    fw_cp16(slot + Slot::B + 16 * (lane + j), gB + ba + 16 * j);
                }
#pragma unroll
            for (uint32_t j = 0; j < 6 * GROUP; j += 32)
                if (lane + j < 6 * ng) fw_cp16(slot + Slot::C + 16 * (lane + j), gC + bc + 16 * j);
            if (hlive && lane <= ntiles(h)) // tile_exc of the next group rides along
                fw_cp4(slot + Slot::TE + 4 * lane, gT + 4 * uint64_t(tile0(h)));
        }
        fw_commit();
    };
    // A group's exception list (its tile_exc entries at ste): checked, then lane e loads entry e.
    auto load_exc = [&](bool live, Grp place, const uint32_t* ste) {
        GemvExc<GROUP> e;
        if (!live) return e;
        const uint32_t ng = ntiles(place);
        uint32_t te[GROUP + 1];
#pragma unroll
        for (int g = 0; g < GROUP; g += 4) {
            const uint4 q = *reinterpret_cast<const uint4*>(ste + g);
            te[g] = q.x;
            if (g + 1 <= GROUP) te[g + 1] = q.y;
            if (g + 2 <= GROUP) te[g + 2] = q.z;
            if (g + 3 <= GROUP) te[g + 3] = q.w;
        }
        te[GROUP] = ste[GROUP];
#pragma unroll
        for (int g = 1; g <= GROUP; ++g) te[g] = static_cast<uint32_t>(g) <= ng ? te[g] : te[g - 1];
        bool ok = te[GROUP] <= n_exc;
#pragma unroll
        for (int g = 0; g < GROUP; ++g) ok = ok && te[g] <= te[g + 1];
        if (!ok) {
            if (lane == 0) atomicOr(p.err, 1u);
            return e;
        }
        e.cnt = te[GROUP] - te[0];
        e.e0 = te[0];
#pragma unroll
        for (int g = 0; g < GROUP; g += 2) e.d[g >> 1] = (te[g] - te[0]) | ((te[g + 1] - te[0]) << 16);
        if (lane < e.cnt) {
            e.gpos = (e.tile_of(lane) << 8) + EPl[e.e0];
            e.word = EWl[e.e0];
        }
        return e;
    };
    // the correction of one escape at column col: (w_true - w_decoded) * x[b][col]
    auto correct = [&](float (&acc)[BATCH], uint32_t col, uint32_t word) {
        const float d = bf_lo(word) - bf_lo(esc_base | (word & 0x7Fu));
#pragma unroll
        for (int b = 0; b < BATCH; ++b) acc[b] = fmaf(d, bf_lo(x[b * cols + col]), acc[b]);
    };

    float acc[BATCH];
#pragma unroll
    for (int b = 0; b < BATCH; ++b) acc[b] = 0.f;
    // places of groups k, k+1, k+2, k+3, and the slots of groups k and k+2
    Grp g0{wg, 0u};
    Grp g1 = next(g0), g2 = next(g1), g3 = next(g2);
    uint32_t slot_k = 0, slot_k2 = 2 * Slot::bytes; // byte offsets in the warp's ring
    // group 0's tile_exc entries go to slot 2 (free until group 2 is queued), as the oldest
    // commit, so that the first wait below covers them
    if (groups > 0 && lane <= ntiles(g0)) fw_cp4(wsm_s + 2 * Slot::bytes + Slot::TE + 4 * lane, gT + 4 * uint64_t(tile0(g0)));
    fw_commit();
    issue(groups > 0, g0, groups > 1, g1, wsm_s);
    issue(groups > 1, g1, groups > 2, g2, wsm_s + Slot::bytes);
    fw_wait_older();
    __syncwarp();
    GemvExc<GROUP> cur = load_exc(groups > 0, g0, reinterpret_cast<const uint32_t*>(wsm + 2 * Slot::bytes + Slot::TE));
    for (uint32_t k = 0; k < groups; ++k) {
        issue(k + 2 < groups, g2, k + 3 < groups, g3, wsm_s + slot_k2);
        fw_wait_older(); // group k has landed
        __syncwarp();
        const uint8_t* sl = wsm + slot_k;
        const GemvExc<GROUP> nxt = load_exc(k + 1 < groups, g1, reinterpret_cast<const uint32_t*>(sl + Slot::TE));
        const uint32_t gi = g0.gi, ng = ntiles(g0), row = g0.row;
        const uint32_t col0 = gi * GROUP * kFwTile; // column of the group's first weight
        const uint32_t* sa = reinterpret_cast<const uint32_t*>(sl + Slot::A) + lane;
        const uint32_t* sb = reinterpret_cast<const uint32_t*>(sl + Slot::B) + lane;
        const uint32_t* sc0 = reinterpret_cast<const uint32_t*>(sl + Slot::C) + cw0;
        const uint32_t* sc1 = reinterpret_cast<const uint32_t*>(sl + Slot::C) + cw1;
        const uint16_t* xg = xl + col0;
        auto tile = [&](int g) {
            const uint4 w = fw_octet(pair_tab, sa[32 * g], sb[32 * g], sc0[24 * g], sc1[24 * g], csh);
#pragma unroll
            for (int b = 0; b < BATCH; ++b) {
                const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xg + b * cols + 256 * g));
                float s = acc[b];
                s = fma_bf16x2(w.x, xv.x, s);
                s = fma_bf16x2(w.y, xv.y, s);
                s = fma_bf16x2(w.z, xv.z, s);
                s = fma_bf16x2(w.w, xv.w, s);
                acc[b] = s;
            }
        };
        if (ng == GROUP) { // a whole group: no per-tile test
#pragma unroll
            for (int g = 0; g < GROUP; ++g) tile(g);
        } else {
            for (uint32_t g = 0; g < ng; ++g) tile(static_cast<int>(g));
        }
        if (lane < cur.cnt) correct(acc, col0 + cur.gpos, cur.word);
        for (uint32_t e = lane + 32; e < cur.cnt; e += 32) // a group with more than 32 escapes
            correct(acc, col0 + (cur.tile_of(e) << 8) + EP[cur.e0 + e], EW[cur.e0 + e]);
        if (gi + 1 == gpr) { // the row is complete
#pragma unroll
            for (int b = 0; b < BATCH; ++b) {
                float s = acc[b];
#pragma unroll
                for (int d = 16; d > 0; d >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, d);
                if (lane == 0) it.y[size_t(b) * rows + row] = s;
                acc[b] = 0.f;
            }
        }
        __syncwarp(); // every lane has read the slot before its refill
        cur = nxt;
        g0 = g1;
        g1 = g2;
        g2 = g3;
        g3 = next(g3);
        slot_k = slot_k == 2 * Slot::bytes ? 0u : slot_k + Slot::bytes;
        slot_k2 = slot_k2 == 2 * Slot::bytes ? 0u : slot_k2 + Slot::bytes;
    }
    fw_wait<0>();
}

// The group size of a product: the largest of 8, 7 and 4 that divides the row's tile count,
// so that every group is whole (else 8, with a shorter last group per row).
inline int gemv_group_for(uint32_t cols) {
    const uint32_t tpr = cols / 256;
    return tpr % 8 == 0 ? 8 : tpr % 7 == 0 ? 7 : tpr % 4 == 0 ? 4 : 8;
}

// The kernel instance for (batch, group), its shared memory, and the CTAs that fit on an SM.
struct GemvKernel {
    void (*fn)(const FwGemvParams);
    uint32_t smem;
};
template <int BATCH, int GROUP>
GemvKernel gemv_kernel_of() {
    return {fw_gemv_kernel<BATCH, GROUP>, gemv_smem<GROUP>()};
}
template <int GROUP>
GemvKernel gemv_kernel_b(uint32_t batch) {
    switch (batch) {
    case 1: return gemv_kernel_of<1, GROUP>();
    case 2: return gemv_kernel_of<2, GROUP>();
    case 3: return gemv_kernel_of<3, GROUP>();
    case 4: return gemv_kernel_of<4, GROUP>();
    case 5: return gemv_kernel_of<5, GROUP>();
    case 6: return gemv_kernel_of<6, GROUP>();
    case 7: return gemv_kernel_of<7, GROUP>();
    default: return gemv_kernel_of<8, GROUP>();
    }
}
GemvKernel gemv_kernel(uint32_t batch, int group) {
    return group == 7 ? gemv_kernel_b<7>(batch) : group == 4 ? gemv_kernel_b<4>(batch) : gemv_kernel_b<8>(batch);
}

} // namespace
} // namespace bs

using namespace bs;
using namespace bs::fw;

extern "C" bs_status bs_fw_gemv(int32_t n, const bs_fw_gemv_item* items, uint32_t batch, uint32_t* d_err,
                                void* stream) {
    if (n < 0 || !d_err || (n > 0 && !items) || batch < 1 || batch > kGemvMaxBatch) return BS_E_ARG;
    for (int32_t k = 0; k < n; ++k) {
        const bs_fw_gemv_item& g = items[k];
        if (!fw_info_ok(g.info) || uint64_t(g.rows) * g.cols != g.info.n_elems) return BS_E_ARG;
        if (g.cols % 256 != 0) return BS_E_ARG;
        if (g.info.n_elems == 0) continue;
        if (!g.d_fw || !g.d_x || !g.d_y || !fw_aligned(g.d_fw, 16) || !fw_aligned(g.d_x, 16) || !fw_aligned(g.d_y, 4))
            return BS_E_ARG;
    }
    bs_status st = fw_device_ok();
    if (st != BS_OK) return st;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // One wave per group size: as many CTAs as fit on the GPU at once, shared among the
    // items in proportion to their rows (a warp per row at a time, at least one row per warp),
    // so that every warp walks many rows and its copy ring stays full. Items whose rows split
    // differently into groups run as separate launches.
    std::vector<FwGemvParams> params(1);
    FwGemvParams& p = params[0];
    p.err = d_err;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    for (int group : {8, 7, 4}) {
        const GemvKernel kern = gemv_kernel(batch, group);
        bool any = false;
        for (int32_t k = 0; k < n && !any; ++k) any = items[k].info.n_elems && gemv_group_for(items[k].cols) == group;
        if (!any) continue;
        cudaError_t e = cudaFuncSetAttribute(kern.fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kern.smem));
        int per_sm = 0;
        if (e == cudaSuccess)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern.fn, kGemvWarps * 32, kern.smem);
        if (e != cudaSuccess) return cuda_status(e);
        const uint64_t wave = uint64_t(std::max(per_sm, 1)) * static_cast<uint64_t>(sms);
        int32_t k = 0;
        while (k < n) {
            p.n_items = 0;
            uint64_t ctas = 0, rows_here = 0;
            for (int32_t q = k, m = 0; q < n && m < kGemvMaxItems; ++q)
                if (items[q].info.n_elems && gemv_group_for(items[q].cols) == group) {
                    rows_here += items[q].rows;
                    ++m;
                }
            for (; k < n && p.n_items < static_cast<uint32_t>(kGemvMaxItems); ++k) {
                const bs_fw_gemv_item& g = items[k];
                if (g.info.n_elems == 0 || gemv_group_for(g.cols) != group) continue;
                const uint64_t share = std::max<uint64_t>(1, wave * g.rows / std::max<uint64_t>(rows_here, 1));
                const uint32_t c =
                    static_cast<uint32_t>(std::min<uint64_t>(share, (g.rows + kGemvWarps - 1) / kGemvWarps));
                if (ctas + c >= (1ull << 31)) break;
                FwGemvItem& it = p.item[p.n_items++];
                it.fw = static_cast<const uint8_t*>(g.d_fw);
                it.x = static_cast<const uint16_t*>(g.d_x);
                it.y = g.d_y;
                it.rows = g.rows;
                it.cols = g.cols;
                it.n_exc = static_cast<uint32_t>(g.info.n_exc);
                it.cta_begin = static_cast<uint32_t>(ctas);
                it.ctas = c;
                std::memcpy(it.table, g.info.table, sizeof(it.table));
                ctas += c;
            }
            if (p.n_items == 0) continue;
            kern.fn<<<static_cast<uint32_t>(ctas), kGemvWarps * 32, kern.smem, s>>>(p);
            count_launch();
            e = cudaGetLastError();
            if (e != cudaSuccess) return cuda_status(e);
        }
    }
    return BS_OK;
}
