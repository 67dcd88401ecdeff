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
// Work split: the rows of W are shared evenly among the item's CTAs, whole rows each (row r
// covers tiles r*cols/256 .. +cols/256). Inside a CTA the tiles of its rows, taken row after
// row, are shared evenly among the 8 warps, so that no warp has more than one tile more than
// another however few rows the CTA has (with whole rows per warp, a projection of 3584 rows
// would leave 1.5 rows per warp and a quarter of the warps idle for the last row). A warp
// walks its tiles in groups of up to 10, 14 or 16 tiles inside one row, through a 2-slot cp.async ring.
// Per tile and lane, the 8 decoded weights meet 8 entries of x (one 16-byte load per batch
// row; x is staged in shared memory when it is small, else served by L1/L2).
//
// Escapes: an escaped weight decodes to (table[0] << 7) | fraction, which is wrong only in its
// sign and exponent. Lane e of the warp holds the group's e-th exception and adds
// (w_true - w_decoded) * x[col] to its row's sum, so there is nothing to route to the lane
// that owns the weight. Each slot carries the next group's tile_exc entries, so a group's
// exception loads are issued one group early.
//
// Each row piece's sum is reduced over the warp. A row held whole by one warp is written
// directly; the pieces of a row split between warps are added in shared memory, in warp order,
// once the CTA is done. So every output is a fixed sum (no atomics), written in fp32.
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
    uint32_t ctas;      // CTAs of this item (at most its rows)
    uint16_t table[16];
    uint32_t pad;
};
static_assert(sizeof(FwGemvItem) == 80, "FwGemvItem layout");
struct FwGemvParams {
    uint32_t n_items;
    uint32_t layouts_resident; // BS_FW_LAYOUTS_RESIDENT: copy W before the dependency wait
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

// A warp walks its tiles in groups of up to GROUP tiles through a ring of two slots: while it
// works on one group, the copies of the next are in flight. One slot: plane A and B words
// (128 B per tile each), plane C (96 B per tile), and the tile_exc entries of the warp's
// NEXT group (GROUP + 1 of them). Groups of 10 to 16 tiles keep the per-group work (copy
// issue, exception list, bookkeeping) small per tile.
constexpr int kGemvStages = 2;
template <int GROUP>
struct GemvSlot {
    static constexpr uint32_t A = 0, B = 128 * GROUP, C = 256 * GROUP, TE = 352 * GROUP;
    static constexpr uint32_t bytes = TE + ((4 * (GROUP + 1) + 15) / 16) * 16;
};
template <int GROUP>
constexpr uint32_t gemv_smem() { return 1024 + kGemvWarps * kGemvStages * GemvSlot<GROUP>::bytes; }
// x is staged in shared memory, once per CTA, when its batch rows take at most this many bytes:
// then two CTAs still fit on an SM, and every load of x (the 16-byte loads of each tile and the
// scattered loads of the escape corrections) is a shared-memory load.
constexpr uint32_t kGemvXsMax = 32768;

// One group's exception list as the lanes hold it: the count, the index of its first entry, and
// for entries lane and lane + 32 the start of the entry's tile in the group (gpos) and its
// position byte and word as loaded (pos, word). The bytes and words are loaded one group
// before they are used and are not touched until then, so the loads' latency hides behind a
// whole group of work.
struct GemvExc {
    uint32_t cnt = 0, e0 = 0;
    uint32_t gpos[2] = {0, 0}, pos[2] = {0, 0}, word[2] = {0, 0};
};

// Two CTAs per SM (at most 128 registers a thread).
// XS: x is copied into shared memory after the ring (kGemvXsMax bytes at most).
template <int BATCH, int GROUP, bool XS>
__global__ void __launch_bounds__(kGemvWarps * 32, 2) fw_gemv_kernel(const __grid_constant__ FwGemvParams p) {
    using Slot = GemvSlot<GROUP>;
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t* pair_tab = reinterpret_cast<uint32_t*>(smem);
    __shared__ int s_item;
    __shared__ float s_first[kGemvWarps][BATCH], s_last[kGemvWarps][BATCH];
    const uint32_t tid = threadIdx.x, lane = tid & 31u, warp = tid >> 5;
    // Programmatic dependent launch: the next kernel of the stream may be scheduled as soon as
    // every CTA of this one has started, so its CTAs take over the SMs that this one leaves
    // and set up while this one finishes. The wait below returns once the kernels before this
    // one have completed and their writes are visible. Before it only the kernel parameters
    // are used, and, when the caller has stated that no work in flight writes the layouts,
    // the first group's copies of W are queued.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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
    uint16_t* xs = reinterpret_cast<uint16_t*>(smem + 1024 + kGemvWarps * kGemvStages * Slot::bytes);

    const uint32_t rows = it.rows, cols = it.cols, tpr = cols >> 8; // tiles per row
    const uint64_t nt = uint64_t(rows) * tpr;
    const uint32_t n_exc = it.n_exc;
    const FwOffsets o = fw_offsets(nt, n_exc);
    const uint8_t* fw = it.fw;
    const uint8_t* EP = fw + o.exc_pos;
    const uint16_t* EW = reinterpret_cast<const uint16_t*>(fw + o.exc_word);
    const uint32_t* TE = reinterpret_cast<const uint32_t*>(fw + o.tile_exc);
    const uint16_t* x = XS ? xs : it.x;
    const uint32_t esc_base = uint32_t(it.table[0]) << 7; // an escape decodes to this | its fraction
    const uint32_t cw0 = (3u * lane) >> 2, csh = (24u * lane) & 31u, cw1 = csh > 8 ? cw0 + 1 : cw0;
    // The CTA's rows [r_begin, r_end) (whole rows, the item's rows shared evenly among its CTAs)
    // and this warp's tiles [tb, te): the CTA's tiles, row after row, split evenly among its
    // warps. Tile indices fit in 32 bits (a layout has at most 2^32 tiles).
    const uint32_t cta = blockIdx.x - it.cta_begin;
    const uint32_t r_begin = static_cast<uint32_t>(uint64_t(rows) * cta / it.ctas);
    const uint32_t r_end = static_cast<uint32_t>(uint64_t(rows) * (cta + 1) / it.ctas);
    const uint64_t cta_tiles = uint64_t(r_end - r_begin) * tpr;
    auto warp_begin = [&](uint32_t w) { return r_begin * tpr + static_cast<uint32_t>(cta_tiles * w / kGemvWarps); };
    const uint32_t tb = warp_begin(warp), te = warp_begin(warp + 1);
    uint8_t* wsm = smem + 1024 + warp * kGemvStages * Slot::bytes;
    const uint32_t wsm_s = static_cast<uint32_t>(__cvta_generic_to_shared(wsm));

    // The warp walks its tiles in groups: runs of at most GROUP tiles that stay inside one row.
    // A Grp is one group's place (tiles k .. k+n-1 of row `row`, that is from tile
    // row * tpr + k on; n = 0 past the end); next() steps to the following one. The loop keeps
    // the places of groups j .. j+2 in a rolling window and works out j+3's when it needs it.
    struct Grp {
        uint32_t row, k, n;
    };
    auto tile0 = [&](Grp g) { return g.row * tpr + g.k; };
    auto ntiles = [&](Grp g) { return g.n; };
    auto run = [&](uint32_t row, uint32_t k) {
        const uint32_t t = row * tpr + k, left = min(tpr - k, te - t);
        return Grp{row, k, t < te ? min(left, static_cast<uint32_t>(GROUP)) : 0u};
    };
    auto next = [&](Grp g) {
        if (g.n == 0) return g;
        return g.k + g.n == tpr ? run(g.row + 1, 0u) : run(g.row, g.k + g.n);
    };
    // this lane's 16-byte share of a group's plane bytes, and of its exception arrays
    const uint8_t* gA = fw + o.a + 16 * lane;
    const uint8_t* gB = fw + o.b + 16 * lane;
    const uint8_t* gC = fw + o.c + 16 * lane;
    const uint8_t* gT = fw + o.tile_exc + 4 * lane;
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
    // A group's exception list (its tile_exc entries at ste): checked, then lane e loads
    // entries e and e + 32. An entry's tile is the number of the group's later tiles whose
    // first entry is at or before it.
    auto load_exc = [&](bool live, Grp place, const uint32_t* ste) {
        GemvExc e;
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
        for (int h = 0; h < 2; ++h) {
            const uint32_t ei = te[0] + lane + 32 * h;
            if (ei < te[GROUP]) {
                uint32_t t = 0;
#pragma unroll
                for (int g = 1; g < GROUP; ++g) t += ei >= te[g];
                e.gpos[h] = t << 8;
                e.pos[h] = EP[ei];
                e.word[h] = EW[ei];
            }
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
    // places of groups j and j+1, and the slot of group j (byte offset in the warp's ring)
    Grp g0 = run(tb / tpr, tb % tpr);
    Grp g1 = next(g0);
    uint32_t slot_k = 0;
    // group 0's tile_exc entries go to slot 1 (free until group 1 is queued), as the oldest
    // commit, so that the first wait below covers them
    if (!p.layouts_resident) asm volatile("griddepcontrol.wait;" ::: "memory");
    if (g0.n > 0 && lane <= g0.n) fw_cp4(wsm_s + Slot::bytes + Slot::TE + 4 * lane, gT + 4 * uint64_t(tile0(g0)));
    fw_commit();
    issue(g0.n > 0, g0, g1.n > 0, g1, wsm_s);
    if (p.layouts_resident) asm volatile("griddepcontrol.wait;" ::: "memory");
    // x is staged while the first group's copies are in flight
    if (XS) { // BATCH * cols BF16 values, a multiple of 256, in 16-byte pieces
        const uint4* src = reinterpret_cast<const uint4*>(it.x);
        for (uint32_t k = tid; k < BATCH * (cols >> 3); k += kGemvWarps * 32) reinterpret_cast<uint4*>(xs)[k] = __ldg(src + k);
    }
    __syncthreads(); // the pair table and x are in place
    fw_wait<1>();
    __syncwarp();
    GemvExc cur = load_exc(g0.n > 0, g0, reinterpret_cast<const uint32_t*>(wsm + Slot::bytes + Slot::TE));
    __syncwarp(); // every lane has read slot 1 before its first fill
    while (g0.n > 0) {
        const Grp g2 = next(g1);
        issue(g1.n > 0, g1, g2.n > 0, g2, wsm_s + (slot_k ^ Slot::bytes));
        fw_wait<1>(); // all but the copies just queued: group j has landed
        __syncwarp();
        const uint8_t* sl = wsm + slot_k;
        const GemvExc nxt = load_exc(g1.n > 0, g1, reinterpret_cast<const uint32_t*>(sl + Slot::TE));
        const uint32_t ng = g0.n, row = g0.row;
        const uint32_t col0 = g0.k * kFwTile; // column of the group's first weight
        const uint32_t* sa = reinterpret_cast<const uint32_t*>(sl + Slot::A) + lane;
        const uint32_t* sb = reinterpret_cast<const uint32_t*>(sl + Slot::B) + lane;
        const uint32_t* sc0 = reinterpret_cast<const uint32_t*>(sl + Slot::C) + cw0;
        const uint32_t* sc1 = reinterpret_cast<const uint32_t*>(sl + Slot::C) + cw1;
        const uint16_t* xg = xl + col0;
        auto tile = [&](int g) {
            const uint4 w = fw_octet(pair_tab, sa[32 * g], sb[32 * g], sc0[24 * g], sc1[24 * g], csh);
#pragma unroll
            for (int b = 0; b < BATCH; ++b) {
                const uint4* xp = reinterpret_cast<const uint4*>(xg + b * cols + 256 * g);
                const uint4 xv = XS ? *xp : __ldg(xp);
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
        if (lane < cur.cnt) correct(acc, col0 + cur.gpos[0] + cur.pos[0], cur.word[0]);
        if (lane + 32 < cur.cnt) correct(acc, col0 + cur.gpos[1] + cur.pos[1], cur.word[1]);
        for (uint32_t e = lane + 64; e < cur.cnt; e += 32) { // a group with more than 64 escapes
            const uint32_t ei = cur.e0 + e, t0 = tile0(g0);
            uint32_t t = 0; // its tile, from the tile_exc entries checked in load_exc
            for (uint32_t g = 1; g < ng; ++g) t += ei >= TE[t0 + g];
            correct(acc, col0 + (t << 8) + EP[ei], EW[ei]);
        }
        const bool row_end = g0.k + ng == tpr;
        if (row_end || tile0(g0) + ng == te) { // the warp's piece of this row is complete
            // a row that the warp holds whole is stored; a piece that starts inside the row
            // goes to s_first, a piece that starts the row and ends inside it to s_last
            const bool starts = row * tpr >= tb;
#pragma unroll
            for (int b = 0; b < BATCH; ++b) {
                float s = acc[b];
#pragma unroll
                for (int d = 16; d > 0; d >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, d);
                if (lane == 0) {
                    if (starts && row_end) it.y[size_t(b) * rows + row] = s;
                    else if (!starts) s_first[warp][b] = s;
                    else s_last[warp][b] = s;
                }
                acc[b] = 0.f;
            }
        }
        __syncwarp(); // every lane has read the slot before its refill
        cur = nxt;
        g0 = g1;
        g1 = g2;
        slot_k ^= Slot::bytes;
    }
    fw_wait<0>();
    // Rows split among the CTA's warps: the warp whose piece starts the row adds, in warp
    // order, the pieces of the following warps that start inside it (warps with no tiles are
    // passed over), so every output is one fixed sum.
    __syncthreads();
    if (tid < kGemvWarps) {
        const uint32_t w = tid, wb = warp_begin(w), we = warp_begin(w + 1);
        if (we > wb) {
            const uint32_t rl = (we - 1) / tpr; // the row of the warp's last tile
            if (rl * tpr >= wb && we < (rl + 1) * tpr) {
                float sum[BATCH];
#pragma unroll
                for (int b = 0; b < BATCH; ++b) sum[b] = s_last[w][b];
                for (uint32_t v = w + 1; v < kGemvWarps; ++v) {
                    const uint32_t vb = warp_begin(v), ve = warp_begin(v + 1);
                    if (ve == vb) continue;
                    if (vb / tpr != rl) break;
#pragma unroll
                    for (int b = 0; b < BATCH; ++b) sum[b] += s_first[v][b];
                }
#pragma unroll
                for (int b = 0; b < BATCH; ++b) it.y[size_t(b) * rows + rl] = sum[b];
            }
        }
    }
}

// The group size of a product: 16, 14 or 10 when it divides the row's tile count (rows of 16,
// 14, 56 tiles in the 9B-shaped model, 20 and 100 in the 27B-shaped one), so that every group
// is whole; else 16 (groups are cut at row ends, so any row length works).
inline int gemv_group_for(uint32_t cols) {
    const uint32_t tpr = cols / 256;
    return tpr % 16 == 0 ? 16 : tpr % 14 == 0 ? 14 : tpr % 10 == 0 ? 10 : 16;
}

// The kernel instance for (batch, group, x staged or not) and its shared memory, without x.
struct GemvKernel {
    void (*fn)(const FwGemvParams);
    uint32_t smem;
};
template <int BATCH, int GROUP>
GemvKernel gemv_kernel_of(bool xs) {
    return {xs ? fw_gemv_kernel<BATCH, GROUP, true> : fw_gemv_kernel<BATCH, GROUP, false>, gemv_smem<GROUP>()};
}
template <int GROUP>
GemvKernel gemv_kernel_b(uint32_t batch, bool xs) {
    switch (batch) {
    case 1: return gemv_kernel_of<1, GROUP>(xs);
    case 2: return gemv_kernel_of<2, GROUP>(xs);
    case 3: return gemv_kernel_of<3, GROUP>(xs);
    case 4: return gemv_kernel_of<4, GROUP>(xs);
    case 5: return gemv_kernel_of<5, GROUP>(xs);
    case 6: return gemv_kernel_of<6, GROUP>(xs);
    case 7: return gemv_kernel_of<7, GROUP>(xs);
    default: return gemv_kernel_of<8, GROUP>(xs);
    }
}
GemvKernel gemv_kernel(uint32_t batch, int group, bool xs) {
    return group == 14 ? gemv_kernel_b<14>(batch, xs) : group == 10 ? gemv_kernel_b<10>(batch, xs) : gemv_kernel_b<16>(batch, xs);
}

} // namespace
} // namespace bs

using namespace bs;
using namespace bs::fw;

extern "C" bs_status bs_fw_gemv(int32_t n, const bs_fw_gemv_item* items, uint32_t batch, uint32_t flags,
                                uint32_t* d_err, void* stream) {
    if (n < 0 || !d_err || (n > 0 && !items) || batch < 1 || batch > kGemvMaxBatch) return BS_E_ARG;
    if (flags & ~BS_FW_LAYOUTS_RESIDENT) return BS_E_ARG;
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
    // items in proportion to their rows (at least one row per CTA). Items whose rows split
    // differently into groups run as separate launches.
    std::vector<FwGemvParams> params(1);
    FwGemvParams& p = params[0];
    p.err = d_err;
    p.layouts_resident = (flags & BS_FW_LAYOUTS_RESIDENT) ? 1u : 0u;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    for (int group : {16, 14, 10}) {
        uint32_t max_cols = 0;
        for (int32_t k = 0; k < n; ++k)
            if (items[k].info.n_elems && gemv_group_for(items[k].cols) == group) max_cols = std::max(max_cols, items[k].cols);
        if (max_cols == 0) continue;
        const uint64_t x_bytes = uint64_t(2) * batch * max_cols;
        const bool xs = x_bytes <= kGemvXsMax;
        GemvKernel kern = gemv_kernel(batch, group, xs);
        if (xs) kern.smem += static_cast<uint32_t>(x_bytes);
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
                const uint32_t c = static_cast<uint32_t>(std::min<uint64_t>(share, g.rows)); // a row at least per CTA
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
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(static_cast<uint32_t>(ctas));
            cfg.blockDim = dim3(kGemvWarps * 32);
            cfg.dynamicSmemBytes = kern.smem;
            cfg.stream = s;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization; // see the kernel's wait
            attr[0].val.programmaticStreamSerializationAllowed = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            e = cudaLaunchKernelEx(&cfg, kern.fn, p);
            count_launch();
            if (e == cudaSuccess) e = cudaGetLastError();
            if (e != cudaSuccess) return cuda_status(e);
        }
    }
    return BS_OK;
}
