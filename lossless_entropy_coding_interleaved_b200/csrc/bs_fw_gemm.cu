// bs_fw_gemm.cu -- Y = X W^T on the tensor cores for a batch of tokens, with W held in the
// fixed-width lane layout (4-bit codes, 7-bit fractions, exceptions) and decoded tile by tile
// into shared memory right before the MMA. No dense copy of W is ever written to device memory.
//
// This is the operand path of the "Qwen3.8-27B-BF16-NVLC-Lossless" card's runtime (compressed
// weights resident, no persistent decoded-weight cache; its runtime accounting and DGX Spark
// tables) for batches of tokens too large for the CUDA-core product of bs_fw_gemv.cu: each token
// adds a multiply-add per weight there (on the 9B-shaped pass it passes this kernel's time at
// about 5 tokens), so the multiply goes to the 5th-generation tensor cores (tcgen05, BF16
// operands, FP32 accumulators in tensor memory).
//
// Work split ("swap AB": the weight rows are the MMA's M, the tokens its N):
//  * A segment's 128 rows of W and up to 64 tokens are walked in slices of 128 columns: half
//    an FW tile of each row. A slice's plane bytes (A, B, C: 176 bytes a row),
//    its tiles' tile_exc entries and the tokens' X slice are copied with cp.async into one of
//    four slots, two slices ahead of the decode. Each copying thread's cp.async completion
//    arrives on the slot's mbarrier.
//  * 16 warps decode a slice from its slot into one of two A stages (BF16, K-major, the
//    128-byte swizzle of the MMA's canonical layout), patch in its exceptions, and arrive on
//    the stage's mbarrier. A tile's exception entries are loaded into registers (four lanes a
//    row, up to 3 each, the rest of a tile's entries read from memory) when its first half is
//    decoded, and serve both halves.
//  * A 17th warp issues each slice's 8 MMAs (M = 128, N = tokens, K = 16 each) into a 128 x N
//    FP32 accumulator in tensor memory once the stage is written, and commits them to the
//    slot's completion barrier. That one barrier frees both the A stage (rewritten two slices
//    later) and the slot (refilled with the slice two ahead). So the decode of a slice, the
//    MMAs of the one before and the copies of the next two all overlap, with no barrier
//    across the CTA inside the loop.
//  * Stream-K work split: a launch's units (item, token tile, 128-row block, FW tile) are shared
//    evenly by one wave of CTAs, one per SM, so no SM idles through a partial last wave. A
//    CTA walks its units as runs of one row block's tiles (segments). Segment g accumulates in
//    tensor-memory accumulator g & 1, so the read-out of one segment overlaps the MMAs of the
//    next. A segment that covers its row block's whole K range stores its sums; one that
//    covers part of it adds them into Y (zeroed by bs_fw_gemm first) with atomic FP32 adds. A
//    row block split between two CTAs gets two such parts, whose sum does not depend on their
//    order; one split among three or more CTAs (tiny launches) can differ in its last bits
//    from run to run.
//  * Four more warps read the accumulators out with tcgen05.ld (warp w reads lanes
//    32(w % 4)..+31, that is 32 rows of W, and every token column) once an extra commit after
//    a segment's last slice has arrived, and write Y[token][row] in FP32, 128 contiguous bytes
//    per warp and token; the decoding warps never wait for it.
//  * Every wait on an mbarrier is bounded. A wait that runs out, or sees that another thread's
//    has, sets the CTA's abort flag and bit 1 of the error word; the threads then skip the
//    remaining work and the tensor memory is still freed. A tile_exc entry out of order or
//    past n_exc sets bit 0 and skips that tile's exceptions.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <memory>
#include <new>

#include "bs_device.cuh"
#include "bs_fw.cuh"

namespace bs {
namespace {
using namespace fw;

constexpr uint32_t kDecWarps = 16;                  // warps that copy and decode
constexpr uint32_t kDecThreads = kDecWarps * 32;
constexpr uint32_t kEpiWarps = 4;                    // warps that read the accumulators out
constexpr uint32_t kGemmThreads = kDecThreads + 32 + kEpiWarps * 32; // + the MMA warp, + those
constexpr uint32_t kBM = 128;                        // rows of W per CTA: the MMA's M
constexpr uint32_t kMaxNt = 64;                      // tokens per CTA: the MMA's N (a multiple of 16)
constexpr uint32_t kAtomA = kBM * 128;               // one 64-wide K atom of an A stage (16 KiB)
constexpr uint32_t kStageA = 2 * kAtomA;             // 128 rows x 128 K x 2 B
constexpr uint32_t kSlots = 4;                       // copy slots: slices in flight + the one decoded
// One slot: the half-tile plane bytes of the CTA's 128 rows (A and B 64 B, C 48 B a row), their
// tiles' two tile_exc entries (8 B a row) and the tokens' X slice (N x 128 K x 2 B, swizzled).
constexpr uint32_t kPlA = 0, kPlB = kBM * 64, kPlC = 2 * kBM * 64, kPlTE = kPlC + kBM * 48, kPlX = kPlTE + kBM * 8;
constexpr uint32_t kSlotBytes = kPlX + kMaxNt * 256; // 39 KiB
static_assert(kPlX % 1024 == 0 && kSlotBytes % 1024 == 0, "the swizzled X atoms start on 1 KiB");
constexpr uint32_t kMaxSegs = 64;                     // segments (runs of one row block's tiles) a CTA
constexpr uint32_t kTabs = 2;                         // pair tables a CTA holds (items it spans)
// pair tables, mbarriers, tensor-memory address
constexpr uint32_t kHead = kTabs * 1024 + 128;
constexpr uint32_t kGemmSmem = kHead + 1024 + 2 * kStageA + kSlots * kSlotBytes; // + slack for 1 KiB alignment
static_assert(kGemmSmem + kMaxSegs * 32 + 64 <= 232448, "shared memory of one CTA");
constexpr uint32_t kTmemCols = 128;                   // two 128 x 64 FP32 accumulators
constexpr uint32_t kSpinLimit = 1u << 20;             // polls of an mbarrier wait (each up to 1 us)
constexpr int kGemmMaxItems = 320;
constexpr uint32_t kExcRegs = 3;                      // exception entries a lane holds in registers

struct FwGemmItem {
    const uint8_t* fw;   // device: the layout of W
    const uint16_t* x;   // device: BF16 [batch][cols]
    float* y;            // device: FP32 [batch][rows], zeroed before the launch
    uint32_t rows, cols;
    uint32_t n_exc;
    uint32_t unit_begin; // first unit of this item in the launch
    uint32_t row_tiles;  // rows / 128
    uint32_t pad;
    uint16_t table[16];
};
static_assert(sizeof(FwGemmItem) == 80, "FwGemmItem layout");
struct FwGemmParams {
    uint32_t n_items;
    uint32_t batch;       // tokens
    uint32_t nt;          // tokens per token tile: min(64, batch rounded up to 16)
    uint32_t token_tiles; // ceil(batch / nt)
    uint32_t units;       // units of the launch: (item, token tile, row block, tile), in that order
    uint32_t ctas;        // CTA c takes units [c * units / ctas, (c + 1) * units / ctas)
    unsigned int* err;    // bit 0: an exception list failed its checks; bit 1: an mbarrier wait ran out
    FwGemmItem item[kGemmMaxItems];
};

// A run of consecutive units of one (item, token tile, row block): tiles kt0 .. kt0 + n - 1 of
// the row block, slices q0 .. q0 + 2n - 1 of the CTA.
struct GemmSeg {
    uint32_t item, row0, tok0, kt0, n, q0, tab, full; // full: the run covers the whole K range
};

// Shared-memory matrix descriptor of a K-major operand in the 128-byte swizzle: rows of 128
// bytes, 8-row groups 1024 bytes apart (SBO), version 1, layout type 2 (SWIZZLE_128B).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) | (static_cast<uint64_t>(2) << 61);
}

__device__ __forceinline__ void mbar_init(uint32_t addr, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(addr), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t addr) {
    asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}" ::"r"(addr) : "memory");
}
// The barrier's arrival for this thread fires once all of the thread's earlier cp.async copies
// have landed (the barrier's count includes it).
__device__ __forceinline__ void mbar_arrive_cp_async(uint32_t addr) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(addr) : "memory");
}
// Waits for the completion of the barrier's phase of this parity. Gives up, sets the CTA's
// abort flag and returns false after kSpinLimit polls (about a second), or within 64 polls of
// another thread giving up.
__device__ __forceinline__ bool mbar_wait(uint32_t addr, uint32_t parity, volatile int* abort_flag) {
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        uint32_t done;
        // the thread may sleep up to 1 us inside one poll, waking as soon as the phase completes
        asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 1000;\n selp.u32 %0, 1, 0, p;\n}"
                     : "=r"(done) : "r"(addr), "r"(parity) : "memory");
        if (done) return true;
        if ((i & 63u) == 63u && *abort_flag) return false;
    }
    *abort_flag = 1;
    return false;
}

__global__ void __launch_bounds__(kGemmThreads, 1) fw_gemm_kernel(const __grid_constant__ FwGemmParams p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ GemmSeg s_seg[kMaxSegs];
    __shared__ int s_nseg, s_abort;
    const uint32_t tid = threadIdx.x, lane = tid & 31u, warp = tid >> 5;
    const uint32_t nt = p.nt, batch = p.batch;
    if (tid == 0) {
        // this CTA's units, cut into segments; the host keeps every CTA within kMaxSegs
        // segments and kTabs items
        s_abort = 0;
        const uint32_t u0 = static_cast<uint32_t>(uint64_t(p.units) * blockIdx.x / p.ctas);
        const uint32_t u1 = static_cast<uint32_t>(uint64_t(p.units) * (blockIdx.x + 1) / p.ctas);
        int k = 0, hi = static_cast<int>(p.n_items) - 1;
        while (k < hi) { // the item holding u0
            const int mid = (k + hi + 1) >> 1;
            if (p.item[mid].unit_begin <= u0) k = mid;
            else hi = mid - 1;
        }
        uint32_t n = 0, q = 0, tab = 0, u = u0;
        int first_item = k;
        while (u < u1 && n < kMaxSegs) {
            while (k + 1 < static_cast<int>(p.n_items) && p.item[k + 1].unit_begin <= u) ++k;
            const FwGemmItem& it = p.item[k];
            const uint32_t tpr = it.cols >> 8, l = u - it.unit_begin, per_tt = it.row_tiles * tpr;
            const uint32_t tt = l / per_tt, rb = (l % per_tt) / tpr, kt = l % tpr;
            const uint32_t len = min(u1 - u, tpr - kt);
            if (k != first_item) tab = 1;
            s_seg[n] = GemmSeg{static_cast<uint32_t>(k), rb * kBM, tt * nt, kt, len, q, tab, (kt == 0 && len == tpr) ? 1u : 0u};
            ++n;
            q += 2 * len;
            u += len;
        }
        if (u < u1) s_abort = 1; // more runs than kMaxSegs: the host's bound was not kept
        s_nseg = static_cast<int>(n);
    }
    __syncthreads();
    volatile int* abort_flag = &s_abort;
    const uint32_t nseg = static_cast<uint32_t>(s_nseg);
    const uint32_t nsl = nseg ? s_seg[nseg - 1].q0 + 2 * s_seg[nseg - 1].n : 0u; // the CTA's slices
    // pair table t (t < kTabs): the first segment's item, and the next item if the CTA spans two
    for (uint32_t t = 0; t < kTabs && nseg > 0; ++t) {
        uint32_t item = s_seg[0].item;
        for (uint32_t g = 0; g < nseg; ++g)
            if (s_seg[g].tab == t) { item = s_seg[g].item; break; }
        uint32_t* pt = reinterpret_cast<uint32_t*>(smem) + 256 * t;
        const FwGemmItem& it = p.item[item];
        for (uint32_t k = tid; k < 256; k += kGemmThreads)
            pt[k] = (uint32_t(it.table[k & 15u]) << 7) | (uint32_t(it.table[k >> 4]) << 23);
    }
    const uint32_t sbase = smem_u32(smem);
    // mbarriers: slot_full[4] (the copies of a slot have landed: one arrival a copying thread),
    // a_full[2] (an A stage is written: one arrival a decoding thread), mma_done[4] (the MMAs
    // of the slice in a slot have completed: the commit), d_free[2] (an accumulator has been
    // read out: one arrival an epilogue thread), seg_done[2] (the MMAs of a segment have
    // completed: an extra commit after its last slice)
    const uint32_t bar_slot = sbase + kTabs * 1024, bar_a = bar_slot + 8 * kSlots, bar_mma = bar_a + 16;
    const uint32_t bar_d = bar_mma + 8 * kSlots, bar_seg = bar_d + 16;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kTabs * 1024 + 8 * (2 * kSlots + 6));
    const uint32_t sA = (sbase + kHead + 1023u) & ~1023u; // 1 KiB aligned, as the swizzle needs
    const uint32_t sS = sA + 2 * kStageA;                  // slot k at sS + k * kSlotBytes
    uint8_t* const gA = smem + (sA - sbase);
    constexpr uint32_t kEpiThreads = kEpiWarps * 32;
    constexpr uint32_t kEpiWarp0 = kDecWarps + 1;          // the read-out warps follow the MMA warp
    if (tid == 0) {
        for (uint32_t k = 0; k < kSlots; ++k) {
            mbar_init(bar_slot + 8 * k, kDecThreads);
            mbar_init(bar_mma + 8 * k, 1);
        }
        mbar_init(bar_a, kDecThreads);
        mbar_init(bar_a + 8, kDecThreads);
        mbar_init(bar_d, kEpiThreads);
        mbar_init(bar_d + 8, kEpiThreads);
        mbar_init(bar_seg, 1);
        mbar_init(bar_seg + 8, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kDecWarps) { // tensor memory: two 128 x (at most 64) FP32 accumulators
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    if (tid < kDecThreads) {
        // The copies of slice q, split over the threads: A and B plane pieces (16 bytes, 4 a
        // row), C pieces (3 a row), tile_exc entries (2 a row) and X pieces (16 a token, placed
        // in the 128-byte swizzle; tokens past the batch are zero-filled, pieces past nt
        // tokens are not copied).
        constexpr uint32_t kPcAB = kBM * 4 / kDecThreads, kPcC = (kBM * 3 + kDecThreads - 1) / kDecThreads;
        constexpr uint32_t kPcTE = (kBM * 2 + kDecThreads - 1) / kDecThreads, kPcX = kMaxNt * 16 / kDecThreads;
        static_assert(kBM * 4 % kDecThreads == 0 && kMaxNt * 16 % kDecThreads == 0, "pieces");
        // The sources of this thread's pieces for the first slice of segment gi (slice q0 + qq
        // of the segment adds 64 qq bytes for A and B, 48 qq for C, 4 (qq / 2) for tile_exc and
        // 128 qq elements for X), worked out once a segment.
        uint32_t gi = 0, gi_end = 0, gi_q0 = 0; // the segment of the slice being queued, its slices
        const uint8_t* srcA[kPcAB];
        const uint8_t* srcC[kPcC];
        const uint8_t* srcT[kPcTE];
        const uint16_t* srcX[kPcX];
        uint64_t gapB = 0;               // plane B's offset from plane A
        uint32_t bytesX = 0, liveX = 0;  // bit i: X piece i reads 16 bytes; piece i is copied
        auto seg_sources = [&](uint32_t g) {
            const GemmSeg sg = s_seg[g];
            const FwGemmItem& it = p.item[sg.item];
            const uint32_t tpr = it.cols >> 8;
            const FwOffsets o = fw_offsets(uint64_t(it.rows) * tpr, it.n_exc);
            const uint64_t tile0 = uint64_t(sg.row0) * tpr + sg.kt0; // the block's first row's tile
            gapB = o.b - o.a;
#pragma unroll
            for (uint32_t i = 0; i < kPcAB; ++i) {
                const uint32_t c = tid + kDecThreads * i;
                srcA[i] = it.fw + o.a + (tile0 + uint64_t(c >> 2) * tpr) * 128u + 16u * (c & 3u);
            }
#pragma unroll
            for (uint32_t i = 0; i < kPcC; ++i) {
                const uint32_t cc = min(tid + kDecThreads * i, kBM * 3 - 1); // the clamped ones are not copied
                srcC[i] = it.fw + o.c + (tile0 + uint64_t(cc / 3u) * tpr) * 96u + 16u * (cc % 3u);
            }
#pragma unroll
            for (uint32_t i = 0; i < kPcTE; ++i) {
                const uint32_t cc = min(tid + kDecThreads * i, kBM * 2 - 1); // likewise
                srcT[i] = it.fw + o.tile_exc + 4 * (tile0 + uint64_t(cc >> 1) * tpr + (cc & 1u));
            }
            bytesX = 0;
            liveX = 0;
#pragma unroll
            for (uint32_t i = 0; i < kPcX; ++i) {
                const uint32_t id = tid + kDecThreads * i, t = id >> 4, c = id & 15u, tok = sg.tok0 + t;
                srcX[i] = tok < batch ? it.x + uint64_t(tok) * it.cols + sg.kt0 * 256 + c * 8 : it.x;
                bytesX |= (tok < batch ? 1u : 0u) << i;
                liveX |= (t < nt ? 1u : 0u) << i;
            }
            gi_q0 = sg.q0;
            gi_end = sg.q0 + 2 * sg.n;
        };
        auto issue = [&](uint32_t q) {
            while (q >= gi_end) seg_sources(++gi);
            const uint32_t qq = q - gi_q0;
            const uint32_t sp = sS + (q % kSlots) * kSlotBytes;
#pragma unroll
            for (uint32_t i = 0; i < kPcAB; ++i) {
                const uint32_t c = tid + kDecThreads * i;
                cp_async16(sp + kPlA + 16 * c, srcA[i] + 64u * qq, 16u);
                cp_async16(sp + kPlB + 16 * c, srcA[i] + gapB + 64u * qq, 16u);
            }
#pragma unroll
            for (uint32_t i = 0; i < kPcC; ++i) {
                const uint32_t c = tid + kDecThreads * i;
                cp_async16_if(c < kBM * 3, sp + kPlC + 16 * c, srcC[i] + 48u * qq, 16u);
            }
#pragma unroll
            for (uint32_t i = 0; i < kPcTE; ++i) {
                const uint32_t c = tid + kDecThreads * i;
                if (c < kBM * 2) fw_cp4(sp + kPlTE + 4 * c, srcT[i] + 4 * (qq >> 1));
            }
#pragma unroll
            for (uint32_t i = 0; i < kPcX; ++i) {
                const uint32_t id = tid + kDecThreads * i, t = id >> 4, c = id & 15u;
                const uint32_t dst = sp + kPlX + (c >> 3) * (nt * 128) + t * 128 + (((c & 7u) ^ (t & 7u)) << 4);
                cp_async16_if((liveX >> i) & 1u, dst, srcX[i] + 128u * qq, ((bytesX >> i) & 1u) * 16u);
            }
            mbar_arrive_cp_async(bar_slot + 8 * (q % kSlots));
        };
        if (nsl > 0) seg_sources(0);
        // decode: warp w writes rows 8w .. 8w+7, two at a time (lanes 0-15 and 16-31), lane
        // octet j = lane & 15 of the half tile
        const uint32_t j = lane & 15u, rsub = lane >> 4;
        const uint32_t cw0 = (3u * j) >> 2, csh = (24u * j) & 31u, cw1 = csh > 8 ? cw0 + 1 : cw0;
        // exceptions: lane holds entries e0 + kExcRegs (lane >> 3) .. of row er's tile, as
        // (position << 16) | word, the first n_ex of them valid
        constexpr uint32_t kRowsW = kBM / kDecWarps; // 8 rows a warp
        const uint32_t er = warp * kRowsW + (lane & (kRowsW - 1u));
        uint32_t ex[kExcRegs];
        uint32_t e0 = 0, eend = 0, n_ex = 0;
        // the segment of the slice being decoded: its first slice and end, its item's exception
        // arrays, exception count and pair table, worked out once a segment
        uint32_t gd = 0, gd_q0 = 0, gd_end = 0, gd_nexc = 0;
        const uint8_t* EP = nullptr;
        const uint16_t* EW = nullptr;
        const uint32_t* pair_tab = nullptr;
        auto seg_decode = [&](uint32_t g) {
            const GemmSeg sg = s_seg[g];
            const FwGemmItem& it = p.item[sg.item];
            const FwOffsets o = fw_offsets(uint64_t(it.rows) * (it.cols >> 8), it.n_exc);
            EP = it.fw + o.exc_pos;
            EW = reinterpret_cast<const uint16_t*>(it.fw + o.exc_word);
            gd_nexc = it.n_exc;
            pair_tab = reinterpret_cast<const uint32_t*>(smem) + 256 * sg.tab;
            gd_q0 = sg.q0;
            gd_end = sg.q0 + 2 * sg.n;
        };
        if (nsl > 0) seg_decode(0);
        for (uint32_t q = 0; q + 1 < kSlots && q < nsl; ++q) issue(q); // slices 0 .. kSlots - 2
        for (uint32_t q = 0; q < nsl && ok; ++q) {
            while (q >= gd_end) seg_decode(++gd);
            const uint32_t s = q % kSlots, st = q & 1u, h = (q - gd_q0) & 1u;
            const uint8_t* slot = smem + (sS - sbase) + s * kSlotBytes;
            if (!mbar_wait(bar_slot + 8 * s, (q / kSlots) & 1u, abort_flag)) { ok = false; break; }
            if (h == 0) { // a new tile: its exception entries, both halves use them
                const uint32_t* te = reinterpret_cast<const uint32_t*>(slot + kPlTE) + 2 * er;
                const uint32_t t0 = te[0], t1 = te[1];
                const bool e_ok = t0 <= t1 && t1 <= gd_nexc;
                if (!e_ok && lane < kRowsW) atomicOr(p.err, 1u);
                e0 = t0;
                eend = e_ok ? t1 : t0;
                const uint32_t ebeg = t0 + kExcRegs * (lane / kRowsW);
                n_ex = ebeg < eend ? min(eend - ebeg, kExcRegs) : 0u;
#pragma unroll
                for (uint32_t i = 0; i < kExcRegs; ++i)
                    ex[i] = i < n_ex ? (uint32_t(__ldg(EP + ebeg + i)) << 16) | __ldg(EW + ebeg + i) : 0u;
            }
            uint32_t pa[4], pb[4], pc0[4], pc1[4];
#pragma unroll
            for (uint32_t i = 0; i < 4; ++i) {
                const uint32_t r = warp * kRowsW + 2 * i + rsub;
                pa[i] = *reinterpret_cast<const uint32_t*>(slot + kPlA + r * 64 + 4 * j);
                pb[i] = *reinterpret_cast<const uint32_t*>(slot + kPlB + r * 64 + 4 * j);
                const uint32_t* cp = reinterpret_cast<const uint32_t*>(slot + kPlC + r * 48);
                pc0[i] = cp[cw0];
                pc1[i] = cp[cw1];
            }
            // A stage st was last read by the MMAs of slice q - 2; once they have completed, a
            // segment that ended with slice q - 2 or before can be read out
            if (q >= 2 && !mbar_wait(bar_mma + 8 * ((q - 2) % kSlots), ((q - 2) / kSlots) & 1u, abort_flag)) {
                ok = false;
                break;
            }
            uint8_t* const stA = gA + st * kStageA;
#pragma unroll
            for (uint32_t i = 0; i < 4; ++i) {
                const uint32_t r = warp * kRowsW + 2 * i + rsub;
                const uint4 w = fw_octet(pair_tab, pa[i], pb[i], pc0[i], pc1[i], csh);
                *reinterpret_cast<uint4*>(stA + (j >> 3) * kAtomA + r * 128 + (((j & 7u) ^ (r & 7u)) << 4)) = w;
            }
            __syncwarp();
            // the exceptions of this half: positions 128 h .. 128 h + 127 of the tile
#pragma unroll
            for (uint32_t i = 0; i < kExcRegs; ++i) {
                if (i >= n_ex) break;
                const uint32_t pos = ex[i] >> 16;
                if ((pos >> 7) == h) {
                    const uint32_t jj = (pos >> 3) & 15u;
                    *reinterpret_cast<uint16_t*>(stA + (jj >> 3) * kAtomA + er * 128 + (((jj & 7u) ^ (er & 7u)) << 4) +
                                                 2 * (pos & 7u)) = static_cast<uint16_t>(ex[i]);
                }
            }
            if (lane < kRowsW) // a tile with more exceptions than the lanes hold: the rest, from memory
                for (uint32_t e = e0 + (32 / kRowsW) * kExcRegs; e < eend; ++e) {
                    const uint32_t pos = __ldg(EP + e);
                    if ((pos >> 7) != h) continue;
                    const uint32_t jj = (pos >> 3) & 15u;
                    *reinterpret_cast<uint16_t*>(stA + (jj >> 3) * kAtomA + er * 128 + (((jj & 7u) ^ (er & 7u)) << 4) +
                                                 2 * (pos & 7u)) = __ldg(EW + e);
                }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); // read by the tensor cores
            mbar_arrive(bar_a + 8 * st);
            // refill: slice q + kSlots - 2 goes into the slot of slice q - 2, whose MMAs have
            // completed (waited for above); slice q - 1's MMAs may still be running
            const uint32_t qn = q + kSlots - 2;
            if (qn < nsl && qn >= kSlots - 1) issue(qn);
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp >= kEpiWarp0) {
        // The read-out warps: warp w reads tensor-memory lanes 32 (w % 4) .. +31 (rows of W) and
        // every token column of segment g's accumulator (g & 1) once the segment's MMAs have
        // completed, and writes Y. A segment that covers its row block's whole K range stores;
        // the others add their part. The accumulator is then free for segment g + 2.
        const uint32_t quarter = warp & 3u;
        for (uint32_t g = 0; g < nseg && ok; ++g) {
            if (!mbar_wait(bar_seg + 8 * (g & 1u), (g >> 1) & 1u, abort_flag)) { ok = false; break; }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const GemmSeg sg = s_seg[g];
            const FwGemmItem& it = p.item[sg.item];
            const uint32_t row = sg.row0 + quarter * 32 + lane;
            for (uint32_t cb = 0; cb < nt; cb += 16) {
                uint32_t v[16];
                const uint32_t taddr = tmem + ((quarter * 32) << 16) + (g & 1u) * 64 + cb;
                asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
                             : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
                               "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
                             : "r"(taddr));
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                for (uint32_t q = 0; q < 16; ++q) {
                    const uint32_t tok = sg.tok0 + cb + q;
                    if (tok < batch) {
                        float* dst = it.y + uint64_t(tok) * it.rows + row;
                        if (sg.full) *dst = __uint_as_float(v[q]);
                        else atomicAdd(dst, __uint_as_float(v[q])); // Y was zeroed; parts add up
                    }
                }
            }
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            mbar_arrive(bar_d + 8 * (g & 1u));
        }
    } else if (tid == kDecThreads) {
        // the MMA thread: M = 128, N = nt, BF16 x BF16 -> FP32, both operands K-major;
        // segment g accumulates into accumulator g & 1, which segment g - 2's read-out frees
        const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((nt >> 3) << 17) | ((kBM >> 4) << 24);
        uint32_t g = 0;
        for (uint32_t q = 0; q < nsl; ++q) {
            while (q >= s_seg[g].q0 + 2 * s_seg[g].n) ++g;
            const uint32_t st = q & 1u, s = q % kSlots, first = q == s_seg[g].q0;
            if (first && g >= 2 && !mbar_wait(bar_d + 8 * (g & 1u), ((g - 2) >> 1) & 1u, abort_flag)) { ok = false; break; }
            if (!mbar_wait(bar_a + 8 * st, (q >> 1) & 1u, abort_flag)) { ok = false; break; }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t a0 = sA + st * kStageA, b0 = sS + s * kSlotBytes + kPlX, d = tmem + (g & 1u) * 64;
#pragma unroll
            for (uint32_t kk = 0; kk < 8; ++kk) { // K = 16 per MMA: atom kk / 4, 32 bytes per step inside it
                const uint64_t ad = sw128_desc(a0 + (kk >> 2) * kAtomA + (kk & 3u) * 32);
                const uint64_t bd = sw128_desc(b0 + (kk >> 2) * (nt * 128) + (kk & 3u) * 32);
                const uint32_t acc = !(first && kk == 0);
                asm volatile("{\n .reg .pred p;\n setp.ne.u32 p, %4, 0;\n"
                             " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}"
                             ::"r"(d), "l"(ad), "l"(bd), "r"(idesc), "r"(acc) : "memory");
            }
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_mma + 8 * s)
                         : "memory");
            if (q + 1 == s_seg[g].q0 + 2 * s_seg[g].n) // the segment's last slice: tell the read-out warps
                asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_seg + 8 * (g & 1u))
                             : "memory");
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (tid == 0 && *abort_flag) atomicOr(p.err, 2u);
    if (warp == kDecWarps)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
}

} // namespace
} // namespace bs

using namespace bs;
using namespace bs::fw;

extern "C" bs_status bs_fw_gemm(int32_t n, const bs_fw_gemv_item* items, uint32_t batch, uint32_t* d_err,
                                void* stream) {
    if (n < 0 || !d_err || (n > 0 && !items) || batch < 1 || batch > (1u << 20)) return BS_E_ARG;
    for (int32_t k = 0; k < n; ++k) {
        const bs_fw_gemv_item& g = items[k];
        if (!fw_info_ok(g.info) || uint64_t(g.rows) * g.cols != g.info.n_elems) return BS_E_ARG;
        if (g.cols % 256 != 0 || g.rows % kBM != 0) return BS_E_ARG;
        if (uint64_t(g.rows) * (g.cols / 256) * 128 >= (1ull << 32)) return BS_E_SIZE; // plane offsets are 32-bit
        if (g.info.n_elems == 0) continue;
        if (!g.d_fw || !g.d_x || !g.d_y || !fw_aligned(g.d_fw, 16) || !fw_aligned(g.d_x, 16) || !fw_aligned(g.d_y, 4))
            return BS_E_ARG;
    }
    bs_status st = fw_device_ok();
    if (st != BS_OK) return st;
    std::unique_ptr<FwGemmParams> pp(new (std::nothrow) FwGemmParams);
    if (!pp) return BS_E_NOMEM;
    FwGemmParams& p = *pp;
    p.err = d_err;
    p.batch = batch;
    p.nt = std::min<uint32_t>(kMaxNt, (batch + 15u) & ~15u);
    p.token_tiles = (batch + p.nt - 1) / p.nt;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaFuncSetAttribute(fw_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kGemmSmem));
    if (e != cudaSuccess) return cuda_status(e);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int32_t k = 0;
    while (k < n) {
        // The items of one launch and their units (token tile, row block, tile). The units are
        // shared evenly by one wave of CTAs (one per SM), so a CTA's range may start or end
        // inside a row block; those parts add into Y, which is zeroed first. A CTA holds at
        // most kMaxSegs runs and two items: launches with small items use more CTAs.
        p.n_items = 0;
        uint64_t units = 0;
        uint32_t min_units = ~0u, min_tpr = ~0u;
        for (; k < n && p.n_items < static_cast<uint32_t>(kGemmMaxItems); ++k) {
            const bs_fw_gemv_item& g = items[k];
            if (g.info.n_elems == 0) continue;
            const uint32_t tpr = g.cols / 256;
            const uint64_t u = uint64_t(g.rows / kBM) * p.token_tiles * tpr;
            if (units + u >= (1ull << 31)) break;
            e = cudaMemsetAsync(g.d_y, 0, sizeof(float) * uint64_t(batch) * g.rows, s);
            if (e != cudaSuccess) return cuda_status(e);
            FwGemmItem& it = p.item[p.n_items++];
            it.fw = static_cast<const uint8_t*>(g.d_fw);
            it.x = static_cast<const uint16_t*>(g.d_x);
            it.y = g.d_y;
            it.rows = g.rows;
            it.cols = g.cols;
            it.n_exc = static_cast<uint32_t>(g.info.n_exc);
            it.unit_begin = static_cast<uint32_t>(units);
            it.row_tiles = g.rows / kBM;
            it.pad = 0;
            std::memcpy(it.table, g.info.table, sizeof(it.table));
            units += u;
            min_units = std::min<uint32_t>(min_units, static_cast<uint32_t>(u));
            min_tpr = std::min(min_tpr, tpr);
        }
        if (p.n_items == 0) continue;
        // one CTA per SM, unless a CTA's share (at most ceil(units / ctas)) would exceed the
        // smallest item's units (so that a CTA spans at most two items) or give more than
        // kMaxSegs runs (a share of L units over rows of at least min_tpr tiles makes at most
        // L / min_tpr + 3 runs)
        const uint64_t bound = std::max<uint64_t>(1, std::min<uint64_t>(min_units, uint64_t(kMaxSegs - 4) * min_tpr));
        const uint64_t ctas = std::max<uint64_t>(std::min<uint64_t>(static_cast<uint64_t>(sms), units), (units + bound - 1) / bound);
        p.units = static_cast<uint32_t>(units);
        p.ctas = static_cast<uint32_t>(ctas);
        fw_gemm_kernel<<<static_cast<uint32_t>(ctas), kGemmThreads, kGemmSmem, s>>>(p);
        count_launch();
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_status(e);
    }
    return BS_OK;
}
