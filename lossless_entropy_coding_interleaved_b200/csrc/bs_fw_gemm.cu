// bs_fw_gemm.cu -- Y = X W^T on the tensor cores for a batch of tokens, with W held in the
// fixed-width lane layout (4-bit codes, 7-bit fractions, exceptions) and decoded tile by tile
// into shared memory right before the MMA. No dense copy of W is ever written to device memory.
//
// This is the operand path of the "Qwen3.8-27B-BF16-NVLC-Lossless" card's runtime (compressed
// weights resident, no persistent decoded-weight cache; its runtime accounting and DGX Spark
// tables) for batches of tokens too large for the CUDA-core product of bs_fw_gemv.cu: at 9 or
// more tokens a product needs more multiply-adds per weight byte than the CUDA cores give, so
// the multiply goes to the 5th-generation tensor cores (tcgen05, BF16 operands, FP32
// accumulators in tensor memory).
//
// Work split ("swap AB": the weight rows are the MMA's M, the tokens its N):
//  * A CTA owns 128 rows of W and up to 64 tokens and walks K in 256-wide slices (one FW tile
//    of each row). The slice kb + 1's plane bytes (A, B, C: 352 bytes a tile), its tile_exc
//    entries and the tokens' X slice are copied into shared memory with cp.async while slice
//    kb is decoded, so the HBM reads run a slice ahead of the work (45 KiB in flight a CTA).
//  * Its 16 warps decode slice kb from shared memory into the A stage (BF16, K-major, the
//    128-byte swizzle of the MMA's canonical layout) and patch in its exceptions. A tile's
//    exception entries are loaded into registers (four lanes a tile, up to 8 each) before the
//    decode, so their latency hides behind it.
//  * A matrix with too few row blocks to fill the GPU splits its K range over several CTAs
//    per row block (up to about two CTAs per SM in all); they add their parts into Y, which
//    bs_fw_gemm zeroes first, with atomic FP32 adds (so the sum's order, and its last bits,
//    can differ between runs).
//  * One thread issues the slice's 16 MMAs (M = 128, N = tokens, K = 16 each) into a 128 x N
//    FP32 accumulator in tensor memory and commits them to an mbarrier. The A stage is
//    rewritten only after that commit has arrived; at these N the MMAs take a small fraction
//    of a slice's time, so one A stage suffices and the shared memory goes to the copies.
//  * The epilogue reads the accumulator with tcgen05.ld (warps 0-7; warp w reads lanes
//    32(w % 4)..+31, that is 32 rows of W, and 32 tokens from column 32(w / 4)) and writes
//    Y[token][row] in FP32, 128 contiguous bytes per warp and token.
//  * Every wait on an mbarrier is bounded. A wait that runs out sets bit 1 of the error word,
//    skips the remaining work and still frees the tensor memory. A tile_exc entry out of order
//    or past n_exc sets bit 0 and skips that tile's exceptions.
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

constexpr int kGemmWarps = 16;
constexpr int kGemmThreads = kGemmWarps * 32;
constexpr uint32_t kBM = 128;                     // rows of W per CTA: the MMA's M
constexpr uint32_t kMaxNt = 64;                   // tokens per CTA: the MMA's N (a multiple of 16)
constexpr uint32_t kAtomA = kBM * 128;            // one 64-wide K atom of the A stage (16 KiB)
constexpr uint32_t kStageA = 4 * kAtomA;          // 128 rows x 256 K x 2 B
constexpr uint32_t kStageB = 4 * kMaxNt * 128;    // up to 64 tokens x 256 K x 2 B
// One slot of copied plane bytes: A and B planes (128 B a tile), C (96 B a tile), and each
// tile's two tile_exc entries (8 B a tile).
constexpr uint32_t kPlA = 0, kPlB = kBM * 128, kPlC = 2 * kBM * 128, kPlTE = kPlC + kBM * 96;
constexpr uint32_t kSlot = kPlTE + kBM * 8;       // 46,080 B
constexpr uint32_t kHead = 2048;                  // pair table, mbarrier, tensor-memory address
// + 1 KiB of slack to align the A stage; then A, two B stages, two plane slots
constexpr uint32_t kGemmSmem = kHead + 1024 + kStageA + 2 * kStageB + 2 * kSlot;
static_assert(kGemmSmem <= 232448, "shared memory of one CTA");
constexpr uint32_t kTmemCols = 64;
constexpr uint32_t kSpinLimit = 1u << 24;
constexpr int kGemmMaxItems = 320;
constexpr uint32_t kExcRegs = 8;                  // exception entries a lane holds in registers

struct FwGemmItem {
    const uint8_t* fw;  // device: the layout of W
    const uint16_t* x;  // device: BF16 [batch][cols]
    float* y;           // device: FP32 [batch][rows]
    uint32_t rows, cols;
    uint32_t n_exc;
    uint32_t cta_begin; // first CTA of this item in the launch
    uint32_t row_tiles; // rows / 128
    uint16_t ksplit;    // CTAs that share a row block's K range, each adding its part into Y
    uint16_t kper;      // 256-wide K slices per such CTA
    uint16_t table[16];
};
static_assert(sizeof(FwGemmItem) == 80, "FwGemmItem layout");
struct FwGemmParams {
    uint32_t n_items;
    uint32_t batch;       // tokens
    uint32_t nt;          // tokens per CTA: min(64, batch rounded up to 16)
    uint32_t token_tiles; // ceil(batch / nt)
    unsigned int* err;    // bit 0: an exception list failed its checks; bit 1: an mbarrier wait ran out
    FwGemmItem item[kGemmMaxItems];
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
// Waits for the completion of the barrier's phase of this parity; false if it ran out.
__device__ __forceinline__ bool mbar_wait(uint32_t addr, uint32_t parity) {
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        uint32_t done;
        asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
                     : "=r"(done) : "r"(addr), "r"(parity) : "memory");
        if (done) return true;
    }
    return false;
}

__global__ void __launch_bounds__(kGemmThreads, 1) fw_gemm_kernel(const __grid_constant__ FwGemmParams p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ int s_item;
    __shared__ int s_abort;
    const uint32_t tid = threadIdx.x, lane = tid & 31u, warp = tid >> 5;
    if (tid == 0) {
        find_item(p, &s_item);
        s_abort = 0;
    }
    __syncthreads();
    const FwGemmItem& it = p.item[s_item];
    uint32_t* pair_tab = reinterpret_cast<uint32_t*>(smem);
    for (uint32_t k = tid; k < 256; k += kGemmThreads)
        pair_tab[k] = (uint32_t(it.table[k & 15u]) << 7) | (uint32_t(it.table[k >> 4]) << 23);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t mbar = sbase + 1024;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + 1040);
    const uint32_t sA = (sbase + kHead + 1023u) & ~1023u; // 1 KiB aligned, as the swizzle needs
    if (tid == 0) {
        mbar_init(mbar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) { // 64 columns of tensor memory: the 128 x (at most 64) FP32 accumulator
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;

    const uint32_t rows = it.rows, K = it.cols, tpr = K >> 8;
    // CTA (row block, token block, K part): K parts innermost, so a row block's parts run together
    const uint32_t local = blockIdx.x - it.cta_begin;
    const uint32_t kpart = local % it.ksplit, rt = local / it.ksplit;
    const uint32_t row0 = (rt % it.row_tiles) * kBM;
    const uint32_t nt = p.nt, tok0 = (rt / it.row_tiles) * nt, batch = p.batch;
    const uint32_t kbeg = kpart * it.kper, kend = min(tpr, kbeg + it.kper);
    const bool split = it.ksplit > 1;
    const uint64_t n_tiles = uint64_t(rows) * tpr;
    const FwOffsets o = fw_offsets(n_tiles, it.n_exc);
    const uint8_t* fw = it.fw;
    const uint8_t* EP = fw + o.exc_pos;
    const uint16_t* EW = reinterpret_cast<const uint16_t*>(fw + o.exc_word);
    const uint32_t cw0 = (3u * lane) >> 2, csh = (24u * lane) & 31u, cw1 = csh > 8 ? cw0 + 1 : cw0;
    // M = 128, N = nt, BF16 x BF16 -> FP32, both operands K-major
    const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((nt >> 3) << 17) | ((kBM >> 4) << 24);
    const uint32_t sB0 = sA + kStageA, bbytes = 4 * nt * 128;      // B stages: sB0 + s * bbytes
    const uint32_t sP0 = sB0 + 2 * bbytes;                           // plane slots: sP0 + s * kSlot
    uint8_t* const pA = smem + (sA - sbase);

    // The copies of a slice, split over the threads so that each thread's share has the same
    // place in every slice: A and B plane pieces (16 bytes, 8 a tile, contiguous in the slot)
    // at piece tid + kGemmThreads i, C plane pieces (6 a tile) likewise, and tile_exc entries.
    // A slice kb's source is the same plus kb * 128 (A, B) or kb * 96 (C) bytes.
    constexpr uint32_t kPiecesAB = kBM * 8 / kGemmThreads, kPiecesC = (kBM * 6 + kGemmThreads - 1) / kGemmThreads;
    static_assert(kBM * 8 % kGemmThreads == 0, "pieces per thread");
    uint32_t offAB[kPiecesAB], offC[kPiecesC]; // byte offsets of slice 0's pieces in the planes
#pragma unroll
    for (uint32_t i = 0; i < kPiecesAB; ++i) {
        const uint32_t c = tid + kGemmThreads * i;
        offAB[i] = (row0 + (c >> 3)) * tpr * 128u + (c & 7u) * 16u;
    }
#pragma unroll
    for (uint32_t i = 0; i < kPiecesC; ++i) {
        const uint32_t c = min(tid + kGemmThreads * i, kBM * 6 - 1); // the guard below skips the clamped ones
        offC[i] = (row0 + c / 6) * tpr * 96u + (c % 6) * 16u;
    }
    const uint8_t* const planeA = fw + o.a;
    const uint8_t* const planeB = fw + o.b;
    const uint8_t* const planeC = fw + o.c;
    const uint8_t* const tex = fw + o.tile_exc;

    // Queue the copies of slice kb into plane slot kb & 1 and B stage kb & 1 (tokens past the
    // batch read as 0).
    auto issue = [&](uint32_t kb) {
        const uint32_t sp = sP0 + (kb & 1u) * kSlot, sb = sB0 + (kb & 1u) * bbytes;
#pragma unroll
        for (uint32_t i = 0; i < kPiecesAB; ++i) {
            const uint32_t c = tid + kGemmThreads * i;
            cp_async16(sp + kPlA + 16 * c, planeA + offAB[i] + kb * 128u, 16u);
            cp_async16(sp + kPlB + 16 * c, planeB + offAB[i] + kb * 128u, 16u);
        }
#pragma unroll
        for (uint32_t i = 0; i < kPiecesC; ++i)
            if (tid + kGemmThreads * i < kBM * 6)
                cp_async16(sp + kPlC + 16 * (tid + kGemmThreads * i), planeC + offC[i] + kb * 96u, 16u);
        if (tid < 2 * kBM) { // tile_exc[T] and tile_exc[T + 1] of row tid >> 1
            const uint64_t T = uint64_t(row0 + (tid >> 1)) * tpr + kb + (tid & 1u);
            fw_cp4(sp + kPlTE + 4 * tid, tex + 4 * T);
        }
        for (uint32_t id = tid; id < nt * 32; id += kGemmThreads) { // X: 16-byte chunks c of token t
            const uint32_t t = id >> 5, c = id & 31u, tok = tok0 + t;
            const uint32_t dst = sb + (c >> 3) * (nt * 128) + t * 128 + (((c & 7u) ^ (t & 7u)) << 4);
            const uint16_t* src = tok < batch ? it.x + uint64_t(tok) * K + kb * 256 + c * 8 : it.x;
            cp_async16(dst, src, tok < batch ? 16u : 0u);
        }
        cp_async_commit();
    };

    bool ok = true;
    if (kbeg < kend) issue(kbeg);
    for (uint32_t kb = kbeg; kb < kend && ok; ++kb) {
        const uint32_t s = kb & 1u, it_k = kb - kbeg; // it_k: this CTA's slice count so far
        const uint32_t sp = sP0 + s * kSlot, sb = sB0 + s * bbytes;
        const uint8_t* slot = smem + (sp - sbase);
        cp_async_wait<0>(); // slice kb's copies (the only group in flight)
        __syncthreads();
        // this lane's share of the exceptions of row (lane & 7) of the warp's 8: entries
        // e0 + 8 (lane >> 3) .. +7, as (position << 16) | word
        constexpr uint32_t kRowsW = kBM / kGemmWarps; // 8 rows a warp
        const uint32_t er = warp * kRowsW + (lane & (kRowsW - 1u));
        const uint32_t* te = reinterpret_cast<const uint32_t*>(slot + kPlTE) + 2 * er;
        const uint32_t e0 = te[0], e1 = te[1];
        const bool e_ok = e0 <= e1 && e1 <= it.n_exc;
        if (!e_ok && lane < kRowsW) atomicOr(p.err, 1u);
        const uint32_t ebeg = e0 + kExcRegs * (lane / kRowsW), eend = e_ok ? e1 : e0;
        uint32_t ex[kExcRegs];
#pragma unroll
        for (uint32_t i = 0; i < kExcRegs; ++i)
            ex[i] = ebeg + i < eend ? (uint32_t(__ldg(EP + ebeg + i)) << 16) | __ldg(EW + ebeg + i) : 0xFFFFFFFFu;
        // the planes of this warp's 8 tiles, read from the slot before anything waits
        uint32_t pa[kRowsW], pb[kRowsW], pc0[kRowsW], pc1[kRowsW];
#pragma unroll
        for (uint32_t i = 0; i < kRowsW; ++i) {
            const uint32_t r = warp * kRowsW + i;
            pa[i] = *reinterpret_cast<const uint32_t*>(slot + kPlA + r * 128 + 4 * lane);
            pb[i] = *reinterpret_cast<const uint32_t*>(slot + kPlB + r * 128 + 4 * lane);
            const uint32_t* cp = reinterpret_cast<const uint32_t*>(slot + kPlC + r * 96);
            pc0[i] = cp[cw0];
            pc1[i] = cp[cw1];
        }
        // the MMAs of slice kb - 1 read the A stage and B stage s ^ 1: one thread waits for
        // them, then slice kb + 1 is queued into the other slot and stage
        if (tid == 0 && it_k >= 1 && !mbar_wait(mbar, (it_k - 1) & 1u)) {
            atomicOr(p.err, 2u);
            s_abort = 1;
        }
        __syncthreads();
        if (kb + 1 < kend) issue(kb + 1);
        // decode: warp w writes rows 8w .. 8w+7, lane j its 8 weights (chunk j of the row)
#pragma unroll
        for (uint32_t i = 0; i < kRowsW; ++i) {
            const uint32_t r = warp * kRowsW + i;
            const uint4 w = fw_octet(pair_tab, pa[i], pb[i], pc0[i], pc1[i], csh);
            *reinterpret_cast<uint4*>(pA + (lane >> 3) * kAtomA + r * 128 + (((lane & 7u) ^ (r & 7u)) << 4)) = w;
        }
        __syncwarp();
#pragma unroll
        for (uint32_t i = 0; i < kExcRegs; ++i) {
            if (ex[i] != 0xFFFFFFFFu) {
                const uint32_t pos = ex[i] >> 16, j = pos >> 3;
                *reinterpret_cast<uint16_t*>(pA + (j >> 3) * kAtomA + er * 128 + (((j & 7u) ^ (er & 7u)) << 4) +
                                             2 * (pos & 7u)) = static_cast<uint16_t>(ex[i]);
            }
        }
        if (lane < kRowsW) // a tile with more than 32 exceptions: the rest, straight from memory
            for (uint32_t e = e0 + (32 / kRowsW) * kExcRegs; e < eend; ++e) {
                const uint32_t pos = __ldg(EP + e), j = pos >> 3;
                *reinterpret_cast<uint16_t*>(pA + (j >> 3) * kAtomA + er * 128 + (((j & 7u) ^ (er & 7u)) << 4) +
                                             2 * (pos & 7u)) = __ldg(EW + e);
            }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); // the stage is read by the tensor cores
        __syncthreads();
        if (s_abort) {
            ok = false;
            break;
        }
        if (tid == 0) {
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
            for (uint32_t kk = 0; kk < 16; ++kk) { // K = 16 per MMA: atom kk / 4, 32 bytes per step inside it
                const uint64_t ad = sw128_desc(sA + (kk >> 2) * kAtomA + (kk & 3u) * 32);
                const uint64_t bd = sw128_desc(sb + (kk >> 2) * (nt * 128) + (kk & 3u) * 32);
                const uint32_t acc = (it_k | kk) != 0;
                asm volatile("{\n .reg .pred p;\n setp.ne.u32 p, %4, 0;\n"
                             " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}"
                             ::"r"(tmem), "l"(ad), "l"(bd), "r"(idesc), "r"(acc) : "memory");
            }
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                         : "memory");
        }
    }
    cp_async_wait<0>();
    // The last commit covers every MMA before it.
    if (ok && kbeg < kend) {
        if (!mbar_wait(mbar, (kend - kbeg - 1) & 1u)) {
            atomicOr(p.err, 2u);
            ok = false;
        }
    }
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (ok && kbeg < kend && warp < 8) {
        // warp w reads tensor-memory lanes 32 (w % 4) .. +31 (rows of W) and columns (tokens)
        // 32 (w / 4) .. +31 of the accumulator
        const uint32_t quarter = warp & 3u, half = warp >> 2;
        const uint32_t row = row0 + quarter * 32 + lane;
        for (uint32_t cb = half * 32; cb < half * 32 + 32 && cb < nt; cb += 16) {
            uint32_t v[16];
            const uint32_t taddr = tmem + ((quarter * 32) << 16) + cb;
            asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
                         : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
                           "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
                         : "r"(taddr));
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
            for (uint32_t q = 0; q < 16; ++q) {
                const uint32_t tok = tok0 + cb + q;
                if (tok < batch) {
                    float* dst = it.y + uint64_t(tok) * rows + row;
                    if (split) atomicAdd(dst, __uint_as_float(v[q])); // Y was zeroed; parts add up
                    else *dst = __uint_as_float(v[q]);
                }
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0)
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
        // the items of one launch; K is split where the row blocks alone would not give about
        // two CTAs per SM
        int32_t k1 = k;
        uint64_t blocks = 0;
        for (uint32_t m = 0; k1 < n && m < static_cast<uint32_t>(kGemmMaxItems); ++k1) {
            if (items[k1].info.n_elems == 0) continue;
            blocks += uint64_t(items[k1].rows / kBM) * p.token_tiles;
            ++m;
        }
        const uint64_t want = 2ull * static_cast<uint64_t>(sms);
        p.n_items = 0;
        uint64_t ctas = 0;
        for (; k < k1; ++k) {
            const bs_fw_gemv_item& g = items[k];
            if (g.info.n_elems == 0) continue;
            const uint32_t tpr = g.cols / 256;
            uint32_t ksplit = blocks >= want ? 1u : static_cast<uint32_t>(std::min<uint64_t>((want + blocks - 1) / blocks, tpr));
            ksplit = std::max<uint32_t>(1u, std::min<uint32_t>(ksplit, 0xFFFFu));
            const uint32_t kper = (tpr + ksplit - 1) / ksplit;
            ksplit = (tpr + kper - 1) / kper; // no empty part
            const uint64_t c = uint64_t(g.rows / kBM) * p.token_tiles * ksplit;
            if (ctas + c >= (1ull << 31) || kper > 0xFFFFu) return BS_E_SIZE;
            if (ksplit > 1) { // the parts add into Y
                e = cudaMemsetAsync(g.d_y, 0, sizeof(float) * uint64_t(batch) * g.rows, s);
                if (e != cudaSuccess) return cuda_status(e);
            }
            FwGemmItem& it = p.item[p.n_items++];
            it.fw = static_cast<const uint8_t*>(g.d_fw);
            it.x = static_cast<const uint16_t*>(g.d_x);
            it.y = g.d_y;
            it.rows = g.rows;
            it.cols = g.cols;
            it.n_exc = static_cast<uint32_t>(g.info.n_exc);
            it.cta_begin = static_cast<uint32_t>(ctas);
            it.row_tiles = g.rows / kBM;
            it.ksplit = static_cast<uint16_t>(ksplit);
            it.kper = static_cast<uint16_t>(kper);
            std::memcpy(it.table, g.info.table, sizeof(it.table));
            ctas += c;
        }
        if (p.n_items == 0) continue;
        fw_gemm_kernel<<<static_cast<uint32_t>(ctas), kGemmThreads, kGemmSmem, s>>>(p);
        count_launch();
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_status(e);
    }
    return BS_OK;
}
