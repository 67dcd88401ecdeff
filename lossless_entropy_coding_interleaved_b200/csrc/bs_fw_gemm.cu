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
//  * A CTA owns 128 rows of W and up to 64 tokens. For each 256-wide slice of K (one FW tile of
//    each row) its 8 warps decode the 128 tiles into the A stage in shared memory (BF16, K-major,
//    the 128-byte swizzle of the MMA's canonical layout), patch in the slice's exceptions, and
//    copy the tokens' X slice into the B stage with cp.async (tokens past the batch read as 0).
//  * One thread issues the slice's 16 MMAs (M = 128, N = tokens, K = 16 each) into a 128 x N
//    FP32 accumulator in tensor memory and commits them to the stage's mbarrier; the warps
//    meanwhile fill the other stage. A stage is refilled only after its MMAs completed.
//  * The epilogue reads the accumulator with tcgen05.ld (warp w reads lanes 32(w % 4)..+31,
//    that is 32 rows of W) and writes Y[token][row] in FP32, 128 contiguous bytes per warp and
//    token.
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

constexpr int kGemmWarps = 8;
constexpr int kGemmThreads = kGemmWarps * 32;
constexpr uint32_t kBM = 128;                     // rows of W per CTA: the MMA's M
constexpr uint32_t kMaxNt = 64;                   // tokens per CTA: the MMA's N (a multiple of 16)
constexpr uint32_t kAtomA = kBM * 128;            // one 64-wide K atom of the A stage (16 KiB)
constexpr uint32_t kStageA = 4 * kAtomA;          // 128 rows x 256 K x 2 B
constexpr uint32_t kStageB = 4 * kMaxNt * 128;    // up to 64 tokens x 256 K x 2 B
constexpr uint32_t kHead = 2048;                  // pair table, mbarriers, tensor-memory address
constexpr uint32_t kGemmSmem = kHead + 1024 + 2 * (kStageA + kStageB); // + slack to align stages to 1 KiB
constexpr uint32_t kTmemCols = 64;
constexpr uint32_t kSpinLimit = 1u << 24;
constexpr int kGemmMaxItems = 320;

struct FwGemmItem {
    const uint8_t* fw;  // device: the layout of W
    const uint16_t* x;  // device: BF16 [batch][cols]
    float* y;           // device: FP32 [batch][rows]
    uint32_t rows, cols;
    uint32_t n_exc;
    uint32_t cta_begin; // first CTA of this item in the launch
    uint32_t row_tiles; // rows / 128
    uint32_t pad;
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
    const uint32_t mbar0 = sbase + 1024, mbar1 = sbase + 1032;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + 1040);
    const uint32_t stage0 = (sbase + kHead + 1023u) & ~1023u; // 1 KiB aligned, as the swizzle needs
    if (tid == 0) {
        mbar_init(mbar0, 1);
        mbar_init(mbar1, 1);
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
    const uint32_t local = blockIdx.x - it.cta_begin;
    const uint32_t row0 = (local % it.row_tiles) * kBM;
    const uint32_t nt = p.nt, tok0 = (local / it.row_tiles) * nt, batch = p.batch;
    const uint64_t n_tiles = uint64_t(rows) * tpr;
    const FwOffsets o = fw_offsets(n_tiles, it.n_exc);
    const uint8_t* fw = it.fw;
    const uint32_t* tile_exc = reinterpret_cast<const uint32_t*>(fw + o.tile_exc);
    const uint8_t* EP = fw + o.exc_pos;
    const uint16_t* EW = reinterpret_cast<const uint16_t*>(fw + o.exc_word);
    const uint32_t cw0 = (3u * lane) >> 2, csh = (24u * lane) & 31u, cw1 = csh > 8 ? cw0 + 1 : cw0;
    // M = 128, N = nt, BF16 x BF16 -> FP32, both operands K-major
    const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((nt >> 3) << 17) | ((kBM >> 4) << 24);
    const uint32_t stage_bytes = kStageA + 4 * nt * 128;

    bool ok = true;
    for (uint32_t kb = 0; kb < tpr && ok; ++kb) {
        const uint32_t s = kb & 1u;
        const uint32_t sa = stage0 + s * stage_bytes, sb = sa + kStageA; // shared addresses
        uint8_t* pa = smem + (sa - sbase);
        if (kb >= 2 && !mbar_wait(s ? mbar1 : mbar0, ((kb - 2) >> 1) & 1u)) { // the MMAs of kb - 2 read this stage
            atomicOr(p.err, 2u);
            s_abort = 1;
        }
        __syncthreads();
        if (s_abort) {
            ok = false;
            break;
        }
        // X slice: nt tokens x 256 K, 16-byte chunks c = 0..31 of each token, swizzled
        for (uint32_t id = tid; id < nt * 32; id += kGemmThreads) {
            const uint32_t t = id >> 5, c = id & 31u, tok = tok0 + t;
            const uint32_t dst = sb + (c >> 3) * (nt * 128) + t * 128 + (((c & 7u) ^ (t & 7u)) << 4);
            const uint16_t* src = tok < batch ? it.x + uint64_t(tok) * K + kb * 256 + c * 8 : it.x;
            cp_async16(dst, src, tok < batch ? 16u : 0u);
        }
        cp_async_commit();
        // W slice: warp w decodes rows 16w .. 16w+15, lane j writes its 8 weights (chunk j)
        for (uint32_t i = 0; i < kBM / kGemmWarps; ++i) {
            const uint32_t r = warp * (kBM / kGemmWarps) + i;
            const uint64_t T = uint64_t(row0 + r) * tpr + kb;
            const uint32_t a = __ldg(reinterpret_cast<const uint32_t*>(fw + o.a + T * 128) + lane);
            const uint32_t b = __ldg(reinterpret_cast<const uint32_t*>(fw + o.b + T * 128) + lane);
            const uint32_t* cp = reinterpret_cast<const uint32_t*>(fw + o.c + T * 96);
            const uint4 w = fw_octet(pair_tab, a, b, __ldg(cp + cw0), __ldg(cp + cw1), csh);
            *reinterpret_cast<uint4*>(pa + (lane >> 3) * kAtomA + r * 128 + (((lane & 7u) ^ (r & 7u)) << 4)) = w;
        }
        __syncwarp();
        for (uint32_t i = 0; i < kBM / kGemmWarps; ++i) { // the exceptions of those tiles
            const uint32_t r = warp * (kBM / kGemmWarps) + i;
            const uint64_t T = uint64_t(row0 + r) * tpr + kb;
            const uint32_t e0 = __ldg(tile_exc + T), e1 = __ldg(tile_exc + T + 1);
            if (e0 > e1 || e1 > it.n_exc) {
                if (lane == 0) atomicOr(p.err, 1u);
                continue;
            }
            for (uint32_t e = e0 + lane; e < e1; e += 32) {
                const uint32_t pos = __ldg(EP + e), j = pos >> 3;
                *reinterpret_cast<uint16_t*>(pa + (j >> 3) * kAtomA + r * 128 + (((j & 7u) ^ (r & 7u)) << 4) + 2 * (pos & 7u)) =
                    __ldg(EW + e);
            }
        }
        cp_async_wait<0>();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); // the stage is read by the tensor cores
        __syncthreads();
        if (tid == 0) {
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
            for (uint32_t kk = 0; kk < 16; ++kk) { // K = 16 per MMA: atom kk / 4, 32 bytes per step inside it
                const uint64_t ad = sw128_desc(sa + (kk >> 2) * kAtomA + (kk & 3u) * 32);
                const uint64_t bd = sw128_desc(sb + (kk >> 2) * (nt * 128) + (kk & 3u) * 32);
                const uint32_t acc = (kb | kk) != 0;
                asm volatile("{\n .reg .pred p;\n setp.ne.u32 p, %4, 0;\n"
                             " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}"
                             ::"r"(tmem), "l"(ad), "l"(bd), "r"(idesc), "r"(acc) : "memory");
            }
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                         ::"r"(s ? mbar1 : mbar0) : "memory");
        }
    }
    // The last commit covers every MMA before it.
    if (ok && tpr > 0) {
        const uint32_t kl = tpr - 1;
        if (!mbar_wait((kl & 1u) ? mbar1 : mbar0, (kl >> 1) & 1u)) {
            atomicOr(p.err, 2u);
            ok = false;
        }
    }
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (ok && tpr > 0) {
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
                if (tok < batch) it.y[uint64_t(tok) * rows + row] = __uint_as_float(v[q]);
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
    int32_t k = 0;
    while (k < n) {
        p.n_items = 0;
        uint64_t ctas = 0;
        for (; k < n && p.n_items < static_cast<uint32_t>(kGemmMaxItems); ++k) {
            const bs_fw_gemv_item& g = items[k];
            if (g.info.n_elems == 0) continue;
            const uint64_t c = uint64_t(g.rows / kBM) * p.token_tiles;
            if (ctas + c >= (1ull << 31)) break;
            FwGemmItem& it = p.item[p.n_items++];
            it.fw = static_cast<const uint8_t*>(g.d_fw);
            it.x = static_cast<const uint16_t*>(g.d_x);
            it.y = g.d_y;
            it.rows = g.rows;
            it.cols = g.cols;
            it.n_exc = static_cast<uint32_t>(g.info.n_exc);
            it.cta_begin = static_cast<uint32_t>(ctas);
            it.row_tiles = g.rows / kBM;
            it.pad = 0;
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
