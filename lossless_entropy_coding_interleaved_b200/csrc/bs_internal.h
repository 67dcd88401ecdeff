// bs_internal.h -- definitions shared by the host planner (bs_plan.cpp) and the kernels
// (bs_kernels.cu) of libbs. Nothing here is shared with the oracle.
#pragma once

#include <cstdint>
#include <string>
#include <vector>

#include <vector_types.h>

#include "bs.h"

namespace bs {

// FORMAT.md sections 2-4
constexpr uint32_t kLanes = 32;
constexpr uint64_t kStateL = 1ull << 32;
constexpr uint32_t kHeaderBytes = 64;
constexpr uint32_t kDirEntryBytes = 144;
constexpr uint32_t kMaxNs = 12, kMaxNf = 11, kMaxRoutes = 15;

// Decode-kernel geometry: a warp decodes kChains chunks at once (two independent state
// chains per lane), and a CTA of kWarps warps covers kWarps*kChains chunks of one tensor.
// Each chunk's word stream goes through its own shared-memory ring of kRingWords 32-bit
// words, in quarters of kRingWords/4 words.
// Three CTA shapes by table size: 20 warps up to 64 KiB of tables, 16 up to 96 KiB, else 8
// (the largest tables, 160 KiB, plus 8 warps of rings fit in the 227 KiB a CTA may use).
constexpr int kChains = 2;
constexpr int kRingWords = 1024;
constexpr int kQuarterWords = kRingWords / 4;
// The rings come first in dynamic shared memory, then the tables. The largest tables
// (160 KiB) plus 8 warps of rings (64 KiB) fit the 227 KiB a CTA may use.
constexpr uint32_t ring_bytes_per_cta(int warps) { return uint32_t(warps) * kChains * kRingWords * 4; }
constexpr uint32_t kBigCtaTableBytes = 96 * 1024;
constexpr uint32_t kHugeCtaTableBytes = 64 * 1024;  // 20 warps: 160 KiB of rings + 64 KiB
inline int warps_for_tables(uint32_t table_bytes) {
    return table_bytes <= kHugeCtaTableBytes ? 20 : table_bytes <= kBigCtaTableBytes ? 16 : 8;
}

// Workspace layout: a 256-byte error block, then 256-aligned tables per RANS tensor.
constexpr uint64_t kErrBlockBytes = 256;

// One tensor of the container as parsed by the planner.
struct Tensor {
    uint32_t kind = 0, ndim = 0, log2_chunk = 0, lanes = 0, ns = 0, nf = 0, n_routes = 0;
    uint64_t n_elems = 0, n_chunks = 0, model_offset = 0, model_bytes = 0, data_offset = 0, data_bytes = 0;
    uint64_t checksum = 0, coded_bytes = 0;
    uint64_t shape[8] = {0};
    std::string name;
    std::vector<uint8_t> model; // RANS: the model section (FORMAT.md 4.3)
    uint64_t ws_offset = 0;   // RANS: byte offset of the decode tables in the workspace
    uint32_t table_bytes = 0; // RANS: bytes of s-table + f-tables (multiple of 16)
};

// ---- Decode tables (built on the host, copied to the workspace, staged in smem) ----
// s-table: 2^ns entries of 8 bytes, indexed by slot = x & (2^ns - 1):
//   .x = freq | (bias << 16)        freq = Fs[s] (<= 4096), bias = slot - cum_s(s)
//   .y = (s << 7) | (frow << 16)    s already in its output position; frow locates the
//                                   f-table row of the route that e = s & 0xFF selects:
//                                   its byte offset when nf <= 10, its word offset when
//                                   nf = 11 (see frow_field)
// f-table: (n_routes + 1) rows of 2^nf u32 entries (the last row is UNIFORM):
//   bits 0-6 fraction, bits 7-18 freq, bits 19-30 bias
inline uint32_t table_bytes_for(uint32_t ns, uint32_t nf, uint32_t n_routes) {
    return (8u << ns) + 4u * (n_routes + 1) * (1u << nf);
}
// The frow field of an s-entry for fraction row `row` (it must fit in 16 bits).
__host__ __device__ inline uint32_t frow_field(uint32_t row, uint32_t nf) {
    return nf <= 10 ? (row << (nf + 2)) : (row << nf);
}

// ---- Kernel launch parameters (passed by value, __grid_constant__) ----
struct DecodeItem {
    const uint8_t* chunk_table; // device: 16-byte chunk entries of this tensor
    const uint8_t* container;   // device: container base (chunk offsets are absolute)
    const uint4* tables;        // device: this tensor's decode tables in the workspace
    uint16_t* out;              // device: decoded words
    uint64_t n_elems;
    uint32_t cta_begin;         // first CTA of this tensor in the launch
    uint32_t tensor_index;      // for error reports
    uint32_t table_bytes;
    uint8_t log2_chunk, ns, nf, pad0;
    uint32_t pad1[2];
};
static_assert(sizeof(DecodeItem) == 64, "DecodeItem layout");

constexpr int kMaxDecodeItems = 500; // 64 B each: the parameters stay under 32 KiB
struct DecodeParams {
    uint32_t n_items;
    uint32_t total_ctas;
    unsigned long long* err; // [0]: flags, [1]: smallest (tensor << 40 | chunk) that failed
    DecodeItem item[kMaxDecodeItems];
};

struct CopyItem {
    const uint8_t* src;
    uint8_t* dst;
    uint64_t bytes;
    uint64_t blk_begin; // first 64 KiB block of this item in the launch
};
constexpr int kMaxCopyItems = 960;
constexpr uint64_t kCopyBlockBytes = 65536;
struct CopyParams {
    uint32_t n_items;
    uint32_t pad;
    uint64_t total_blocks;
    CopyItem item[kMaxCopyItems];
};

// ---- Encoder (bs_encode.cpp, bs_encode_kernels.cu) ----
// Encode tables of one tensor, in u32 words:
//   [0, 512)                s-table: qs | (cum_s << 16)
//   [512, 512 + 128*rows)   fraction rows (the last one UNIFORM): qf | (cum_f << 16)
//   [.., + 64)              route: 256 bytes, row index per exponent
inline uint32_t enc_table_words(uint32_t n_routes) { return 512 + 128 * (n_routes + 1) + 64; }

struct EncItem {
    const uint16_t* in;         // device: original words
    const uint32_t* tables;     // device: encode tables (layout above)
    uint32_t* n_words;          // device: words per chunk (count pass writes, write pass checks)
    const uint64_t* chunk_off;  // device: absolute container offset per chunk (write pass)
    uint64_t n_elems;
    uint32_t cta_begin;
    uint32_t table_words;
    uint16_t pad_word;
    uint8_t log2_chunk, ns, nf, n_routes, pad0, pad1;
};
static_assert(sizeof(EncItem) == 56, "EncItem layout");

constexpr int kEncWarps = 8;
constexpr int kMaxEncItems = 512;
struct EncParams {
    uint32_t n_items;
    uint32_t total_ctas;
    uint32_t write;             // 0: count words per chunk; 1: write states and words
    uint32_t pad;
    uint8_t* container;         // device (write pass)
    unsigned int* err;          // device: set when the write pass disagrees with the count pass
    EncItem item[kMaxEncItems];
};

constexpr uint32_t kHistBins = 512 + 256 * 128; // s counts, then (exponent, fraction) counts
int launch_histogram(const uint16_t* in, uint64_t n, unsigned long long* d_hist, void* stream);
int launch_encode(const EncParams& p, void* stream);

// Keeps the cudaError_t behind a BS_E_CUDA for bs_last_cuda_error (bs_plan.cpp).
void record_cuda_error(int e);
// Counts kernel launches for bs_launch_counter (bs_plan.cpp).
void count_launch();

// Kernel launchers (bs_kernels.cu). They return a cudaError_t as int.
int launch_decode(const DecodeParams& p, int warps, bool default_precision, uint32_t smem_bytes, void* stream);
int launch_copy(const CopyParams& p, void* stream);
int launch_checksum(const void* data, uint64_t n, int raw_bytes, unsigned long long* d_sum, void* stream);
int max_dynamic_smem();

} // namespace bs
