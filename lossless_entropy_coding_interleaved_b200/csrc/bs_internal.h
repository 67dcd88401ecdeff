// bs_internal.h -- definitions shared by the host planner (bs_plan.cpp) and the kernels
// (bs_kernels.cu) of libbs. Nothing here is shared with the oracle.
#pragma once

#include <cstdint>
#include <string>
#include <vector>

#include <vector_types.h>

#include "bs.h"

namespace bs {

// The BF16RANS container, version 2: 32 lanes per chunk, 32-bit states in [2^16, 2^32),
// 64-byte header, 144-byte directory entries
constexpr uint32_t kFormatVersion = 2;
constexpr uint32_t kLanes = 32;
constexpr uint32_t kStateL = 1u << 16;
constexpr uint32_t kHeaderBytes = 64;
constexpr uint32_t kDirEntryBytes = 144;
constexpr uint32_t kMaxNs = 12, kMinNh = 3, kMaxNh = 5, kMaxPrecision = 16, kMaxRoutes = 15;
// The JOINT kind: one table over the 4096 pairs j = (s << 3) | h,
// precision nj. Its decode table (2^nj entries of 8 bytes) sits at offset 0 of shared
// memory, and the rings follow at kJointRegion.
constexpr uint32_t kJointPairs = 4096, kMinNj = 8, kMaxNj = 13;
constexpr uint32_t kJointRegion = 8u << kMaxNj;
// A JOINT tensor whose frequencies are all below 256 (every large tensor of normally
// distributed weights) gets 4-byte slot entries instead: the word j << 4 in the low half
// (its low nibble zero), the slot's rank in byte 2 and F in byte 3.
// A random 4-byte gather of 32 lanes costs about 3.5 shared-memory wavefronts against about
// 6 for the 8-byte one. The table region is then at most 32 KiB.
constexpr uint32_t kCompactMaxF = 255;
constexpr uint32_t kJoint4Region = 4u << kMaxNj;
inline uint32_t joint4_table_bytes(uint32_t nj) { return 4u << nj; }
inline bool is_coded(uint32_t kind) { return kind == BS_KIND_RANS || kind == BS_KIND_JOINT; }
// joint table entry for slot (cum(j) + k): .x = F | (word << 16) with word = j << 4, .y = k
inline uint32_t joint_table_bytes(uint32_t nj) { return 8u << nj; }
// Bytes of a chunk payload: 32 start states, the nibble words when stored, the 16-bit
// words, padded to 16.
inline uint64_t payload_bytes(uint64_t n_c, uint32_t n_words, bool nib_stored) {
    const uint64_t blocks = (n_c + 255) / 256;
    return (128 + (nib_stored ? 128 * blocks : 0) + 2ull * n_words + 15) & ~uint64_t(15);
}

// Decode-kernel geometry: a warp decodes `chains` chunks at once (independent state chains
// per lane), and a CTA of `warps` warps covers warps*chains chunks of one tensor. Kind RANS
// at the default precisions uses 24 warps of 2 chains; kind JOINT at nj = 13 uses 32 warps of
// 2 with 4-byte table entries (kWarpsJoint4, bs_joint4.cu) and 28 warps of 2 with 8-byte ones
// (kWarpsJoint below); the other precisions use 20 warps of 2 (ns = 12 tables leave room for
// 40 rings).
// Each chunk's 16-bit word stream goes through its own shared-memory ring of kRingBytes,
// in quarters of kQuarterBytes (one 16-byte cp.async per lane fills a quarter), and its
// nibble words through a ring of kNibRingBlocks blocks (128 bytes each).
constexpr int kWarpsDefault = 24, kChainsDefault = 2, kWarpsGeneric = 20, kChainsGeneric = 2;
// JOINT at the default precision (nj = 13) with 8-byte entries (a pair frequency above 255):
// the table takes the first 64 KiB, then 56 rings of each kind (204 KiB in all). 28 warps
// hold 72 registers a thread, the most that fits.
constexpr int kWarpsJoint = 28, kChainsJoint = 2;
inline bool is_default_precision(uint32_t ns, uint32_t nh) { return ns == 11 && nh == 5; }
inline int warps_for(uint32_t ns, uint32_t nh) { return is_default_precision(ns, nh) ? kWarpsDefault : kWarpsGeneric; }
inline int chains_for(uint32_t ns, uint32_t nh) { return is_default_precision(ns, nh) ? kChainsDefault : kChainsGeneric; }
inline uint64_t chunks_per_cta(uint32_t ns, uint32_t nh) { return uint64_t(warps_for(ns, nh)) * chains_for(ns, nh); }
// Warps per CTA for one launch of `chunks` chunks: the largest shape when the grid covers the
// SMs several times over; fewer warps when a small launch (one layer, one tensor) would
// otherwise leave SMs idle, so that its CTAs spread over every SM in one wave.
constexpr uint32_t kMinWarps = 4;
inline uint32_t launch_warps(uint64_t chunks, uint32_t max_warps, uint32_t chains, uint32_t sms) {
    const uint64_t per_sm = (chunks + sms - 1) / sms;
    const uint64_t w = (per_sm + chains - 1) / chains;
    return static_cast<uint32_t>(w < kMinWarps ? kMinWarps : w > max_warps ? max_warps : w);
}
constexpr uint32_t kRingBytes = 2048;
constexpr uint32_t kQuarterBytes = kRingBytes / 4;
static_assert(kQuarterBytes == 32 * 16, "one cp.async of 16 bytes per lane fills a quarter");
constexpr uint32_t kNibRingBlocks = 4;
constexpr uint32_t kNibRingBytes = kNibRingBlocks * 128;
// Shared memory of a CTA:
//   [0, kHRegion)                 fraction rows, one copy per lane (row r, slot j, lane c at
//                                 byte ((r << nh) + j) * 128 + 4c): conflict-free lookups
//   [kHRegion, + 8 << ns)         s-table (its size rounded up to 2 KiB)
//   then the word rings (kRingBytes each, so each starts at a multiple of kRingBytes) and
//   the nibble rings
// The fraction region is reserved at its largest (16 rows of 2^5 slots) so that the s-table
// sits at a constant offset. Default precisions: 80 KiB of tables + 144 KiB of rings for 48
// chains; ns = 12: 96 KiB + 120 KiB for 40 chains.
constexpr uint32_t kHRegion = 16u * 32u * 128u;
__host__ __device__ inline uint32_t s_region_bytes(uint32_t ns) { return ((8u << ns) + kRingBytes - 1) & ~(kRingBytes - 1); }
inline uint32_t smem_bytes_for(uint32_t ns, uint32_t nh) {
    return kHRegion + s_region_bytes(ns) + uint32_t(chunks_per_cta(ns, nh)) * (kRingBytes + kNibRingBytes);
}
inline uint32_t smem_bytes_for(uint32_t ns, uint32_t warps, uint32_t chains) {
    return kHRegion + s_region_bytes(ns) + warps * chains * (kRingBytes + kNibRingBytes);
}
// JOINT: the table region (kJointRegion, the largest table), then the same rings.
inline uint32_t joint_smem_bytes(uint32_t warps, uint32_t chains) {
    return kJointRegion + warps * chains * (kRingBytes + kNibRingBytes);
}

inline uint32_t joint4_smem_bytes(uint32_t warps, uint32_t chains) {
    return kJoint4Region + warps * chains * (kRingBytes + kNibRingBytes);
}

// Workspace layout: a 256-byte error block, then 256-aligned tables per RANS tensor.
constexpr uint64_t kErrBlockBytes = 256;

// One tensor of the container as parsed by the planner.
struct Tensor {
    uint32_t kind = 0, ndim = 0, log2_chunk = 0, lanes = 0, ns = 0, nh = 0, n_routes = 0, nib_mode = 0;
    uint64_t n_elems = 0, n_chunks = 0, model_offset = 0, model_bytes = 0, data_offset = 0, data_bytes = 0;
    uint64_t checksum = 0, coded_bytes = 0;
    uint64_t shape[8] = {0};
    std::string name;
    std::vector<uint8_t> model; // coded kinds: the model section as stored
    uint32_t joint_compact = 0; // JOINT: 4-byte slot entries (every frequency <= kCompactMaxF)
    uint64_t ws_offset = 0;   // RANS: byte offset of the decode tables in the workspace
    uint32_t table_bytes = 0; // RANS: bytes of s-table + compact fraction rows (multiple of 16)
};

// ---- Decode tables (built on the host, copied to the workspace, staged in smem) ----
// s-table: 2^ns entries of 8 bytes, indexed by js, the high ns bits of the P-bit slot:
//   .x = Fs | (bs << 16)            Fs = Fs[s] (<= 8192), bs = js - cum_s(s)
//   .y = (s << 7) | (frow << 16)    s already in its output position; frow = the byte
//                                   offset in shared memory of the fraction row that
//                                   e = s & 0xFF selects: row * (2^nh * 128)
// fraction rows (compact in the workspace, one copy per lane in shared memory):
//   (n_routes + 1) rows of 2^nh u32 entries (the last row is UNIFORM), indexed by jh:
//   bits 4-6 h, bits 16-23 Fh, bits 24-31 bh = jh - cum_h(h); bits 0-3 and 7-15 are zero,
//   so (s << 7) | (h << 4) is one bitwise select of the two entries
inline uint32_t table_bytes_for(uint32_t ns, uint32_t nh, uint32_t n_routes) {
    return (8u << ns) + 4u * (n_routes + 1) * (1u << nh);
}
__host__ __device__ inline uint32_t frow_field(uint32_t row, uint32_t nh) { return row << (nh + 7); }
__host__ __device__ inline uint32_t h_entry(uint32_t h, uint32_t Fh, uint32_t bh) {
    return (h << 4) | (Fh << 16) | (bh << 24);
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
    uint8_t log2_chunk, ns, nh, n_routes;
    uint8_t nib_mode, pad0[3];
    uint32_t chunk_base;        // a range of a tensor: its first chunk (error reports add it)
};
static_assert(sizeof(DecodeItem) == 64, "DecodeItem layout");

constexpr int kMaxDecodeItems = 500; // 64 B each: the parameters stay under 32 KiB
struct DecodeParams {
    uint32_t n_items;
    uint32_t total_ctas;
    unsigned long long* err; // [0]: flags, [1]: smallest (tensor << 40 | chunk) that failed
    // Multipliers the decode loop uses in multiply-adds. Read from the parameters, they stay
    // opaque to the compiler, so those steps run as IMAD on the FMA pipe (which has spare
    // issue slots) instead of becoming shifts on the integer ALU pipe, the kernel's bound.
    uint32_t mul2 = 2, mul65536 = 65536;
    uint32_t warps = 0; // warps per CTA of this launch (at most the kernel's WARPS)
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
//   [512, 512 + 8*rows)     fraction rows over h (the last one UNIFORM): qh | (cum_h << 16)
//   [.., + 64)              route: 256 bytes, row index per exponent
inline uint32_t enc_table_words(uint32_t n_routes) { return 512 + 8 * (n_routes + 1) + 64; }
// JOINT encode table: Fj | (cum << 16) per pair j
constexpr uint32_t kEncJointWords = 4096;
constexpr uint32_t kEncTableWordsMax = kEncJointWords; // larger than enc_table_words(kMaxRoutes)

struct EncItem {
    const uint16_t* in;         // device: original words
    const uint32_t* tables;     // device: encode tables (layout above)
    uint32_t* n_words;          // device: words per chunk (count pass writes, write pass checks)
    const uint64_t* chunk_off;  // device: absolute container offset per chunk (write pass)
    uint64_t n_elems;
    uint32_t cta_begin;
    uint32_t table_words;
    uint16_t pad_word;
    uint8_t log2_chunk, ns, nh, n_routes, nib_stored, joint; // JOINT: ns = nj, nh = n_routes = 0
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

// (s, h) pair counts (j = w >> 4, from which the s and (exponent, h) counts follow), then
// the low-nibble counts
constexpr uint32_t kHistBins = 4096 + 16;
int launch_histogram(const uint16_t* in, uint64_t n, unsigned long long* d_hist, void* stream);
int launch_encode(const EncParams& p, void* stream);

// Keeps the cudaError_t behind a BS_E_CUDA for bs_last_cuda_error (bs_plan.cpp).
void record_cuda_error(int e);
// Counts kernel launches for bs_launch_counter (bs_plan.cpp).
void count_launch();

// Kernel launchers (bs_kernels.cu). They return a cudaError_t as int.
// Which decode_kernel instance a launch uses: the default precisions (ns 11, nh 5), any
// other factored precisions, or the JOINT kind.
// JOINT at nj = 13 (the default) has a compile-time instance; other nj use a generic one.
// JointCompact: JOINT with 4-byte slot entries, any nj.
enum class DecodeMode { Default = 0, Generic = 1, Joint = 2, JointGeneric = 3, JointCompact = 4 };
constexpr int kDecodeModes = 5;
// JOINT with 4-byte entries: 32 warps of 2 chunks at 64 registers a thread; the 32 KiB table
// and 64 rings of each kind take 192 KiB of shared memory.
constexpr int kWarpsJoint4 = 32, kChainsJoint4 = 2;
constexpr uint32_t kDefaultNj = 13;
// The largest CTA shape of each mode (small launches take fewer warps, see launch_warps).
inline uint32_t max_warps_of(DecodeMode m) {
    return m == DecodeMode::Default ? kWarpsDefault : m == DecodeMode::Joint ? kWarpsJoint
         : m == DecodeMode::JointCompact ? kWarpsJoint4 : kWarpsGeneric;
}
inline uint32_t chains_of(DecodeMode m) {
    return m == DecodeMode::Default ? kChainsDefault : m == DecodeMode::Joint ? kChainsJoint
         : m == DecodeMode::JointCompact ? kChainsJoint4 : kChainsGeneric;
}
int launch_decode(const DecodeParams& p, DecodeMode mode, uint32_t smem_bytes, void* stream);
int launch_decode_joint4(const DecodeParams& p, uint32_t smem_bytes, void* stream); // bs_joint4.cu
int launch_copy(const CopyParams& p, void* stream);
int launch_checksum(const void* data, uint64_t n, int raw_bytes, unsigned long long* d_sum, void* stream);
int max_dynamic_smem();

} // namespace bs
