// bs_host.h -- host-side pieces of libbs shared by the planner (bs_plan.cpp) and the layer
// streamer (bs_stream.cpp): container parsing, the workspace image, and the batching of
// decode and copy work into kernel launches.
#pragma once

#include <cstdint>
#include <memory>
#include <vector>

#include "bs_internal.h"

namespace bs {

inline uint64_t up256(uint64_t v) { return (v + 255) & ~uint64_t(255); }

// ---- Validation (bs_validate.cpp): one copy of each rule for every host path ----
struct HeaderInfo {
    uint32_t n_tensors = 0;
    uint64_t dir = 0, names = 0, names_bytes = 0;
};
// The 64-byte header of a container of len bytes: magic, version, sizes, reserved field,
// 16-byte aligned directory and names inside the container. BS_E_SIZE if total_bytes != len.
bs_status check_header(const uint8_t* hdr, uint64_t len, HeaderInfo* h);
// One 144-byte directory entry: fills t's directory fields and the name's place in the names
// section, and checks every field that needs no other section (kind, shape, chunking,
// precisions, section bounds and alignment).
bs_status check_entry(const uint8_t* d, uint64_t len, const HeaderInfo& h, Tensor* t, uint32_t* name_off,
                      uint32_t* name_len);
// The model section (t->model_bytes bytes at m) of a coded entry that passed check_entry:
// ascending symbols or pairs, nonzero frequencies, table sums, routes. Sets t->table_bytes
// and, for JOINT, t->joint_compact.
bs_status check_model(const uint8_t* m, Tensor* t);
// The chunk table (16 * n_chunks bytes at ct): aligned payloads inside the container, zero
// reserved words. Sets t->coded_bytes.
bs_status check_chunk_table(const uint8_t* ct, uint64_t len, Tensor* t);
// Expand the model (at m) of a coded tensor that passed check_model into its decode tables,
// t.table_bytes bytes at dst.
void build_tables(const Tensor& t, const uint8_t* m, uint8_t* dst);
// Dynamic shared memory of a decode launch of this mode and shape (s_region: the largest
// s-table region of a factored launch).
uint32_t decode_smem_bytes(DecodeMode mode, uint32_t warps, uint32_t chains, uint32_t s_region);

// Parse and validate a container held in host memory.
bs_status parse_host_container(const uint8_t* h, uint64_t len, std::vector<Tensor>& out);

// Bytes of the decode workspace: the error block, then each RANS tensor's tables.
uint64_t workspace_bytes_for(const std::vector<Tensor>& ts);

// Assign each RANS tensor its ws_offset and write the workspace image. The image holds
// the error block (no flag set, first_bad = all ones) and the decode tables.
// Returns BS_E_UNSUPPORTED when a tensor's tables and rings exceed the device's shared
// memory per block.
bs_status build_workspace(std::vector<Tensor>& ts, std::vector<uint8_t>& image);

// Bins decode work by kernel instance (factored at the default precisions or any other,
// JOINT at nj = 13 or any other), and
// verbatim copies into one
// copy list. It launches a bin when the bin is full,
// and launches every bin on flush().
// The decode kernel instance (and CTA shape) of a coded tensor.
inline DecodeMode decode_mode_of(const Tensor& t) {
    if (t.kind == BS_KIND_JOINT)
        return t.joint_compact ? DecodeMode::JointCompact : t.ns == kDefaultNj ? DecodeMode::Joint : DecodeMode::JointGeneric;
    return is_default_precision(t.ns, t.nh) ? DecodeMode::Default : DecodeMode::Generic;
}

class DecodeBatch {
  public:
    // d_err: the workspace's error block.
    explicit DecodeBatch(unsigned long long* d_err) : err_(d_err) {}
    bs_status init(); // allocates the parameter blocks (about 220 KB of host memory)
    // Queue tensor t, whose chunk offsets are relative to d_container, for decoding into d_out.
    // Launches on `stream` when a bin fills up. [begin, begin + count) selects a range of the
    // tensor's elements (bytes for RAW); for coded kinds begin is a multiple of the chunk size
    // and the range ends on a chunk boundary or at the tensor's end (checked by the caller).
    bs_status add(const Tensor& t, uint32_t tensor_index, const uint8_t* d_container, const uint8_t* d_ws,
                  void* d_out, void* stream, uint64_t begin = 0, uint64_t count = ~0ull);
    bs_status flush(void* stream);

  private:
    struct Bin {
        std::unique_ptr<DecodeParams> p;
        DecodeMode mode = DecodeMode::Default;
        uint32_t s_region = 0;  // largest s-table region of the queued tensors
        uint64_t chunks = 0;    // chunks queued; the CTA shape is chosen at flush
    };
    bs_status flush_bin(Bin& b, void* stream);
    bs_status flush_copy(void* stream);
    unsigned long long* err_;
    uint32_t sms_ = 148;
    Bin bins_[kDecodeModes];
    std::unique_ptr<CopyParams> cp_;
};

// bs_tensor_info for tensor t; the name points into t.
void fill_tensor_info(const Tensor& t, bs_tensor_info* o);

// Records e for bs_last_cuda_error and returns BS_E_CUDA.
bs_status cuda_status(int e);

} // namespace bs
