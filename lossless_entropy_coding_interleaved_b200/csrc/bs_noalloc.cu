// bs_noalloc.cu -- bs_decode_tensor_noalloc: decode one tensor without any device
// memory from the caller beyond the container and the output.
//
// Who needs this: code that cannot call cudaMalloc or ask an allocator for a workspace.
// Examples are a plugin running inside another runtime whose allocator owns every byte of
// device memory, or a callback on a path where an allocation would synchronise the device
// or is forbidden. Such callers still hand in the container and the output buffer. The
// decode tables and the error block live in the static device array below instead of a
// caller workspace.
//
// The array is file-scope device memory: every GPU that loads libbs holds it until the
// process exits. Host code must not pass the symbol itself to a kernel, because on the host
// it is only a stand-in. The device address is looked up once per device with
// cudaGetSymbolAddress, on the first call made with that device current.
//
// The tensor is validated in place in the caller's host copy by the same rules as bs_plan
// (bs_validate.cpp), and its tables are built by the same builder into a static host image,
// which one cudaMemcpyAsync puts into the array. So the two entry points agree on what a
// valid container is and decode from identical tables.
#include <cuda_runtime.h>

#include <atomic>
#include <cstring>
#include <mutex>

#include "bs_host.h"

namespace bs {

// Largest decode tables the array holds: the JOINT table at nj = 13 with 8-byte entries
// (64 KiB), which is larger than any other (its 4-byte form takes 32 KiB; the factored
// s-table at ns = 12 takes 32 KiB plus 16 compact fraction rows of 2^5 entries, 2 KiB). That
// is every tensor a valid container can hold; larger tables would get BS_E_SIZE.
constexpr uint32_t kNoAllocFactoredBytes = (8u << kMaxNs) + 4u * (kMaxRoutes + 1) * (1u << kMaxNh);
constexpr uint32_t kNoAllocTableBytes = (8u << kMaxNj) > kNoAllocFactoredBytes ? (8u << kMaxNj) : kNoAllocFactoredBytes;
constexpr uint32_t kNoAllocBytes = 256 + kNoAllocTableBytes; // error block, then tables

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_addr_mutex;
unsigned char* g_addr[kMaxDevices] = {nullptr};

// The host image of the array's contents (error block, then tables), built under g_image_mutex
// and copied in with one cudaMemcpyAsync. A static buffer: no host allocation either.
std::mutex g_image_mutex;
alignas(256) unsigned char g_image[kNoAllocBytes];

// Device address of g_noalloc_scratch for the current device (looked up once per device).
cudaError_t scratch_address(unsigned char** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_addr_mutex);
    if (!g_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_addr[dev] = static_cast<unsigned char*>(p);
    }
    *out = g_addr[dev];
    return cudaSuccess;
}

bs_status cuda_error(cudaError_t e) {
    record_cuda_error(e);
    return BS_E_CUDA;
}

} // namespace

} // namespace bs

using namespace bs;

extern "C" bs_status bs_decode_tensor_noalloc(const void* h_container_v, size_t len, const void* d_container_v,
                                              int32_t idx, void* d_out, size_t out_bytes, void* stream_v) {
    const uint8_t* b = static_cast<const uint8_t*>(h_container_v);
    const uint8_t* d_container = static_cast<const uint8_t*>(d_container_v);
    cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
    if (!b || !d_container || idx < 0) return BS_E_ARG;
    if (reinterpret_cast<uintptr_t>(d_container) & 15u) return BS_E_ARG;
    // --- validate the header and this tensor in place, by bs_plan's rules ---
    HeaderInfo h;
    bs_status st = check_header(b, len, &h);
    if (st != BS_OK) return st;
    if (static_cast<uint32_t>(idx) >= h.n_tensors) return BS_E_ARG;
    Tensor t; // its name and model stay empty: nothing is allocated
    uint32_t name_off = 0, name_len = 0;
    st = check_entry(b + h.dir + uint64_t(kDirEntryBytes) * idx, len, h, &t, &name_off, &name_len);
    if (st != BS_OK) return st;
    const uint64_t want = t.kind == BS_KIND_RAW ? t.n_elems : 2 * t.n_elems;
    if (out_bytes != want) return BS_E_SIZE;
    if (want && (!d_out || (reinterpret_cast<uintptr_t>(d_out) & 15u))) return BS_E_ARG;

    if (!is_coded(t.kind)) { // verbatim: no scratch needed, the copy kernel does it
        if (want == 0) return BS_OK;
        CopyParams cp;
        cp.n_items = 1;
        cp.total_blocks = (want + kCopyBlockBytes - 1) / kCopyBlockBytes;
        cp.item[0] = CopyItem{d_container + t.data_offset, static_cast<uint8_t*>(d_out), want, 0};
        int e = launch_copy(cp, stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
        return e ? cuda_error(static_cast<cudaError_t>(e)) : BS_OK;
    }
    const uint8_t* model = b + t.model_offset;
    if ((st = check_model(model, &t)) != BS_OK) return st;
    if ((st = check_chunk_table(b + t.data_offset, len, &t)) != BS_OK) return st;
    if (t.table_bytes > kNoAllocTableBytes) return BS_E_SIZE; // larger than the static array holds

    // --- set-up: the array's device address on this device ---
    unsigned char* scratch = nullptr;
    cudaError_t ce = scratch_address(&scratch);
    if (ce != cudaSuccess) return cuda_error(ce);
    // The array keeps the previous call's bytes: its error block (flags = 0, first_bad = all
    // ones) and the tables are rewritten whole. A copy from pageable host memory returns once
    // the image is staged, so the image is free again when the call returns.
    {
        std::lock_guard<std::mutex> lock(g_image_mutex);
        std::memset(g_image, 0, 256);
        std::memset(g_image + 8, 0xFF, 8);
        build_tables(t, model, g_image + 256);
        ce = cudaMemcpyAsync(scratch, g_image, 256 + t.table_bytes, cudaMemcpyHostToDevice, stream);
    }
    if (ce != cudaSuccess) return cuda_error(ce);

    // --- the decode kernel of bs_decode_tensor, with its tables and error block in the array ---
    DecodeParams p; // about 31 KiB of launch parameters, on the stack (no heap use)
    p.n_items = 1;
    const DecodeMode mode = decode_mode_of(t);
    const uint32_t chains = chains_of(mode);
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        sms = 148;
    p.warps = launch_warps(t.n_chunks, max_warps_of(mode), chains, static_cast<uint32_t>(sms));
    const uint64_t per_cta = uint64_t(p.warps) * chains;
    p.total_ctas = static_cast<uint32_t>((t.n_chunks + per_cta - 1) / per_cta);
    p.err = reinterpret_cast<unsigned long long*>(scratch);
    DecodeItem& it = p.item[0];
    std::memset(&it, 0, sizeof(it));
    it.chunk_table = d_container + t.data_offset;
    it.container = d_container;
    it.tables = reinterpret_cast<const uint4*>(scratch + 256);
    it.out = static_cast<uint16_t*>(d_out);
    it.n_elems = t.n_elems;
    it.cta_begin = 0;
    it.tensor_index = static_cast<uint32_t>(idx);
    it.table_bytes = t.table_bytes;
    it.log2_chunk = static_cast<uint8_t>(t.log2_chunk);
    it.ns = static_cast<uint8_t>(t.ns);
    it.nh = static_cast<uint8_t>(t.nh);
    it.n_routes = static_cast<uint8_t>(t.n_routes);
    it.nib_mode = static_cast<uint8_t>(t.nib_mode);
    const int e = launch_decode(p, mode, decode_smem_bytes(mode, p.warps, chains, s_region_bytes(t.ns)), stream);
    if (e) return cuda_error(static_cast<cudaError_t>(e));
    unsigned long long flags = 0;
    ce = cudaMemcpyAsync(&flags, scratch, 8, cudaMemcpyDeviceToHost, stream);
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(stream);
    if (ce != cudaSuccess) return cuda_error(ce);
    return flags ? BS_E_CORRUPT : BS_OK;
}
