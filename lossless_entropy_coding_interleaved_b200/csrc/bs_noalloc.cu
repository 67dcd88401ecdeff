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
#include <cuda_runtime.h>

#include <atomic>
#include <cstring>
#include <mutex>

#include "bs_internal.h"

namespace bs {

// Largest decode tables the array holds: the JOINT table at nj = 13 (64 KiB), which is
// larger than any factored one (the s-table at ns = 12, 32 KiB, plus 16 compact fraction
// rows of 2^5 entries, 2 KiB). That is every tensor a valid container can hold; larger
// tables would get BS_E_SIZE.
constexpr uint32_t kNoAllocFactoredBytes = (8u << kMaxNs) + 4u * (kMaxRoutes + 1) * (1u << kMaxNh);
constexpr uint32_t kNoAllocTableBytes = (8u << kMaxNj) > kNoAllocFactoredBytes ? (8u << kMaxNj) : kNoAllocFactoredBytes;
constexpr uint32_t kNoAllocBytes = 256 + kNoAllocTableBytes; // error block, then tables

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_addr_mutex;
unsigned char* g_addr[kMaxDevices] = {nullptr};

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

uint64_t rd64(const uint8_t* p) {
    uint64_t v;
    std::memcpy(&v, p, 8);
    return v;
}
uint32_t rd32(const uint8_t* p) {
    uint32_t v;
    std::memcpy(&v, p, 4);
    return v;
}
uint16_t rd16(const uint8_t* p) {
    uint16_t v;
    std::memcpy(&v, p, 2);
    return v;
}
bool in_range(uint64_t off, uint64_t n, uint64_t len) { return off <= len && n <= len - off; }

} // namespace

// Expand a tensor's model (read from the container on the device) into the decode-table
// layout that decode_kernel stages (bs_internal.h): the s-table, then the compact fraction
// rows with the UNIFORM row last. One CTA. It writes into the tables part of the array above.
// The host validated the model in its own copy. The device copy is read defensively: the
// caller zeroes the table region first, n_present comes from the host, every write is
// bounded by its table, and a route index out of range reads as UNIFORM. So the decode
// kernel's lookups stay inside the tables even if the two copies differ.
__global__ void __launch_bounds__(512) noalloc_tables_kernel(const uint8_t* model, uint32_t n_present, uint32_t ns,
                                                             uint32_t nh, uint32_t n_routes) {
    __shared__ uint32_t s_cum[513];
    __shared__ uint16_t h_cum[16][9];
    unsigned char* tab = g_noalloc_scratch + 256;
    const uint8_t* pairs = model + 4;
    const uint8_t* route = model + 4 + 4 * n_present;
    const uint8_t* rows = route + 256;
    const uint32_t Mh = 1u << nh;
    if (threadIdx.x == 0) {
        uint32_t acc = 0;
        for (uint32_t i = 0; i < n_present; ++i) {
            s_cum[i] = acc;
            acc += pairs[4 * i + 2] | (pairs[4 * i + 3] << 8);
        }
        s_cum[n_present] = acc;
    }
    if (threadIdx.x >= 32 && threadIdx.x < 32 + n_routes + 1) {
        const uint32_t r = threadIdx.x - 32;
        uint32_t acc = 0;
        for (uint32_t h = 0; h < 8; ++h) {
            h_cum[r][h] = static_cast<uint16_t>(acc);
            acc += (r == n_routes) ? Mh / 8 : (rows[16 * r + 2 * h] | (rows[16 * r + 2 * h + 1] << 8));
        }
        h_cum[r][8] = static_cast<uint16_t>(acc);
    }
    __syncthreads();
    uint32_t* st = reinterpret_cast<uint32_t*>(tab);
    const uint32_t Ms = 1u << ns;
    for (uint32_t i = threadIdx.x; i < n_present; i += blockDim.x) {
        const uint32_t s = (pairs[4 * i] | (pairs[4 * i + 1] << 8)) & 0x1FFu;
        const uint32_t q = s_cum[i + 1] - s_cum[i];
        const uint8_t r = route[s & 0xFF];
        const uint32_t frow = frow_field(r < n_routes ? r : n_routes, nh);
        for (uint32_t k = 0; k < q && s_cum[i] + k < Ms; ++k) {
            st[2 * (s_cum[i] + k)] = q | (k << 16);
            st[2 * (s_cum[i] + k) + 1] = (s << 7) | (frow << 16);
        }
    }
    uint32_t* ht = reinterpret_cast<uint32_t*>(tab + (8u << ns));
    for (uint32_t j = threadIdx.x; j < (n_routes + 1) * 8; j += blockDim.x) {
        const uint32_t r = j >> 3, h = j & 7u;
        const uint32_t c0 = h_cum[r][h], q = static_cast<uint16_t>(h_cum[r][h + 1] - c0);
        for (uint32_t k = 0; k < q && c0 + k < Mh; ++k) ht[r * Mh + c0 + k] = h_entry(h, q, k);
    }
}

// The JOINT table (bs_internal.h): for the pair of slot cum(j) + k, .x = F | ((j << 4) << 16)
// and .y = k. One CTA; thread 0 takes the running sums, then every thread fills pairs.
// Writes are bounded by 2^nj slots, so a device copy that differs from the host's validated
// one cannot write outside the table.
__global__ void __launch_bounds__(512) noalloc_joint_kernel(const uint8_t* model, uint32_t n_pairs, uint32_t nj) {
    __shared__ uint32_t cum[kJointPairs + 1];
    uint32_t* jt = reinterpret_cast<uint32_t*>(g_noalloc_scratch + 256);
    const uint8_t* pairs = model + 4;
    if (threadIdx.x == 0) {
        uint32_t acc = 0;
        for (uint32_t i = 0; i < n_pairs; ++i) {
            cum[i] = acc;
            acc += pairs[4 * i + 2] | (pairs[4 * i + 3] << 8);
        }
        cum[n_pairs] = acc;
    }
    __syncthreads();
    const uint32_t M = 1u << nj;
    for (uint32_t i = threadIdx.x; i < n_pairs; i += blockDim.x) {
        const uint32_t j = (pairs[4 * i] | (pairs[4 * i + 1] << 8)) & (kJointPairs - 1u);
        const uint32_t q = cum[i + 1] - cum[i];
        for (uint32_t k = 0; k < q && cum[i] + k < M; ++k) {
            jt[2 * (cum[i] + k)] = (q & 0xFFFFu) | ((j << 4) << 16);
            jt[2 * (cum[i] + k) + 1] = k;
        }
    }
}

} // namespace bs

using namespace bs;

extern "C" bs_status bs_decode_tensor_noalloc(const void* h_container_v, size_t len, const void* d_container_v,
                                              int32_t idx, void* d_out, size_t out_bytes, void* stream_v) {
    const uint8_t* b = static_cast<const uint8_t*>(h_container_v);
    const uint8_t* d_container = static_cast<const uint8_t*>(d_container_v);
    cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
    if (!b || !d_container || idx < 0) return BS_E_ARG;
    if (reinterpret_cast<uintptr_t>(d_container) & 15u) return BS_E_ARG;
    // --- validate the header and this tensor in place (the container's validation rules) ---
    if (len < kHeaderBytes || std::memcmp(b, "BF16RANS", 8) != 0) return BS_E_FORMAT;
    if (rd32(b + 8) != kFormatVersion) return BS_E_VERSION;
    if (rd32(b + 12) != kHeaderBytes || rd32(b + 20) != kDirEntryBytes || rd64(b + 56) != 0) return BS_E_FORMAT;
    if (rd64(b + 48) != len) return BS_E_SIZE;
    const uint32_t nt = rd32(b + 16);
    const uint64_t dir = rd64(b + 24), names_bytes = rd64(b + 40);
    if (dir % 16 || !in_range(dir, uint64_t(kDirEntryBytes) * nt, len) || !in_range(rd64(b + 32), names_bytes, len))
        return BS_E_FORMAT;
    if (static_cast<uint32_t>(idx) >= nt) return BS_E_ARG;
    const uint8_t* d = b + dir + uint64_t(kDirEntryBytes) * idx;
    const uint32_t kind = d[0], ndim = d[1], log2c = d[2], lanes = d[3], ns = d[4], nh = d[5], n_routes = d[6];
    const uint32_t nib_mode = d[7];
    const uint64_t n = rd64(d + 16), n_chunks = rd64(d + 24), model_off = rd64(d + 32), model_bytes = rd64(d + 40);
    const uint64_t data_off = rd64(d + 48), data_bytes = rd64(d + 56);
    if (kind > BS_KIND_JOINT || ndim > 8 || rd64(d + 72) != 0) return BS_E_FORMAT;
    if (!is_coded(kind) && nib_mode != 0) return BS_E_FORMAT;
    if (uint64_t(rd32(d + 8)) + rd32(d + 12) > names_bytes) return BS_E_FORMAT;
    unsigned __int128 prod = 1;
    for (uint32_t i = 0; i < 8; ++i) {
        const uint64_t v = rd64(d + 80 + 8 * i);
        if (i >= ndim) {
            if (v) return BS_E_FORMAT;
            continue;
        }
        prod *= v;
        if (prod > (static_cast<unsigned __int128>(1) << 64)) return BS_E_FORMAT;
    }
    if (prod != n || data_off % 16 || !in_range(data_off, data_bytes, len)) return BS_E_FORMAT;
    const uint64_t want = kind == BS_KIND_RAW ? n : 2 * n;
    if (kind == BS_KIND_STORED && n > (1ull << 62)) return BS_E_FORMAT;
    if (out_bytes != want) return BS_E_SIZE;
    if (want && (!d_out || (reinterpret_cast<uintptr_t>(d_out) & 15u))) return BS_E_ARG;

    if (!is_coded(kind)) { // verbatim: no scratch needed, the copy kernel does it
        if (data_bytes != want) return BS_E_FORMAT;
        if (want == 0) return BS_OK;
        CopyParams cp;
        cp.n_items = 1;
        cp.total_blocks = (want + kCopyBlockBytes - 1) / kCopyBlockBytes;
        cp.item[0] = CopyItem{d_container + data_off, static_cast<uint8_t*>(d_out), want, 0};
        int e = launch_copy(cp, stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
        if (e) {
            record_cuda_error(e);
            return BS_E_CUDA;
        }
        return BS_OK;
    }
    const bool joint = kind == BS_KIND_JOINT;
    if (lanes != kLanes || log2c < 8 || log2c > 24 || n == 0 || n > (1ull << 40)) return BS_E_FORMAT;
    if (joint ? (ns < kMinNj || ns > kMaxNj || nh != 0 || n_routes != 0)
              : (ns < 1 || ns > kMaxNs || nh < kMinNh || nh > kMaxNh || ns + nh > kMaxPrecision || n_routes > kMaxRoutes))
        return BS_E_FORMAT;
    if (nib_mode != 0 && (nib_mode & 0xF0u) != 0x10u) return BS_E_FORMAT;
    if (n_chunks != ((n + (1ull << log2c) - 1) >> log2c) || data_bytes != 16 * n_chunks) return BS_E_FORMAT;
    if (model_off % 16 || !in_range(model_off, model_bytes, len) || model_bytes < (joint ? 8u : 264u))
        return BS_E_FORMAT;
    const uint8_t* m = b + model_off;
    const uint32_t n_present = joint ? 0 : rd16(m);
    uint32_t n_pairs = 0;
    if (joint) { // the JOINT model: n_pairs, reserved, then (j, Fj) with j ascending
        n_pairs = rd16(m);
        if (n_pairs < 1 || n_pairs > kJointPairs || rd16(m + 2) != 0 || model_bytes != 4 + 4ull * n_pairs)
            return BS_E_FORMAT;
        uint64_t sumj = 0;
        int prevj = -1;
        for (uint32_t i = 0; i < n_pairs; ++i) {
            const int j = rd16(m + 4 + 4 * i);
            const uint32_t q = rd16(m + 6 + 4 * i);
            if (j <= prevj || j >= static_cast<int>(kJointPairs) || q == 0) return BS_E_FORMAT;
            prevj = j;
            sumj += q;
        }
        if (sumj != (1ull << ns)) return BS_E_FORMAT;
    } else {
    if (n_present < 1 || n_present > 512 || model_bytes != 260 + 4ull * n_present + 16ull * n_routes)
        return BS_E_FORMAT;
    uint64_t sum = 0;
    int prev = -1;
    for (uint32_t i = 0; i < n_present; ++i) {
        const int s = rd16(m + 4 + 4 * i);
        const uint32_t q = rd16(m + 6 + 4 * i);
        if (s <= prev || s > 511 || q == 0) return BS_E_FORMAT;
        prev = s;
        sum += q;
    }
    if (sum != (1ull << ns)) return BS_E_FORMAT;
    const uint8_t* route = m + 4 + 4 * n_present;
    for (int e = 0; e < 256; ++e)
        if (route[e] != 0xFF && route[e] >= n_routes) return BS_E_FORMAT;
    for (uint32_t r = 0; r < n_routes; ++r) {
        sum = 0;
        for (int h = 0; h < 8; ++h) sum += rd16(route + 256 + 16 * r + 2 * h);
        if (sum != (1ull << nh)) return BS_E_FORMAT;
    }
    }
    const uint64_t C = 1ull << log2c;
    for (uint64_t c = 0; c < n_chunks; ++c) {
        const uint8_t* e = b + data_off + 16 * c;
        const uint64_t nc = (n - c * C < C) ? n - c * C : C;
        if (rd64(e) % 16 || rd32(e + 12) != 0 || !in_range(rd64(e), payload_bytes(nc, rd32(e + 8), nib_mode == 0), len))
            return BS_E_FORMAT;
    }
    const uint32_t tb = joint ? joint_table_bytes(ns) : table_bytes_for(ns, nh, n_routes);
    if (tb > kNoAllocTableBytes) return BS_E_SIZE; // larger than the static array holds

    // --- set-up: the array's device address on this device ---
    unsigned char* scratch = nullptr;
    cudaError_t ce = scratch_address(&scratch);
    if (ce != cudaSuccess) {
        record_cuda_error(ce);
        return BS_E_CUDA;
    }
    // error block: flags = 0, first_bad = all ones; tables zeroed (the array keeps the
    // previous call's bytes)
    ce = cudaMemsetAsync(scratch, 0, 256 + tb, stream);
    if (ce == cudaSuccess) ce = cudaMemsetAsync(scratch + 8, 0xFF, 8, stream);
    if (ce != cudaSuccess) {
        record_cuda_error(ce);
        return BS_E_CUDA;
    }
    if (joint) noalloc_joint_kernel<<<1, 512, 0, stream>>>(d_container + model_off, n_pairs, ns);
    else noalloc_tables_kernel<<<1, 512, 0, stream>>>(d_container + model_off, n_present, ns, nh, n_routes);
    count_launch();
    ce = cudaGetLastError();
    if (ce != cudaSuccess) {
        record_cuda_error(ce);
        return BS_E_CUDA;
    }
    // --- the decode kernel, unchanged, with its tables and error block in the array ---
    DecodeParams p; // about 31 KiB of launch parameters, on the stack (no heap use)
    p.n_items = 1;
    const bool dflt = joint ? ns == kDefaultNj : is_default_precision(ns, nh); // the larger shape
    const DecodeMode mode = joint ? (dflt ? DecodeMode::Joint : DecodeMode::JointGeneric)
                                  : dflt ? DecodeMode::Default : DecodeMode::Generic;
    const uint32_t chains = chains_of(mode);
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        sms = 148;
    p.warps = launch_warps(n_chunks, max_warps_of(mode), chains, static_cast<uint32_t>(sms));
    const uint64_t per_cta = uint64_t(p.warps) * chains;
    p.total_ctas = static_cast<uint32_t>((n_chunks + per_cta - 1) / per_cta);
    p.err = reinterpret_cast<unsigned long long*>(scratch);
    DecodeItem& it = p.item[0];
    std::memset(&it, 0, sizeof(it));
    it.chunk_table = d_container + data_off;
    it.container = d_container;
    it.tables = reinterpret_cast<const uint4*>(scratch + 256);
    it.out = static_cast<uint16_t*>(d_out);
    it.n_elems = n;
    it.cta_begin = 0;
    it.tensor_index = static_cast<uint32_t>(idx);
    it.table_bytes = tb;
    it.log2_chunk = static_cast<uint8_t>(log2c);
    it.ns = static_cast<uint8_t>(ns);
    it.nh = static_cast<uint8_t>(nh);
    it.n_routes = static_cast<uint8_t>(n_routes);
    it.nib_mode = static_cast<uint8_t>(nib_mode);
    int e = launch_decode(p, mode, joint ? joint_smem_bytes(p.warps, chains) : smem_bytes_for(ns, p.warps, chains), stream);
    if (e) {
        record_cuda_error(e);
        return BS_E_CUDA;
    }
    unsigned long long flags = 0;
    ce = cudaMemcpyAsync(&flags, scratch, 8, cudaMemcpyDeviceToHost, stream);
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(stream);
    if (ce != cudaSuccess) {
        record_cuda_error(ce);
        return BS_E_CUDA;
    }
    return flags ? BS_E_CORRUPT : BS_OK;
}
