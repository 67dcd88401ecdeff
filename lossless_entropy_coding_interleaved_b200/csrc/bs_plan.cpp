// bs_plan.cpp -- host side of libbs: container parsing and validation, decode-table
// construction, and the C ABI of include/bs.h. The GPU work lives in bs_kernels.cu.
//
// The container is BF16RANS version 2. This parser is written against that
// document. It shares no code with the oracle (oracle/bsoracle.c).
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstring>
#include <memory>
#include <new>
#include <vector>

#include "bs_host.h"

using namespace bs;

struct bs_plan_t {
    std::vector<Tensor> tensors;
    const uint8_t* d_container = nullptr;
    uint64_t container_bytes = 0;
    uint8_t* d_ws = nullptr;
    uint64_t ws_bytes = 0;
    int device = 0;
    std::vector<uint8_t> host_tables; // staging copy of the workspace tables (kept until destroy)
};

namespace {
thread_local int g_last_cuda = 0;
} // namespace

void bs::record_cuda_error(int e) { g_last_cuda = e; }

static std::atomic<unsigned long long> g_launches{0};
void bs::count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

namespace {

bs_status cuda_fail(cudaError_t e) { return cuda_status(static_cast<int>(e)); }

uint64_t get_u64(const uint8_t* p) {
    uint64_t v;
    std::memcpy(&v, p, 8);
    return v;
}
uint32_t get_u32(const uint8_t* p) {
    uint32_t v;
    std::memcpy(&v, p, 4);
    return v;
}
uint16_t get_u16(const uint8_t* p) {
    uint16_t v;
    std::memcpy(&v, p, 2);
    return v;
}
bool inside(uint64_t off, uint64_t bytes, uint64_t len) { return off <= len && bytes <= len - off; }
uint64_t up16(uint64_t v) { return (v + 15) & ~uint64_t(15); }

// Reads container bytes from a host copy or, without one, from device memory.
struct Reader {
    const uint8_t* host = nullptr;
    const uint8_t* dev = nullptr;
    cudaStream_t stream = nullptr;
    uint64_t len = 0;
    bool cuda_error = false;
    bool read(uint64_t off, uint64_t n, void* dst) {
        if (!inside(off, n, len)) return false;
        if (n == 0) return true;
        if (host) {
            std::memcpy(dst, host + off, n);
            return true;
        }
        cudaError_t e = cudaMemcpyAsync(dst, dev + off, n, cudaMemcpyDeviceToHost, stream);
        if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
        if (e != cudaSuccess) {
            g_last_cuda = static_cast<int>(e);
            cuda_error = true;
            return false;
        }
        return true;
    }
};

// Byte layout and validation rules of the container. Fills `out` with every tensor, or returns
// the first error.
bs_status parse(Reader& rd, std::vector<Tensor>& out) {
    const uint64_t len = rd.len;
    uint8_t hdr[kHeaderBytes];
    auto fail = [&](bs_status st) { return rd.cuda_error ? BS_E_CUDA : st; };
    if (len < kHeaderBytes || !rd.read(0, kHeaderBytes, hdr)) return fail(BS_E_FORMAT);
    const uint8_t* b = hdr;
    if (std::memcmp(b, "BF16RANS", 8) != 0) return BS_E_FORMAT;
    if (get_u32(b + 8) != kFormatVersion) return BS_E_VERSION;
    if (get_u32(b + 12) != kHeaderBytes || get_u32(b + 20) != kDirEntryBytes || get_u64(b + 56) != 0)
        return BS_E_FORMAT;
    if (get_u64(b + 48) != len) return BS_E_SIZE;
    const uint32_t nt = get_u32(b + 16);
    const uint64_t dir = get_u64(b + 24), names = get_u64(b + 32), names_bytes = get_u64(b + 40);
    if (dir % 16 || names % 16) return BS_E_FORMAT;
    if (!inside(dir, uint64_t(kDirEntryBytes) * nt, len) || !inside(names, names_bytes, len)) return BS_E_FORMAT;
    std::vector<uint8_t> dbuf, nbuf, tbuf;
    try {
        dbuf.resize(uint64_t(kDirEntryBytes) * nt);
        nbuf.resize(names_bytes);
    } catch (...) {
        return BS_E_NOMEM;
    }
    if (!rd.read(dir, dbuf.size(), dbuf.data()) || !rd.read(names, names_bytes, nbuf.data())) return fail(BS_E_FORMAT);
    out.clear();
    out.reserve(nt);
    for (uint32_t k = 0; k < nt; ++k) {
        const uint8_t* d = dbuf.data() + uint64_t(kDirEntryBytes) * k;
        Tensor t;
        t.kind = d[0];
        t.ndim = d[1];
        t.log2_chunk = d[2];
        t.lanes = d[3];
        t.ns = d[4];
        t.nh = d[5];
        t.n_routes = d[6];
        t.nib_mode = d[7];
        if (get_u64(d + 72) != 0) return BS_E_FORMAT;
        const uint32_t name_off = get_u32(d + 8), name_len = get_u32(d + 12);
        t.n_elems = get_u64(d + 16);
        t.n_chunks = get_u64(d + 24);
        t.model_offset = get_u64(d + 32);
        t.model_bytes = get_u64(d + 40);
        t.data_offset = get_u64(d + 48);
        t.data_bytes = get_u64(d + 56);
        t.checksum = get_u64(d + 64);
        for (int i = 0; i < 8; ++i) t.shape[i] = get_u64(d + 80 + 8 * i);
        if (t.kind > BS_KIND_JOINT || t.ndim > 8) return BS_E_FORMAT;
        if (!is_coded(t.kind) && t.nib_mode != 0) return BS_E_FORMAT;
        if (uint64_t(name_off) + name_len > names_bytes) return BS_E_FORMAT;
        t.name.assign(reinterpret_cast<const char*>(nbuf.data() + name_off), name_len);
        unsigned __int128 prod = 1;
        for (uint32_t i = 0; i < t.ndim; ++i) {
            prod *= t.shape[i];
            if (prod > (static_cast<unsigned __int128>(1) << 64)) return BS_E_FORMAT;
        }
        for (uint32_t i = t.ndim; i < 8; ++i)
            if (t.shape[i] != 0) return BS_E_FORMAT;
        if (prod != t.n_elems) return BS_E_FORMAT;
        if (t.data_offset % 16 || !inside(t.data_offset, t.data_bytes, len)) return BS_E_FORMAT;
        if (!is_coded(t.kind)) {
            if (t.kind == BS_KIND_STORED && t.n_elems > (1ull << 62)) return BS_E_FORMAT;
            const uint64_t want = t.kind == BS_KIND_STORED ? 2 * t.n_elems : t.n_elems;
            if (t.data_bytes != want) return BS_E_FORMAT;
            t.coded_bytes = want;
            out.push_back(std::move(t));
            continue;
        }
        // RANS and JOINT
        const bool joint = t.kind == BS_KIND_JOINT;
        if (t.lanes != kLanes || t.log2_chunk < 8 || t.log2_chunk > 24) return BS_E_FORMAT;
        if (joint) {
            if (t.ns < kMinNj || t.ns > kMaxNj || t.nh != 0 || t.n_routes != 0) return BS_E_FORMAT;
        } else if (t.ns < 1 || t.ns > kMaxNs || t.nh < kMinNh || t.nh > kMaxNh || t.ns + t.nh > kMaxPrecision ||
                   t.n_routes > kMaxRoutes) {
            return BS_E_FORMAT;
        }
        if (t.nib_mode != 0 && (t.nib_mode & 0xF0u) != 0x10u) return BS_E_FORMAT;
        if (t.n_elems == 0 || t.n_elems > (1ull << 40)) return BS_E_FORMAT;
        const uint64_t C = 1ull << t.log2_chunk;
        if (t.n_chunks != (t.n_elems + C - 1) / C || t.data_bytes != 16 * t.n_chunks) return BS_E_FORMAT;
        const uint64_t model_min = joint ? 8 : 264, model_max = joint ? 4 + 4 * kJointPairs : 260 + 4 * 512 + 16 * kMaxRoutes;
        if (t.model_offset % 16 || !inside(t.model_offset, t.model_bytes, len) || t.model_bytes < model_min ||
            t.model_bytes > model_max)
            return BS_E_FORMAT;
        t.model.resize(t.model_bytes);
        if (!rd.read(t.model_offset, t.model_bytes, t.model.data())) return fail(BS_E_FORMAT);
        const uint8_t* m = t.model.data();
        if (joint) { // the JOINT model: n_pairs, reserved, then (j, Fj) with j ascending
            const uint32_t n_pairs = get_u16(m);
            if (n_pairs < 1 || n_pairs > kJointPairs || get_u16(m + 2) != 0) return BS_E_FORMAT;
            if (t.model_bytes != 4 + 4ull * n_pairs) return BS_E_FORMAT;
            uint64_t sumj = 0;
            int prevj = -1;
            for (uint32_t i = 0; i < n_pairs; ++i) {
                const int j = get_u16(m + 4 + 4 * i);
                const uint32_t q = get_u16(m + 6 + 4 * i);
                if (j <= prevj || j >= static_cast<int>(kJointPairs) || q == 0) return BS_E_FORMAT;
                prevj = j;
                sumj += q;
            }
            if (sumj != (1ull << t.ns)) return BS_E_FORMAT;
        }
        const uint32_t n_present = joint ? 0 : get_u16(m);
        if (!joint) {
        if (n_present < 1 || n_present > 512) return BS_E_FORMAT;
        if (t.model_bytes != 260 + 4ull * n_present + 16ull * t.n_routes) return BS_E_FORMAT;
        uint64_t sum = 0;
        int prev = -1;
        for (uint32_t i = 0; i < n_present; ++i) {
            const int s = get_u16(m + 4 + 4 * i);
            const uint32_t q = get_u16(m + 6 + 4 * i);
            if (s <= prev || s > 511 || q == 0) return BS_E_FORMAT;
            prev = s;
            sum += q;
        }
        if (sum != (1ull << t.ns)) return BS_E_FORMAT;
        const uint8_t* route = m + 4 + 4 * n_present;
        for (int e = 0; e < 256; ++e)
            if (route[e] != 0xFF && route[e] >= t.n_routes) return BS_E_FORMAT;
        for (uint32_t r = 0; r < t.n_routes; ++r) {
            sum = 0;
            for (int h = 0; h < 8; ++h) sum += get_u16(route + 256 + 16 * r + 2 * h);
            if (sum != (1ull << t.nh)) return BS_E_FORMAT;
        }
        }
        (void)n_present;
        try {
            tbuf.resize(t.data_bytes);
        } catch (...) {
            return BS_E_NOMEM;
        }
        if (!rd.read(t.data_offset, t.data_bytes, tbuf.data())) return fail(BS_E_FORMAT);
        t.coded_bytes = t.model_bytes + t.data_bytes;
        for (uint64_t c = 0; c < t.n_chunks; ++c) {
            const uint8_t* e = tbuf.data() + 16 * c;
            const uint64_t off = get_u64(e);
            const uint32_t nw = get_u32(e + 8);
            const uint64_t nc = std::min<uint64_t>(C, t.n_elems - c * C);
            const uint64_t bytes = payload_bytes(nc, nw, t.nib_mode == 0);
            if (off % 16 || get_u32(e + 12) != 0 || !inside(off, bytes, len)) return BS_E_FORMAT;
            t.coded_bytes += bytes;
        }
        if (joint) {
            uint32_t max_f = 0;
            for (uint32_t i = 0; i < get_u16(t.model.data()); ++i) max_f = std::max<uint32_t>(max_f, get_u16(t.model.data() + 6 + 4 * i));
            t.joint_compact = max_f <= kCompactMaxF;
        }
        t.table_bytes = !joint ? table_bytes_for(t.ns, t.nh, t.n_routes)
                      : t.joint_compact ? joint4_table_bytes(t.ns) : joint_table_bytes(t.ns);
        out.push_back(std::move(t));
    }
    return BS_OK;
}

// Expand one tensor's model into the decode tables (layout in bs_internal.h): the s-table,
// then the compact fraction rows with the UNIFORM row last. For JOINT, one entry per slot:
// .x = F | ((j << 4) << 16), .y = the slot's rank k within its pair.
void build_tables(const Tensor& t, uint8_t* dst) {
    const uint8_t* m = t.model.data();
    if (t.kind == BS_KIND_JOINT) {
        const uint32_t n_pairs = get_u16(m);
        uint32_t* jt = reinterpret_cast<uint32_t*>(dst);
        uint32_t cum = 0;
        for (uint32_t i = 0; i < n_pairs; ++i) {
            const uint32_t j = get_u16(m + 4 + 4 * i), q = get_u16(m + 6 + 4 * i);
            for (uint32_t k = 0; k < q; ++k) {
                if (t.joint_compact) { // F | rank << 8 | j << 20 (q <= 255, so k < 255)
                    jt[cum + k] = q | (k << 8) | (j << 20);
                } else {
                    jt[2 * (cum + k)] = q | ((j << 4) << 16);
                    jt[2 * (cum + k) + 1] = k;
                }
            }
            cum += q;
        }
        return;
    }
    const uint32_t n_present = get_u16(m);
    const uint8_t* route = m + 4 + 4 * n_present;
    const uint32_t Mh = 1u << t.nh;
    auto frow = [&](uint32_t s) -> uint32_t {
        const uint8_t r = route[s & 0xFF];
        return frow_field(r == 0xFF ? t.n_routes : r, t.nh);
    };
    uint32_t* st = reinterpret_cast<uint32_t*>(dst);
    uint32_t cum = 0;
    for (uint32_t i = 0; i < n_present; ++i) {
        const uint32_t s = get_u16(m + 4 + 4 * i), q = get_u16(m + 6 + 4 * i);
        for (uint32_t k = 0; k < q; ++k) {
            st[2 * (cum + k)] = q | (k << 16);
            st[2 * (cum + k) + 1] = (s << 7) | (frow(s) << 16);
        }
        cum += q;
    }
    uint32_t* ht = reinterpret_cast<uint32_t*>(dst + (8u << t.ns));
    for (uint32_t r = 0; r <= t.n_routes; ++r) {
        uint32_t* row = ht + r * Mh;
        cum = 0;
        for (uint32_t h = 0; h < 8; ++h) {
            const uint32_t q = (r == t.n_routes) ? Mh / 8 : get_u16(route + 256 + 16 * r + 2 * h);
            for (uint32_t k = 0; k < q; ++k) row[cum + k] = h_entry(h, q, k);
            cum += q;
        }
    }
}

} // namespace

uint64_t bs::workspace_bytes_for(const std::vector<Tensor>& ts) {
    uint64_t ws = kErrBlockBytes;
    for (const Tensor& t : ts)
        if (is_coded(t.kind)) ws += up256(t.table_bytes);
    return ws;
}

bs_status bs::cuda_status(int e) {
    g_last_cuda = e;
    return BS_E_CUDA;
}

bs_status bs::parse_host_container(const uint8_t* h, uint64_t len, std::vector<Tensor>& out) {
    if (!h) return BS_E_ARG;
    Reader rd;
    rd.host = h;
    rd.len = len;
    return parse(rd, out);
}

bs_status bs::build_workspace(std::vector<Tensor>& ts, std::vector<uint8_t>& image) {
    const int smem_cap = max_dynamic_smem();
    try {
        image.assign(workspace_bytes_for(ts), 0);
    } catch (...) {
        return BS_E_NOMEM;
    }
    uint64_t pos = kErrBlockBytes;
    for (Tensor& t : ts) {
        if (!is_coded(t.kind)) continue;
        const uint32_t need = t.kind != BS_KIND_JOINT ? smem_bytes_for(t.ns, t.nh)
                            : t.joint_compact ? joint4_smem_bytes(kWarpsJoint4, kChainsJoint4)
                                              : joint_smem_bytes(kWarpsJoint, kChainsJoint);
        if (static_cast<int>(need) > smem_cap) return BS_E_UNSUPPORTED;
        t.ws_offset = pos;
        build_tables(t, image.data() + pos);
        pos += up256(t.table_bytes);
    }
    std::memset(image.data() + 8, 0xFF, 8); // error block: flags = 0, first_bad = all ones
    return BS_OK;
}

void bs::fill_tensor_info(const Tensor& t, bs_tensor_info* o) {
    std::memset(o, 0, sizeof(*o));
    o->n_elems = t.n_elems;
    o->out_bytes = t.kind == BS_KIND_RAW ? t.n_elems : 2 * t.n_elems;
    o->coded_bytes = t.coded_bytes;
    o->n_chunks = t.n_chunks;
    o->checksum = t.checksum;
    for (int i = 0; i < 8; ++i) o->shape[i] = t.shape[i];
    o->kind = t.kind;
    o->ndim = t.ndim;
    o->ns = t.ns;
    o->nh = t.nh;
    o->nib_mode = t.nib_mode;
    o->n_routes = t.n_routes;
    o->log2_chunk = t.log2_chunk;
    o->name = t.name.data();
    o->name_bytes = static_cast<uint32_t>(t.name.size());
}

bs_status DecodeBatch::init() {
    for (int k = 0; k < kDecodeModes; ++k) {
        bins_[k].p.reset(new (std::nothrow) DecodeParams);
        if (!bins_[k].p) return BS_E_NOMEM;
        bins_[k].mode = static_cast<DecodeMode>(k);
        bins_[k].p->n_items = 0;
        bins_[k].p->total_ctas = 0;
        bins_[k].p->err = err_;
    }
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0)
        sms_ = static_cast<uint32_t>(sms);
    cp_.reset(new (std::nothrow) CopyParams);
    if (!cp_) return BS_E_NOMEM;
    cp_->n_items = 0;
    cp_->total_blocks = 0;
    return BS_OK;
}

// Chooses the CTA shape for the queued chunks, assigns each item its CTA range and launches.
bs_status DecodeBatch::flush_bin(Bin& b, void* stream) {
    DecodeParams& p = *b.p;
    if (p.n_items == 0) return BS_OK;
    const uint32_t chains = chains_of(b.mode), max_warps = max_warps_of(b.mode);
    p.warps = launch_warps(b.chunks, max_warps, chains, sms_);
    // Every item rounds up to whole CTAs. If that pushes a launch that would fit one wave into
    // a second one, widen the CTAs until it fits again. A launch that needs more than one wave
    // even at the largest shape (many small tensors: each takes a CTA) keeps its shape.
    auto ctas_at = [&](uint32_t warps) {
        uint64_t n = 0;
        for (uint32_t k = 0; k < p.n_items; ++k) {
            const DecodeItem& it = p.item[k];
            const uint64_t C = 1ull << it.log2_chunk, n_chunks = (it.n_elems + C - 1) / C;
            n += (n_chunks + uint64_t(warps) * chains - 1) / (uint64_t(warps) * chains);
        }
        return n;
    };
    if (ctas_at(p.warps) > sms_ && ctas_at(max_warps) <= sms_)
        while (ctas_at(p.warps) > sms_) ++p.warps;
    const uint64_t per_cta = uint64_t(p.warps) * chains;
    uint64_t ctas = 0;
    for (uint32_t k = 0; k < p.n_items; ++k) {
        DecodeItem& it = p.item[k];
        const uint64_t C = 1ull << it.log2_chunk, n_chunks = (it.n_elems + C - 1) / C;
        it.cta_begin = static_cast<uint32_t>(ctas);
        ctas += (n_chunks + per_cta - 1) / per_cta;
    }
    p.total_ctas = static_cast<uint32_t>(ctas); // at most 2^31 / 8 + kMaxDecodeItems (see add)
    const bool joint = b.mode == DecodeMode::Joint || b.mode == DecodeMode::JointGeneric;
    const uint32_t smem = b.mode == DecodeMode::JointCompact ? joint4_smem_bytes(p.warps, chains)
                        : joint ? joint_smem_bytes(p.warps, chains)
                                : kHRegion + b.s_region + p.warps * chains * (kRingBytes + kNibRingBytes);
    const int e = launch_decode(p, b.mode, smem, stream);
    p.n_items = 0;
    p.total_ctas = 0;
    b.s_region = 0;
    b.chunks = 0;
    return e ? cuda_status(e) : BS_OK;
}

bs_status DecodeBatch::flush_copy(void* stream) {
    if (cp_->n_items == 0) return BS_OK;
    const int e = launch_copy(*cp_, stream);
    cp_->n_items = 0;
    cp_->total_blocks = 0;
    return e ? cuda_status(e) : BS_OK;
}

bs_status DecodeBatch::add(const Tensor& t, uint32_t tensor_index, const uint8_t* d_container,
                           const uint8_t* d_ws, void* d_out, void* stream, uint64_t begin, uint64_t count) {
    const uint64_t n_units = t.n_elems; // elements, or bytes for RAW
    if (begin > n_units) begin = n_units;
    if (count > n_units - begin) count = n_units - begin;
    if (is_coded(t.kind)) {
        // a range is decoded as a tensor of its own: its chunk entries, its length, its output
        const uint64_t c0 = begin >> t.log2_chunk;
        const uint64_t range_chunks = (count + (1ull << t.log2_chunk) - 1) >> t.log2_chunk;
        const DecodeMode mode = decode_mode_of(t);
        Bin& b = bins_[static_cast<int>(mode)];
        // the smallest CTA holds kMinWarps * 2 chunks, so 2^31 chunks keep the grid below 2^31 CTAs
        if (range_chunks == 0) return BS_OK;
        if (b.p->n_items == kMaxDecodeItems || b.chunks + range_chunks > (1ull << 31)) {
            bs_status s = flush_bin(b, stream);
            if (s) return s;
        }
        DecodeItem& it = b.p->item[b.p->n_items++];
        std::memset(&it, 0, sizeof(it));
        it.chunk_table = d_container + t.data_offset + 16 * c0;
        it.container = d_container;
        it.tables = reinterpret_cast<const uint4*>(d_ws + t.ws_offset);
        it.out = static_cast<uint16_t*>(d_out);
        it.n_elems = count;
        it.tensor_index = tensor_index;
        it.chunk_base = static_cast<uint32_t>(c0); // c0 < n_chunks <= 2^32
        it.table_bytes = t.table_bytes;
        it.log2_chunk = static_cast<uint8_t>(t.log2_chunk);
        it.ns = static_cast<uint8_t>(t.ns);
        it.nh = static_cast<uint8_t>(t.nh);
        it.n_routes = static_cast<uint8_t>(t.n_routes);
        it.nib_mode = static_cast<uint8_t>(t.nib_mode);
        b.chunks += range_chunks;
        b.s_region = std::max<uint32_t>(b.s_region, s_region_bytes(t.ns));
    } else if (count) {
        const uint64_t unit = t.kind == BS_KIND_RAW ? 1 : 2;
        const uint64_t bytes = unit * count;
        const uint64_t blks = (bytes + kCopyBlockBytes - 1) / kCopyBlockBytes;
        if (cp_->n_items == kMaxCopyItems || cp_->total_blocks + blks > 0x7FFFFFFFull) {
            bs_status s = flush_copy(stream);
            if (s) return s;
        }
        CopyItem& it = cp_->item[cp_->n_items++];
        it.src = d_container + t.data_offset + unit * begin;
        it.dst = static_cast<uint8_t*>(d_out);
        it.bytes = bytes;
        it.blk_begin = cp_->total_blocks;
        cp_->total_blocks += blks;
    }
    return BS_OK;
}

bs_status DecodeBatch::flush(void* stream) {
    for (Bin& b : bins_) {
        bs_status s = flush_bin(b, stream);
        if (s) return s;
    }
    return flush_copy(stream);
}

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

} // namespace

extern "C" {

size_t bs_plan_workspace_bytes(const void* h_container, size_t container_bytes) {
    if (!h_container) return 0;
    std::vector<Tensor> ts;
    Reader rd;
    rd.host = static_cast<const uint8_t*>(h_container);
    rd.len = container_bytes;
    if (parse(rd, ts) != BS_OK) return 0;
    return workspace_bytes_for(ts);
}

size_t bs_plan_workspace_bytes_device(const void* d_container, size_t container_bytes, void* stream) {
    if (!d_container) return 0;
    std::vector<Tensor> ts;
    Reader rd;
    rd.dev = static_cast<const uint8_t*>(d_container);
    rd.stream = static_cast<cudaStream_t>(stream);
    rd.len = container_bytes;
    if (parse(rd, ts) != BS_OK) return 0;
    return workspace_bytes_for(ts);
}

bs_status bs_plan(const void* h_container, size_t container_bytes, const void* d_container, void* d_workspace,
                  size_t workspace_bytes, void* stream, bs_plan_t** out) {
    if (!out || !d_container || !d_workspace) return BS_E_ARG;
    *out = nullptr;
    if (!aligned(d_container, 16) || !aligned(d_workspace, 256)) return BS_E_ARG;
    int dev = 0, major = 0, minor = 0;
    cudaError_t ce = cudaGetDevice(&dev);
    if (ce != cudaSuccess) return cuda_fail(ce);
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0) return BS_E_UNSUPPORTED;

    std::unique_ptr<bs_plan_t> p(new (std::nothrow) bs_plan_t);
    if (!p) return BS_E_NOMEM;
    Reader rd;
    rd.host = static_cast<const uint8_t*>(h_container);
    rd.dev = static_cast<const uint8_t*>(d_container);
    rd.stream = static_cast<cudaStream_t>(stream);
    rd.len = container_bytes;
    bs_status st = parse(rd, p->tensors);
    if (st != BS_OK) return st;
    const uint64_t ws = workspace_bytes_for(p->tensors);
    if (workspace_bytes < ws) return BS_E_SIZE;
    st = build_workspace(p->tensors, p->host_tables);
    if (st != BS_OK) return st;
    ce = cudaMemcpyAsync(d_workspace, p->host_tables.data(), ws, cudaMemcpyHostToDevice,
                         static_cast<cudaStream_t>(stream));
    if (ce != cudaSuccess) return cuda_fail(ce);
    p->d_container = static_cast<const uint8_t*>(d_container);
    p->container_bytes = container_bytes;
    p->d_ws = static_cast<uint8_t*>(d_workspace);
    p->ws_bytes = ws;
    p->device = dev;
    *out = p.release();
    return BS_OK;
}

void bs_plan_destroy(bs_plan_t* plan) { delete plan; }

bs_status bs_tensor_count(const bs_plan_t* plan, int32_t* n) {
    if (!plan || !n) return BS_E_ARG;
    *n = static_cast<int32_t>(plan->tensors.size());
    return BS_OK;
}

bs_status bs_tensor_info_get(const bs_plan_t* plan, int32_t idx, bs_tensor_info* o) {
    if (!plan || !o || idx < 0 || idx >= static_cast<int32_t>(plan->tensors.size())) return BS_E_ARG;
    fill_tensor_info(plan->tensors[idx], o);
    return BS_OK;
}

bs_status bs_decode_batch(const bs_plan_t* plan, const int32_t* idx, void* const* d_out, const size_t* out_bytes,
                          int32_t n, void* stream) {
    if (!plan || n < 0 || (n > 0 && (!idx || !d_out || !out_bytes))) return BS_E_ARG;
    const int32_t nt = static_cast<int32_t>(plan->tensors.size());
    for (int32_t k = 0; k < n; ++k) {
        if (idx[k] < 0 || idx[k] >= nt) return BS_E_ARG;
        const Tensor& t = plan->tensors[idx[k]];
        const uint64_t want = t.kind == BS_KIND_RAW ? t.n_elems : 2 * t.n_elems;
        if (out_bytes[k] != want) return BS_E_SIZE;
        if (want && !d_out[k]) return BS_E_ARG;
        if (is_coded(t.kind) && !aligned(d_out[k], 16)) return BS_E_ARG;
    }
    DecodeBatch batch(reinterpret_cast<unsigned long long*>(plan->d_ws));
    bs_status st = batch.init();
    if (st) return st;
    for (int32_t k = 0; k < n; ++k) {
        st = batch.add(plan->tensors[idx[k]], static_cast<uint32_t>(idx[k]), plan->d_container, plan->d_ws,
                       d_out[k], stream);
        if (st) return st;
    }
    return batch.flush(stream);
}

bs_status bs_decode_ranges(const bs_plan_t* plan, const bs_range* ranges, int32_t n, void* stream) {
    if (!plan || n < 0 || (n > 0 && !ranges)) return BS_E_ARG;
    const int32_t nt = static_cast<int32_t>(plan->tensors.size());
    for (int32_t k = 0; k < n; ++k) {
        const bs_range& r = ranges[k];
        if (r.idx < 0 || r.idx >= nt || r.reserved) return BS_E_ARG;
        const Tensor& t = plan->tensors[r.idx];
        if (r.begin > t.n_elems || r.count > t.n_elems - r.begin) return BS_E_ARG;
        if (is_coded(t.kind) && r.count) { // whole chunks: the start and the end on chunk boundaries (or the tensor's end)
            const uint64_t mask = (1ull << t.log2_chunk) - 1;
            if ((r.begin & mask) || (r.begin + r.count != t.n_elems && (r.count & mask))) return BS_E_ARG;
            if (!aligned(r.d_out, 16)) return BS_E_ARG;
        }
        const uint64_t want = t.kind == BS_KIND_RAW ? r.count : 2 * r.count;
        if (r.out_bytes != want) return BS_E_SIZE;
        if (want && !r.d_out) return BS_E_ARG;
    }
    DecodeBatch batch(reinterpret_cast<unsigned long long*>(plan->d_ws));
    bs_status st = batch.init();
    if (st) return st;
    for (int32_t k = 0; k < n; ++k) {
        const bs_range& r = ranges[k];
        st = batch.add(plan->tensors[r.idx], static_cast<uint32_t>(r.idx), plan->d_container, plan->d_ws, r.d_out,
                       stream, r.begin, r.count);
        if (st) return st;
    }
    return batch.flush(stream);
}

bs_status bs_decode_geometry(const bs_plan_t* plan, int32_t idx, uint32_t* chunks_per_cta, uint32_t* ctas_per_wave) {
    if (!plan || !chunks_per_cta || !ctas_per_wave || idx < 0 || idx >= static_cast<int32_t>(plan->tensors.size()))
        return BS_E_ARG;
    const Tensor& t = plan->tensors[idx];
    *chunks_per_cta = is_coded(t.kind) ? max_warps_of(decode_mode_of(t)) * chains_of(decode_mode_of(t)) : 0;
    int dev = 0, sms = 0;
    cudaError_t ce = cudaGetDevice(&dev);
    if (ce == cudaSuccess) ce = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (ce != cudaSuccess || sms <= 0) return cuda_fail(ce == cudaSuccess ? cudaErrorInvalidDevice : ce);
    *ctas_per_wave = static_cast<uint32_t>(sms); // every decode shape takes over half an SM's shared memory
    return BS_OK;
}

bs_status bs_decode_tensor(const bs_plan_t* plan, int32_t idx, void* d_out, size_t out_bytes, void* stream) {
    return bs_decode_batch(plan, &idx, &d_out, &out_bytes, 1, stream);
}

bs_status bs_verify_tensor(const bs_plan_t* plan, int32_t idx, const void* d_out, size_t out_bytes, void* d_scratch,
                           void* stream, uint64_t* got) {
    if (!plan || idx < 0 || idx >= static_cast<int32_t>(plan->tensors.size()) || !d_scratch ||
        !aligned(d_scratch, 8))
        return BS_E_ARG;
    const Tensor& t = plan->tensors[idx];
    const uint64_t want = t.kind == BS_KIND_RAW ? t.n_elems : 2 * t.n_elems;
    if (out_bytes != want) return BS_E_SIZE;
    if (want && !d_out) return BS_E_ARG;
    auto* sum = static_cast<unsigned long long*>(d_scratch);
    int e = launch_checksum(d_out, t.n_elems, t.kind == BS_KIND_RAW, sum, stream);
    if (e) return cuda_fail(static_cast<cudaError_t>(e));
    unsigned long long h = 0;
    cudaError_t ce = cudaMemcpyAsync(&h, sum, 8, cudaMemcpyDeviceToHost, static_cast<cudaStream_t>(stream));
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (ce != cudaSuccess) return cuda_fail(ce);
    if (got) *got = h;
    return h == t.checksum ? BS_OK : BS_E_CORRUPT;
}

bs_status bs_check(const bs_plan_t* plan, void* stream, int64_t* first_bad) {
    if (!plan) return BS_E_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned long long h[2] = {0, 0};
    cudaError_t ce = cudaMemcpyAsync(h, plan->d_ws, 16, cudaMemcpyDeviceToHost, s);
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(s);
    if (ce != cudaSuccess) return cuda_fail(ce);
    if (first_bad) *first_bad = h[0] ? static_cast<int64_t>(h[1]) : -1;
    if (!h[0]) return BS_OK;
    static const unsigned long long reset[2] = {0, ~0ull};
    ce = cudaMemcpyAsync(plan->d_ws, reset, 16, cudaMemcpyHostToDevice, s);
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(s);
    if (ce != cudaSuccess) return cuda_fail(ce);
    return BS_E_CORRUPT;
}

const char* bs_status_str(bs_status s) {
    switch (s) {
    case BS_OK: return "ok";
    case BS_E_ARG: return "bad argument";
    case BS_E_FORMAT: return "container fails validation";
    case BS_E_VERSION: return "unknown container version";
    case BS_E_SIZE: return "wrong buffer size";
    case BS_E_CUDA: return "CUDA runtime error";
    case BS_E_CORRUPT: return "corrupt chunk or checksum mismatch";
    case BS_E_NOMEM: return "host allocation failed";
    case BS_E_UNSUPPORTED: return "unsupported device or model size";
    }
    return "unknown status";
}

int bs_last_cuda_error(void) { return g_last_cuda; }

uint64_t bs_launch_counter(void) { return g_launches.load(std::memory_order_relaxed); }

} // extern "C"
