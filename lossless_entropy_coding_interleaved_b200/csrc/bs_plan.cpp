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

bool inside(uint64_t off, uint64_t bytes, uint64_t len) { return off <= len && bytes <= len - off; }

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

// Reads and validates the whole container (the rules are in bs_validate.cpp). Fills `out`
// with every tensor, or returns the first error.
bs_status parse(Reader& rd, std::vector<Tensor>& out) {
    const uint64_t len = rd.len;
    uint8_t hdr[kHeaderBytes];
    auto fail = [&](bs_status st) { return rd.cuda_error ? BS_E_CUDA : st; };
    if (len < kHeaderBytes || !rd.read(0, kHeaderBytes, hdr)) return fail(BS_E_FORMAT);
    HeaderInfo h;
    bs_status st = check_header(hdr, len, &h);
    if (st != BS_OK) return st;
    std::vector<uint8_t> dbuf, nbuf, tbuf;
    try {
        dbuf.resize(uint64_t(kDirEntryBytes) * h.n_tensors);
        nbuf.resize(h.names_bytes);
    } catch (...) {
        return BS_E_NOMEM;
    }
    if (!rd.read(h.dir, dbuf.size(), dbuf.data()) || !rd.read(h.names, h.names_bytes, nbuf.data()))
        return fail(BS_E_FORMAT);
    out.clear();
    out.reserve(h.n_tensors);
    for (uint32_t k = 0; k < h.n_tensors; ++k) {
        Tensor t;
        uint32_t name_off = 0, name_len = 0;
        st = check_entry(dbuf.data() + uint64_t(kDirEntryBytes) * k, len, h, &t, &name_off, &name_len);
        if (st != BS_OK) return st;
        t.name.assign(reinterpret_cast<const char*>(nbuf.data() + name_off), name_len);
        if (is_coded(t.kind)) {
            try {
                t.model.resize(t.model_bytes);
                tbuf.resize(t.data_bytes);
            } catch (...) {
                return BS_E_NOMEM;
            }
            if (!rd.read(t.model_offset, t.model_bytes, t.model.data())) return fail(BS_E_FORMAT);
            if ((st = check_model(t.model.data(), &t)) != BS_OK) return st;
            if (!rd.read(t.data_offset, t.data_bytes, tbuf.data())) return fail(BS_E_FORMAT);
            if ((st = check_chunk_table(tbuf.data(), len, &t)) != BS_OK) return st;
        }
        out.push_back(std::move(t));
    }
    return BS_OK;
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
        const DecodeMode mode = decode_mode_of(t);
        const uint32_t need = decode_smem_bytes(mode, max_warps_of(mode), chains_of(mode), s_region_bytes(t.ns));
        if (static_cast<int>(need) > smem_cap) return BS_E_UNSUPPORTED;
        t.ws_offset = pos;
        build_tables(t, t.model.data(), image.data() + pos);
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
    const uint32_t smem = decode_smem_bytes(b.mode, p.warps, chains, b.s_region);
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
