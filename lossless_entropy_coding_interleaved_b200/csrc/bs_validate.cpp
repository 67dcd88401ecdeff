// bs_validate.cpp -- the container's validation rules and the decode-table builder, shared by
// every host path of libbs: the planner (bs_plan.cpp, which reads the container from host or
// device memory), the layer streamer (bs_stream.cpp) and the allocation-free entry point
// (bs_noalloc.cu, which checks one tensor in place in the caller's host copy). One copy of
// each rule, so the paths cannot disagree on what a valid container is.
//
// The container is BF16RANS version 2, this library's own layout (the pages give none):
//   header (64 bytes): magic, version, header and entry sizes, tensor count, the directory
//     and names offsets, the total size;
//   directory entries (144 bytes): kind, shape, chunking, precisions, model and data
//     sections, checksum;
//   per coded tensor: its model (RANS: s-table, routes, h tables; JOINT: the pair table) and
//     a chunk table of 16-byte entries (payload offset, word count).
// Nothing here is shared with the oracle, which has its own parser.
#include <algorithm>
#include <cstring>

#include "bs_host.h"

namespace bs {

namespace {

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

} // namespace

bs_status check_header(const uint8_t* b, uint64_t len, HeaderInfo* h) {
    if (len < kHeaderBytes || std::memcmp(b, "BF16RANS", 8) != 0) return BS_E_FORMAT;
    if (get_u32(b + 8) != kFormatVersion) return BS_E_VERSION;
    if (get_u32(b + 12) != kHeaderBytes || get_u32(b + 20) != kDirEntryBytes || get_u64(b + 56) != 0)
        return BS_E_FORMAT;
    if (get_u64(b + 48) != len) return BS_E_SIZE;
    h->n_tensors = get_u32(b + 16);
    h->dir = get_u64(b + 24);
    h->names = get_u64(b + 32);
    h->names_bytes = get_u64(b + 40);
    if (h->dir % 16 || h->names % 16) return BS_E_FORMAT;
    if (!inside(h->dir, uint64_t(kDirEntryBytes) * h->n_tensors, len) || !inside(h->names, h->names_bytes, len))
        return BS_E_FORMAT;
    return BS_OK;
}

bs_status check_entry(const uint8_t* d, uint64_t len, const HeaderInfo& h, Tensor* t, uint32_t* name_off,
                      uint32_t* name_len) {
    t->kind = d[0];
    t->ndim = d[1];
    t->log2_chunk = d[2];
    t->lanes = d[3];
    t->ns = d[4];
    t->nh = d[5];
    t->n_routes = d[6];
    t->nib_mode = d[7];
    *name_off = get_u32(d + 8);
    *name_len = get_u32(d + 12);
    t->n_elems = get_u64(d + 16);
    t->n_chunks = get_u64(d + 24);
    t->model_offset = get_u64(d + 32);
    t->model_bytes = get_u64(d + 40);
    t->data_offset = get_u64(d + 48);
    t->data_bytes = get_u64(d + 56);
    t->checksum = get_u64(d + 64);
    for (int i = 0; i < 8; ++i) t->shape[i] = get_u64(d + 80 + 8 * i);
    if (get_u64(d + 72) != 0 || t->kind > BS_KIND_JOINT || t->ndim > 8) return BS_E_FORMAT;
    if (!is_coded(t->kind) && t->nib_mode != 0) return BS_E_FORMAT;
    if (uint64_t(*name_off) + *name_len > h.names_bytes) return BS_E_FORMAT;
    unsigned __int128 prod = 1;
    for (uint32_t i = 0; i < t->ndim; ++i) {
        prod *= t->shape[i];
        if (prod > (static_cast<unsigned __int128>(1) << 64)) return BS_E_FORMAT;
    }
    for (uint32_t i = t->ndim; i < 8; ++i)
        if (t->shape[i] != 0) return BS_E_FORMAT;
    if (prod != t->n_elems) return BS_E_FORMAT;
    if (t->data_offset % 16 || !inside(t->data_offset, t->data_bytes, len)) return BS_E_FORMAT;
    if (!is_coded(t->kind)) { // STORED words or RAW bytes, verbatim
        if (t->kind == BS_KIND_STORED && t->n_elems > (1ull << 62)) return BS_E_FORMAT;
        const uint64_t want = t->kind == BS_KIND_STORED ? 2 * t->n_elems : t->n_elems;
        if (t->data_bytes != want) return BS_E_FORMAT;
        t->coded_bytes = want;
        return BS_OK;
    }
    const bool joint = t->kind == BS_KIND_JOINT;
    if (t->lanes != kLanes || t->log2_chunk < 8 || t->log2_chunk > 24) return BS_E_FORMAT;
    if (joint) {
        if (t->ns < kMinNj || t->ns > kMaxNj || t->nh != 0 || t->n_routes != 0) return BS_E_FORMAT;
    } else if (t->ns < 1 || t->ns > kMaxNs || t->nh < kMinNh || t->nh > kMaxNh || t->ns + t->nh > kMaxPrecision ||
               t->n_routes > kMaxRoutes) {
        return BS_E_FORMAT;
    }
    if (t->nib_mode != 0 && (t->nib_mode & 0xF0u) != 0x10u) return BS_E_FORMAT;
    if (t->n_elems == 0 || t->n_elems > (1ull << 40)) return BS_E_FORMAT;
    const uint64_t C = 1ull << t->log2_chunk;
    if (t->n_chunks != (t->n_elems + C - 1) / C || t->data_bytes != 16 * t->n_chunks) return BS_E_FORMAT;
    const uint64_t model_min = joint ? 8 : 264;
    const uint64_t model_max = joint ? 4 + 4 * kJointPairs : 260 + 4 * 512 + 16 * kMaxRoutes;
    if (t->model_offset % 16 || !inside(t->model_offset, t->model_bytes, len) || t->model_bytes < model_min ||
        t->model_bytes > model_max)
        return BS_E_FORMAT;
    return BS_OK;
}

bs_status check_model(const uint8_t* m, Tensor* t) {
    if (t->kind == BS_KIND_JOINT) { // n_pairs, reserved, then (j, Fj) with j ascending, sum 2^nj
        const uint32_t n_pairs = get_u16(m);
        if (n_pairs < 1 || n_pairs > kJointPairs || get_u16(m + 2) != 0) return BS_E_FORMAT;
        if (t->model_bytes != 4 + 4ull * n_pairs) return BS_E_FORMAT;
        uint64_t sumj = 0;
        uint32_t max_f = 0;
        int prevj = -1;
        for (uint32_t i = 0; i < n_pairs; ++i) {
            const int j = get_u16(m + 4 + 4 * i);
            const uint32_t q = get_u16(m + 6 + 4 * i);
            if (j <= prevj || j >= static_cast<int>(kJointPairs) || q == 0) return BS_E_FORMAT;
            prevj = j;
            sumj += q;
            max_f = std::max(max_f, q);
        }
        if (sumj != (1ull << t->ns)) return BS_E_FORMAT;
        t->joint_compact = max_f <= kCompactMaxF;
        t->table_bytes = t->joint_compact ? joint4_table_bytes(t->ns) : joint_table_bytes(t->ns);
        return BS_OK;
    }
    // RANS: n_present, reserved, (s, Fs) with s ascending and sum 2^ns, route[256], the
    // route tables over h (each sums to 2^nh)
    const uint32_t n_present = get_u16(m);
    if (n_present < 1 || n_present > 512 || get_u16(m + 2) != 0) return BS_E_FORMAT;
    if (t->model_bytes != 260 + 4ull * n_present + 16ull * t->n_routes) return BS_E_FORMAT;
    uint64_t sum = 0;
    int prev = -1;
    for (uint32_t i = 0; i < n_present; ++i) {
        const int s = get_u16(m + 4 + 4 * i);
        const uint32_t q = get_u16(m + 6 + 4 * i);
        if (s <= prev || s > 511 || q == 0) return BS_E_FORMAT;
        prev = s;
        sum += q;
    }
    if (sum != (1ull << t->ns)) return BS_E_FORMAT;
    const uint8_t* route = m + 4 + 4 * n_present;
    for (int e = 0; e < 256; ++e)
        if (route[e] != 0xFF && route[e] >= t->n_routes) return BS_E_FORMAT;
    for (uint32_t r = 0; r < t->n_routes; ++r) {
        sum = 0;
        for (int h = 0; h < 8; ++h) sum += get_u16(route + 256 + 16 * r + 2 * h);
        if (sum != (1ull << t->nh)) return BS_E_FORMAT;
    }
    t->table_bytes = table_bytes_for(t->ns, t->nh, t->n_routes);
    return BS_OK;
}

bs_status check_chunk_table(const uint8_t* ct, uint64_t len, Tensor* t) {
    const uint64_t C = 1ull << t->log2_chunk;
    t->coded_bytes = t->model_bytes + t->data_bytes;
    for (uint64_t c = 0; c < t->n_chunks; ++c) {
        const uint8_t* e = ct + 16 * c;
        const uint64_t off = get_u64(e);
        const uint32_t nw = get_u32(e + 8);
        const uint64_t nc = std::min<uint64_t>(C, t->n_elems - c * C);
        const uint64_t bytes = payload_bytes(nc, nw, t->nib_mode == 0);
        if (off % 16 || get_u32(e + 12) != 0 || !inside(off, bytes, len)) return BS_E_FORMAT;
        t->coded_bytes += bytes;
    }
    return BS_OK;
}

// Expand one coded tensor's model into its decode tables (layouts in bs_internal.h):
//  * RANS: the s-table, then the compact fraction rows with the UNIFORM row last;
//  * JOINT, 8-byte entries: .x = F | ((j << 4) << 16), .y = the slot's rank k within its pair;
//  * JOINT, 4-byte entries: (j << 4) | k << 16 | F << 24.
void build_tables(const Tensor& t, const uint8_t* m, uint8_t* dst) {
    if (t.kind == BS_KIND_JOINT) {
        const uint32_t n_pairs = get_u16(m);
        uint32_t* jt = reinterpret_cast<uint32_t*>(dst);
        uint32_t cum = 0;
        for (uint32_t i = 0; i < n_pairs; ++i) {
            const uint32_t j = get_u16(m + 4 + 4 * i), q = get_u16(m + 6 + 4 * i);
            for (uint32_t k = 0; k < q; ++k) {
                if (t.joint_compact) { // q <= 255, so k < 255
                    jt[cum + k] = (j << 4) | (k << 16) | (q << 24);
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

uint32_t decode_smem_bytes(DecodeMode mode, uint32_t warps, uint32_t chains, uint32_t s_region) {
    const uint32_t rings = warps * chains * (kRingBytes + kNibRingBytes);
    switch (mode) {
    case DecodeMode::JointCompact: return kJoint4Region + rings;
    case DecodeMode::Joint:
    case DecodeMode::JointGeneric: return kJointRegion + rings;
    default: return kHRegion + s_region + rings;
    }
}

} // namespace bs
