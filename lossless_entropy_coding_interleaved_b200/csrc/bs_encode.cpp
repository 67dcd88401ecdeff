// bs_encode.cpp -- host side of the device encoder (include/bs.h, bs_encoder_*).
//
// It implements the container's integer encoder rules (quantiser, route rule, joint model, pad word, STORED
// fallback)
// and the canonical layout of section 4.6 from that document. It shares no code with the
// oracle. The statistics come from histogram_kernel and the per-chunk word counts from the
// count pass of encode_kernel (bs_encode_kernels.cu). The write pass then places every
// chunk at its final offset.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <memory>
#include <new>
#include <string>
#include <vector>

#include "bs_internal.h"

using namespace bs;

namespace {

bs_status enc_cuda(cudaError_t e) {
    record_cuda_error(static_cast<int>(e));
    return BS_E_CUDA;
}

uint64_t up16(uint64_t v) { return (v + 15) & ~uint64_t(15); }
uint64_t up256(uint64_t v) { return (v + 255) & ~uint64_t(255); }
void put_u64(uint8_t* p, uint64_t v) { std::memcpy(p, &v, 8); }
void put_u32(uint8_t* p, uint32_t v) { std::memcpy(p, &v, 4); }
void put_u16(uint8_t* p, uint16_t v) { std::memcpy(p, &v, 2); }

// Quantiser: proportional rounding with a floor of one slot per present
// symbol, then one-slot moves in the direction of the sum, chosen by the first-order change
// of sum(c * log q) (c/(2q+1) to add, c/(2q-1) to remove), lowest index on ties.
bool quantise(const uint64_t* c, int K, uint32_t M, uint32_t* q) {
    uint64_t n = 0;
    int present = 0;
    for (int k = 0; k < K; ++k) {
        n += c[k];
        present += c[k] != 0;
    }
    if (n == 0 || static_cast<uint64_t>(present) > M) return false;
    using u128 = unsigned __int128;
    int64_t total = 0;
    for (int k = 0; k < K; ++k) {
        if (!c[k]) {
            q[k] = 0;
            continue;
        }
        const uint64_t r = static_cast<uint64_t>((u128(2) * c[k] * M + n) / (u128(2) * n));
        q[k] = static_cast<uint32_t>(std::max<uint64_t>(1, r));
        total += q[k];
    }
    // a/b > c/d for positive b, d
    auto gt = [](uint64_t a, uint64_t b, uint64_t cc, uint64_t d) { return u128(a) * d > u128(cc) * b; };
    while (total < static_cast<int64_t>(M)) {
        int best = -1;
        for (int k = 0; k < K; ++k)
            if (c[k] && (best < 0 || gt(c[k], 2ull * q[k] + 1, c[best], 2ull * q[best] + 1))) best = k;
        ++q[best];
        ++total;
    }
    while (total > static_cast<int64_t>(M)) {
        int best = -1;
        for (int k = 0; k < K; ++k)
            if (c[k] && q[k] >= 2 && (best < 0 || gt(c[best], 2ull * q[best] - 1, c[k], 2ull * q[k] - 1))) best = k;
        if (best < 0) return false;
        --q[best];
        --total;
    }
    return true;
}

// Routes: Pearson's statistic of the fraction's top three bits against
// the uniform distribution, chi2 * n_e = 8 * sum c^2 - n_e^2. Exponents with chi2 > 256
// compete, the largest chi2 (lower exponent on ties) win up to max_routes, numbered in
// ascending exponent.
void choose_routes(const uint64_t* ceh, uint32_t max_routes, uint8_t* route, std::vector<int>& route_e) {
    using u128 = unsigned __int128;
    u128 num[256];
    uint64_t ne[256];
    bool cand[256], taken[256];
    for (int e = 0; e < 256; ++e) {
        u128 sq = 0;
        uint64_t n = 0;
        for (int h = 0; h < 8; ++h) {
            n += ceh[e * 8 + h];
            sq += u128(ceh[e * 8 + h]) * ceh[e * 8 + h];
        }
        ne[e] = n;
        num[e] = u128(8) * sq - u128(n) * n;
        cand[e] = n > 0 && num[e] > u128(256) * n;
        taken[e] = false;
        route[e] = 0xFF;
    }
    for (uint32_t r = 0; r < max_routes; ++r) {
        int best = -1;
        for (int e = 0; e < 256; ++e) {
            if (!cand[e] || taken[e]) continue;
            if (best < 0 || num[e] * ne[best] > num[best] * ne[e]) best = e;
        }
        if (best < 0) break;
        taken[best] = true;
    }
    route_e.clear();
    for (int e = 0; e < 256; ++e)
        if (taken[e]) {
            route[e] = static_cast<uint8_t>(route_e.size());
            route_e.push_back(e);
        }
}

struct EncTensor {
    bs_enc_item item{};
    std::string name;
    uint32_t kind = BS_KIND_STORED; // decided in run
    bool candidate = false;         // a BF16 tensor with weights: try RANS
    uint64_t n_chunks = 0;
    uint32_t n_routes = 0;
    uint32_t nib_mode = 0;          // 0 = stored nibble words, 0x10 + c = every low nibble is c
    uint16_t pad_word = 0;
    std::vector<uint8_t> model;     // the serialised model section
    std::vector<uint32_t> tables;   // encode tables (bs_internal.h)
    std::vector<uint32_t> n_words;  // per chunk, from the count pass
    uint64_t checksum = 0;
    uint64_t coded = 0;
    // layout
    uint64_t model_offset = 0, data_offset = 0;
    std::vector<uint64_t> chunk_off;
    // scratch placement
    uint64_t sc_tables = 0, sc_words = 0, sc_offs = 0;
};

} // namespace

struct bs_encoder_t {
    bs_enc_params prm{};
    std::vector<EncTensor> t;
    uint64_t sc_hist = 0, sc_err = 0, sc_sums = 0, sc_total = 0;
    bool ran = false;
    uint64_t total_bytes = 0, dir_offset = 0, names_offset = 0, names_bytes = 0;
};

namespace {

// Build the model bytes and the encode tables of one tensor from its histogram (pair
// counts j = (s << 3) | h, then low-nibble counts).
bool build_model(EncTensor& T, const bs_enc_params& P, const unsigned long long* hist) {
    const unsigned long long* cnib = hist + 4096;
    // nibble mode: constant when only one low nibble occurs
    int seen = 0, only = 0;
    for (int u = 0; u < 16; ++u)
        if (cnib[u]) {
            ++seen;
            only = u;
        }
    T.nib_mode = seen == 1 ? 0x10u | static_cast<uint32_t>(only) : 0u;
    if (P.model == 1) { // joint model: Fj = quantise(pair counts, 2^nj); the pad pair has the largest Fj
        std::vector<uint64_t> cj(hist, hist + kJointPairs);
        std::vector<uint32_t> Fj(kJointPairs);
        if (!quantise(cj.data(), kJointPairs, 1u << P.nj, Fj.data())) return false;
        uint32_t j_pad = 0, n_pairs = 0;
        for (uint32_t j = 0; j < kJointPairs; ++j) {
            if (Fj[j] > Fj[j_pad]) j_pad = j;
            n_pairs += Fj[j] != 0;
        }
        T.pad_word = static_cast<uint16_t>(j_pad << 4);
        T.n_routes = 0;
        T.model.assign(4 + 4ull * n_pairs, 0); // n_pairs, reserved, then (j, Fj) pairs
        uint8_t* m = T.model.data();
        put_u16(m, static_cast<uint16_t>(n_pairs));
        uint64_t o = 4;
        T.tables.assign(kEncJointWords, 0);
        uint32_t cum = 0;
        for (uint32_t j = 0; j < kJointPairs; ++j) {
            T.tables[j] = Fj[j] | (cum << 16);
            cum += Fj[j];
            if (Fj[j]) {
                put_u16(m + o, static_cast<uint16_t>(j));
                put_u16(m + o + 2, static_cast<uint16_t>(Fj[j]));
                o += 4;
            }
        }
        return true;
    }
    uint64_t cs[512] = {}, ceh[256 * 8] = {};
    for (uint32_t j = 0; j < kJointPairs; ++j) {
        cs[j >> 3] += hist[j];
        ceh[((j >> 3) & 0xFFu) * 8 + (j & 7u)] += hist[j]; // the sign is folded
    }
    uint32_t Fs[512];
    if (!quantise(cs, 512, 1u << P.ns, Fs)) return false;
    uint8_t route[256];
    std::vector<int> route_e;
    choose_routes(ceh, P.max_routes, route, route_e);
    const uint32_t R = static_cast<uint32_t>(route_e.size());
    std::vector<uint32_t> Fh(8 * R);
    for (uint32_t r = 0; r < R; ++r)
        if (!quantise(ceh + 8 * route_e[r], 8, 1u << P.nh, Fh.data() + 8 * r)) return false;
    T.n_routes = R;
    // pad word: most frequent s (lowest on ties), then its table's most frequent h
    int s_pad = 0;
    for (int s = 1; s < 512; ++s)
        if (cs[s] > cs[s_pad]) s_pad = s;
    int h_pad = 0;
    if (route[s_pad & 0xFF] != 0xFF) {
        const uint32_t* row = Fh.data() + 8 * route[s_pad & 0xFF];
        for (int h = 1; h < 8; ++h)
            if (row[h] > row[h_pad]) h_pad = h;
    }
    T.pad_word = static_cast<uint16_t>((s_pad << 7) | (h_pad << 4));
    // model bytes: n_present, reserved, (s, Fs) pairs, route[256], the route tables
    uint32_t n_present = 0;
    for (int s = 0; s < 512; ++s) n_present += Fs[s] != 0;
    T.model.assign(260 + 4ull * n_present + 16ull * R, 0);
    uint8_t* m = T.model.data();
    put_u16(m, static_cast<uint16_t>(n_present));
    uint64_t o = 4;
    for (int s = 0; s < 512; ++s)
        if (Fs[s]) {
            put_u16(m + o, static_cast<uint16_t>(s));
            put_u16(m + o + 2, static_cast<uint16_t>(Fs[s]));
            o += 4;
        }
    std::memcpy(m + o, route, 256);
    o += 256;
    for (uint32_t k = 0; k < 8 * R; ++k, o += 2) put_u16(m + o, static_cast<uint16_t>(Fh[k]));
    // encode tables
    T.tables.assign(enc_table_words(R), 0);
    uint32_t cum = 0;
    for (int s = 0; s < 512; ++s) {
        T.tables[s] = Fs[s] | (cum << 16);
        cum += Fs[s];
    }
    const uint32_t Mh = 1u << P.nh;
    for (uint32_t r = 0; r <= R; ++r) {
        cum = 0;
        for (int h = 0; h < 8; ++h) {
            const uint32_t q = r == R ? Mh / 8 : Fh[8 * r + h];
            T.tables[512 + 8 * r + h] = q | (cum << 16);
            cum += q;
        }
    }
    uint8_t* rt = reinterpret_cast<uint8_t*>(T.tables.data() + 512 + 8 * (R + 1));
    for (int e = 0; e < 256; ++e) rt[e] = route[e] == 0xFF ? static_cast<uint8_t>(R) : route[e];
    return true;
}

template <class F>
bs_status run_encode_launches(bs_encoder_t* enc, uint8_t* d_scratch, uint8_t* d_container, uint32_t write,
                              void* stream, F&& want) {
    std::unique_ptr<EncParams> p(new (std::nothrow) EncParams);
    if (!p) return BS_E_NOMEM;
    p->n_items = 0;
    p->total_ctas = 0;
    p->write = write;
    p->container = d_container;
    p->err = reinterpret_cast<unsigned int*>(d_scratch + enc->sc_err);
    auto flush = [&]() -> bs_status {
        if (!p->n_items) return BS_OK;
        const int e = launch_encode(*p, stream);
        p->n_items = 0;
        p->total_ctas = 0;
        return e ? enc_cuda(static_cast<cudaError_t>(e)) : BS_OK;
    };
    for (EncTensor& T : enc->t) {
        if (!want(T)) continue;
        const uint64_t ctas = (T.n_chunks + kEncWarps - 1) / kEncWarps;
        if (p->n_items == kMaxEncItems || p->total_ctas + ctas > 0x7FFFFFFFull) {
            bs_status s = flush();
            if (s) return s;
        }
        EncItem& it = p->item[p->n_items++];
        std::memset(&it, 0, sizeof(it));
        it.in = static_cast<const uint16_t*>(T.item.d_data);
        it.tables = reinterpret_cast<const uint32_t*>(d_scratch + T.sc_tables);
        it.n_words = reinterpret_cast<uint32_t*>(d_scratch + T.sc_words);
        it.chunk_off = reinterpret_cast<const uint64_t*>(d_scratch + T.sc_offs);
        it.n_elems = T.item.n_elems;
        it.cta_begin = p->total_ctas;
        it.table_words = static_cast<uint32_t>(T.tables.size());
        it.pad_word = T.pad_word;
        const bool joint = enc->prm.model == 1;
        it.log2_chunk = static_cast<uint8_t>(enc->prm.log2_chunk);
        it.ns = static_cast<uint8_t>(joint ? enc->prm.nj : enc->prm.ns);
        it.nh = static_cast<uint8_t>(joint ? 0 : enc->prm.nh);
        it.n_routes = static_cast<uint8_t>(T.n_routes);
        it.nib_stored = T.nib_mode == 0;
        it.joint = joint;
        p->total_ctas += static_cast<uint32_t>(ctas);
    }
    return flush();
}

} // namespace

extern "C" {

bs_status bs_encoder_create(const bs_enc_item* items, int32_t n, const bs_enc_params* prm, bs_encoder_t** out) {
    if (!out || n < 0 || (n && !items) || !prm) return BS_E_ARG;
    *out = nullptr;
    const bs_enc_params& P = *prm;
    if (P.log2_chunk < 8 || P.log2_chunk > 24 || P.ns < 1 || P.ns > kMaxNs || P.nh < kMinNh || P.nh > kMaxNh ||
        P.ns + P.nh > kMaxPrecision || P.max_routes > kMaxRoutes || P.model > 1 ||
        (P.model == 1 && (P.nj < kMinNj || P.nj > kMaxNj)))
        return BS_E_ARG;
    std::unique_ptr<bs_encoder_t> enc(new (std::nothrow) bs_encoder_t);
    if (!enc) return BS_E_NOMEM;
    enc->prm = P;
    try {
        enc->t.resize(n);
    } catch (...) {
        return BS_E_NOMEM;
    }
    uint64_t sc = 0;
    enc->sc_hist = sc;
    sc += up256(8ull * kHistBins);
    enc->sc_err = sc;
    sc += 256;
    enc->sc_sums = sc;
    sc += up256(8ull * n);
    for (int32_t k = 0; k < n; ++k) {
        const bs_enc_item& it = items[k];
        EncTensor& T = enc->t[k];
        T.item = it;
        if (it.ndim > 8 || (it.kind != 0 && it.kind != 2) || (it.n_elems && !it.d_data) ||
            (it.name_bytes && !it.name))
            return BS_E_ARG;
        unsigned __int128 prod = 1;
        for (uint32_t d = 0; d < it.ndim; ++d) prod *= it.shape[d];
        if (prod != it.n_elems) return BS_E_ARG;
        T.name.assign(it.name ? it.name : "", it.name_bytes);
        T.item.name = nullptr;
        if (it.kind == 2) {
            T.kind = BS_KIND_RAW;
            continue;
        }
        if (it.n_elems > (1ull << 40)) return BS_E_ARG;
        if (reinterpret_cast<uintptr_t>(it.d_data) & 15u) return BS_E_ARG;
        T.kind = BS_KIND_STORED;
        T.candidate = it.n_elems > 0;
        if (!T.candidate) continue;
        T.n_chunks = (it.n_elems + (1ull << P.log2_chunk) - 1) >> P.log2_chunk;
        T.sc_tables = sc;
        sc += up256(4ull * kEncTableWordsMax);
        T.sc_words = sc;
        sc += up256(4ull * T.n_chunks);
        T.sc_offs = sc;
        sc += up256(8ull * T.n_chunks);
    }
    enc->sc_total = sc;
    *out = enc.release();
    return BS_OK;
}

bs_status bs_encoder_scratch_bytes(const bs_encoder_t* enc, size_t* bytes) {
    if (!enc || !bytes) return BS_E_ARG;
    *bytes = enc->sc_total;
    return BS_OK;
}

bs_status bs_encoder_run(bs_encoder_t* enc, void* d_scratch_v, size_t scratch_bytes, void* stream,
                         size_t* container_bytes) {
    if (!enc || !d_scratch_v || !container_bytes || scratch_bytes < enc->sc_total) return BS_E_ARG;
    if (reinterpret_cast<uintptr_t>(d_scratch_v) & 255u) return BS_E_ARG;
    uint8_t* d_scratch = static_cast<uint8_t*>(d_scratch_v);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bs_enc_params& P = enc->prm;
    std::vector<unsigned long long> hist(kHistBins);
    auto* d_hist = reinterpret_cast<unsigned long long*>(d_scratch + enc->sc_hist);
    auto* d_sums = reinterpret_cast<unsigned long long*>(d_scratch + enc->sc_sums);
    cudaError_t ce = cudaMemsetAsync(d_scratch + enc->sc_err, 0, 256, s);
    if (ce != cudaSuccess) return enc_cuda(ce);
    for (size_t k = 0; k < enc->t.size(); ++k) {
        EncTensor& T = enc->t[k];
        int e = launch_checksum(T.item.d_data, T.item.n_elems, T.kind == BS_KIND_RAW, d_sums + k, stream);
        if (e) return enc_cuda(static_cast<cudaError_t>(e));
        if (!T.candidate) continue;
        e = launch_histogram(static_cast<const uint16_t*>(T.item.d_data), T.item.n_elems, d_hist, stream);
        if (e) return enc_cuda(static_cast<cudaError_t>(e));
        ce = cudaMemcpyAsync(hist.data(), d_hist, 8ull * kHistBins, cudaMemcpyDeviceToHost, s);
        if (ce == cudaSuccess) ce = cudaStreamSynchronize(s);
        if (ce != cudaSuccess) return enc_cuda(ce);
        if (P.model == 1) { // more distinct pairs than 2^nj slots: no JOINT table, so STORED
            uint32_t n_pairs = 0;
            for (uint32_t j = 0; j < kJointPairs; ++j) n_pairs += hist[j] != 0;
            if (n_pairs > (1u << P.nj)) {
                T.candidate = false;
                T.kind = BS_KIND_STORED;
                continue;
            }
        }
        if (!build_model(T, P, hist.data())) return BS_E_ARG;
        ce = cudaMemcpyAsync(d_scratch + T.sc_tables, T.tables.data(), 4ull * T.tables.size(), cudaMemcpyHostToDevice, s);
        if (ce != cudaSuccess) return enc_cuda(ce);
        ce = cudaStreamSynchronize(s); // T.tables must outlive the copy; it does, but keep the order plain
        if (ce != cudaSuccess) return enc_cuda(ce);
    }
    // count pass
    bs_status st = run_encode_launches(enc, d_scratch, nullptr, 0, stream, [](const EncTensor& T) { return T.candidate; });
    if (st) return st;
    std::vector<unsigned long long> sums(enc->t.size());
    if (!sums.empty()) {
        ce = cudaMemcpyAsync(sums.data(), d_sums, 8ull * sums.size(), cudaMemcpyDeviceToHost, s);
        if (ce != cudaSuccess) return enc_cuda(ce);
    }
    for (EncTensor& T : enc->t) {
        if (!T.candidate) continue;
        T.n_words.resize(T.n_chunks);
        ce = cudaMemcpyAsync(T.n_words.data(), d_scratch + T.sc_words, 4ull * T.n_chunks, cudaMemcpyDeviceToHost, s);
        if (ce != cudaSuccess) return enc_cuda(ce);
    }
    ce = cudaStreamSynchronize(s);
    if (ce != cudaSuccess) return enc_cuda(ce);
    // STORED fallback and canonical layout (header, directory, names, then each tensor's sections)
    uint64_t names_bytes = 0;
    for (size_t k = 0; k < enc->t.size(); ++k) {
        EncTensor& T = enc->t[k];
        T.checksum = sums[k];
        names_bytes += T.name.size();
        if (!T.candidate) continue;
        T.coded = T.model.size() + 16 * T.n_chunks;
        const uint64_t C = 1ull << P.log2_chunk;
        for (uint64_t c = 0; c < T.n_chunks; ++c)
            T.coded += payload_bytes(std::min(C, T.item.n_elems - c * C), T.n_words[c], T.nib_mode == 0);
        T.kind = (!P.force_rans && T.coded >= 2 * T.item.n_elems) ? BS_KIND_STORED
                 : P.model == 1                                       ? BS_KIND_JOINT
                                                                      : BS_KIND_RANS;
    }
    enc->dir_offset = kHeaderBytes;
    enc->names_offset = up16(enc->dir_offset + uint64_t(kDirEntryBytes) * enc->t.size());
    enc->names_bytes = names_bytes;
    uint64_t pos = up16(enc->names_offset + names_bytes);
    for (EncTensor& T : enc->t) {
        if (is_coded(T.kind)) {
            T.model_offset = pos;
            pos = up16(pos + T.model.size());
            T.data_offset = pos;
            pos = up16(pos + 16 * T.n_chunks);
            T.chunk_off.resize(T.n_chunks);
            const uint64_t C = 1ull << enc->prm.log2_chunk;
            for (uint64_t c = 0; c < T.n_chunks; ++c) {
                T.chunk_off[c] = pos;
                pos += payload_bytes(std::min(C, T.item.n_elems - c * C), T.n_words[c], T.nib_mode == 0);
            }
        } else {
            const uint64_t bytes = T.kind == BS_KIND_STORED ? 2 * T.item.n_elems : T.item.n_elems;
            T.data_offset = pos;
            pos = up16(pos + bytes);
        }
    }
    enc->total_bytes = pos;
    enc->ran = true;
    *container_bytes = pos;
    return BS_OK;
}

bs_status bs_encoder_emit(bs_encoder_t* enc, void* d_scratch_v, void* d_container_v, size_t container_bytes,
                          void* h_container, void* stream) {
    if (!enc || !enc->ran || !d_scratch_v || !d_container_v || container_bytes != enc->total_bytes) return BS_E_ARG;
    if (reinterpret_cast<uintptr_t>(d_container_v) & 15u) return BS_E_ARG;
    uint8_t* d_scratch = static_cast<uint8_t*>(d_scratch_v);
    uint8_t* d_container = static_cast<uint8_t*>(d_container_v);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bs_enc_params& P = enc->prm;
    cudaError_t ce = cudaMemsetAsync(d_container, 0, container_bytes, s);
    if (ce != cudaSuccess) return enc_cuda(ce);
    // chunk offsets for the write pass
    for (EncTensor& T : enc->t) {
        if (!is_coded(T.kind)) continue;
        ce = cudaMemcpyAsync(d_scratch + T.sc_offs, T.chunk_off.data(), 8ull * T.n_chunks, cudaMemcpyHostToDevice, s);
        if (ce != cudaSuccess) return enc_cuda(ce);
    }
    bs_status st = run_encode_launches(enc, d_scratch, d_container, 1, stream,
                                       [](const EncTensor& T) { return is_coded(T.kind); });
    if (st) return st;
    // verbatim data
    for (EncTensor& T : enc->t) {
        if (is_coded(T.kind) || T.item.n_elems == 0) continue;
        const uint64_t bytes = T.kind == BS_KIND_STORED ? 2 * T.item.n_elems : T.item.n_elems;
        ce = cudaMemcpyAsync(d_container + T.data_offset, T.item.d_data, bytes, cudaMemcpyDeviceToDevice, s);
        if (ce != cudaSuccess) return enc_cuda(ce);
    }
    // metadata: header, directory and names in one block; model + chunk table per RANS tensor
    std::vector<uint8_t> head(enc->names_offset + enc->names_bytes, 0);
    uint8_t* h = head.data();
    std::memcpy(h, "BF16RANS", 8);
    put_u32(h + 8, kFormatVersion);
    put_u32(h + 12, kHeaderBytes);
    put_u32(h + 16, static_cast<uint32_t>(enc->t.size()));
    put_u32(h + 20, kDirEntryBytes);
    put_u64(h + 24, enc->dir_offset);
    put_u64(h + 32, enc->names_offset);
    put_u64(h + 40, enc->names_bytes);
    put_u64(h + 48, enc->total_bytes);
    uint64_t name_pos = 0;
    std::vector<std::vector<uint8_t>> meta(enc->t.size());
    for (size_t k = 0; k < enc->t.size(); ++k) {
        EncTensor& T = enc->t[k];
        uint8_t* d = h + enc->dir_offset + uint64_t(kDirEntryBytes) * k;
        d[0] = static_cast<uint8_t>(T.kind);
        d[1] = static_cast<uint8_t>(T.item.ndim);
        put_u32(d + 8, static_cast<uint32_t>(name_pos));
        put_u32(d + 12, static_cast<uint32_t>(T.name.size()));
        put_u64(d + 16, T.item.n_elems);
        put_u64(d + 48, T.data_offset);
        put_u64(d + 64, T.checksum);
        for (uint32_t i = 0; i < T.item.ndim; ++i) put_u64(d + 80 + 8 * i, T.item.shape[i]);
        std::memcpy(h + enc->names_offset + name_pos, T.name.data(), T.name.size());
        name_pos += T.name.size();
        if (is_coded(T.kind)) {
            d[2] = static_cast<uint8_t>(P.log2_chunk);
            d[3] = kLanes;
            d[4] = static_cast<uint8_t>(T.kind == BS_KIND_JOINT ? P.nj : P.ns);
            d[5] = static_cast<uint8_t>(T.kind == BS_KIND_JOINT ? 0 : P.nh);
            d[6] = static_cast<uint8_t>(T.n_routes);
            d[7] = static_cast<uint8_t>(T.nib_mode);
            put_u64(d + 24, T.n_chunks);
            put_u64(d + 32, T.model_offset);
            put_u64(d + 40, T.model.size());
            put_u64(d + 56, 16 * T.n_chunks);
            // model, padding, chunk table: contiguous from model_offset
            std::vector<uint8_t>& mb = meta[k];
            mb.assign(T.data_offset - T.model_offset + 16 * T.n_chunks, 0);
            std::memcpy(mb.data(), T.model.data(), T.model.size());
            uint8_t* tab = mb.data() + (T.data_offset - T.model_offset);
            for (uint64_t c = 0; c < T.n_chunks; ++c) {
                put_u64(tab + 16 * c, T.chunk_off[c]);
                put_u32(tab + 16 * c + 8, T.n_words[c]);
            }
            ce = cudaMemcpyAsync(d_container + T.model_offset, mb.data(), mb.size(), cudaMemcpyHostToDevice, s);
            if (ce != cudaSuccess) return enc_cuda(ce);
        } else {
            put_u64(d + 56, T.kind == BS_KIND_STORED ? 2 * T.item.n_elems : T.item.n_elems);
        }
    }
    ce = cudaMemcpyAsync(d_container, head.data(), head.size(), cudaMemcpyHostToDevice, s);
    if (ce != cudaSuccess) return enc_cuda(ce);
    unsigned int err = 0;
    ce = cudaMemcpyAsync(&err, d_scratch + enc->sc_err, 4, cudaMemcpyDeviceToHost, s);
    if (ce == cudaSuccess && h_container)
        ce = cudaMemcpyAsync(h_container, d_container, container_bytes, cudaMemcpyDeviceToHost, s);
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(s);
    if (ce != cudaSuccess) return enc_cuda(ce);
    return err ? BS_E_CORRUPT : BS_OK;
}

void bs_encoder_destroy(bs_encoder_t* enc) { delete enc; }

} // extern "C"
