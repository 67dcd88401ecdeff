// bs_stream.cpp -- layer streaming. Groups of tensors (for example the layers of a
// checkpoint) are decoded on demand from a container held in host memory into a device
// cache that lives in an arena the caller provides. It is the device-side counterpart of
// the low-VRAM streaming loader on the "Gemma 2 9B Instruct -- Lossless Compressed" card
// (section "Low-VRAM streaming": decode layer by layer under an LRU cap on device memory).
//
// Arena layout: two staging slots of stage_bytes each, then the cache. Loading a group
// takes three steps, all on one stream:
//  1. copy the group's compressed byte range host-to-device into the next staging slot;
//  2. decode it, with the kernels bs_decode_batch uses, into a cache block;
//  3. record the group's `ready` event and the slot's `done` event.
// The cache is managed first-fit. When room is needed, unpinned groups leave it in
// least-recently-used order, except that a prefetched group is kept until it has been
// acquired once (it goes only when nothing else can). Groups between acquire and release
// are pinned.
//
// Ordering uses CUDA events only, so no call blocks the host:
//  * an evicted block is reused after the evicted group's `released` event, which follows
//    the consumer's last use. A group that was never acquired waits on its `ready` event.
//  * a staging slot is refilled after its `done` event, which follows the decode that read it.
//  * acquire makes the consumer's stream wait for the group's `ready` event.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <map>
#include <memory>
#include <mutex>
#include <new>
#include <vector>

#include "bs_host.h"

using namespace bs;

namespace {

bs_status cuda_err(cudaError_t e) { return cuda_status(static_cast<int>(e)); }

// First-fit allocator over [0, size) in 256-byte units.
class Arena {
  public:
    explicit Arena(uint64_t size) {
        if (size) free_[0] = size;
    }
    // The block's offset, or UINT64_MAX when no free block is large enough.
    uint64_t alloc(uint64_t bytes) {
        bytes = up256(bytes);
        for (auto it = free_.begin(); it != free_.end(); ++it) {
            if (it->second < bytes) continue;
            const uint64_t off = it->first, rest = it->second - bytes;
            free_.erase(it);
            if (rest) free_[off + bytes] = rest;
            used_ += bytes;
            return off;
        }
        return UINT64_MAX;
    }
    void release(uint64_t off, uint64_t bytes) {
        bytes = up256(bytes);
        used_ -= bytes;
        auto it = free_.emplace(off, bytes).first;
        auto next = std::next(it);
        if (next != free_.end() && it->first + it->second == next->first) {
            it->second += next->second;
            free_.erase(next);
        }
        if (it != free_.begin()) {
            auto prev = std::prev(it);
            if (prev->first + prev->second == it->first) {
                prev->second += it->second;
                free_.erase(it);
            }
        }
    }
    uint64_t used() const { return used_; }

  private:
    std::map<uint64_t, uint64_t> free_; // offset -> bytes; no two blocks are adjacent
    uint64_t used_ = 0;
};

struct Group {
    std::vector<int32_t> tensors;  // ascending tensor index
    std::vector<uint64_t> out_off; // each tensor's output offset inside the group's block
    uint64_t c_begin = 0, c_end = 0, out_bytes = 0;
    bool resident = false;
    uint64_t block = 0; // cache offset of the decoded block
    int pins = 0;
    bool fresh = false; // loaded by prefetch and not acquired since
    uint64_t last_use = 0;
    cudaEvent_t ready = nullptr, released = nullptr;
    bool released_recorded = false;
};

uint64_t out_bytes_of(const Tensor& t) { return t.kind == BS_KIND_RAW ? t.n_elems : 2 * t.n_elems; }

// The container bytes that tensor t's decode reads: [begin, end), begin 16-byte aligned.
// For RANS and JOINT: the chunk table and each chunk's payload: states, nibble words and words (the
// model is expanded into the workspace at create time and is not read again).
void coded_range(const Tensor& t, const uint8_t* h, uint64_t* begin, uint64_t* end) {
    uint64_t b = t.data_offset, e = t.data_offset + t.data_bytes;
    if (is_coded(t.kind)) {
        const uint64_t C = 1ull << t.log2_chunk;
        for (uint64_t c = 0; c < t.n_chunks; ++c) {
            uint64_t off;
            uint32_t nw;
            std::memcpy(&off, h + t.data_offset + 16 * c, 8);
            std::memcpy(&nw, h + t.data_offset + 16 * c + 8, 4);
            b = std::min(b, off);
            e = std::max<uint64_t>(e, off + payload_bytes(std::min(C, t.n_elems - c * C), nw, t.nib_mode == 0));
        }
    }
    *begin = b & ~uint64_t(15);
    *end = e;
}

// Groups from the caller's tensor -> group map. Group numbers must be 0..G-1, each used.
bs_status make_groups(const std::vector<Tensor>& ts, const uint8_t* h, const int32_t* group_of_tensor,
                      std::vector<Group>& groups, uint64_t* max_stage, uint64_t* max_out) {
    int32_t n_groups = 0;
    for (size_t k = 0; k < ts.size(); ++k) {
        if (group_of_tensor[k] < 0 || group_of_tensor[k] >= static_cast<int32_t>(ts.size())) return BS_E_ARG;
        n_groups = std::max(n_groups, group_of_tensor[k] + 1);
    }
    groups.clear();
    groups.resize(n_groups);
    for (size_t k = 0; k < ts.size(); ++k) {
        Group& g = groups[group_of_tensor[k]];
        uint64_t b, e;
        coded_range(ts[k], h, &b, &e);
        if (e > b) {
            const bool first = g.c_end == g.c_begin;
            g.c_begin = first ? b : std::min(g.c_begin, b);
            g.c_end = first ? e : std::max(g.c_end, e);
        }
        g.tensors.push_back(static_cast<int32_t>(k));
        g.out_off.push_back(g.out_bytes);
        g.out_bytes += up256(out_bytes_of(ts[k]));
    }
    *max_stage = *max_out = 0;
    for (Group& g : groups) {
        if (g.tensors.empty()) return BS_E_ARG;
        *max_stage = std::max(*max_stage, up256(g.c_end - g.c_begin));
        *max_out = std::max(*max_out, up256(g.out_bytes));
    }
    return BS_OK;
}

} // namespace

struct bs_streamer_t {
    std::vector<Tensor> tensors;
    std::vector<Group> groups;
    const uint8_t* h = nullptr;
    uint8_t* d_ws = nullptr;
    uint8_t* d_arena = nullptr;
    uint64_t stage_bytes = 0; // one staging slot
    std::unique_ptr<Arena> cache;
    std::unique_ptr<DecodeBatch> batch;
    cudaEvent_t stage_done[2] = {nullptr, nullptr};
    bool stage_used[2] = {false, false};
    int next_stage = 0;
    uint64_t tick = 0;
    bs_streamer_stats_t st{};
    std::mutex mu;
    ~bs_streamer_t() {
        for (Group& g : groups) {
            if (g.ready) cudaEventDestroy(g.ready);
            if (g.released) cudaEventDestroy(g.released);
        }
        for (cudaEvent_t e : stage_done)
            if (e) cudaEventDestroy(e);
    }
    uint8_t* cache_base() const { return d_arena + 2 * stage_bytes; }
};

namespace {

// A cache block of `bytes`, evicting unpinned groups until one fits: first the least
// recently used among those acquired since they were loaded, then prefetched groups not yet
// acquired (oldest first). Stream s waits for each evicted group's last use. UINT64_MAX
// when pinned groups leave no room.
uint64_t cache_alloc(bs_streamer_t* S, uint64_t bytes, cudaStream_t s, cudaError_t* ce) {
    *ce = cudaSuccess;
    for (;;) {
        const uint64_t off = S->cache->alloc(bytes);
        if (off != UINT64_MAX) return off;
        Group* victim = nullptr;
        for (Group& g : S->groups)
            if (g.resident && g.pins == 0 &&
                (!victim || g.fresh < victim->fresh || (g.fresh == victim->fresh && g.last_use < victim->last_use)))
                victim = &g;
        if (!victim) return UINT64_MAX;
        *ce = cudaStreamWaitEvent(s, victim->released_recorded ? victim->released : victim->ready, 0);
        if (*ce != cudaSuccess) return UINT64_MAX;
        S->cache->release(victim->block, victim->out_bytes);
        victim->resident = false;
        victim->released_recorded = false;
        ++S->st.evictions;
        --S->st.resident_groups;
    }
}

// Stage group g's compressed bytes and decode them into a new cache block, on stream s.
bs_status load_group(bs_streamer_t* S, Group& g, cudaStream_t s) {
    cudaError_t ce;
    const uint64_t block = cache_alloc(S, g.out_bytes, s, &ce);
    if (ce != cudaSuccess) return cuda_err(ce);
    if (block == UINT64_MAX) return BS_E_SIZE;
    const int slot = S->next_stage;
    if (S->stage_used[slot]) {
        ce = cudaStreamWaitEvent(s, S->stage_done[slot], 0);
        if (ce != cudaSuccess) {
            S->cache->release(block, g.out_bytes); // nothing was queued
            return cuda_err(ce);
        }
    }
    // From here on work may be queued into the slot and the block. On failure the block is
    // not given back (a later group could be decoded into it while this work still runs),
    // and the slot counts as used.
    S->next_stage ^= 1;
    S->stage_used[slot] = true;
    uint8_t* stage = S->d_arena + slot * S->stage_bytes;
    const uint64_t cb = g.c_end - g.c_begin;
    if (cb) {
        ce = cudaMemcpyAsync(stage, S->h + g.c_begin, cb, cudaMemcpyHostToDevice, s);
        if (ce != cudaSuccess) return cuda_err(ce);
    }
    // The slot stands in for the container: container offset o is read at base + o, for
    // every o in [c_begin, c_end), which holds all the bytes this group's decode reads.
    const uint8_t* base = reinterpret_cast<const uint8_t*>(reinterpret_cast<uintptr_t>(stage) - g.c_begin);
    uint8_t* out = S->cache_base() + block;
    for (size_t k = 0; k < g.tensors.size(); ++k) {
        bs_status st = S->batch->add(S->tensors[g.tensors[k]], static_cast<uint32_t>(g.tensors[k]), base, S->d_ws,
                                     out + g.out_off[k], s);
        if (st) return st;
    }
    bs_status st = S->batch->flush(s);
    if (st) return st;
    ce = cudaEventRecord(S->stage_done[slot], s);
    if (ce == cudaSuccess) ce = cudaEventRecord(g.ready, s);
    if (ce != cudaSuccess) return cuda_err(ce);
    g.block = block;
    g.resident = true;
    g.released_recorded = false;
    ++S->st.loads;
    ++S->st.resident_groups;
    S->st.h2d_bytes += cb;
    S->st.decoded_bytes += g.out_bytes;
    return BS_OK;
}

bool valid_group(const bs_streamer_t* S, int32_t group) {
    return S && group >= 0 && group < static_cast<int32_t>(S->groups.size());
}

} // namespace

extern "C" {

size_t bs_streamer_workspace_bytes(const void* h_container, size_t container_bytes) {
    std::vector<Tensor> ts;
    if (!h_container || parse_host_container(static_cast<const uint8_t*>(h_container), container_bytes, ts) != BS_OK)
        return 0;
    return workspace_bytes_for(ts);
}

size_t bs_streamer_min_arena_bytes(const void* h_container, size_t container_bytes, const int32_t* group_of_tensor) {
    std::vector<Tensor> ts;
    const uint8_t* h = static_cast<const uint8_t*>(h_container);
    if (!h || !group_of_tensor || parse_host_container(h, container_bytes, ts) != BS_OK) return 0;
    std::vector<Group> groups;
    uint64_t max_stage, max_out;
    if (make_groups(ts, h, group_of_tensor, groups, &max_stage, &max_out) != BS_OK) return 0;
    return 2 * max_stage + max_out;
}

bs_status bs_streamer_create(const void* h_container, size_t container_bytes, const int32_t* group_of_tensor,
                             void* d_workspace, size_t workspace_bytes, void* d_arena, size_t arena_bytes,
                             void* stream, bs_streamer_t** out) {
    if (!out) return BS_E_ARG;
    *out = nullptr;
    if (!h_container || !group_of_tensor || !d_workspace || !d_arena) return BS_E_ARG;
    if ((reinterpret_cast<uintptr_t>(d_workspace) | reinterpret_cast<uintptr_t>(d_arena)) & 255u) return BS_E_ARG;
    const uint8_t* h = static_cast<const uint8_t*>(h_container);
    std::unique_ptr<bs_streamer_t> S(new (std::nothrow) bs_streamer_t);
    if (!S) return BS_E_NOMEM;
    bs_status st = parse_host_container(h, container_bytes, S->tensors);
    if (st) return st;
    if (workspace_bytes < workspace_bytes_for(S->tensors)) return BS_E_SIZE;
    uint64_t max_stage, max_out;
    st = make_groups(S->tensors, h, group_of_tensor, S->groups, &max_stage, &max_out);
    if (st) return st;
    if (arena_bytes < 2 * max_stage + max_out) return BS_E_SIZE;
    int dev = 0, major = 0, minor = 0;
    cudaError_t ce = cudaGetDevice(&dev);
    if (ce != cudaSuccess) return cuda_err(ce);
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0) return BS_E_UNSUPPORTED;
    std::vector<uint8_t> image;
    st = build_workspace(S->tensors, image);
    if (st) return st;
    S->h = h;
    S->d_ws = static_cast<uint8_t*>(d_workspace);
    S->d_arena = static_cast<uint8_t*>(d_arena);
    S->stage_bytes = max_stage;
    S->cache.reset(new (std::nothrow) Arena(arena_bytes - 2 * max_stage));
    S->batch.reset(new (std::nothrow) DecodeBatch(reinterpret_cast<unsigned long long*>(S->d_ws)));
    if (!S->cache || !S->batch) return BS_E_NOMEM;
    st = S->batch->init();
    if (st) return st;
    S->st.cache_bytes = arena_bytes - 2 * max_stage;
    S->st.stage_bytes = max_stage;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    ce = cudaMemcpyAsync(d_workspace, image.data(), image.size(), cudaMemcpyHostToDevice, s);
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(s); // `image` is freed on return
    if (ce != cudaSuccess) return cuda_err(ce);
    for (Group& g : S->groups) {
        ce = cudaEventCreateWithFlags(&g.ready, cudaEventDisableTiming);
        if (ce == cudaSuccess) ce = cudaEventCreateWithFlags(&g.released, cudaEventDisableTiming);
        if (ce != cudaSuccess) return cuda_err(ce);
    }
    for (cudaEvent_t& e : S->stage_done) {
        ce = cudaEventCreateWithFlags(&e, cudaEventDisableTiming);
        if (ce != cudaSuccess) return cuda_err(ce);
    }
    *out = S.release();
    return BS_OK;
}

bs_status bs_streamer_group_count(const bs_streamer_t* S, int32_t* n) {
    if (!S || !n) return BS_E_ARG;
    *n = static_cast<int32_t>(S->groups.size());
    return BS_OK;
}

bs_status bs_streamer_tensor_info_get(const bs_streamer_t* S, int32_t idx, bs_tensor_info* o) {
    if (!S || !o || idx < 0 || idx >= static_cast<int32_t>(S->tensors.size())) return BS_E_ARG;
    fill_tensor_info(S->tensors[idx], o);
    return BS_OK;
}

bs_status bs_streamer_prefetch(bs_streamer_t* S, int32_t group, void* stream) {
    if (!valid_group(S, group)) return BS_E_ARG;
    std::lock_guard<std::mutex> lock(S->mu);
    Group& g = S->groups[group];
    if (g.resident) return BS_OK;
    bs_status st = load_group(S, g, static_cast<cudaStream_t>(stream));
    if (st == BS_OK) {
        g.fresh = true;
        g.last_use = ++S->tick;
    }
    return st;
}

bs_status bs_streamer_acquire(bs_streamer_t* S, int32_t group, void** d_ptrs, int32_t n_ptrs, void* stream) {
    if (!valid_group(S, group) || !d_ptrs) return BS_E_ARG;
    std::lock_guard<std::mutex> lock(S->mu);
    Group& g = S->groups[group];
    if (n_ptrs != static_cast<int32_t>(g.tensors.size())) return BS_E_SIZE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (!g.resident) {
        bs_status st = load_group(S, g, s);
        if (st) return st;
    } else {
        cudaError_t ce = cudaStreamWaitEvent(s, g.ready, 0); // it may still be loading on another stream
        if (ce != cudaSuccess) return cuda_err(ce);
        ++S->st.hits;
    }
    ++g.pins;
    g.fresh = false;
    g.last_use = ++S->tick;
    uint8_t* out = S->cache_base() + g.block;
    for (size_t k = 0; k < g.tensors.size(); ++k) d_ptrs[k] = out + g.out_off[k];
    return BS_OK;
}

bs_status bs_streamer_release(bs_streamer_t* S, int32_t group, void* stream) {
    if (!valid_group(S, group)) return BS_E_ARG;
    std::lock_guard<std::mutex> lock(S->mu);
    Group& g = S->groups[group];
    if (!g.resident || g.pins <= 0) return BS_E_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t ce = cudaSuccess;
    // With several pins on several streams, each release point must follow the earlier
    // ones, because the event keeps only its latest record.
    if (g.released_recorded) ce = cudaStreamWaitEvent(s, g.released, 0);
    if (ce == cudaSuccess) ce = cudaEventRecord(g.released, s);
    if (ce != cudaSuccess) return cuda_err(ce);
    g.released_recorded = true;
    --g.pins;
    return BS_OK;
}

bs_status bs_streamer_get_stats(bs_streamer_t* S, bs_streamer_stats_t* out) {
    if (!S || !out) return BS_E_ARG;
    std::lock_guard<std::mutex> lock(S->mu);
    *out = S->st;
    out->cache_bytes_used = S->cache->used();
    return BS_OK;
}

bs_status bs_streamer_check(bs_streamer_t* S, void* stream, int64_t* first_bad) {
    if (!S) return BS_E_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned long long hbuf[2] = {0, 0};
    cudaError_t ce = cudaMemcpyAsync(hbuf, S->d_ws, 16, cudaMemcpyDeviceToHost, s);
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(s);
    if (ce != cudaSuccess) return cuda_err(ce);
    if (first_bad) *first_bad = hbuf[0] ? static_cast<int64_t>(hbuf[1]) : -1;
    if (!hbuf[0]) return BS_OK;
    static const unsigned long long reset[2] = {0, ~0ull};
    ce = cudaMemcpyAsync(S->d_ws, reset, 16, cudaMemcpyHostToDevice, s);
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(s);
    if (ce != cudaSuccess) return cuda_err(ce);
    return BS_E_CORRUPT;
}

void bs_streamer_destroy(bs_streamer_t* S) { delete S; }

} // extern "C"
